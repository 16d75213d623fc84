"""ctypes bindings of the fp64 oracle.  Test infrastructure only."""
from __future__ import annotations

import ctypes as C
from typing import Dict, Optional, Sequence

import numpy as np
import torch

from .build import build_oracle

ORC_F32, ORC_BF16, ORC_FP8, ORC_MXFP4 = 0, 1, 2, 3

_lib = None


class Dims(C.Structure):
    _fields_ = [("n_layers", C.c_int32), ("hidden", C.c_int32), ("n_q_heads", C.c_int32),
                ("n_kv_heads", C.c_int32), ("head_dim", C.c_int32), ("ffn", C.c_int32),
                ("vocab", C.c_int32), ("n_experts", C.c_int32), ("top_k", C.c_int32),
                ("expert_ffn", C.c_int32), ("rms_eps", C.c_double), ("rope_theta", C.c_double),
                ("qk_norm", C.c_int32), ("rope_factor", C.c_double), ("rope_low_freq_factor", C.c_double),
                ("rope_high_freq_factor", C.c_double), ("rope_original_max_pos", C.c_double)]


class Layer(C.Structure):
    _fields_ = [("attn_norm", C.c_void_p), ("wqkv", C.c_void_p), ("wo", C.c_void_p),
                ("ffn_norm", C.c_void_p), ("w_gate_up", C.c_void_p), ("w_down", C.c_void_p),
                ("w_router", C.c_void_p), ("we_gate_up", C.c_void_p), ("we_down", C.c_void_p),
                ("q_norm", C.c_void_p), ("k_norm", C.c_void_p)]


class Model(C.Structure):
    _fields_ = [("d", Dims), ("dtype", C.c_int32), ("embed", C.c_void_p), ("lm_head", C.c_void_p),
                ("final_norm", C.c_void_p), ("layers", C.POINTER(Layer)), ("mat_dtype", C.c_int32)]


class Fp8(C.Structure):
    """orc_fp8: E4M3 codes [rows][K] and one fp32 scale per row."""
    _fields_ = [("codes", C.c_void_p), ("scale", C.c_void_p)]


class Mx4(C.Structure):
    """orc_mxfp4: packed E2M1 codes [rows][K/2], block exponents [K/128][rows][4],
    one fp32 scale per row, and the matrix's row count."""
    _fields_ = [("codes", C.c_void_p), ("bscale", C.c_void_p), ("scale", C.c_void_p), ("rows", C.c_int64)]


class Spec(C.Structure):
    _fields_ = [("target", Model), ("drafter", Model), ("block_size", C.c_int32),
                ("n_taps", C.c_int32), ("tap_layers", C.POINTER(C.c_int32)),
                ("mask_token_id", C.c_int32), ("w_fc", C.c_void_p), ("fc_norm", C.c_void_p)]


_dp = C.POINTER(C.c_double)
_ip = C.POINTER(C.c_int32)


def load_lib():
    global _lib
    if _lib is not None:
        return _lib
    lib = C.CDLL(build_oracle())
    lib.orc_rmsnorm.argtypes = [C.c_void_p, C.c_void_p, C.c_int32, C.c_double, C.c_void_p]
    lib.orc_rope.argtypes = [C.c_void_p, C.c_int32, C.c_int64, C.c_double]
    lib.orc_rope_inv_freq.argtypes = [C.POINTER(Dims), C.c_int32]
    lib.orc_rope_inv_freq.restype = C.c_double
    lib.orc_rope_dims.argtypes = [C.c_void_p, C.POINTER(Dims), C.c_int64]
    lib.orc_matmul.argtypes = [C.c_void_p, C.c_int32, C.c_int32, C.c_int32, C.c_void_p, C.c_int32, C.c_void_p]
    lib.orc_matmul_rows.argtypes = [C.c_void_p, C.c_int32, C.c_int32, C.c_int32, C.c_int32, C.c_void_p, C.c_int32,
                                    C.c_void_p]
    lib.orc_e4m3_value.argtypes = [C.c_uint8]
    lib.orc_e4m3_value.restype = C.c_double
    lib.orc_e2m1_value.argtypes = [C.c_uint8]
    lib.orc_e2m1_value.restype = C.c_double
    lib.orc_attend.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int64, C.c_int32, C.c_int32, C.c_void_p]
    lib.orc_argmax.argtypes = [C.c_void_p, C.c_int32, C.c_void_p]
    lib.orc_argmax.restype = C.c_int32
    lib.orc_accept.argtypes = [C.c_void_p, C.c_void_p, C.c_int32]
    lib.orc_accept.restype = C.c_int32
    lib.orc_ffn.argtypes = [C.POINTER(Model), C.c_int32, C.c_void_p, C.c_void_p]
    lib.orc_fuse.argtypes = [C.POINTER(Spec), C.c_void_p, C.c_void_p]
    lib.orc_session_new.argtypes = [C.POINTER(Spec), C.c_int32]
    lib.orc_session_new.restype = C.c_void_p
    lib.orc_session_free.argtypes = [C.c_void_p]
    lib.orc_session_len.argtypes = [C.c_void_p]
    lib.orc_session_len.restype = C.c_int32
    lib.orc_prefill.argtypes = [C.c_void_p, C.c_void_p, C.c_int32, C.c_void_p, C.c_void_p]
    lib.orc_prefill.restype = C.c_int32
    lib.orc_draft.argtypes = [C.c_void_p, C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p]
    lib.orc_verify.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]
    lib.orc_commit.argtypes = [C.c_void_p, C.c_int32]
    lib.orc_commit.restype = C.c_int32
    lib.orc_last_taps.argtypes = [C.c_void_p]
    lib.orc_last_taps.restype = C.c_void_p
    lib.orc_ctx_kv.argtypes = [C.c_void_p, C.c_int32, C.c_int32, C.c_void_p, C.c_void_p]
    lib.orc_target_kv.argtypes = [C.c_void_p, C.c_int32, C.c_int32, C.c_void_p, C.c_void_p]
    lib.orc_generate_ar.argtypes = [C.POINTER(Spec), C.c_void_p, C.c_int32, C.c_int32, C.c_void_p, C.c_void_p]
    lib.orc_generate_spec.argtypes = [C.POINTER(Spec), C.c_void_p, C.c_int32, C.c_int32, C.c_void_p,
                                      C.c_void_p, C.c_void_p]
    lib.orc_generate_spec.restype = C.c_int32
    _lib = lib
    return lib


def _ptr(a) -> int:
    if isinstance(a, np.ndarray):
        return a.ctypes.data
    return a.data_ptr()


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _wtensor(t: torch.Tensor) -> torch.Tensor:
    """Host tensor in a storage type the oracle reads (fp32, bf16 bits or FP8 codes)."""
    t = t.detach().to("cpu").contiguous()
    if t.dtype not in (torch.float32, torch.bfloat16, torch.uint8):
        raise TypeError(t.dtype)
    return t


def dims(d) -> Dims:
    """The oracle's view of one model's shape and settings."""
    f, lo, hi, orig = (float(x) for x in d.rope_scaling)
    return Dims(d.n_layers, d.hidden, d.n_q_heads, d.n_kv_heads, d.head_dim, d.ffn, d.vocab,
                d.n_experts, d.top_k, d.expert_ffn, float(d.rms_eps), float(d.rope_theta),
                1 if d.qk_norm else 0, f, lo, hi, orig)


class OracleSpec:
    """A target + drafter + fuse weight set, viewed by the C oracle (no copies)."""

    def __init__(self, cfg, weights: Dict[str, torch.Tensor]):
        self.cfg = cfg
        self.lib = load_lib()
        self._keep = []
        w = {k: _wtensor(v) for k, v in weights.items()}
        self._keep.append(w)
        dtype = ORC_BF16 if w["embed"].dtype == torch.bfloat16 else ORC_F32
        if w["lm_head"].dtype == torch.uint8:
            self.mat_dtype = ORC_MXFP4 if "lm_head.bscale" in w else ORC_FP8
        else:
            self.mat_dtype = dtype
        for k, v in w.items():
            if k == "embed" or k.endswith(".scale") or k.endswith(".bscale"):
                continue
            if v.dim() > 1 and v.dtype != {ORC_BF16: torch.bfloat16, ORC_F32: torch.float32,
                                           ORC_FP8: torch.uint8, ORC_MXFP4: torch.uint8}[self.mat_dtype]:
                raise TypeError(f"{k}: mixed storage types")
            if v.dim() == 1 and v.dtype != torch.float32:
                raise TypeError(f"{k}: norm gains must be fp32")
        self._w = w
        self.spec = Spec()
        self.spec.target = self._model("target", cfg.target, w, dtype)
        self.spec.drafter = self._model("drafter", cfg.drafter, w, dtype)
        self.spec.block_size = cfg.block_size
        taps = _i32(cfg.tap_layers)
        self._keep.append(taps)
        self.spec.n_taps = len(cfg.tap_layers)
        self.spec.tap_layers = taps.ctypes.data_as(_ip)
        self.spec.mask_token_id = cfg.mask_id
        self.spec.w_fc = self._mat("fuse.w_fc")
        self.spec.fc_norm = _ptr(w["fuse.norm"])

    def _mat(self, name):
        """Address the oracle reads matrix `name` from: its storage, or for FP8 /
        MXFP4 weights a descriptor of its codes and scales."""
        if self.mat_dtype == ORC_FP8:
            q = Fp8(_ptr(self._w[name]), _ptr(self._w[name + ".scale"]))
        elif self.mat_dtype == ORC_MXFP4:
            q = Mx4(_ptr(self._w[name]), _ptr(self._w[name + ".bscale"]), _ptr(self._w[name + ".scale"]),
                    self._w[name].shape[0])
        else:
            return _ptr(self._w[name])
        self._keep.append(q)
        return C.addressof(q)

    def _model(self, prefix, d, w, dtype) -> Model:
        m = Model()
        m.d = dims(d)
        m.dtype = dtype
        m.mat_dtype = self.mat_dtype
        if self.mat_dtype in (ORC_FP8, ORC_MXFP4) and d.n_experts > 0:
            raise ValueError("the oracle reads FP8 / MXFP4 weights for dense models only")
        m.embed = _ptr(w["embed"])
        m.lm_head = self._mat("lm_head")
        m.final_norm = _ptr(w[f"{prefix}.final_norm"])
        layers = (Layer * max(1, d.n_layers))()
        for l in range(d.n_layers):
            p = f"{prefix}.L{l}."
            L = layers[l]
            L.attn_norm = _ptr(w[p + "attn_norm"])
            L.wqkv = self._mat(p + "wqkv")
            L.wo = self._mat(p + "wo")
            L.ffn_norm = _ptr(w[p + "ffn_norm"])
            if d.qk_norm:
                L.q_norm = _ptr(w[p + "q_norm"])
                L.k_norm = _ptr(w[p + "k_norm"])
            if d.n_experts > 0:
                L.w_router = _ptr(w[p + "w_router"])
                L.we_gate_up = _ptr(w[p + "we_gate_up"])
                L.we_down = _ptr(w[p + "we_down"])
            else:
                L.w_gate_up = self._mat(p + "w_gate_up")
                L.w_down = self._mat(p + "w_down")
        self._keep.append(layers)
        m.layers = C.cast(layers, C.POINTER(Layer))
        return m

    # ---- whole generations ----
    def generate_ar(self, prompt, max_new: int, with_margins: bool = False):
        p = _i32(prompt)
        out = np.zeros(max_new, np.int32)
        mg = np.zeros(max_new, np.float64) if with_margins else None
        self.lib.orc_generate_ar(C.byref(self.spec), p.ctypes.data, len(p), max_new, out.ctypes.data,
                                 mg.ctypes.data if mg is not None else None)
        return (out, mg) if with_margins else out

    def generate_spec(self, prompt, max_new: int, forced: Optional[Sequence[int]] = None):
        p = _i32(prompt)
        out = np.zeros(max_new, np.int32)
        acc = np.zeros(max(1, max_new), np.int32)
        f = _i32(forced) if forced is not None else None
        if f is not None and len(f) < max_new + self.cfg.block_size:
            raise ValueError("forced script must hold max_new + block_size tokens")
        it = self.lib.orc_generate_spec(C.byref(self.spec), p.ctypes.data, len(p), max_new,
                                        f.ctypes.data if f is not None else None,
                                        out.ctypes.data, acc.ctypes.data)
        return out, acc[:it]

    def session(self, max_len: int) -> "OracleSession":
        return OracleSession(self, max_len)

    def fuse(self, taps) -> np.ndarray:
        t = _f64(taps)
        c = np.zeros(self.cfg.drafter.hidden, np.float64)
        self.lib.orc_fuse(C.byref(self.spec), t.ctypes.data, c.ctypes.data)
        return c

    def ffn(self, which: str, layer: int, x) -> np.ndarray:
        m = self.spec.target if which == "target" else self.spec.drafter
        xx = _f64(x)
        out = np.zeros_like(xx)
        self.lib.orc_ffn(C.byref(m), layer, xx.ctypes.data, out.ctypes.data)
        return out


class OracleSession:
    """One sequence's oracle state: target KV, drafter context KV, taps."""

    def __init__(self, spec: OracleSpec, max_len: int):
        self.spec = spec
        self.lib = spec.lib
        self.cfg = spec.cfg
        self.h = self.lib.orc_session_new(C.byref(spec.spec), max_len)

    def __del__(self):
        if getattr(self, "h", None):
            self.lib.orc_session_free(self.h)
            self.h = None

    @property
    def len(self) -> int:
        return self.lib.orc_session_len(self.h)

    def prefill(self, prompt, want_logits: bool = False):
        p = _i32(prompt)
        V = self.cfg.target.vocab
        lg = np.zeros(V, np.float64) if want_logits else None
        mg = np.zeros(1, np.float64)
        tok = self.lib.orc_prefill(self.h, p.ctypes.data, len(p),
                                   lg.ctypes.data if lg is not None else None, mg.ctypes.data)
        return tok, mg[0], lg

    def draft(self, anchor: int, want_logits: bool = False):
        B, V = self.cfg.block_size, self.cfg.target.vocab
        d = np.zeros(max(1, B - 1), np.int32)
        mg = np.zeros(max(1, B - 1), np.float64)
        lg = np.zeros((B - 1, V), np.float64) if want_logits else None
        self.lib.orc_draft(self.h, int(anchor), d.ctypes.data,
                           lg.ctypes.data if lg is not None else None, mg.ctypes.data)
        return d[:B - 1], mg[:B - 1], lg

    def verify(self, tokens, want_logits: bool = False):
        B, V = self.cfg.block_size, self.cfg.target.vocab
        t = _i32(tokens)
        assert len(t) == B
        g = np.zeros(B, np.int32)
        mg = np.zeros(B, np.float64)
        lg = np.zeros((B, V), np.float64) if want_logits else None
        self.lib.orc_verify(self.h, t.ctypes.data, g.ctypes.data,
                            lg.ctypes.data if lg is not None else None, mg.ctypes.data)
        return g, mg, lg

    def commit(self, a: int) -> int:
        return self.lib.orc_commit(self.h, int(a))

    def ctx_kv(self, layer: int, pos: int):
        d = self.cfg.drafter
        n = d.n_kv_heads * d.head_dim
        k = np.zeros(n, np.float64)
        v = np.zeros(n, np.float64)
        self.lib.orc_ctx_kv(self.h, layer, pos, k.ctypes.data, v.ctypes.data)
        return k, v

    def target_kv(self, layer: int, pos: int):
        d = self.cfg.target
        n = d.n_kv_heads * d.head_dim
        k = np.zeros(n, np.float64)
        v = np.zeros(n, np.float64)
        self.lib.orc_target_kv(self.h, layer, pos, k.ctypes.data, v.ctypes.data)
        return k, v


# ---- building blocks, for pinning ----
def rmsnorm(x, g, eps: float) -> np.ndarray:
    lib = load_lib()
    xx = _f64(x)
    gg = np.ascontiguousarray(np.asarray(g, np.float32))
    y = np.zeros_like(xx)
    lib.orc_rmsnorm(xx.ctypes.data, gg.ctypes.data, len(xx), eps, y.ctypes.data)
    return y


def rope_inv_freq(d, i: int) -> float:
    """Inverse frequency of RoPE pair i of model shape d (with its rescaling, if any)."""
    dd = dims(d)
    return load_lib().orc_rope_inv_freq(C.byref(dd), i)


def rope_dims(v, pos: int, d) -> np.ndarray:
    """RoPE of one head vector at pos under model shape d's settings."""
    out = _f64(v).copy()
    dd = dims(d)
    load_lib().orc_rope_dims(out.ctypes.data, C.byref(dd), pos)
    return out


def rope(v, pos: int, theta: float) -> np.ndarray:
    lib = load_lib()
    vv = _f64(v).copy()
    lib.orc_rope(vv.ctypes.data, len(vv), pos, theta)
    return vv


def matmul(W: torch.Tensor, X) -> np.ndarray:
    lib = load_lib()
    W = _wtensor(W)
    dt = ORC_BF16 if W.dtype == torch.bfloat16 else ORC_F32
    N, K = W.shape
    XX = _f64(X).reshape(-1, K)
    Y = np.zeros((XX.shape[0], N), np.float64)
    lib.orc_matmul(_ptr(W), dt, N, K, XX.ctypes.data, XX.shape[0], Y.ctypes.data)
    return Y


def matmul_fp8(codes: torch.Tensor, scale: torch.Tensor, X, row0: int = 0, n_rows: Optional[int] = None) -> np.ndarray:
    """Y[r][n] = sum_k scale[row0+n] * e4m3(codes[row0+n][k]) * X[r][k] through the oracle."""
    lib = load_lib()
    codes, scale = _wtensor(codes), _wtensor(scale)
    N, K = codes.shape
    n = N - row0 if n_rows is None else n_rows
    q = Fp8(_ptr(codes), _ptr(scale))
    XX = _f64(X).reshape(-1, K)
    Y = np.zeros((XX.shape[0], n), np.float64)
    lib.orc_matmul_rows(C.addressof(q), ORC_FP8, row0, n, K, XX.ctypes.data, XX.shape[0], Y.ctypes.data)
    return Y


def e4m3_value(code: int) -> float:
    return load_lib().orc_e4m3_value(int(code) & 0xFF)


def e2m1_value(code: int) -> float:
    return load_lib().orc_e2m1_value(int(code) & 0xF)


def matmul_mxfp4(codes: torch.Tensor, bscale: torch.Tensor, scale: torch.Tensor, X, row0: int = 0,
                 n_rows: Optional[int] = None) -> np.ndarray:
    """Y[r][n] = sum_k W_q[row0+n][k] * X[r][k] through the oracle (W_q the MXFP4
    matrix's quantised weights)."""
    lib = load_lib()
    codes, bscale, scale = _wtensor(codes), _wtensor(bscale), _wtensor(scale)
    N, K2 = codes.shape
    K = 2 * K2
    n = N - row0 if n_rows is None else n_rows
    q = Mx4(_ptr(codes), _ptr(bscale), _ptr(scale), N)
    XX = _f64(X).reshape(-1, K)
    Y = np.zeros((XX.shape[0], n), np.float64)
    lib.orc_matmul_rows(C.addressof(q), ORC_MXFP4, row0, n, K, XX.ctypes.data, XX.shape[0], Y.ctypes.data)
    return Y


def attend(q, keys, vals) -> np.ndarray:
    lib = load_lib()
    qq = _f64(q)
    kk = _f64(keys)
    vv = _f64(vals)
    n, hd = kk.shape
    out = np.zeros(hd, np.float64)
    lib.orc_attend(qq.ctypes.data, kk.ctypes.data, vv.ctypes.data, hd, n, hd, out.ctypes.data)
    return out


def argmax(x):
    lib = load_lib()
    xx = _f64(x)
    m = np.zeros(1, np.float64)
    i = lib.orc_argmax(xx.ctypes.data, len(xx), m.ctypes.data)
    return i, m[0]


def accept(drafts, g, block_size: int) -> int:
    lib = load_lib()
    d = _i32(drafts)
    gg = _i32(g)
    return lib.orc_accept(d.ctypes.data, gg.ctypes.data, block_size)
