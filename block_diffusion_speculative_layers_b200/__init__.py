"""Python binding of libdflash (the DFlash draft-and-verify decode library).

Argument marshalling only: every step of prefill, drafting, verification and
commit runs in the library's CUDA kernels.  PyTorch supplies device memory (the
two arenas) and the CUDA stream.  The library must be built
(``python -m block_diffusion_speculative_layers_b200.build``); importing the
binding without it raises instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Dict, Optional, Sequence

import numpy as np
import torch

from .build import lib_path

DFLASH_OK, DFLASH_EINVAL, DFLASH_ESTATE, DFLASH_ECAPACITY = 0, 1, 2, 3
DFLASH_ECUDA, DFLASH_ENUMERIC, DFLASH_ETIMEOUT, DFLASH_EUNSUPPORTED = 4, 5, 6, 7
DFLASH_FP32, DFLASH_BF16, DFLASH_BF16_FAST, DFLASH_FP8, DFLASH_FP4, DFLASH_UE8M0 = 0, 1, 2, 3, 4, 5
_SLOT_TYPES = {DFLASH_FP32: (torch.float32, 4), DFLASH_BF16: (torch.bfloat16, 2), DFLASH_FP8: (torch.uint8, 1),
               DFLASH_FP4: (torch.uint8, 1), DFLASH_UE8M0: (torch.uint8, 1)}
DFLASH_DRAFT_MODEL, DFLASH_DRAFT_SCRIPT = 0, 1
MAX_TAPS, MAX_BLOCK = 8, 32
# dflash_profile_read classes, in the order of the DFLASH_PROF_* values
PROF_CLASSES = ("projection", "attention", "gate_up", "qkv", "o", "down", "lm_head", "fuse", "other_proj",
                "draft_pass", "verify_pass")

STATUS_NAMES = {0: "OK", 1: "EINVAL", 2: "ESTATE", 3: "ECAPACITY", 4: "ECUDA", 5: "ENUMERIC",
                6: "ETIMEOUT", 7: "EUNSUPPORTED"}

# Every symbol include/dflash.h declares.
EXPORTS = [
    "dflash_workspace_size", "dflash_create", "dflash_destroy", "dflash_last_error",
    "dflash_weight_count", "dflash_weight_info", "dflash_weight_slot", "dflash_prefill",
    "dflash_draft_block", "dflash_verify_commit", "dflash_generate", "dflash_generate_ar",
    "dflash_set_draft_mode", "dflash_set_script", "dflash_debug_logits", "dflash_seq_state",
    "dflash_debug_kv", "dflash_decode_iters", "dflash_get_stats", "dflash_reset_stats",
    "dflash_profile", "dflash_profile_read", "dflash_head_argmax_noalloc", "dflash_set_sampling",
]


class DFlashError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str = ""):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} {msg}".strip())


class ModelCfg(C.Structure):
    _fields_ = [("n_layers", C.c_int32), ("hidden", C.c_int32), ("n_q_heads", C.c_int32),
                ("n_kv_heads", C.c_int32), ("head_dim", C.c_int32), ("ffn", C.c_int32),
                ("vocab", C.c_int32), ("n_experts", C.c_int32), ("top_k", C.c_int32),
                ("expert_ffn", C.c_int32), ("rms_eps", C.c_double), ("rope_theta", C.c_double),
                ("qk_norm", C.c_int32), ("reserved", C.c_int32), ("rope_factor", C.c_double),
                ("rope_low_freq_factor", C.c_double), ("rope_high_freq_factor", C.c_double),
                ("rope_original_max_pos", C.c_double)]


class Config(C.Structure):
    _fields_ = [("target", ModelCfg), ("drafter", ModelCfg), ("block_size", C.c_int32),
                ("n_taps", C.c_int32), ("tap_layers", C.c_int32 * MAX_TAPS),
                ("mask_token_id", C.c_int32), ("max_batch", C.c_int32), ("max_len", C.c_int32),
                ("prefill_chunk", C.c_int32), ("dtype", C.c_int32), ("keep_logits", C.c_int32),
                ("timeout_ms", C.c_int32), ("sampling", C.c_int32)]


class Stats(C.Structure):
    _fields_ = [("iterations", C.c_int64), ("tokens", C.c_int64),
                ("accept_hist", C.c_int64 * MAX_BLOCK), ("mean_tau", C.c_double),
                ("ms_prefill", C.c_double), ("ms_decode", C.c_double),
                ("kernel_launches", C.c_int64)]


class KernelProf(C.Structure):
    _fields_ = [("launches", C.c_int64), ("ms", C.c_double), ("bytes", C.c_double)]


_lib = None
_vp, _i32, _i64, _sz = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t
_ip = C.POINTER(C.c_int32)


def load_library(path: Optional[str] = None):
    """Load libdflash.so; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or lib_path()
    if not os.path.exists(path):
        raise ImportError(f"libdflash.so not built at {path}: run "
                          "`python -m block_diffusion_speculative_layers_b200.build`")
    lib = C.CDLL(path)
    sig = {
        "dflash_workspace_size": (_i32, [C.POINTER(Config), C.POINTER(_sz), C.POINTER(_sz)]),
        "dflash_create": (_i32, [C.POINTER(Config), _vp, _sz, _vp, _sz, _vp, C.POINTER(_vp)]),
        "dflash_destroy": (None, [_vp]),
        "dflash_last_error": (C.c_char_p, [_vp]),
        "dflash_weight_count": (_i32, [_vp]),
        "dflash_weight_info": (_i32, [_vp, _i32, C.POINTER(C.c_char_p), C.POINTER(_sz), C.POINTER(_sz),
                                      _ip, _ip, C.POINTER(_i64)]),
        "dflash_weight_slot": (_i32, [_vp, C.c_char_p, C.POINTER(_sz), C.POINTER(_sz), _ip]),
        "dflash_prefill": (_i32, [_vp, _i32, _ip, _i32, _ip]),
        "dflash_draft_block": (_i32, [_vp, _ip, _i32, _ip]),
        "dflash_verify_commit": (_i32, [_vp, _ip, _i32, _ip, _ip, _ip, _ip]),
        "dflash_generate": (_i32, [_vp, C.POINTER(_ip), _ip, _i32, _i32, _ip, C.POINTER(Stats)]),
        "dflash_generate_ar": (_i32, [_vp, C.POINTER(_ip), _ip, _i32, _i32, _ip, C.POINTER(C.c_double)]),
        "dflash_set_draft_mode": (_i32, [_vp, _i32, _i32]),
        "dflash_set_script": (_i32, [_vp, _i32, _ip, _i32]),
        "dflash_debug_logits": (_i32, [_vp, _i32, C.POINTER(C.c_float), _i64, C.POINTER(_i64)]),
        "dflash_seq_state": (_i32, [_vp, _i32, _ip, _ip, _ip]),
        "dflash_debug_kv": (_i32, [_vp, _i32, _i32, _i32, _i32, _i32, C.POINTER(C.c_float),
                                   C.POINTER(C.c_float)]),
        "dflash_decode_iters": (_i32, [_vp, _i32, _i32]),
        "dflash_get_stats": (_i32, [_vp, C.POINTER(Stats)]),
        "dflash_reset_stats": (_i32, [_vp]),
        "dflash_profile": (_i32, [_vp, _i32]),
        "dflash_profile_read": (_i32, [_vp, C.POINTER(KernelProf)]),
        "dflash_head_argmax_noalloc": (_i32, [_vp, _i32, _ip, _ip]),
        "dflash_set_sampling": (_i32, [_vp, C.c_double, C.c_uint64]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _model_cfg(d) -> ModelCfg:
    f, lo, hi, orig = (float(x) for x in getattr(d, "rope_scaling", (0.0, 0.0, 0.0, 0.0)))
    return ModelCfg(d.n_layers, d.hidden, d.n_q_heads, d.n_kv_heads, d.head_dim, d.ffn, d.vocab,
                    d.n_experts, d.top_k, d.expert_ffn, float(d.rms_eps), float(d.rope_theta),
                    1 if getattr(d, "qk_norm", False) else 0, 0, f, lo, hi, orig)


def make_config(spec, max_batch: int = 1, max_len: int = 4096, prefill_chunk: int = 0,
                keep_logits: bool = False, timeout_ms: int = 0, bf16_act: str = "split",
                sampling: bool = False) -> Config:
    """dflash_config from any object with target/drafter dims, block_size, tap_layers,
    mask_id and dtype ("bf16" / "fp32") attributes.  bf16_act selects how a bf16
    model carries its activations: "split" (two bf16 planes, DFLASH_BF16) or
    "fast" (one plane, DFLASH_BF16_FAST)."""
    if bf16_act not in ("split", "fast"):
        raise ValueError("bf16_act must be 'split' or 'fast'")
    c = Config()
    c.target = _model_cfg(spec.target)
    c.drafter = _model_cfg(spec.drafter)
    c.block_size = spec.block_size
    taps = list(spec.tap_layers)
    if len(taps) > MAX_TAPS:
        raise ValueError("too many tap layers")
    c.n_taps = len(taps)
    for i, t in enumerate(taps):
        c.tap_layers[i] = t
    c.mask_token_id = spec.mask_id
    c.max_batch = max_batch
    c.max_len = max_len
    c.prefill_chunk = prefill_chunk
    if spec.dtype == "bf16":
        c.dtype = DFLASH_BF16 if bf16_act == "split" else DFLASH_BF16_FAST
    elif spec.dtype == "fp8":
        c.dtype = DFLASH_FP8
    elif spec.dtype == "fp4":
        c.dtype = DFLASH_FP4
    else:
        c.dtype = DFLASH_FP32
    c.keep_logits = 1 if keep_logits else 0
    c.sampling = 1 if sampling else 0
    c.timeout_ms = timeout_ms
    return c


def _ints(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _iptr(a: np.ndarray):
    return a.ctypes.data_as(_ip)


class DFlash:
    """One dflash context with torch-owned device arenas on the current CUDA device."""

    def __init__(self, spec, max_batch: int = 1, max_len: int = 4096, prefill_chunk: int = 0,
                 keep_logits: bool = False, device: Optional[torch.device] = None,
                 stream: Optional[torch.cuda.Stream] = None, timeout_ms: int = 0, bf16_act: str = "split",
                 sampling: bool = False):
        self.lib = load_library()
        self.spec = spec
        self.cfg = make_config(spec, max_batch, max_len, prefill_chunk, keep_logits, timeout_ms, bf16_act,
                               sampling)
        self.device = torch.device(device or "cuda")
        wb, sb = _sz(), _sz()
        self._check(self.lib.dflash_workspace_size(C.byref(self.cfg), C.byref(wb), C.byref(sb)),
                    "dflash_workspace_size")
        self.weight_bytes, self.state_bytes = wb.value, sb.value
        self.warena = torch.empty(self.weight_bytes + 256, dtype=torch.uint8, device=self.device)
        self.sarena = torch.empty(self.state_bytes + 256, dtype=torch.uint8, device=self.device)
        self._woff = (-self.warena.data_ptr()) % 256
        self._soff = (-self.sarena.data_ptr()) % 256
        self.stream = stream or torch.cuda.current_stream(self.device)
        h = _vp()
        with torch.cuda.device(self.device):
            st = self.lib.dflash_create(C.byref(self.cfg), self.warena.data_ptr() + self._woff, self.weight_bytes,
                                        self.sarena.data_ptr() + self._soff, self.state_bytes,
                                        self.stream.cuda_stream, C.byref(h))
        self._check(st, "dflash_create")
        self.h = h
        self.block_size = spec.block_size
        self.vocab = spec.target.vocab

    def __del__(self):
        h = getattr(self, "h", None)
        if h:
            self.lib.dflash_destroy(h)
            self.h = None

    def close(self):
        self.__del__()

    def _check(self, st: int, where: str):
        if st != DFLASH_OK:
            msg = ""
            if getattr(self, "h", None):
                msg = (self.lib.dflash_last_error(self.h) or b"").decode()
            raise DFlashError(st, where, msg)

    # ---- weights ----
    def weight_slots(self):
        out = {}
        for i in range(self.lib.dflash_weight_count(self.h)):
            name, off, numel = C.c_char_p(), _sz(), _sz()
            dt, nd = C.c_int32(), C.c_int32()
            shape = (_i64 * 3)()
            self._check(self.lib.dflash_weight_info(self.h, i, C.byref(name), C.byref(off), C.byref(numel),
                                                    C.byref(dt), C.byref(nd), shape), "dflash_weight_info")
            out[name.value.decode()] = (off.value, numel.value, dt.value, tuple(shape[:nd.value]))
        return out

    def weight_view(self, name: str) -> torch.Tensor:
        off, numel, dt, shape = self.weight_slots()[name]
        tdt, es = _SLOT_TYPES[dt]
        base = self._woff + off
        return self.warena[base:base + numel * es].view(tdt).view(shape)

    def load_weights(self, weights: Dict[str, torch.Tensor]):
        slots = self.weight_slots()
        missing = set(slots) - set(weights)
        if missing:
            raise KeyError(f"missing weights: {sorted(missing)[:5]}")
        for name, (off, numel, dt, shape) in slots.items():
            t = weights[name]
            tdt, es = _SLOT_TYPES[dt]
            if tuple(t.shape) != shape or t.dtype != tdt:
                raise ValueError(f"{name}: expected {shape} {tdt}, got {tuple(t.shape)} {t.dtype}")
            base = self._woff + off
            self.warena[base:base + numel * es].view(tdt).view(shape).copy_(t, non_blocking=False)
        torch.cuda.synchronize(self.device)

    # ---- decode steps ----
    def prefill(self, seq: int, prompt: Sequence[int]) -> int:
        p = _ints(prompt)
        first = C.c_int32()
        self._check(self.lib.dflash_prefill(self.h, seq, _iptr(p), len(p), C.byref(first)), "dflash_prefill")
        return first.value

    def draft_block(self, seqs: Sequence[int]) -> np.ndarray:
        s = _ints(seqs)
        d = np.zeros(max(1, len(s) * (self.block_size - 1)), np.int32)
        self._check(self.lib.dflash_draft_block(self.h, _iptr(s), len(s), _iptr(d)), "dflash_draft_block")
        return d[:len(s) * (self.block_size - 1)].reshape(len(s), self.block_size - 1)

    def verify_commit(self, seqs: Sequence[int], drafts=None):
        s = _ints(seqs)
        n, B = len(s), self.block_size
        dptr = None
        if drafts is not None:
            dd = _ints(drafts).reshape(-1)
            if len(dd) != n * (B - 1):
                raise ValueError("drafts must hold n*(B-1) ids")
            dptr = _iptr(dd) if len(dd) else None
        acc = np.zeros(n, np.int32)
        com = np.zeros(n * B, np.int32)
        nl = np.zeros(n, np.int32)
        self._check(self.lib.dflash_verify_commit(self.h, _iptr(s), n, dptr, _iptr(acc), _iptr(com), _iptr(nl)),
                    "dflash_verify_commit")
        return acc, com.reshape(n, B), nl

    def generate(self, prompts, max_new: int):
        n = len(prompts)
        arrs = [_ints(p) for p in prompts]
        ptrs = (_ip * n)(*[_iptr(a) for a in arrs])
        lens = _ints([len(a) for a in arrs])
        out = np.zeros(n * max_new, np.int32)
        st = Stats()
        self._check(self.lib.dflash_generate(self.h, ptrs, _iptr(lens), n, max_new, _iptr(out), C.byref(st)),
                    "dflash_generate")
        return out.reshape(n, max_new), st

    def generate_ar(self, prompts, max_new: int):
        n = len(prompts)
        arrs = [_ints(p) for p in prompts]
        ptrs = (_ip * n)(*[_iptr(a) for a in arrs])
        lens = _ints([len(a) for a in arrs])
        out = np.zeros(n * max_new, np.int32)
        ms = C.c_double()
        self._check(self.lib.dflash_generate_ar(self.h, ptrs, _iptr(lens), n, max_new, _iptr(out), C.byref(ms)),
                    "dflash_generate_ar")
        return out.reshape(n, max_new), ms.value

    def decode_iters(self, n_seqs: int, iters: int):
        """Enqueue draft+verify iterations on slots 0..n_seqs-1 (asynchronous)."""
        self._check(self.lib.dflash_decode_iters(self.h, n_seqs, iters), "dflash_decode_iters")

    def stats(self) -> Stats:
        st = Stats()
        self._check(self.lib.dflash_get_stats(self.h, C.byref(st)), "dflash_get_stats")
        return st

    def reset_stats(self):
        self._check(self.lib.dflash_reset_stats(self.h), "dflash_reset_stats")

    def profile(self, mode):
        """mode: False/0 off, True/1 events around every kernel launch, 2 around passes, 3 both."""
        self._check(self.lib.dflash_profile(self.h, int(mode)), "dflash_profile")

    def profile_read(self):
        """{class name: (launches, ms, algorithmic bytes)} of the current record."""
        out = (KernelProf * len(PROF_CLASSES))()
        self._check(self.lib.dflash_profile_read(self.h, out), "dflash_profile_read")
        return {name: (out[i].launches, out[i].ms, out[i].bytes) for i, name in enumerate(PROF_CLASSES)}

    def load_weights_from(self, make_one, names=None):
        """Fill each weight slot from make_one(name) (one tensor alive at a time)."""
        slots = self.weight_slots()
        for name in (names or slots):
            off, numel, dt, shape = slots[name]
            t = make_one(name)
            tdt, es = _SLOT_TYPES[dt]
            if tuple(t.shape) != shape or t.dtype != tdt:
                raise ValueError(f"{name}: expected {shape} {tdt}, got {tuple(t.shape)} {t.dtype}")
            base = self._woff + off
            self.warena[base:base + numel * es].view(tdt).view(shape).copy_(t)
            del t
        torch.cuda.synchronize(self.device)

    def head_argmax_noalloc(self, which: int) -> np.ndarray:
        """Greedy ids of the rows of the last pass (0 draft, 1 verify, 2 prefill),
        computed without any caller-provided scratch (see dflash.h)."""
        cap = max(64, self.cfg.max_batch * self.block_size)
        out = np.zeros(cap, np.int32)
        n = C.c_int32()
        self._check(self.lib.dflash_head_argmax_noalloc(self.h, which, _iptr(out), C.byref(n)),
                    "dflash_head_argmax_noalloc")
        return out[:n.value].copy()

    def set_draft_mode(self, mode: int, tau: int = 1):
        self._check(self.lib.dflash_set_draft_mode(self.h, mode, tau), "dflash_set_draft_mode")

    def set_sampling(self, temperature: float, seed: int = 0):
        """Temperature sampling (needs sampling=True at construction); 0 = greedy."""
        self._check(self.lib.dflash_set_sampling(self.h, float(temperature), int(seed) & (2 ** 64 - 1)),
                    "dflash_set_sampling")

    def set_script(self, seq: int, script: Sequence[int]):
        s = _ints(script)
        self._check(self.lib.dflash_set_script(self.h, seq, _iptr(s), len(s)), "dflash_set_script")

    def debug_logits(self, which: int, n_rows: int) -> np.ndarray:
        V = self.vocab
        out = np.zeros((max(1, n_rows), V), np.float32)
        rows = _i64()
        self._check(self.lib.dflash_debug_logits(self.h, which, out.ctypes.data_as(C.POINTER(C.c_float)),
                                                 out.size, C.byref(rows)), "dflash_debug_logits")
        return out[:rows.value]

    def seq_state(self, seq: int):
        a, b, c = C.c_int32(), C.c_int32(), C.c_int32()
        self._check(self.lib.dflash_seq_state(self.h, seq, C.byref(a), C.byref(b), C.byref(c)), "dflash_seq_state")
        return a.value, b.value, c.value

    def debug_kv(self, which: int, layer: int, seq: int, p0: int, n: int):
        d = self.spec.target if which == 0 else self.spec.drafter
        w = d.n_kv_heads * d.head_dim
        k = np.zeros((n, w), np.float32)
        v = np.zeros((n, w), np.float32)
        fp = C.POINTER(C.c_float)
        self._check(self.lib.dflash_debug_kv(self.h, which, layer, seq, p0, n, k.ctypes.data_as(fp),
                                             v.ctypes.data_as(fp)), "dflash_debug_kv")
        return k, v


__all__ = ["DFlash", "DFlashError", "load_library", "make_config", "Config", "Stats", "EXPORTS",
           "DFLASH_DRAFT_MODEL", "DFLASH_DRAFT_SCRIPT", "DFLASH_FP32", "DFLASH_BF16", "DFLASH_BF16_FAST",
           "DFLASH_FP8", "DFLASH_FP4"]
