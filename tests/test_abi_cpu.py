"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad configurations before touching the device."""
from __future__ import annotations

import ctypes as C
import os
import re
import subprocess
from dataclasses import replace

import pytest

import block_diffusion_speculative_layers_b200 as dfl
from block_diffusion_speculative_layers_b200.build import build, lib_path
from synthetic import get_config

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return dfl.load_library()


def _declared():
    src = open(os.path.join(ROOT, "include", "dflash.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dflash_[a-z_]+)\s*\(", src)))


def test_header_declares_binding_exports():
    assert _declared() == sorted(dfl.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", lib_path()], capture_output=True, text=True, check=True).stdout
    syms = set(l.split()[-1] for l in out.splitlines() if l.strip())
    for name in _declared():
        assert name in syms, name
        assert getattr(lib, name) is not None


def _sizes(cfg, **kw):
    c = dfl.make_config(cfg, **kw)
    wb, sb = C.c_size_t(), C.c_size_t()
    st = dfl.load_library().dflash_workspace_size(C.byref(c), C.byref(wb), C.byref(sb))
    return st, wb.value, sb.value


def test_workspace_size_matches_weight_count(lib):
    from synthetic.weights import weight_shapes
    cfg = get_config("tiny")
    st, wb, sb = _sizes(cfg, max_batch=2, max_len=256)
    assert st == 0 and sb > 0
    n = sum(int(__import__("numpy").prod(s)) * (4 if k == "norm" or cfg.dtype == "fp32" else 2)
            for s, k in weight_shapes(cfg).values())
    assert n <= wb <= n + 256 * len(weight_shapes(cfg))
    cfg2 = get_config("qwen3_8b")
    st, wb2, _ = _sizes(cfg2, max_batch=1, max_len=3000)
    assert st == 0 and 18.0e9 < wb2 < 19.0e9  # embed + head + 36 + 5 layers + fuse


@pytest.mark.parametrize("mutate", [
    lambda c: c.with_(block_size=0),
    lambda c: c.with_(block_size=33),
    lambda c: c.with_(tap_layers=(0, 5)),
    lambda c: c.with_(mask_token_id=5000),
    lambda c: c.with_(target=replace(c.target, head_dim=96)),
    lambda c: c.with_(target=replace(c.target, n_q_heads=3)),
    lambda c: c.with_(drafter=replace(c.drafter, hidden=128)),
])
def test_bad_configs_rejected(lib, mutate):
    st, _, _ = _sizes(mutate(get_config("tiny")), max_batch=1, max_len=128)
    assert st == dfl.DFLASH_EINVAL if hasattr(dfl, "DFLASH_EINVAL") else st == 1


def test_create_rejects_missing_arenas(lib):
    c = dfl.make_config(get_config("tiny"), max_batch=1, max_len=128)
    h = C.c_void_p()
    assert lib.dflash_create(C.byref(c), None, 0, None, 0, None, C.byref(h)) == 1
    assert lib.dflash_create(C.byref(c), 256, 1 << 40, 256, 1, None, C.byref(h)) == 1  # too small state arena
    assert not h.value


def test_struct_layouts_match_the_header(tmp_path):
    """The ctypes mirrors of dflash_model_cfg / dflash_config / dflash_stats /
    dflash_kernel_prof have the C header's size and field offsets (gcc)."""
    import ctypes as C
    import subprocess
    structs = {"dflash_model_cfg": dfl.ModelCfg, "dflash_config": dfl.Config, "dflash_stats": dfl.Stats,
               "dflash_kernel_prof": dfl.KernelProf}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "dflash.h"', 'int main(void) {']
    for cname, py in structs.items():
        lines.append(f'printf("{cname} size %zu\\n", sizeof({cname}));')
        for f, _ in py._fields_:
            lines.append(f'printf("{cname} {f} %zu\\n", offsetof({cname}, {f}));')
    lines.append("return 0; }")
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    got = {tuple(ln.split()[:2]): int(ln.split()[2]) for ln in out if ln.strip()}
    for cname, py in structs.items():
        assert got[(cname, "size")] == C.sizeof(py), cname
        for f, _ in py._fields_:
            assert got[(cname, f)] == getattr(py, f).offset, (cname, f)


def test_fidelity_toggles_reach_the_library():
    """QK-norm adds the q_norm / k_norm slots of every layer; RoPE rescaling
    needs 0 < low < high and a positive original length (EINVAL otherwise)."""
    import ctypes as C
    from dataclasses import replace
    from synthetic import get_config
    lib = dfl.load_library()
    base = get_config("tiny")

    def sizes(cfg):
        c = dfl.make_config(cfg)
        wb, sb = C.c_size_t(), C.c_size_t()
        return lib.dflash_workspace_size(C.byref(c), C.byref(wb), C.byref(sb)), wb.value

    st0, w0 = sizes(base)
    qk = base.with_(target=replace(base.target, qk_norm=True), drafter=replace(base.drafter, qk_norm=True))
    st1, w1 = sizes(qk)
    assert st0 == st1 == dfl.DFLASH_OK
    n_layers = base.target.n_layers + base.drafter.n_layers
    assert w0 < w1 <= w0 + n_layers * 2 * (base.target.head_dim * 4 + 256)
    ok = base.with_(target=replace(base.target, rope_scaling=(8.0, 1.0, 4.0, 256.0)))
    assert sizes(ok)[0] == dfl.DFLASH_OK
    bad = base.with_(target=replace(base.target, rope_scaling=(8.0, 4.0, 1.0, 256.0)))
    assert sizes(bad)[0] == dfl.DFLASH_EINVAL


def test_quantised_weight_storage_sizes():
    """FP8 and FP4 weight arenas hold what the header describes: the stored bytes
    of every slot synthetic.weights lays out (FP4: codes two per byte, a block
    exponent byte per 32 values, an fp32 scale per row), each slot 256-byte
    aligned; at the Qwen3-8B shape the quantised arenas shrink accordingly; FP4
    refuses widths off the 128 grid and MoE targets."""
    import numpy as np
    from synthetic.weights import weight_shapes
    tiny = get_config("tiny")
    sizes = {}
    for dt in ("bf16", "fp8", "fp4"):
        cfg = tiny.with_(dtype=dt)
        st, wb, _ = _sizes(cfg, max_batch=1, max_len=128)
        assert st == dfl.DFLASH_OK, dt
        stored = 0
        for shape, kind in weight_shapes(cfg).values():
            es = {"norm": 4, "scale": 4, "matrix": 2, "fp8": 1, "fp4": 1, "bscale": 1}[kind]
            stored += int(np.prod(shape)) * es
        n_slots = len(weight_shapes(cfg))
        assert stored <= wb <= stored + 256 * n_slots, dt
        sizes[dt] = wb
    assert sizes["fp4"] < sizes["fp8"] < sizes["bf16"]
    q = {dt: _sizes(get_config("qwen3_8b").with_(dtype=dt), max_batch=1, max_len=3000)[1] for dt in ("fp8", "fp4")}
    # every matrix but the embedding: 1 byte (FP8) or 0.5 + 1/32 byte (FP4) per weight; the embedding stays bf16
    emb = 151936 * 4096 * 2
    assert 8.5e9 < q["fp8"] - emb < 8.8e9  # LM head 0.62 GB + 41 layers x 0.19 GB + fuse
    assert 0.5 * (q["fp8"] - emb) < q["fp4"] - emb < 0.56 * (q["fp8"] - emb)
    off_grid = tiny.with_(dtype="fp4", target=replace(tiny.target, hidden=192, ffn=576),
                          drafter=replace(tiny.drafter, hidden=192, ffn=576))
    assert _sizes(off_grid, max_batch=1, max_len=128)[0] == dfl.DFLASH_EINVAL
    moe = tiny.with_(dtype="fp4", target=replace(tiny.target, n_experts=8, top_k=2, expert_ffn=128))
    assert _sizes(moe, max_batch=1, max_len=128)[0] == dfl.DFLASH_EINVAL
