"""Host-side pieces of bench.py, checked without a GPU: the algorithmic bytes of
one draft+verify step (the roofline's numerator) against a hand count from the
model shapes, and the JSON workload description."""
import math
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
from synthetic import get_config  # noqa: E402


def _dense_layer_params(m):
    qkv = (m.n_q_heads + 2 * m.n_kv_heads) * m.head_dim * m.hidden
    o = m.hidden * m.n_q_heads * m.head_dim
    return qkv + o + 3 * m.hidden * m.ffn


def test_qwen3_8b_step_bytes_hand_count():
    cfg = get_config("qwen3_8b")
    t, d = cfg.target, cfg.drafter
    weights = (t.n_layers * _dense_layer_params(t) + d.n_layers * _dense_layer_params(d)
               + 2 * t.vocab * t.hidden                      # LM head, drafter pass + verify pass
               + d.hidden * cfg.n_taps * t.hidden) * 2       # fuse
    ctx = 1536.0
    kv = (ctx + cfg.block_size) * 2 * 2 * (t.n_layers * t.n_kv_heads + d.n_layers * d.n_kv_heads) * t.head_dim
    got = bench.iteration_bytes(cfg, 1, ctx, kv_planes=1)
    assert got == pytest.approx(weights + kv, rel=1e-9)
    # the figure the step roofline quotes for this shape: about 18.7 GB
    assert 18.5e9 < got < 18.9e9
    # two-plane K/V doubles only the K/V part
    assert bench.iteration_bytes(cfg, 1, ctx, kv_planes=2) - got == pytest.approx(kv, rel=1e-9)


def test_moe_step_counts_touched_experts_only():
    cfg = get_config("qwen3_coder_30b_a3b")
    t = cfg.target
    rows = cfg.block_size
    touched = t.n_experts * (1.0 - (1.0 - t.top_k / t.n_experts) ** rows)
    assert 80 < touched < 85                                  # ~82 of 128 experts per layer at batch 1
    with_experts = bench.iteration_bytes(cfg, 1, 2048.0, kv_planes=1)
    expert_bytes = t.n_layers * touched * 3 * t.hidden * t.expert_ffn * 2
    all_experts = t.n_layers * t.n_experts * 3 * t.hidden * t.expert_ffn * 2
    assert expert_bytes < all_experts
    assert 41e9 < with_experts < 43e9
    # batch 8: 128 rows touch nearly every expert
    b8 = bench.iteration_bytes(cfg, 8, 2048.0, kv_planes=1)
    assert b8 > with_experts
    touched8 = t.n_experts * (1.0 - (1.0 - t.top_k / t.n_experts) ** (8 * rows))
    assert touched8 > 127


def test_workload_config_and_threads():
    cfg = get_config("qwen3_8b")

    class A:
        bf16_act = "split"

    c = bench.workload_config(cfg, A, 2)
    assert c["global_batch"] == 2 * cfg.batch and c["parallelism"] == "replicas x2"
    assert "512-token prompt" in c["workload"] and "36-layer target" in c["workload"]
    assert c["activations"].startswith("bf16 hi+lo")
    assert c["l2"] == "inputs larger than L2 (18.6 GB streamed per step)"
    moe = bench.workload_config(get_config("qwen3_coder_30b_a3b"), A, 1)
    assert moe["l2"] == "inputs larger than L2 (41.6 GB streamed per step)"
    assert bench.workload_config(get_config("tiny"), A, 1)["l2"].startswith("inputs fit in L2")
    assert bench.omp_threads() >= 1
