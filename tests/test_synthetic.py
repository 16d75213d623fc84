"""The two implementations of the synthetic weight generator agree bit for bit."""
import time

import torch

from synthetic import get_config, make_weight, make_prompt
from synthetic.fast import make_weight_host, make_weights_host


def test_fast_generator_matches_torch_generator():
    for cfg in (get_config("tiny"), get_config("tiny").with_(dtype="bf16"), get_config("qwen3_8b")):
        for name in ("embed", "target.L0.wqkv", "target.L1.attn_norm", "fuse.w_fc"):
            if name == "embed" and cfg.name == "qwen3_8b":
                continue  # large; covered by the layer tensors
            a = make_weight(cfg, name, random_gains=True)
            b = make_weight_host(cfg, name, random_gains=True)
            assert a.dtype == b.dtype and a.shape == b.shape
            assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32),
                               b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32)), (cfg.name, name)


def test_generator_statistics():
    w = make_weight_host(get_config("qwen3_8b"), "target.L3.wo").float()
    assert abs(w.mean().item()) < 1e-4
    assert abs(w.std().item() - 0.02) < 2e-4


def test_prompts_are_seeded_and_in_range():
    a = make_prompt("zipf", 512, 151936, 2)
    b = make_prompt("zipf", 512, 151936, 2)
    assert (a == b).all() and a.min() >= 0 and a.max() < 151936
    assert (a < 100).mean() > 0.4   # Zipf(1.1): most mass on frequent ids
