"""Model shapes of the synthetic workloads.

Each shape is a Llama/Qwen-style pre-norm decoder.  The drafter is a short
decoder of the target's width that shares the target's token embedding and
output head; its context comes from hidden states tapped at several target
layers (DFlash page "DFlash: Decodificação Especulativa com Blocos em Paralelo",
section "O alvo sabe mais").  Block size 16 means the anchor token plus 15
mask positions (the serving snippet on the same page sets
num_speculative_tokens to 15; the ceviu newsletter says 16 tokens per pass).
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Dict, List, Optional, Tuple


@dataclass(frozen=True)
class ModelDims:
    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    rms_eps: float = 1e-6
    rope_theta: float = 1e6
    n_experts: int = 0      # 0 = dense SwiGLU FFN
    top_k: int = 0
    expert_ffn: int = 0
    # fidelity toggles (not on the pages; off by default): per-head RMSNorm of
    # q and k before RoPE as in Qwen3 layers, and the Llama 3.1 RoPE frequency
    # rescaling (factor, low_freq_factor, high_freq_factor, original max
    # position; factor <= 1 leaves the frequencies as they are)
    qk_norm: bool = False
    rope_scaling: Tuple[float, float, float, float] = (0.0, 0.0, 0.0, 0.0)

    @property
    def q_dim(self) -> int:
        return self.n_q_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    @property
    def qkv_dim(self) -> int:
        return self.q_dim + 2 * self.kv_dim

    @property
    def is_moe(self) -> bool:
        return self.n_experts > 0


@dataclass(frozen=True)
class SpecConfig:
    """One draft-and-verify workload: target, drafter, block and taps."""
    name: str
    target: ModelDims
    drafter: ModelDims
    block_size: int
    tap_layers: Tuple[int, ...]
    dtype: str = "bf16"               # "bf16" or "fp32" storage/compute type
    mask_token_id: Optional[int] = None  # None -> vocab - 1
    batch: int = 1
    prompt_len: int = 512
    max_new: int = 2048
    prompt_kind: str = "zipf"         # "zipf" (exponent 1.1) or "uniform"
    seed: int = 0
    weight_std: float = 0.02

    @property
    def mask_id(self) -> int:
        return self.target.vocab - 1 if self.mask_token_id is None else self.mask_token_id

    @property
    def n_taps(self) -> int:
        return len(self.tap_layers)

    def with_(self, **kw) -> "SpecConfig":
        return replace(self, **kw)


def tap_layers_evenly(n_layers: int, n_taps: int = 5) -> Tuple[int, ...]:
    """Evenly spaced tap layers 1 + floor(i*(L-4)/(n-1)), i = 0..n-1.

    The pages only say "several layers"; this spacing is our reading of
    "evenly spaced" and is a plain parameter of the configuration.
    """
    if n_taps == 1:
        return (n_layers // 2,)
    return tuple(1 + (i * (n_layers - 4)) // (n_taps - 1) for i in range(n_taps))


def _qwen3_8b() -> ModelDims:
    return ModelDims(n_layers=36, hidden=4096, n_q_heads=32, n_kv_heads=8, head_dim=128,
                     ffn=12288, vocab=151936, rms_eps=1e-6, rope_theta=1e6)


def _llama31_8b() -> ModelDims:
    return ModelDims(n_layers=32, hidden=4096, n_q_heads=32, n_kv_heads=8, head_dim=128,
                     ffn=14336, vocab=128256, rms_eps=1e-5, rope_theta=5e5)


def _qwen3_coder_30b_a3b() -> ModelDims:
    return ModelDims(n_layers=48, hidden=2048, n_q_heads=32, n_kv_heads=4, head_dim=128,
                     ffn=768, vocab=151936, rms_eps=1e-6, rope_theta=1e6,
                     n_experts=128, top_k=8, expert_ffn=768)


_TINY = ModelDims(n_layers=2, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64,
                  ffn=768, vocab=1024, rms_eps=1e-6, rope_theta=1e4)


def _drafter_of(t: ModelDims, n_layers: int, ffn: Optional[int] = None) -> ModelDims:
    return ModelDims(n_layers=n_layers, hidden=t.hidden, n_q_heads=t.n_q_heads,
                     n_kv_heads=t.n_kv_heads, head_dim=t.head_dim,
                     ffn=t.ffn if ffn is None else ffn, vocab=t.vocab,
                     rms_eps=t.rms_eps, rope_theta=t.rope_theta)


def _build() -> Dict[str, SpecConfig]:
    q = _qwen3_8b()
    l = _llama31_8b()
    c = _qwen3_coder_30b_a3b()
    cfgs = {
        # Tiny correctness case, fp32: 2-layer target, 1-layer drafter, block 4.
        "tiny": SpecConfig(name="tiny", target=_TINY, drafter=_drafter_of(_TINY, 1),
                           block_size=4, tap_layers=(0, 1), dtype="fp32", batch=1,
                           prompt_len=32, max_new=64, prompt_kind="uniform", seed=0),
        # Qwen3-8B shape, 5-layer block-16 drafter, batch 1.
        "qwen3_8b": SpecConfig(name="qwen3_8b", target=q, drafter=_drafter_of(q, 5),
                               block_size=16, tap_layers=tap_layers_evenly(36),
                               dtype="bf16", batch=1, prompt_len=512, max_new=2048,
                               prompt_kind="zipf", seed=2),
        # Same model, concurrency sweep (batch is overridden per sweep point).
        "qwen3_8b_sweep": SpecConfig(name="qwen3_8b_sweep", target=q, drafter=_drafter_of(q, 5),
                                     block_size=16, tap_layers=tap_layers_evenly(36),
                                     dtype="bf16", batch=1, prompt_len=1024, max_new=1024,
                                     prompt_kind="zipf", seed=3),
        # Llama-3.1-8B shape, long reasoning: 8192-token uniform prompt.
        "llama31_8b": SpecConfig(name="llama31_8b", target=l, drafter=_drafter_of(l, 5),
                                 block_size=16, tap_layers=tap_layers_evenly(32),
                                 dtype="bf16", batch=1, prompt_len=8192, max_new=4096,
                                 prompt_kind="uniform", seed=4),
        # Qwen3-Coder-30B-A3B-shaped MoE target with a dense 8-layer drafter.
        "qwen3_coder_30b_a3b": SpecConfig(
            name="qwen3_coder_30b_a3b", target=c,
            drafter=ModelDims(n_layers=8, hidden=2048, n_q_heads=32, n_kv_heads=4, head_dim=128,
                              ffn=6144, vocab=151936, rms_eps=1e-6, rope_theta=1e6),
            block_size=16, tap_layers=tap_layers_evenly(48), dtype="bf16", batch=1,
            prompt_len=2048, max_new=2048, prompt_kind="zipf", seed=5),
    }
    return cfgs


CONFIGS: Dict[str, SpecConfig] = _build()


def get_config(name: str, **overrides) -> SpecConfig:
    cfg = CONFIGS[name]
    return cfg.with_(**overrides) if overrides else cfg


def shrink(cfg: SpecConfig, target_layers: int = 2, drafter_layers: int = 1,
           vocab: Optional[int] = None, n_experts: Optional[int] = None,
           tap_layers: Optional[Tuple[int, ...]] = None, **kw) -> SpecConfig:
    """Same widths, fewer layers (and optionally a smaller vocab / expert count)."""
    t = replace(cfg.target, n_layers=target_layers)
    d = replace(cfg.drafter, n_layers=drafter_layers)
    if vocab is not None:
        t = replace(t, vocab=vocab)
        d = replace(d, vocab=vocab)
    if n_experts is not None and t.is_moe:
        t = replace(t, n_experts=n_experts, top_k=min(t.top_k, n_experts))
    if tap_layers is None:
        # keep the number of taps (and so the fuse matrix shape); repeats are allowed
        tap_layers = tuple(min(x, target_layers - 1) for x in cfg.tap_layers)
    return cfg.with_(name=cfg.name + f"_L{target_layers}", target=t, drafter=d,
                     tap_layers=tap_layers, **kw)
