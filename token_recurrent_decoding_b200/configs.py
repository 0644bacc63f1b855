"""Model shapes and synthetic workloads of the Recurrent Looped Transformer (RLT).

Plain data only: no arithmetic of the method lives here.

Citation key used across this package:
  [RLT-96]  "RLT Runs 96 Blocks Per Token With Recurrent State, No Resets"
            (aimastery.page news item)
  [RLT-TC]  "Recurrent Looped Transformer (RLT): prompts in parallel, depth in
            sequence" (thakicloud.com tech blog)
  [RLT-FT]  "Recurrent Looped Transformer debunked" (flowtivity.ai blog)
  [RLT-PV]  "Per-token recurrence, no quality gain" (news.promtvault.app story)

Shapes follow [RLT-PV] body (widths 512 / 768, 6+6 and 12+12 layers, window 64,
one feedback gate) and [RLT-96] "Architecture: encoder memory meets recurrent
decoder" (48 + 48 tied layers, G = 1 or G = L_D).
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field

GELU = 0
SWIGLU = 1
F32 = 0
BF16 = 1


@dataclass(frozen=True)
class RLTConfig:
    """Architecture of one RLT model (names follow the pages' notation)."""

    d: int                 # model width
    n_heads: int           # H, heads of every attention (self and cross)
    head_dim: int          # dh = d / H
    n_enc: int             # L_E, causal encoder blocks
    n_dec: int             # L_D, recurrent decoder blocks
    ffn_dim: int           # F
    ffn_kind: int          # GELU or SWIGLU
    vocab: int             # V
    window: int            # W, includes the current token
    mem_groups: int        # G: 1 (shared memory) or L_D (one per decoder layer)
    tied: bool             # decoder layer l reuses encoder layer l's attention/FFN
    dtype: int             # F32 or BF16 storage of weights / K / V / memory
    alpha: float = 1.0     # feedback scale of the gated merge
    rms_eps: float = 1e-6
    rope_theta: float = 10000.0

    def __post_init__(self):
        assert self.d == self.n_heads * self.head_dim
        assert self.mem_groups in (1, self.n_dec)
        assert self.window >= 1
        if self.tied:
            assert self.n_dec <= self.n_enc

    def replace(self, **kw) -> "RLTConfig":
        return dataclasses.replace(self, **kw)


@dataclass(frozen=True)
class Workload:
    """A batch of independent sequences: model + per-sequence token counts.

    ``lengths[i]`` is the number of tokens of sequence i. Every token runs
    through the encoder and every position runs one decoder transition (the
    decoder also steps over prompt tokens: [RLT-FT] "How slow is per-token
    recurrence to train?").
    """

    name: str
    model: RLTConfig
    lengths: tuple
    prompt_lengths: tuple = field(default=())

    @property
    def batch(self) -> int:
        return len(self.lengths)

    @property
    def max_len(self) -> int:
        return max(self.lengths)

    @property
    def seq_steps(self) -> int:
        return int(sum(self.lengths))


TINY = RLTConfig(d=64, n_heads=4, head_dim=16, n_enc=2, n_dec=2, ffn_dim=256,
                 ffn_kind=GELU, vocab=256, window=8, mem_groups=1, tied=False,
                 dtype=F32)
M50 = RLTConfig(d=512, n_heads=8, head_dim=64, n_enc=6, n_dec=6, ffn_dim=2048,
                ffn_kind=GELU, vocab=32768, window=64, mem_groups=1, tied=False,
                dtype=BF16)
M140 = RLTConfig(d=768, n_heads=12, head_dim=64, n_enc=12, n_dec=12,
                 ffn_dim=3072, ffn_kind=GELU, vocab=32768, window=128,
                 mem_groups=12, tied=False, dtype=BF16)
TIED = RLTConfig(d=2048, n_heads=16, head_dim=128, n_enc=48, n_dec=48,
                 ffn_dim=5632, ffn_kind=SWIGLU, vocab=32768, window=256,
                 mem_groups=1, tied=True, dtype=BF16)
RAGGED_MODEL = M140.replace(mem_groups=1)


def ragged_prompt_lengths(n: int = 1024, lo: int = 128, hi: int = 2048,
                          seed: int = 2):
    """Prompt lengths uniform in [lo, hi] (inclusive) from numpy PCG64(seed)."""
    import numpy as np
    return tuple(int(x) for x in np.random.default_rng(seed).integers(lo, hi + 1, n))


def workloads():
    """The five synthetic workloads, by name."""
    pl = ragged_prompt_lengths()
    return {
        "tiny_fp32": Workload("tiny_fp32", TINY, (64,) * 2),
        "m50_bf16": Workload("m50_bf16", M50, (1024,) * 64),
        "m50_bf16_alpha0": Workload("m50_bf16_alpha0", M50.replace(alpha=0.0), (1024,) * 64),
        "m140_bf16": Workload("m140_bf16", M140, (1024,) * 256, (768,) * 256),
        "tied_bf16": Workload("tied_bf16", TIED, (4096,) * 32, (3072,) * 32),
        "ragged_bf16": Workload("ragged_bf16", RAGGED_MODEL,
                                tuple(p + 256 for p in pl), pl),
    }


def model_from_dict(d: dict) -> RLTConfig:
    return RLTConfig(**d)
