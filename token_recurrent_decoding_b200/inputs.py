"""Seeded synthetic inputs shared by the CUDA path, the oracle and the bench.

This module holds random draws and dtype rounding only; none of the method's
arithmetic. Everything is drawn from numpy PCG64 (``default_rng``) so that both
sides receive the same values.

Weights (seed 0), drawn in this order, each ``standard_normal(float32) * 0.02``
in row-major ``[out][in]`` layout (y = W x):

  embed [V][d]
  for l < L_E: enc.l.wqkv [3d][d] (rows q | k | v), enc.l.wo [d][d],
               GELU: enc.l.w1 [F][d], enc.l.w2 [d][F]
               SwiGLU: enc.l.wa [F][d], enc.l.wb [F][d], enc.l.w2 [d][F]
  for g < G:   mem.g.wk [d][d], mem.g.wv [d][d]
  gate.w [d][2d]   (columns 0..d-1 multiply e_t, d..2d-1 multiply s_{t-1})
  sstar [d]        (standard_normal, scale 1: the learned start state s*)
  for l < L_D: dec.l.wqkv, dec.l.wo   (skipped when tied)
               dec.l.wqx [d][d], dec.l.wox [d][d]
               dec.l.w1, dec.l.w2 / wa, wb, w2 (skipped when tied)

Norm gains (enc.l.ln1, enc.l.ln2, enc.lnf, dec.l.ln1..ln3, dec.lnf) are ones and
the gate bias gate.b is zero, not drawn. With ``perturb=True`` they are instead
drawn from PCG64(seed + 100) as 1 + 0.1 N(0,1) and 0.1 N(0,1), after the
matrices, so tests can see a dropped gain or bias.

bf16 models round every fp32 draw to bf16 with round-to-nearest-even; the
returned float32 arrays hold those bf16 values exactly.

Tokens (seed 1): ``integers(0, V, (B, T_max))``; sequence i uses row i's first
``lengths[i]`` entries. Ragged prompt lengths come from seed 2 (configs module).
"""
from __future__ import annotations

from typing import Dict, Iterator, Tuple

import numpy as np

from .configs import BF16, SWIGLU, RLTConfig

WEIGHT_STD = 0.02


def round_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 -> nearest bf16 value (ties to even), returned as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values that are already bf16-representable."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def _ffn_names(cfg: RLTConfig, prefix: str):
    if cfg.ffn_kind == SWIGLU:
        return [(f"{prefix}.wa", (cfg.ffn_dim, cfg.d)),
                (f"{prefix}.wb", (cfg.ffn_dim, cfg.d)),
                (f"{prefix}.w2", (cfg.d, cfg.ffn_dim))]
    return [(f"{prefix}.w1", (cfg.ffn_dim, cfg.d)),
            (f"{prefix}.w2", (cfg.d, cfg.ffn_dim))]


def drawn_matrices(cfg: RLTConfig):
    """(name, shape, scale) of every drawn tensor, in draw order."""
    d = cfg.d
    out = [("embed", (cfg.vocab, d), WEIGHT_STD)]
    for l in range(cfg.n_enc):
        out += [(f"enc.{l}.wqkv", (3 * d, d), WEIGHT_STD),
                (f"enc.{l}.wo", (d, d), WEIGHT_STD)]
        out += [(n, s, WEIGHT_STD) for n, s in _ffn_names(cfg, f"enc.{l}")]
    for g in range(cfg.mem_groups):
        out += [(f"mem.{g}.wk", (d, d), WEIGHT_STD),
                (f"mem.{g}.wv", (d, d), WEIGHT_STD)]
    out += [("gate.w", (d, 2 * d), WEIGHT_STD), ("sstar", (d,), 1.0)]
    for l in range(cfg.n_dec):
        if not cfg.tied:
            out += [(f"dec.{l}.wqkv", (3 * d, d), WEIGHT_STD),
                    (f"dec.{l}.wo", (d, d), WEIGHT_STD)]
        out += [(f"dec.{l}.wqx", (d, d), WEIGHT_STD),
                (f"dec.{l}.wox", (d, d), WEIGHT_STD)]
        if not cfg.tied:
            out += [(n, s, WEIGHT_STD) for n, s in _ffn_names(cfg, f"dec.{l}")]
    return out


def vector_params(cfg: RLTConfig):
    """(name, shape, base) of the norm gains (base 1) and gate bias (base 0)."""
    d = cfg.d
    out = []
    for l in range(cfg.n_enc):
        out += [(f"enc.{l}.ln1", (d,), 1.0), (f"enc.{l}.ln2", (d,), 1.0)]
    out += [("enc.lnf", (d,), 1.0), ("gate.b", (d,), 0.0)]
    for l in range(cfg.n_dec):
        out += [(f"dec.{l}.ln1", (d,), 1.0), (f"dec.{l}.ln2", (d,), 1.0),
                (f"dec.{l}.ln3", (d,), 1.0)]
    out += [("dec.lnf", (d,), 1.0)]
    return out


def tied_aliases(cfg: RLTConfig) -> Dict[str, str]:
    """Decoder tensor name -> encoder tensor it shares in the tied layout."""
    if not cfg.tied:
        return {}
    out = {}
    for l in range(cfg.n_dec):
        out[f"dec.{l}.wqkv"] = f"enc.{l}.wqkv"
        out[f"dec.{l}.wo"] = f"enc.{l}.wo"
        for n, _ in _ffn_names(cfg, f"dec.{l}"):
            out[n] = n.replace("dec.", "enc.", 1)
    return out


def iter_weights(cfg: RLTConfig, seed: int = 0, perturb: bool = False
                 ) -> Iterator[Tuple[str, np.ndarray]]:
    """Yield (name, float32 array) one tensor at a time (bounded host memory)."""
    rng = np.random.default_rng(seed)
    for name, shape, scale in drawn_matrices(cfg):
        x = rng.standard_normal(shape, dtype=np.float32)
        if scale != 1.0:
            x *= np.float32(scale)
        if cfg.dtype == BF16:
            x = round_bf16(x)
        yield name, x
    prng = np.random.default_rng(seed + 100) if perturb else None
    for name, shape, base in vector_params(cfg):
        if prng is None:
            x = np.full(shape, base, dtype=np.float32)
        else:
            x = (np.float32(base)
                 + np.float32(0.1) * prng.standard_normal(shape, dtype=np.float32))
        if cfg.dtype == BF16:
            x = round_bf16(x)
        yield name, x


def make_weights(cfg: RLTConfig, seed: int = 0, perturb: bool = False
                 ) -> Dict[str, np.ndarray]:
    """All weights by name; tied decoder names alias the encoder arrays."""
    w = dict(iter_weights(cfg, seed, perturb))
    for dst, src in tied_aliases(cfg).items():
        w[dst] = w[src]
    return w


def make_tokens(vocab: int, lengths, seed: int = 1) -> np.ndarray:
    """int32 [B][T_max]; row i is valid on its first lengths[i] entries."""
    lengths = list(lengths)
    rng = np.random.default_rng(seed)
    return rng.integers(0, vocab, (len(lengths), max(lengths))).astype(np.int32)


def random_like_state(cfg: RLTConfig, seed: int):
    """A random decoder state H = (s, window cache) for set/get round trips.

    Returns s [d] and cache [L_D][2][W-1][d] as float32 (bf16 values for bf16
    models).
    """
    rng = np.random.default_rng(seed)
    s = rng.standard_normal(cfg.d, dtype=np.float32)
    c = rng.standard_normal((cfg.n_dec, 2, max(cfg.window - 1, 0), cfg.d),
                            dtype=np.float32)
    if cfg.dtype == BF16:
        c = round_bf16(c)
    return s, c
