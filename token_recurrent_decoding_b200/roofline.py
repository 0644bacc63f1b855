"""Algorithmic bytes and FLOPs of the decoder step and the encoder prefill.

Counting rules (everything once per step):
  * decoder weights: read once per step launch, whatever the batch size;
  * per sequence: e_t (model dtype) and s_{t-1} (fp32) in, s_t (fp32) out;
  * per decoder layer: the retained window, 2 * min(t, W-1) rows of d, read,
    and the new (k, v) written;
  * memory M<=t: 2 * (t + 1) rows of d read once per group. With G = 1 the
    shared memory counts once per step even though every layer reads it
    (the strict count); ``mem_reread`` counts it once per layer.
FLOPs: 2 x decoder matmul parameters per sequence, plus 4 d (min(t+1, W) +
(t+1)) per layer for the two attentions.
"""
from __future__ import annotations

import numpy as np

from .configs import BF16, SWIGLU, RLTConfig


def elem_bytes(cfg: RLTConfig) -> int:
    return 2 if cfg.dtype == BF16 else 4


def ffn_params(cfg: RLTConfig) -> int:
    return (3 if cfg.ffn_kind == SWIGLU else 2) * cfg.d * cfg.ffn_dim


def dec_matmul_params(cfg: RLTConfig) -> int:
    d = cfg.d
    per_layer = 3 * d * d + d * d + d * d + d * d + ffn_params(cfg)
    return cfg.n_dec * per_layer + (2 * d * d if cfg.alpha != 0 else 0)


def enc_matmul_params(cfg: RLTConfig) -> int:
    d = cfg.d
    return cfg.n_enc * (4 * d * d + ffn_params(cfg)) + cfg.mem_groups * 2 * d * d


def decoder_step_bytes(cfg: RLTConfig, ts, mem_reread: bool = False) -> float:
    """Bytes of one batched step whose slots sit at positions ``ts``."""
    ts = np.asarray(ts, dtype=np.float64)
    es, d, L, W = elem_bytes(cfg), cfg.d, cfg.n_dec, cfg.window
    g_eff = L if (cfg.mem_groups == L or mem_reread) else 1
    weights = dec_matmul_params(cfg) * es
    per_seq = d * es + d * 4 + d * 4
    ring = L * (2 * np.minimum(ts, W - 1) * d * es + 2 * d * es)
    mem = g_eff * 2 * (ts + 1) * d * es
    return float(weights + np.sum(per_seq + ring + mem))


def decoder_step_flops(cfg: RLTConfig, ts) -> float:
    ts = np.asarray(ts, dtype=np.float64)
    d, L, W = cfg.d, cfg.n_dec, cfg.window
    attn = L * 4 * d * (np.minimum(ts + 1, W) + (ts + 1))
    return float(np.sum(2 * dec_matmul_params(cfg) + attn))


def encoder_flops(cfg: RLTConfig, lengths) -> float:
    """Encoder + memory projection FLOPs of full sequences (causal attention
    over positions 0..t)."""
    tot = 0.0
    for T in lengths:
        t = np.arange(T, dtype=np.float64)
        tot += 2 * enc_matmul_params(cfg) * T + np.sum(cfg.n_enc * 4 * cfg.d * (t + 1))
    return float(tot)


def run_roofline(cfg: RLTConfig, lengths, hbm_gbs: float, tensor_tflops: float,
                 mem_reread: bool = False):
    """Roofline time of a full lock-step run (sequences drop out as they
    finish) and of the encoder prefill; returns a dict of seconds/bytes/FLOPs."""
    lengths = np.asarray(lengths)
    T = int(lengths.max())
    dec_t = 0.0
    dec_bytes = 0.0
    dec_flops = 0.0
    for t in range(T):
        n = int(np.sum(lengths > t))
        ts = np.full(n, t)
        b = decoder_step_bytes(cfg, ts, mem_reread)
        f = decoder_step_flops(cfg, ts)
        dec_bytes += b
        dec_flops += f
        dec_t += max(b / (hbm_gbs * 1e9), f / (tensor_tflops * 1e12))
    enc_f = encoder_flops(cfg, lengths)
    return {"decoder_s": dec_t, "decoder_bytes": dec_bytes, "decoder_flops": dec_flops,
            "encoder_s": enc_f / (tensor_tflops * 1e12), "encoder_flops": enc_f,
            "seq_steps": int(lengths.sum())}


def decoder_parallel_roofline(cfg: RLTConfig, lengths, hbm_gbs: float, tensor_tflops: float):
    """Roofline of the token-parallel decoder pass (feedback off) over full
    sequences: FLOPs = 2 x decoder matmul parameters per token plus the
    window-masked and prefix attention, bytes = weights once, e_t and the
    memory rows read once per group, s_t written; the larger time bounds."""
    lengths = np.asarray(lengths)
    es = elem_bytes(cfg)
    d, W = cfg.d, cfg.window
    flops = 0.0
    for T in lengths:
        t = np.arange(T, dtype=np.float64)
        flops += 2 * dec_matmul_params(cfg) * T
        flops += np.sum(cfg.n_dec * 4 * d * (np.minimum(t + 1, W) + t + 1))
    tok = float(lengths.sum())
    byts = dec_matmul_params(cfg) * es + tok * d * (es + 4) + cfg.mem_groups * tok * 2 * d * es
    return {"seconds": max(flops / (tensor_tflops * 1e12), byts / (hbm_gbs * 1e9)),
            "flops": float(flops), "bytes": float(byts), "seq_steps": int(tok)}


def backward_flops(cfg: RLTConfig, lengths) -> float:
    """FLOPs of one backpropagation through time over full sequences: the
    recomputed forward (the step's FLOPs) plus twice that for the gradients
    of every matmul (activations and weights) and of the attentions, plus the
    recorded forward itself: 4 x the decoder run's FLOPs. The memory
    projection's backward adds 2 x 2 x 2 d^2 G per position."""
    lengths = np.asarray(lengths)
    tot = 0.0
    for T in lengths:
        t = np.arange(T, dtype=np.float64)
        tot += 4 * decoder_step_flops(cfg, t) + 8.0 * cfg.d * cfg.d * cfg.mem_groups * T
    return float(tot)


def backward_roofline(cfg: RLTConfig, lengths, hbm_gbs: float, tensor_tflops: float):
    """Roofline of rlt_backward over full sequences (lock-step): per step the
    recorded forward, the recomputed forward and the backward each move about
    one forward step's bytes (weights, the window and memory rows; the
    backward reads W^T and the same keys and values again), and the FLOPs are
    backward_flops; the larger time bounds each step."""
    lengths = np.asarray(lengths)
    T = int(lengths.max())
    sec = 0.0
    tot_b = 0.0
    for t in range(T):
        n = int(np.sum(lengths > t))
        ts = np.full(n, t)
        b = 3.0 * decoder_step_bytes(cfg, ts)
        f = 4.0 * decoder_step_flops(cfg, ts) + 8.0 * cfg.d * cfg.d * cfg.mem_groups * n
        tot_b += b
        sec += max(b / (hbm_gbs * 1e9), f / (tensor_tflops * 1e12))
    return {"seconds": sec, "bytes": tot_b, "flops": backward_flops(cfg, lengths),
            "seq_steps": int(lengths.sum())}
