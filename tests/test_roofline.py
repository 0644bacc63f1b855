"""Algorithmic byte / FLOP counts of the measurement (host logic, CPU):
checked against the model's actual weight arrays, against an enumeration of
the rows each attention reads, and against the step-roofline figures derived
independently for the five workloads (HBM 6443.2 GB/s, bf16 1410 TFLOP/s)."""
import numpy as np
import pytest

from token_recurrent_decoding_b200 import configs, inputs, roofline

HBM, TC = 6443.2, 1410.0


@pytest.mark.parametrize("cfg", [configs.TINY, configs.M50, configs.M50.replace(alpha=0.0),
                                 configs.TIED.replace(n_enc=2, n_dec=2)],
                         ids=["tiny", "m50", "m50_alpha0", "tied_2layers"])
def test_decoder_parameter_count_matches_the_weights(cfg):
    """2 x matmul parameters per token: the matrices a decoder step multiplies."""
    w = inputs.make_weights(cfg, 0, False)
    enc_or_dec = "enc" if cfg.tied else "dec"
    total = 0
    for l in range(cfg.n_dec):
        ffn = ("wa", "wb", "w2") if cfg.ffn_kind == configs.SWIGLU else ("w1", "w2")
        names = [f"{enc_or_dec}.{l}.{k}" for k in ("wqkv", "wo") + ffn]
        names += [f"dec.{l}.wqx", f"dec.{l}.wox"]
        total += sum(w[k].size for k in names)
    if cfg.alpha != 0:
        total += w["gate.w"].size
    assert roofline.dec_matmul_params(cfg) == total


def enumerate_step(cfg, ts, mem_reread=False):
    """Bytes and FLOPs of one step by walking the rows every attention reads."""
    es, d, W = roofline.elem_bytes(cfg), cfg.d, cfg.window
    byts = roofline.dec_matmul_params(cfg) * es
    flops = 0.0
    for t in ts:
        byts += d * es + 4 * d + 4 * d  # e_t in, s_{t-1} in, s_t out
        flops += 2 * roofline.dec_matmul_params(cfg)
        window = [p for p in range(max(0, t - W + 1), t + 1)]
        prefix = list(range(0, t + 1))
        for l in range(cfg.n_dec):
            old = [p for p in window if p != t]  # retained rows; row t is written
            byts += 2 * len(old) * d * es + 2 * d * es
            flops += 2 * 2 * d * (len(window) + len(prefix))
        groups = cfg.n_dec if (cfg.mem_groups == cfg.n_dec or mem_reread) else 1
        byts += groups * 2 * len(prefix) * d * es
    return byts, flops


@pytest.mark.parametrize("cfg", [configs.TINY, configs.M50, configs.M140])
@pytest.mark.parametrize("reread", [False, True])
def test_step_counts_match_an_enumeration(cfg, reread):
    ts = [0, 1, cfg.window - 2, cfg.window - 1, cfg.window, 3 * cfg.window + 5]
    b, f = enumerate_step(cfg, ts, reread)
    assert roofline.decoder_step_bytes(cfg, ts, reread) == pytest.approx(b, rel=1e-12)
    assert roofline.decoder_step_flops(cfg, ts) == pytest.approx(f, rel=1e-12)


@pytest.mark.parametrize("name,seconds", [("m50_bf16", 0.0256), ("m140_bf16", 0.981),
                                          ("tied_bf16", 5.98), ("ragged_bf16", 1.56)])
def test_run_roofline_matches_the_derived_figures(name, seconds):
    wl = configs.workloads()[name]
    r = roofline.run_roofline(wl.model, wl.lengths, HBM, TC)
    assert r["decoder_s"] == pytest.approx(seconds, rel=5e-3)
    assert r["seq_steps"] == int(np.sum(wl.lengths))


def test_parallel_pass_flops_match_an_enumeration():
    cfg = configs.M50.replace(alpha=0.0, n_dec=2, window=4)
    lengths = [7, 3]
    f = 0.0
    for T in lengths:
        for t in range(T):
            f += 2 * roofline.dec_matmul_params(cfg)
            band = len(range(max(0, t - cfg.window + 1), t + 1))
            f += cfg.n_dec * 2 * 2 * cfg.d * (band + (t + 1))
    r = roofline.decoder_parallel_roofline(cfg, lengths, HBM, TC)
    assert r["flops"] == pytest.approx(f, rel=1e-12)
    assert r["seq_steps"] == sum(lengths)
    assert r["seconds"] == pytest.approx(max(f / (TC * 1e12), r["bytes"] / (HBM * 1e9)))


def test_backward_roofline_counts_three_forward_steps_of_bytes():
    """The backward's bytes are three forward steps' per step (recorded,
    recomputed, differentiated); its FLOPs four forward steps' plus the
    memory projection's backward."""
    cfg = configs.M140
    lengths = [40, 40]
    br = roofline.backward_roofline(cfg, lengths, 6650.0, 1400.0)
    fw = roofline.run_roofline(cfg, lengths, 6650.0, 1400.0)
    assert abs(br["bytes"] - 3 * fw["decoder_bytes"]) <= 1e-9 * br["bytes"]
    extra = 8.0 * cfg.d * cfg.d * cfg.mem_groups * sum(lengths)
    assert abs(br["flops"] - (4 * fw["decoder_flops"] + extra)) <= 1e-9 * br["flops"]
    assert br["seconds"] >= 3 * fw["decoder_s"] * (1 - 1e-9)
