"""Full-size checks in the launch configuration the bench times, with sampled
step-wise comparisons against the fp64 oracle fed the GPU's own state, and
size-independent invariants:
  * the ~140M workload (B = 256, T = 1024, W = 128, G = L_D), one run call
    over all 256 sequences;
  * the tied 48 + 48 workload (d = 2048, SwiGLU, W = 256, G = 1, B = 32,
    3072 prompt + 1024 response positions), sampled past the prompt;
  * the ragged 1024-sequence workload through the ready-set scheduler, probe
    sequences checked at ticks where the batch has shrunk."""
import gc

import numpy as np
import pytest
import torch

import oracle
from rlt_cases import STEP_TOL, CACHE_TOL, prefill_all, rms, to_np
from token_recurrent_decoding_b200 import configs, inputs
from token_recurrent_decoding_b200.rlt import Model

pytestmark = pytest.mark.gpu


def _check_step(o, enc, t, before, after, dtype, what):
    e_g, mem_g = enc
    s_ref, win_ref = o.step(e_g[t], mem_g, t, *before)
    s_new, c_new = after
    err = np.abs(s_new - s_ref).max() / rms(s_ref)
    assert err <= STEP_TOL[dtype], (what, t, err)
    if c_new.shape[2]:
        newest = c_new[:, :, -1]
        ref = win_ref[:, :, -1]
        assert np.abs(newest - ref).max() <= CACHE_TOL[dtype] * rms(ref), (what, t)


def test_m140_full_size_sampled_stepwise():
    wl = configs.workloads()["m140_bf16"]
    cfg, B, T = wl.model, wl.batch, wl.max_len
    w = inputs.make_weights(cfg)
    tok = inputs.make_tokens(cfg.vocab, wl.lengths)
    m = Model(cfg, w, B, T)
    prefill_all(m, tok, wl.lengths)
    o = oracle.Oracle(cfg, w)
    probe = [0, 131, 255]
    enc = {i: [to_np(x) for x in m.get_encoder_output(i)] for i in probe}
    ids = list(range(B))
    done = 0
    for t in (0, 129, 767, 1023):
        m.run_sequence(ids, t - done)
        before = {i: [to_np(x) for x in m.get_state(i)[:2]] for i in probe}
        m.run_sequence(ids, 1)
        done = t + 1
        for i in probe:
            after = [to_np(x) for x in m.get_state(i)[:2]]
            _check_step(o, enc[i], t, before[i], after, cfg.dtype, ("m140", i))
    # states stay finite and normalised (s_t is RMS-normalised, gain 1)
    for i in probe:
        s = to_np(m.get_state(i)[0])
        assert np.isfinite(s).all() and abs(rms(s) - 1) < 1e-3


def test_tied_full_size_sampled_stepwise():
    wl = configs.workloads()["tied_bf16"]
    cfg, B, T = wl.model, wl.batch, wl.max_len
    w = inputs.make_weights(cfg)
    tok = inputs.make_tokens(cfg.vocab, wl.lengths)
    m = Model(cfg, w, B, T)
    o = oracle.Oracle(cfg, w)
    del w
    gc.collect()
    prefill_all(m, tok, wl.lengths)
    probe = [0, 31]
    enc = {i: [to_np(x) for x in m.get_encoder_output(i)] for i in probe}
    ids = list(range(B))
    done = 0
    for t in (0, 1100, 3071, 3072, 4095):
        m.run_sequence(ids, t - done)
        before = {i: [to_np(x) for x in m.get_state(i)[:2]] for i in probe}
        m.run_sequence(ids, 1)
        done = t + 1
        for i in probe:
            after = [to_np(x) for x in m.get_state(i)[:2]]
            _check_step(o, enc[i], t, before[i], after, cfg.dtype, ("tied", i))
    assert m.poll_device_error() == 0


def test_ragged_full_size_sampled_stepwise():
    wl = configs.workloads()["ragged_bf16"]
    cfg, B = wl.model, wl.batch
    lengths = np.asarray(wl.lengths)
    w = inputs.make_weights(cfg)
    tok = inputs.make_tokens(cfg.vocab, wl.lengths)
    m = Model(cfg, w, B, wl.max_len)
    prefill_all(m, tok, wl.lengths)
    o = oracle.Oracle(cfg, w)
    order = np.argsort(lengths, kind="stable")
    probe = [int(order[0]), int(order[B // 2]), int(order[-1])]  # shortest, middle, longest
    enc = {i: [to_np(x) for x in m.get_encoder_output(i)] for i in probe}
    ids = np.arange(B, dtype=np.int32)
    done = 0
    # ticks: before anyone finishes, after the shortest finished, near the end
    ticks = [100, int(lengths.min()) - 1, int(np.median(lengths)) + 3, int(lengths.max()) - 1]
    for k in ticks:
        m.run_ragged(ids, np.clip(lengths, 0, k) - np.clip(lengths, 0, done))
        live = [i for i in probe if lengths[i] > k]
        before = {i: [to_np(x) for x in m.get_state(i)[:2]] for i in live}
        step = (lengths > k).astype(np.int32)
        assert 0 < step.sum() <= B
        m.run_ragged(ids, step)
        done = k + 1
        for i in live:
            after = [to_np(x) for x in m.get_state(i)[:2]]
            _check_step(o, enc[i], k, before[i], after, cfg.dtype, ("ragged", i, int(step.sum())))
    for i in probe:
        assert m.get_state(i)[2] == min(int(lengths[i]), done)
    assert m.poll_device_error() == 0
