"""Full-size checks: the ~140M workload (B = 256, T = 1024, W = 128, G = L_D)
in the launch configuration the bench times (one run call over all 256
sequences), with sampled step-wise comparisons against the fp64 oracle fed the
GPU's own state, and the size-independent invariants."""
import numpy as np
import pytest
import torch

import oracle
from rlt_cases import STEP_TOL, prefill_all, rms, to_np
from token_recurrent_decoding_b200 import configs, inputs
from token_recurrent_decoding_b200.rlt import Model

pytestmark = pytest.mark.gpu


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
            s_new = to_np(m.get_state(i)[0])
            e_g, mem_g = enc[i]
            s_ref, _ = o.step(e_g[t], mem_g, t, *before[i])
            err = np.abs(s_new - s_ref).max() / rms(s_ref)
            assert err <= STEP_TOL[cfg.dtype], (i, t, err)
    # states stay finite and normalised (s_t is RMS-normalised, gain 1)
    for i in probe:
        s = to_np(m.get_state(i)[0])
        assert np.isfinite(s).all() and abs(rms(s) - 1) < 1e-3
