"""Token-parallel decoder pass for feedback off (alpha = 0), through the C ABI,
against the oracle's own parallel pass (every s_t) and its recurrent decode
(the state after the pass), both fed the GPU's encoder output e and memory M
as the step-wise recurrent tests feed the GPU's own state; and recurrent steps
continued from the parallel state against the oracle's run from tokens.
Tolerances as for the recurrent path: step-wise max|err| <= 1e-5 RMS(s)
(fp32) or 2e-2 RMS(s) (bf16); cache entries 1e-5 / 5e-2 RMS; trajectory
rel-L2 1e-4 / 5e-2."""
import numpy as np
import pytest
import torch

import oracle
from rlt_cases import SMALL, STEP_TOL, TRAJ_TOL, make_model, rel_l2, rms, to_np
from token_recurrent_decoding_b200 import configs
from token_recurrent_decoding_b200.rlt import RLTError

pytestmark = pytest.mark.gpu

CACHE_TOL = {configs.F32: 1e-5, configs.BF16: 5e-2}


@pytest.mark.parametrize("name", ["tiny_fp32", "m50_like", "m140_like", "tied_like",
                                  "ragged_like"])
def test_parallel_pass_matches_oracle(name):
    cfg = SMALL[name].replace(alpha=0.0)
    T, more, n = 100, 12, 3  # two 64-row query blocks; the window lies inside
    m, w, tok = make_model(cfg, [T + more] * n)
    o = oracle.Oracle(cfg, w)
    s_all = torch.full((n, T, cfg.d), float("nan"), dtype=torch.float32, device="cuda")
    m.decoder_parallel(list(range(n)), T, s_all)
    step_tol = STEP_TOL[cfg.dtype]
    for i in range(n):
        e, mem = (to_np(x) for x in m.get_encoder_output(i))
        ref = o.decode_parallel_nofeedback(e, mem, T)
        got = to_np(s_all[i])
        err = np.abs(got - ref).max() / rms(ref)
        assert err <= step_tol, (name, i, err)
        # the recurrent state after the pass
        s, cache, t = m.get_state(i)
        assert t == T
        s0, w0 = o.init_state()
        _, s_ref, win_ref = o.decode(e, mem, 0, T, s0, w0)
        assert np.abs(to_np(s) - s_ref).max() / rms(s_ref) <= step_tol, (name, i)
        if cfg.window > 1:
            c = to_np(cache)
            assert np.abs(c - win_ref).max() <= CACHE_TOL[cfg.dtype] * rms(win_ref), (name, i)
    # recurrent steps continue from the parallel state
    m.run_sequence(list(range(n)), more)
    for i in range(n):
        s, _, t = m.get_state(i)
        assert t == T + more
        assert rel_l2(to_np(s), o.run(tok[i, :T + more])[1]) <= TRAJ_TOL[cfg.dtype], (name, i)


def test_parallel_pass_short_and_chunked():
    """Lengths below the window and more sequences than one prefill chunk."""
    cfg = SMALL["m50_like"].replace(alpha=0.0)
    n, T = 5, 6  # T < W = 8: a partial window
    m, w, tok = make_model(cfg, [T] * n, max_prefill_tokens=2 * T)
    o = oracle.Oracle(cfg, w)
    s_all = torch.empty((n, T, cfg.d), dtype=torch.float32, device="cuda")
    m.decoder_parallel(list(range(n)), T, s_all)
    for i in range(n):
        e, mem = (to_np(x) for x in m.get_encoder_output(i))
        ref = o.decode_parallel_nofeedback(e, mem, T)
        assert np.abs(to_np(s_all[i]) - ref).max() / rms(ref) <= STEP_TOL[cfg.dtype]
        s0, w0 = o.init_state()
        _, s_ref, win_ref = o.decode(e, mem, 0, T, s0, w0)
        s, cache, t = m.get_state(i)
        assert t == T
        assert np.abs(to_np(cache) - win_ref).max() <= CACHE_TOL[cfg.dtype] * rms(win_ref)


def test_parallel_pass_errors():
    cfg = SMALL["m50_like"]  # alpha = 1: s_{t-1} feeds step t
    m, _, _ = make_model(cfg, [20, 20])
    with pytest.raises(RLTError) as ei:
        m.decoder_parallel([0], 10)
    assert ei.value.status == 2  # UNSUPPORTED
    m, _, _ = make_model(cfg.replace(alpha=0.0), [20, 20], max_len=32)
    with pytest.raises(RLTError) as ei:
        m.decoder_parallel([0], 21)
    assert ei.value.status == 3  # NOT_READY: t_enc = 20
    with pytest.raises(RLTError) as ei:
        m.decoder_parallel([0], 33)
    assert ei.value.status == 4  # CAPACITY: beyond max_len
    with pytest.raises(RLTError) as ei:
        m.decoder_parallel([0, 0], 5)
    assert ei.value.status == 5  # DUPLICATE_ID
    m.decoder_step([1])
    with pytest.raises(RLTError) as ei:
        m.decoder_parallel([1], 5)
    assert ei.value.status == 1  # INVALID_ARG: not a fresh sequence
    m.decoder_parallel([0], 0)  # no steps: nothing to do
    assert m.get_state(0)[2] == 0
