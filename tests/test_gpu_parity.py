"""GPU path (through the C ABI) against the fp64 CPU oracle on the same seeded
inputs. Tolerances: step-wise max|err| <= 1e-5 RMS(s) (fp32 models) or
2e-2 RMS(s) (bf16 weights, fp32 accumulation), fed the GPU's own H_{t-1};
trajectory rel-L2 of s_t <= 1e-4 / 5e-2 from tokens alone."""
import numpy as np
import pytest
import torch

import oracle
from rlt_cases import (CACHE_TOL, SMALL, STEP_TOL, TRAJ_TOL, make_model, prefill_all, rel_l2,
                       rms, to_np)
from token_recurrent_decoding_b200 import configs, inputs
from token_recurrent_decoding_b200.rlt import Model, RLTError

pytestmark = pytest.mark.gpu

# encoder outputs e_t and memory rows: stored in the model dtype, so bf16
# adds one storage rounding (2^-9 relative) on top of the residual-stream
# error; bound max|err| / RMS and rel-L2.
ENC_TOL = {configs.F32: (1e-5, 1e-6), configs.BF16: (6e-2, 1.5e-2)}


@pytest.mark.parametrize("name,lengths", [(n, [37, 70, 5, 1]) for n in SMALL]
                         + [("m50_like", [300, 257, 128, 1, 64]),
                            ("tied_like", [200, 129, 63])])
def test_encoder_and_memory_parity(name, lengths):
    cfg = SMALL[name]
    m, w, tok = make_model(cfg, lengths)
    o = oracle.Oracle(cfg, w)
    tmax, trel = ENC_TOL[cfg.dtype]
    for i, L in enumerate(lengths):
        e_g, mem_g = m.get_encoder_output(i)
        e_r, mem_r = o.encode(tok[i, :L])
        e_g, mem_g = to_np(e_g), to_np(mem_g)
        assert e_g.shape == (L, cfg.d)
        assert np.abs(e_g - e_r).max() <= tmax * rms(e_r), name
        assert rel_l2(e_g, e_r) <= trel
        mr = mem_r[:, :L]
        assert np.abs(mem_g - mr).max() <= tmax * rms(mr), name
        assert rel_l2(mem_g, mr) <= trel


KERNELS = [(n, k) for n in SMALL for k in ("fused", "chain")
           if k == "chain" or SMALL[n].dtype == configs.BF16]


def _use(m, kernel):
    from token_recurrent_decoding_b200 import rlt as R
    assert m.get_step_kernel() == R.STEP_CHAIN  # the default
    if m.cfg.dtype == configs.BF16:
        assert m.step_kernel_ctas() > 0  # the persistent step covers the model
    m.set_step_kernel(R.STEP_FUSED if kernel == "fused" else R.STEP_CHAIN)
    assert m.get_step_kernel() == (R.STEP_FUSED if kernel == "fused" else R.STEP_CHAIN)


@pytest.mark.parametrize("name,kernel", KERNELS)
def test_stepwise_parity_on_gpu_state(name, kernel):
    """Both step kernels of a bf16 model (the persistent one-launch step and
    the chain of kernels), and the fp32 chain."""
    cfg = SMALL[name]
    T = 40
    m, w, tok = make_model(cfg, [T] * 3)
    _use(m, kernel)
    o = oracle.Oracle(cfg, w)
    e_g, mem_g = (to_np(x) for x in m.get_encoder_output(1))
    checks = sorted({0, 1, cfg.window - 1, cfg.window, cfg.window + 1, 23, T - 1})
    tol = STEP_TOL[cfg.dtype]
    for t in range(T):
        if t in checks:
            s_prev, c_prev, tt = m.get_state(1)
            assert tt == t
            s_prev, c_prev = to_np(s_prev), to_np(c_prev)
        m.decoder_step([0, 1, 2])
        if t in checks:
            s_new, c_new, tt = m.get_state(1)
            assert tt == t + 1
            s_ref, win_ref = o.step(e_g[t], mem_g, t, s_prev, c_prev)
            err = np.abs(to_np(s_new) - s_ref).max() / rms(s_ref)
            assert err <= tol, (name, t, err)
            if cfg.window > 1:
                newest_g = to_np(c_new)[:, :, -1]
                newest_r = win_ref[:, :, -1]
                assert np.abs(newest_g - newest_r).max() <= CACHE_TOL[cfg.dtype] * rms(newest_r)
                # older entries are the previous window shifted by one
                np.testing.assert_array_equal(to_np(c_new)[:, :, :-1], c_prev[:, :, 1:])


@pytest.mark.parametrize("name,kernel", KERNELS)
def test_trajectory_parity_from_tokens(name, kernel):
    cfg = SMALL[name]
    B, T = 2, 64
    m, w, tok = make_model(cfg, [T] * B)
    _use(m, kernel)
    o = oracle.Oracle(cfg, w)
    tol = TRAJ_TOL[cfg.dtype]
    ref0, _, _ = o.run(tok[0])
    # sequence 0 step by step (every s_t), sequence 1 in one run call
    for t in range(T):
        m.decoder_step([0])
        s_t = to_np(m.get_state(0)[0])
        assert rel_l2(s_t, ref0[t]) <= tol, (name, t)
    m.run_sequence([1], T)
    s1, _, t1 = m.get_state(1)
    assert t1 == T
    assert rel_l2(to_np(s1), o.run(tok[1])[1]) <= tol


def test_tiny_fp32_workload_full_size():
    """The tiny fp32 workload at its own size (B = 2, T = 64), batched."""
    w0 = configs.workloads()["tiny_fp32"]
    cfg = w0.model
    m, w, tok = make_model(cfg, list(w0.lengths), perturb=False)
    m.run_sequence([0, 1], w0.max_len)
    o = oracle.Oracle(cfg, w)
    for i in range(2):
        assert rel_l2(to_np(m.get_state(i)[0]), o.run(tok[i])[1]) <= TRAJ_TOL[cfg.dtype]


def test_batch_composition_is_bitwise_invariant():
    cfg = SMALL["m140_like"]
    lengths = [48] * 6
    w = inputs.make_weights(cfg, 0, True)
    tok = inputs.make_tokens(cfg.vocab, lengths)
    a = Model(cfg, w, 6, 48)
    prefill_all(a, tok, lengths)
    a.run_sequence([2], 48)
    a.run_sequence([0, 1, 3, 4, 5], 48)
    b = Model(cfg, w, 6, 48)
    prefill_all(b, tok, lengths)
    b.run_sequence(list(range(6)), 48)
    for i in range(6):
        assert torch.equal(a.get_state(i)[0], b.get_state(i)[0])
        assert torch.equal(a.get_state(i)[1], b.get_state(i)[1])


@pytest.mark.parametrize("k", [1, 7, 16, 33])
def test_split_invariance_snapshot_roundtrip(k):
    """Proposition 3.1: carrying H_t = (s_t, C_t) across a split (export to
    host and import into another slot) equals one uninterrupted pass."""
    cfg = SMALL["m50_like"]
    T = 48
    w = inputs.make_weights(cfg, 0, True)
    tok = inputs.make_tokens(cfg.vocab, [T])
    m = Model(cfg, w, 3, T)
    both = np.concatenate([tok, tok, tok])
    prefill_all(m, both, [T] * 3)
    m.run_sequence([0], T)
    m.run_sequence([1], k)
    s, c, t = m.get_state(1)
    s_h, c_h = s.cpu().pin_memory(), c.cpu().pin_memory()  # snapshot through host memory
    torch.cuda.synchronize()
    m.set_state(2, s_h, c_h, t)
    m.run_sequence([2], T - k)
    assert torch.equal(m.get_state(0)[0], m.get_state(2)[0])
    assert torch.equal(m.get_state(0)[1], m.get_state(2)[1])


def test_alpha_zero_ignores_previous_output_on_gpu():
    cfg = SMALL["m50_like"].replace(alpha=0.0)
    T = 30
    w = inputs.make_weights(cfg, 0, True)
    tok = inputs.make_tokens(cfg.vocab, [T])
    m = Model(cfg, w, 2, T)
    prefill_all(m, np.concatenate([tok, tok]), [T, T])
    m.run_sequence([0, 1], 11)
    s, c, t = m.get_state(1)
    m.set_state(1, torch.randn_like(s) * 5, c, t)
    m.run_sequence([0, 1], T - 11)
    assert torch.equal(m.get_state(0)[0], m.get_state(1)[0])
    o = oracle.Oracle(cfg, w)
    assert rel_l2(to_np(m.get_state(0)[0]), o.run(tok[0])[1]) <= TRAJ_TOL[cfg.dtype]


def test_ragged_scheduler_parity_and_invariance():
    cfg = SMALL["ragged_like"]
    lengths = [13, 40, 1, 27, 40, 8, 33]
    w = inputs.make_weights(cfg, 0, True)
    tok = inputs.make_tokens(cfg.vocab, lengths)
    m = Model(cfg, w, len(lengths), max(lengths))
    prefill_all(m, tok, lengths)
    m.run_ragged(list(range(len(lengths))), lengths)
    alone = Model(cfg, w, len(lengths), max(lengths))
    prefill_all(alone, tok, lengths)
    o = oracle.Oracle(cfg, w)
    for i, L in enumerate(lengths):
        alone.run_sequence([i], L)
        s, _, t = m.get_state(i)
        assert t == L
        assert torch.equal(s, alone.get_state(i)[0])
        assert rel_l2(to_np(s), o.run(tok[i, :L])[1]) <= TRAJ_TOL[cfg.dtype]


def test_api_errors_change_no_state():
    cfg = SMALL["m50_like"]
    m, w, tok = make_model(cfg, [10, 10], max_len=12)
    s0 = m.get_state(0)[0].clone()
    cases = [
        (lambda: m.decoder_step([0, 0]), 5),
        (lambda: m.decoder_step([2]), 1),
        (lambda: m.decoder_step([-1]), 1),
        (lambda: m.run_sequence([0, 1], 11), 3),
        (lambda: m.run_ragged([0, 1], [3, 11]), 3),
        (lambda: m.set_state(0, s0, None, 13), 1),
        (lambda: m.prefill_encoder(torch.zeros(13, dtype=torch.int32, device="cuda"),
                                   [0], [0], [13]), 4),
        (lambda: m.prefill_encoder(torch.zeros(4, dtype=torch.int32, device="cuda"),
                                   [1, 1], [0, 2], [2, 2]), 5),
    ]
    for fn, code in cases:
        with pytest.raises(RLTError) as ei:
            fn()
        assert ei.value.status == code
    s, c, t = m.get_state(0)
    assert t == 0 and torch.equal(s, s0)
    m.run_sequence([0, 1], 10)  # still usable
    assert m.get_state(1)[2] == 10


def test_bad_token_sets_device_error():
    cfg = SMALL["m50_like"]
    m, w, tok = make_model(cfg, [4], prefill=False)
    bad = torch.tensor([1, cfg.vocab, 2, 3], dtype=torch.int32, device="cuda")
    m.prefill_encoder(bad, [0], [0], [4])
    assert m.poll_device_error() == 8
    assert m.poll_device_error() == 0


def test_window_one_and_short_sequences():
    """W = 1 (only the current token) and sequences shorter than the window."""
    for cfg, T in ((SMALL["m50_like"].replace(window=1), 20),
                   (SMALL["m50_like"].replace(window=64), 20)):
        m, w, tok = make_model(cfg, [T])
        m.run_sequence([0], T)
        ref = oracle.Oracle(cfg, w).run(tok[0])[1]
        assert rel_l2(to_np(m.get_state(0)[0]), ref) <= TRAJ_TOL[cfg.dtype]


def test_graph_replay_equals_direct_launches():
    """Steps on a side stream replay captured CUDA graphs; results are bitwise
    those of direct launches on the legacy stream (same kernels, same order)."""
    cfg = SMALL["m140_like"]
    lengths = [300, 300, 290]
    w = inputs.make_weights(cfg, 0, True)
    tok = inputs.make_tokens(cfg.vocab, lengths)
    a = Model(cfg, w, 3, 300)
    prefill_all(a, tok, lengths)
    a.run_ragged([0, 1, 2], lengths)
    side = torch.cuda.Stream()
    b = Model(cfg, w, 3, 300, stream=side)
    with torch.cuda.stream(side):
        prefill_all(b, tok, lengths)
    b.run_ragged([0, 1, 2], lengths)
    side.synchronize()
    for i in range(3):
        sa = a.get_state(i)
        with torch.cuda.stream(side):
            sb = b.get_state(i)
        side.synchronize()
        assert sa[2] == sb[2] == lengths[i]
        assert torch.equal(sa[0], sb[0]) and torch.equal(sa[1], sb[1])
    assert a.poll_device_error() == 0 and b.poll_device_error() == 0


def test_encoder_is_causal_at_full_size_bitwise():
    """Changing tokens after position k changes no e_<=k and no memory row
    <= k, at the ~140M workload's size (256 x 1024 tokens, 131072-row chunks)."""
    wl = configs.workloads()["m140_bf16"]
    cfg = wl.model
    B, T = 8, wl.max_len
    w = inputs.make_weights(cfg)
    tok = inputs.make_tokens(cfg.vocab, [T] * B)
    m = Model(cfg, w, B, T)
    prefill_all(m, tok, [T] * B)
    before = [m.get_encoder_output(i) for i in (0, 5)]
    k = 700
    tok2 = tok.copy()
    tok2[:, k + 1:] = (tok2[:, k + 1:] + 7) % cfg.vocab
    prefill_all(m, tok2, [T] * B)
    for (e0, m0), i in zip(before, (0, 5)):
        e1, m1 = m.get_encoder_output(i)
        assert torch.equal(e0[: k + 1], e1[: k + 1])
        assert torch.equal(m0[:, : k + 1], m1[:, : k + 1])
        assert not torch.equal(e0[k + 1:], e1[k + 1:])


@pytest.mark.parametrize("name,kernel", [("ragged_like", "fused"), ("tied_like", "fused"),
                                         ("m140_like", "fused"), ("m140_like", "chain")])
def test_stepwise_parity_past_one_memory_chunk(name, kernel):
    """Positions past 1024: the cross-attention over M<=t splits into several
    1024-row chunks (partials merged in chunk order, a ragged tail chunk);
    step-wise against the oracle fed the GPU's own state."""
    cfg = SMALL[name]
    T = 2100
    m, w, tok = make_model(cfg, [T] * 2)
    _use(m, kernel)
    o = oracle.Oracle(cfg, w)
    e_g, mem_g = (to_np(x) for x in m.get_encoder_output(1))
    tol = STEP_TOL[cfg.dtype]
    done = 0
    for t in (1023, 1024, 1025, 2047, 2048, T - 1):
        m.run_sequence([0, 1], t - done)
        s_prev, c_prev, tt = m.get_state(1)
        assert tt == t
        m.run_sequence([0, 1], 1)
        done = t + 1
        s_ref, win_ref = o.step(e_g[t], mem_g, t, to_np(s_prev), to_np(c_prev))
        s_new, c_new, _ = m.get_state(1)
        err = np.abs(to_np(s_new) - s_ref).max() / rms(s_ref)
        assert err <= tol, (name, t, err)
        newest = to_np(c_new)[:, :, -1]
        assert np.abs(newest - win_ref[:, :, -1]).max() <= CACHE_TOL[cfg.dtype] * rms(
            win_ref[:, :, -1])


@pytest.mark.parametrize("kernel", ["fused", "chain"])
def test_bounded_wait_timeout_is_reported_and_model_recovers(kernel):
    """Failure detection without faulting the GPU: a planted fault makes the
    decoder attention's producer fill nothing, so its consumers' bounded waits
    (limited to 2 ms for the test) run out; the step returns, the device error
    word reads RLT_ERR_TIMEOUT, and after the fault is cleared and the slots
    are prefilled again the model computes the same states as a fresh one."""
    from token_recurrent_decoding_b200 import rlt as R
    cfg = SMALL["m50_like"]
    lengths = [24, 24]
    m, w, tok = make_model(cfg, lengths)
    _use(m, kernel)
    m.set_fault(R.FAULT_SKIP_ATTN_PRODUCER, 2_000_000)
    m.decoder_step([0, 1])
    assert m.poll_device_error() == 7  # RLT_ERR_TIMEOUT
    assert m.poll_device_error() == 0  # the poll cleared it
    m.set_fault(R.FAULT_NONE, 0)
    prefill_all(m, tok, lengths)
    m.run_sequence([0, 1], 24)
    assert m.poll_device_error() == 0
    ref, _, _ = make_model(cfg, lengths)
    _use(ref, kernel)
    ref.run_sequence([0, 1], 24)
    for i in range(2):
        assert torch.equal(m.get_state(i)[0], ref.get_state(i)[0])
    with pytest.raises(RLTError):
        m.set_fault(99, 0)


def test_fused_and_chain_kernels_agree():
    """The persistent one-launch step and the chain of kernels compute the
    same transition (bf16 tolerance: different split-K partitions), on a
    batch of more than one 128-row tile, for a whole trajectory."""
    cfg = SMALL["m140_like"]
    lengths = [70] * 200
    a, w, tok = make_model(cfg, lengths)
    b, _, _ = make_model(cfg, lengths)
    _use(a, "fused")
    _use(b, "chain")
    ids = list(range(len(lengths)))
    a.run_sequence(ids, 70)
    b.run_sequence(ids, 70)
    for i in (0, 99, 127, 128, 199):
        assert rel_l2(to_np(a.get_state(i)[0]), to_np(b.get_state(i)[0])) <= TRAJ_TOL[cfg.dtype]
    o = oracle.Oracle(cfg, w)
    for i in (0, 150):
        assert rel_l2(to_np(a.get_state(i)[0]), o.run(tok[i])[1]) <= TRAJ_TOL[cfg.dtype]
    assert a.poll_device_error() == 0
