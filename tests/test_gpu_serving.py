"""Serving state and the autoregressive loop, through the C ABI, against the
fp64 oracle: exact prefix snapshots (restore continues bit for bit; other
weights or another configuration are refused), one-token encoder appends
(equal to a whole-sequence encoding of the longer prompt), the next-token
head and the sampler, and whole serve loops."""
import numpy as np
import pytest
import torch

import oracle
from rlt_cases import (SMALL, STEP_TOL, TRAJ_TOL, make_model, prefill_all, rel_l2, rms,
                       to_np)
from token_recurrent_decoding_b200 import configs, inputs
from token_recurrent_decoding_b200.rlt import Model, RLTError

pytestmark = pytest.mark.gpu

# encoder outputs and memory rows are stored in the model dtype (see
# test_gpu_parity.ENC_TOL): max|err| / RMS and rel-L2
ENC_TOL = {configs.F32: (1e-5, 1e-6), configs.BF16: (6e-2, 1.5e-2)}
STATUS_STALE = 9


def _header(buf):
    """(t_dec, t_enc) of a snapshot held in a uint8 tensor."""
    raw = buf[:256].cpu().numpy()
    t_dec, t_enc = np.frombuffer(raw[64:80].tobytes(), dtype=np.int64)
    return int(t_dec), int(t_enc)


@pytest.mark.parametrize("name,enc_cache", [("m50_like", True), ("m140_like", False),
                                            ("tiny_fp32", True), ("tied_like", True)])
def test_snapshot_restore_continues_exactly(name, enc_cache):
    """Proposition 3.1 for a whole serving state: slot 1 runs k steps, its
    snapshot goes through pinned host memory into slot 2 of ANOTHER model with
    the same weights, which runs the rest; states and encoder outputs equal an
    uninterrupted run bit for bit."""
    cfg = SMALL[name]
    T, k = 48, 19
    w = inputs.make_weights(cfg, 0, True)
    tok = inputs.make_tokens(cfg.vocab, [T])
    both = np.concatenate([tok, tok, tok])
    a = Model(cfg, w, 3, T, enc_cache=enc_cache)
    prefill_all(a, both, [T, T, T])
    a.run_sequence([0], T)
    a.run_sequence([1], k)
    snap = a.get_snapshot(1, torch.empty(a.snapshot_bytes(1), dtype=torch.uint8).pin_memory())
    torch.cuda.synchronize()
    assert _header(snap) == (k, T)
    b = Model(cfg, w, 3, T, enc_cache=enc_cache)
    b.set_snapshot(2, snap)
    assert b.get_state(2)[2] == k
    eb, mb = b.get_encoder_output(2)
    ea, ma = a.get_encoder_output(1)
    assert torch.equal(eb, ea) and torch.equal(mb, ma)
    b.run_sequence([2], T - k)
    assert torch.equal(a.get_state(0)[0], b.get_state(2)[0])
    assert torch.equal(a.get_state(0)[1], b.get_state(2)[1])
    # a device-memory snapshot round-trips too
    snap_d = b.get_snapshot(2)
    a.set_snapshot(1, snap_d)
    assert torch.equal(a.get_state(1)[0], a.get_state(0)[0])


def test_snapshot_refused_for_other_weights_or_configuration():
    cfg = SMALL["m50_like"]
    T = 24
    a, w, tok = make_model(cfg, [T], enc_cache=True)
    a.run_sequence([0], 5)
    snap = a.get_snapshot(0)
    torch.cuda.synchronize()
    f0 = a.fingerprint()
    # other weight values
    w2 = inputs.make_weights(cfg, 1, True)
    other = Model(cfg, w2, 1, T, enc_cache=True)
    with pytest.raises(RLTError) as e:
        other.set_snapshot(0, snap)
    assert e.value.status == STATUS_STALE
    # the same model after a weight update in place
    b = Model(cfg, w, 1, T, enc_cache=True)
    assert b.fingerprint() == f0
    b.set_snapshot(0, snap)
    t = next(iter(b._dev.values()))
    t.view(-1)[0] += 1
    assert b.fingerprint() != f0
    with pytest.raises(RLTError) as e:
        b.set_snapshot(0, snap)
    assert e.value.status == STATUS_STALE
    # another window convention
    c = Model(cfg.replace(window=cfg.window + 1), w, 1, T, enc_cache=True)
    with pytest.raises(RLTError) as e:
        c.set_snapshot(0, snap)
    assert e.value.status == STATUS_STALE
    # not a snapshot
    junk = torch.zeros(snap.numel(), dtype=torch.uint8, device="cuda")
    with pytest.raises(RLTError) as e:
        b.set_snapshot(0, junk)
    assert e.value.status == 1


@pytest.mark.parametrize("name,P,k", [("m140_like", 40, 9), ("tied_like", 250, 12),
                                      ("tiny_fp32", 30, 6), ("ragged_like", 1020, 8)])
def test_encoder_append_equals_whole_prompt_encoding(name, P, k):
    """Appending tokens one at a time extends e and M<=t exactly as encoding
    the longer prompt does (the encoder is causal): against the oracle's
    whole-sequence encoding, across a cross-attention chunk boundary for the
    longer prompts."""
    cfg = SMALL[name]
    L = P + k
    w = inputs.make_weights(cfg, 0, True)
    tok = inputs.make_tokens(cfg.vocab, [L])
    m = Model(cfg, w, 2, L, enc_cache=True)
    prefill_all(m, tok, [P])
    for j in range(P, L):
        m.append_encoder(torch.tensor([tok[0, j]], dtype=torch.int32, device="cuda"), [0])
    e_g, mem_g = (to_np(x) for x in m.get_encoder_output(0))
    assert e_g.shape[0] == L
    e_r, mem_r = oracle.Oracle(cfg, w).encode(tok[0])
    tmax, trel = ENC_TOL[cfg.dtype]
    assert np.abs(e_g - e_r).max() <= tmax * rms(e_r)
    assert rel_l2(e_g, e_r) <= trel
    mr = mem_r[:, :L]
    assert np.abs(mem_g - mr).max() <= tmax * rms(mr)
    # the appended positions agree with the GPU's own whole prefill
    prefill_all(m, np.concatenate([tok, tok]), [L, L], ids=[1, 0])
    e_p = to_np(m.get_encoder_output(1)[0])
    assert rel_l2(e_g[P:], e_p[P:]) <= trel
    assert m.poll_device_error() == 0


def _check_sample(logits64, tau, u, got):
    """The GPU's draw from its own logits: the oracle's draw, or (fp32 sums
    against fp64 sums) a token whose cumulative weight brackets the target
    within rounding."""
    ref = oracle.sample(logits64, tau, u)
    if got == ref:
        return
    if tau == 0:
        assert logits64[got] == logits64.max(), (got, ref)
        return
    p = np.exp((logits64 - logits64.max()) / tau)
    cum = np.cumsum(p)
    target = u * cum[-1]
    lo = cum[got - 1] if got > 0 else 0.0
    assert lo - 1e-5 * cum[-1] <= target <= cum[got] + 1e-5 * cum[-1], (got, ref)


@pytest.mark.parametrize("name", ["tiny_fp32", "m50_like", "tied_like"])
def test_lm_head_and_sampler(name):
    cfg = SMALL[name]
    T = 20
    m, w, tok = make_model(cfg, [T] * 3, enc_cache=True)
    m.run_sequence([0, 1, 2], 11)
    o = oracle.Oracle(cfg, w)
    ids = [2, 0, 1]
    logits = m.lm_head(ids)
    lg = to_np(logits)
    tol = STEP_TOL[cfg.dtype]
    for r, i in enumerate(ids):
        ref = o.lm_head(to_np(m.get_state(i)[0]))
        assert np.abs(lg[r] - ref).max() <= tol * rms(ref), (name, i)
    g = torch.Generator(device="cpu").manual_seed(7)
    for tau in (0.0, 0.7, 1.5):
        u = torch.rand(3, generator=g).cuda()
        got = m.sample(logits, tau, u).cpu().numpy()
        for r in range(3):
            _check_sample(lg[r], tau, float(u[r]), int(got[r]))
    with pytest.raises(RLTError):
        m.sample(logits, -1.0, None)


@pytest.mark.parametrize("name,tau", [("tiny_fp32", 0.9), ("m50_like", 0.0),
                                      ("m140_like", 1.0)])
def test_serve_loop_against_oracle(name, tau):
    """Prompt prefill, the decoder over the prompt, then serve steps (step,
    head, draw, append) against the oracle fed the same tokens: every s_t and
    the logits step-wise on the GPU's state, every draw valid for the GPU's
    logits, and the final encoder output and decoder trajectory of the whole
    generated sequence from tokens alone."""
    cfg = SMALL[name]
    P, G = 17, 10
    L = P + G
    w = inputs.make_weights(cfg, 0, True)
    tok = inputs.make_tokens(cfg.vocab, [L] * 2)
    m = Model(cfg, w, 2, L, enc_cache=True)
    prefill_all(m, tok, [P, P])
    m.run_sequence([0, 1], P - 1)
    o = oracle.Oracle(cfg, w)
    gen = [list(tok[0, :P]), list(tok[1, :P])]
    g = torch.Generator(device="cpu").manual_seed(3)
    for step in range(G):
        u = torch.rand(2, generator=g).cuda()
        out, logits = m.serve_step([0, 1], tau, u)
        toks = out.cpu().numpy()
        lg = to_np(logits)
        for i in range(2):
            ref = o.lm_head(to_np(m.get_state(i)[0]))
            assert np.abs(lg[i] - ref).max() <= STEP_TOL[cfg.dtype] * rms(ref)
            _check_sample(lg[i], tau, float(u[i]), int(toks[i]))
            gen[i].append(int(toks[i]))
    assert m.poll_device_error() == 0
    for i in range(2):
        seq = np.asarray(gen[i], dtype=np.int32)
        e_g = to_np(m.get_encoder_output(i)[0])
        e_r, _ = o.encode(seq)
        assert rel_l2(e_g, e_r) <= ENC_TOL[cfg.dtype][1]
        # decoder: P - 1 + G transitions; the oracle runs them from tokens
        s_all, _, _ = o.run(seq)
        assert m.get_state(i)[2] == P - 1 + G
        assert rel_l2(to_np(m.get_state(i)[0]), s_all[P - 2 + G]) <= TRAJ_TOL[cfg.dtype]


def test_snapshot_mid_generation_replays_the_same_tokens():
    """A snapshot taken between serve steps (encoder cache included) restored
    into another model continues with the same draws, bit for bit."""
    cfg = SMALL["m50_like"]
    P, G = 12, 6
    w = inputs.make_weights(cfg, 0, True)
    tok = inputs.make_tokens(cfg.vocab, [P + 2 * G])
    a = Model(cfg, w, 1, P + 2 * G, enc_cache=True)
    prefill_all(a, tok, [P])
    a.run_sequence([0], P - 1)
    g = torch.Generator(device="cpu").manual_seed(11)
    us = [torch.rand(1, generator=g).cuda() for _ in range(2 * G)]
    for k in range(G):
        a.serve_step([0], 0.8, us[k])
    snap = a.get_snapshot(0)
    rest_a = [int(a.serve_step([0], 0.8, us[G + k])[0].item()) for k in range(G)]
    b = Model(cfg, w, 1, P + 2 * G, enc_cache=True)
    b.set_snapshot(0, snap)
    rest_b = [int(b.serve_step([0], 0.8, us[G + k])[0].item()) for k in range(G)]
    assert rest_a == rest_b
    assert torch.equal(a.get_state(0)[0], b.get_state(0)[0])


def test_serving_errors_change_no_state():
    cfg = SMALL["m50_like"]
    m, w, tok = make_model(cfg, [10, 10], enc_cache=False)
    with pytest.raises(RLTError) as e:
        m.append_encoder(torch.zeros(1, dtype=torch.int32, device="cuda"), [0])
    assert e.value.status == 2  # UNSUPPORTED without the encoder cache
    m2, _, _ = make_model(cfg, [10, 10], enc_cache=True, max_len=12)
    u = torch.rand(1).cuda()
    with pytest.raises(RLTError) as e:
        m2.serve_step([0], 1.0, u)  # the decoder has not reached the last prompt token
    assert e.value.status == 3
    m2.run_sequence([0], 9)
    with pytest.raises(RLTError) as e:
        m2.serve_step([0, 0], 1.0, torch.rand(2).cuda())
    assert e.value.status == 5
    assert m2.get_state(0)[2] == 9
    m2.serve_step([0], 1.0, u)  # appends position 10
    m2.serve_step([0], 1.0, u)  # appends position 11: the arena is full
    with pytest.raises(RLTError) as e:
        m2.serve_step([0], 1.0, u)
    assert e.value.status == 4
    assert m2.get_state(0)[2] == 11
    assert m2.get_encoder_output(0)[0].shape[0] == 12


def test_serve_step_on_a_two_chain_batch():
    """Batches of 128 rows and more step as two half-batch chains; the serve
    step's head, draw and append follow the same rows: greedy draws equal the
    argmax of the logits the oracle reads from the GPU's s_t."""
    cfg = SMALL["m140_like"]
    B, P = 160, 6
    w = inputs.make_weights(cfg, 0, True)
    tok = inputs.make_tokens(cfg.vocab, [P + 3] * B)
    m = Model(cfg, w, B, P + 3, enc_cache=True)
    prefill_all(m, tok, [P] * B)
    ids = list(range(B))
    m.run_sequence(ids, P - 1)
    o = oracle.Oracle(cfg, w)
    for step in range(3):
        out, logits = m.serve_step(ids, 0.0)
        toks = out.cpu().numpy()
        lg = to_np(logits)
        for i in (0, 79, 80, 159):
            ref = o.lm_head(to_np(m.get_state(i)[0]))
            assert np.abs(lg[i] - ref).max() <= STEP_TOL[cfg.dtype] * rms(ref)
            assert lg[i][toks[i]] == lg[i].max()
    assert m.get_state(0)[2] == P + 2
    assert m.poll_device_error() == 0
