"""GPU parity of backpropagation through time (rlt_backward) against the
gradient oracle (oracle/bptt.py: float64 forward, reverse mode by autograd,
pinned by finite differences of the C oracle).

The oracle is fed the GPU's own encoder output e (so the encoder's rounding
is not charged to the backward) and the same upstream gradients. Per
gradient tensor the bar is the trajectory tolerance of the forward parity, as a
relative L2 error: the gradient is a smooth function of the trajectory, and
the GPU's trajectory is the product forward's (bf16 storage of K/V, memory
and GEMM inputs for bf16 models), within that tolerance of the oracle's.
"""
import numpy as np
import pytest
import torch

from oracle import bptt
from rlt_cases import SMALL, TRAJ_TOL, make_model, to_np
from token_recurrent_decoding_b200 import configs

pytestmark = pytest.mark.gpu


def _sgrad(n, T, d, seed=5):
    g = np.random.default_rng(seed).standard_normal((n, T, d)).astype(np.float32)
    return g, torch.from_numpy(g).cuda()


def _oracle(m, cfg, w, ids, T, G, t0=0, s0=None, win0=None, carry_s=None, carry_win=None):
    """Oracle gradients summed over the listed sequences (parameters), per
    sequence for e and the carried state."""
    tot, per = None, []
    for b, i in enumerate(ids):
        e = to_np(m.get_encoder_output(i)[0])
        s_start = w["sstar"] if s0 is None else s0[b]
        wz = np.zeros((cfg.n_dec, 2, max(cfg.window - 1, 0), cfg.d)) if win0 is None else win0[b]
        r = bptt.chunk_grads(cfg, w, e, s_start, wz, t0, t0 + T, G[b],
                             None if carry_s is None else carry_s[b],
                             None if carry_win is None else carry_win[b])
        per.append(r)
        if tot is None:
            tot = {k: np.array(v, np.float64) for k, v in r.items() if k in bptt.param_names(cfg)}
        else:
            for k in tot:
                tot[k] += r[k]
    return tot, per


def _rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / nb) if nb > 0 else float(np.linalg.norm(a))


CASES = ["tiny_fp32", "m50_like", "m140_like", "tied_like"]


@pytest.mark.parametrize("name", CASES)
def test_backward_matches_oracle(name):
    cfg = SMALL[name]
    T, B = (12, 2) if cfg.dtype == configs.F32 else (20, 3)
    m, w, tok = make_model(cfg, [T] * B)
    ids = list(range(B))
    G, Gd = _sgrad(B, T, cfg.d)
    grads, egrad, carry = m.backward(ids, Gd)
    torch.cuda.synchronize()
    assert m.poll_device_error() == 0
    ref, per = _oracle(m, cfg, w, ids, T, G)
    tol = TRAJ_TOL[cfg.dtype]
    worst = {}
    for k, v in ref.items():
        worst[k] = _rel(to_np(grads[k]), v)
    bad = {k: e for k, e in worst.items() if not e <= tol}
    print(name, "worst relative L2 error", max(worst.values()), max(worst, key=worst.get))
    assert not bad, (name, bad)
    eg = to_np(egrad)
    for b in range(B):
        assert _rel(eg[b, :T], per[b]["e"]) <= tol, (name, "e", b)
    # the state's gradient entering position 0 is s*'s gradient (carried out too)
    c = to_np(carry)
    for b in range(B):
        assert _rel(c[b, :cfg.d], per[b]["s0"]) <= tol, (name, "s0", b)


def test_backward_alpha_zero_and_window_one():
    cfg = SMALL["m50_like"].replace(alpha=0.0, window=1)
    T, B = 10, 2
    m, w, tok = make_model(cfg, [T] * B)
    G, Gd = _sgrad(B, T, cfg.d, seed=6)
    grads, egrad, carry = m.backward([0, 1], Gd)
    ref, per = _oracle(m, cfg, w, [0, 1], T, G)
    for k in ("gate.w", "gate.b", "sstar"):
        assert not torch.any(grads[k]).item(), k
    for k, v in ref.items():
        if k in ("gate.w", "gate.b", "sstar"):
            continue
        assert _rel(to_np(grads[k]), v) <= TRAJ_TOL[cfg.dtype], k


@pytest.mark.parametrize("name", ["tiny_fp32", "m140_like"])
def test_chunked_backward_composes(name):
    """Chunks in reverse order chained by the carried gradient equal one pass
    over the whole sequence (exact backpropagation through time), and the
    state left behind equals rlt_run_sequence's."""
    cfg = SMALL[name]
    T, k, B = 14, 9, 2
    m, w, tok = make_model(cfg, [T] * B)
    ids = [0, 1]
    G, Gd = _sgrad(B, T, cfg.d, seed=8)
    start = [m.get_state(i) for i in ids]
    full, e_full, _ = m.backward(ids, Gd)
    end_full = [m.get_state(i) for i in ids]
    for i, (s, c, t) in zip(ids, start):
        m.set_state(i, s, c, t)
    m.run_sequence(ids, k)
    mid = [m.get_state(i) for i in ids]
    late, e_acc, carry = m.backward(ids, Gd[:, k:].contiguous())
    end_late = [m.get_state(i) for i in ids]
    for i, (s, c, t) in zip(ids, start):
        m.set_state(i, s, c, t)
    m.backward(ids, Gd[:, :k].contiguous(), grads=late, egrad=e_acc, carry_in=carry)
    torch.cuda.synchronize()
    # fp32: the same arithmetic regrouped; bf16: each chunk rounds its own
    # partial memory-row gradients to bf16 for the projection's tensor-core
    # GEMMs (2^-9 relative per element, on either side)
    bound = 1e-5 if cfg.dtype == configs.F32 else 1e-2
    for key in full:
        assert _rel(to_np(late[key]), to_np(full[key])) <= bound, key
    assert _rel(to_np(e_acc), to_np(e_full)) <= bound
    for a, b in zip(end_full, end_late):
        assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1]) and a[2] == b[2] == T
    # against the oracle as two chunks too: the late chunk from the GPU's state at k
    s0 = np.stack([to_np(x[0]) for x in mid])
    win0 = np.stack([to_np(x[1]) for x in mid])
    ref_late, per_late = _oracle(m, cfg, w, ids, T - k, G[:, k:], t0=k, s0=s0, win0=win0)
    for key, v in ref_late.items():
        if key == "sstar":
            continue
        assert np.isfinite(v).all()
    c = to_np(carry)
    tol = TRAJ_TOL[cfg.dtype]
    for b in range(B):
        assert _rel(c[b, :cfg.d], per_late[b]["s0"]) <= tol
        assert _rel(c[b, cfg.d:], per_late[b]["win0"].reshape(-1)) <= tol


def test_backward_argument_checks():
    cfg = SMALL["tiny_fp32"]
    m, w, tok = make_model(cfg, [8, 8])
    G, Gd = _sgrad(2, 4, cfg.d)
    m.run_sequence([1], 1)  # sequences at different positions
    with pytest.raises(RuntimeError):
        m.backward([0, 1], Gd)
    with pytest.raises(RuntimeError):  # past the encoder output
        m.backward([0], torch.zeros((1, 9, cfg.d), device="cuda"))
    with pytest.raises(RuntimeError):  # workspace too small
        m.backward([0], Gd[:1].contiguous(), workspace=torch.empty(256, dtype=torch.uint8,
                                                                   device="cuda"))
    assert m.get_state(0)[2] == 0  # refused calls changed nothing


def test_backward_full_size_m140_late_chunk():
    """The ~140M model at its real shapes (d = 768, 12 + 12 layers, W = 128,
    G = L_D, SwiGLU-free GELU FFN 3072) for two sequences: a chunk of
    positions 1000 .. 1007 after 1000 recurrent steps (memory rows up to
    1007, full windows), every parameter gradient, dL/de and the carried
    state against the gradient oracle started from the GPU's own state."""
    wl = configs.workloads()["m140_bf16"]
    cfg = wl.model
    T, t0, NS, B = 1024, 1000, 8, 2
    m, w, tok = make_model(cfg, [T] * B)
    ids = [0, 1]
    m.run_sequence(ids, t0)
    state = [m.get_state(i) for i in ids]
    G, Gd = _sgrad(B, NS, cfg.d, seed=9)
    grads, egrad, carry = m.backward(ids, Gd)
    torch.cuda.synchronize()
    assert m.poll_device_error() == 0
    s0 = np.stack([to_np(x[0]) for x in state])
    win0 = np.stack([to_np(x[1]) for x in state])
    ref, per = _oracle(m, cfg, w, ids, NS, G, t0=t0, s0=s0, win0=win0)
    tol = TRAJ_TOL[cfg.dtype]
    worst = {k: _rel(to_np(grads[k]), v) for k, v in ref.items() if k != "sstar"}
    print("m140 full size worst relative L2 error", max(worst.values()), max(worst, key=worst.get))
    assert all(e <= tol for e in worst.values()), {k: e for k, e in worst.items() if e > tol}
    eg = to_np(egrad)
    c = to_np(carry)
    for b in range(B):
        assert _rel(eg[b, :t0 + NS], per[b]["e"]) <= tol
        assert _rel(c[b, :cfg.d], per[b]["s0"]) <= tol
        assert _rel(c[b, cfg.d:], per[b]["win0"].reshape(-1)) <= tol
