"""Pins of the gradient oracle (oracle/bptt.py), CPU only.

The gradient is pinned to things other than itself:
  * its forward equals the C oracle's forward (an independent implementation
    pinned by test_oracle_invariants / test_oracle_pieces) step for step;
  * every gradient, tensor by tensor, equals the central finite difference of
    the C oracle's float64 loss along a random direction;
  * chunks run backwards and chained by their carried gradient equal one
    pass over the whole sequence (exact backpropagation through time);
  * alpha = 0 gives exactly zero gradient to the gate and to s ([RLT-PV]
    body: alpha = 0 strips the recurrent path);
  * with s detached between steps, a window of one position cuts every path
    between steps, while W >= 2 leaves the cache paths open ([RLT-96]
    "Training and serving implications": the state-to-state Jacobian has
    cross-terms through the decoder's cache).
"""
import numpy as np
import pytest

import oracle
from oracle import bptt
from token_recurrent_decoding_b200 import configs, inputs


def tiny(**kw):
    base = dict(d=16, n_heads=2, head_dim=8, n_enc=1, n_dec=2, ffn_dim=24,
                ffn_kind=configs.GELU, vocab=32, window=3, mem_groups=1, tied=False,
                dtype=configs.F32, alpha=1.0)
    base.update(kw)
    return configs.RLTConfig(**base)


def weights(cfg, seed=0, scale=10.0):
    """Generator weights with matrices scaled up so every nonlinearity bites."""
    w = inputs.make_weights(cfg, seed, perturb=True)
    out = {}
    for k, v in w.items():
        v = np.asarray(v, np.float64)
        out[k] = v * scale if v.ndim == 2 and k != "embed" else v.copy()
    out["gate.b"] = out["gate.b"] + 0.3
    return out


def problem(cfg, T, t0, seed=1):
    rng = np.random.default_rng(seed)
    d = cfg.d
    e = rng.standard_normal((T, d))
    s0 = rng.standard_normal(d)
    win0 = rng.standard_normal((cfg.n_dec, 2, max(cfg.window - 1, 0), d))
    # entries of positions < 0 are zero in a real state
    for i in range(cfg.window - 1):
        if t0 - (cfg.window - 1) + i < 0:
            win0[:, :, i] = 0.0
    G = rng.standard_normal((T - t0, d))
    cs = rng.standard_normal(d)
    cw = rng.standard_normal(win0.shape)
    return e, s0, win0, G, cs, cw


def memory(cfg, w, e, T):
    mem = np.zeros((cfg.mem_groups, T, 2, cfg.d))
    for g in range(cfg.mem_groups):
        for j in range(T):
            mem[g, j, 0] = oracle.linear(w[f"mem.{g}.wk"], e[j])
            mem[g, j, 1] = oracle.linear(w[f"mem.{g}.wv"], e[j])
    return mem


def c_loss(cfg, w, e, s0, win0, t0, t1, G, cs=None, cw=None):
    """The chunk loss with the C oracle's float64 forward."""
    orc = oracle.Oracle(cfg, w)
    s_start = w["sstar"] if t0 == 0 else s0
    out, s, win = orc.decode(e, memory(cfg, w, e, t1), t0, t1, s_start, win0)
    L = float(np.sum(out * G))
    if cs is not None:
        L += float(np.dot(s, cs))
    if cw is not None and cfg.window > 1:
        pos = t1 - (cfg.window - 1) + np.arange(cfg.window - 1)
        L += float(np.sum(win * cw * (pos >= 0)[None, None, :, None]))
    return L


FORWARD_CASES = [
    dict(),
    dict(ffn_kind=configs.SWIGLU, mem_groups=2, window=2),
    dict(window=1, alpha=0.5),
    dict(window=8, alpha=0.0, n_dec=3, mem_groups=3),
]


@pytest.mark.parametrize("kw", FORWARD_CASES)
@pytest.mark.parametrize("t0", [0, 3])
def test_forward_matches_c_oracle(kw, t0):
    import torch
    cfg = tiny(**kw)
    w = weights(cfg)
    T = 7
    e, s0, win0, *_ = problem(cfg, T, t0)
    s_start = w["sstar"] if t0 == 0 else s0
    orc = oracle.Oracle(cfg, w)
    ref, s_ref, win_ref = orc.decode(e, memory(cfg, w, e, T), t0, T, s_start, win0)
    P = {n: torch.tensor(w[n]) for n in bptt.param_names(cfg)}
    out, s, win = bptt.chunk_forward(cfg, P, torch.tensor(e), torch.tensor(s_start),
                                     torch.tensor(win0), t0, T)
    assert np.max(np.abs(out.numpy() - ref)) < 1e-12 * max(1.0, np.max(np.abs(ref)))
    assert np.max(np.abs(s.numpy() - s_ref)) < 1e-12
    if cfg.window > 1:
        pos = T - (cfg.window - 1) + np.arange(cfg.window - 1)
        keep = pos >= 0
        assert np.max(np.abs(win.numpy()[:, :, keep] - win_ref[:, :, keep])) < 1e-11


FD_CASES = [
    (dict(), 6, 0),
    (dict(ffn_kind=configs.SWIGLU, mem_groups=2, window=2), 5, 0),
    (dict(window=1, alpha=0.5), 5, 2),
    (dict(window=4), 7, 3),
]


def fd_mismatches(cfg, T, t0, tol=1e-6):
    """Names whose oracle gradient disagrees with the central finite difference
    of the C oracle's loss along a random direction."""
    w = weights(cfg)
    e, s0, win0, G, cs, cw = problem(cfg, T, t0)
    res = bptt.chunk_grads(cfg, w, e, s0, win0, t0, T, G, cs, cw)
    rng = np.random.default_rng(7)
    h = 1e-5
    bad = []
    targets = list(bptt.param_names(cfg)) + ["e", "win0"] + ([] if t0 == 0 else ["s0"])
    for name in targets:
        if name == "win0" and cfg.window == 1:
            continue
        base = {"e": e, "win0": win0, "s0": s0}.get(name)
        if base is None:
            base = w[name]
        delta = rng.standard_normal(base.shape)
        if name == "win0":  # entries of positions < 0 are not part of the state
            for i in range(cfg.window - 1):
                if t0 - (cfg.window - 1) + i < 0:
                    delta[:, :, i] = 0.0

        def loss_at(sign):
            ww, ee, ss, wn = dict(w), e, s0, win0
            if name == "e":
                ee = e + sign * h * delta
            elif name == "win0":
                wn = win0 + sign * h * delta
            elif name == "s0":
                ss = s0 + sign * h * delta
            else:
                ww[name] = w[name] + sign * h * delta
            return c_loss(cfg, ww, ee, ss, wn, t0, T, G, cs, cw)

        fd = (loss_at(1) - loss_at(-1)) / (2 * h)
        an = float(np.sum(res[name] * delta))
        scale = float(np.linalg.norm(res[name]) * np.linalg.norm(delta)) + 1e-12
        if not abs(fd - an) <= tol * scale:
            bad.append(name)
    return bad


@pytest.mark.parametrize("kw,T,t0", FD_CASES)
def test_gradients_match_finite_differences(kw, T, t0):
    assert fd_mismatches(tiny(**kw), T, t0) == []


def test_planted_mistakes_fail_the_pins(monkeypatch):
    """A cache detached from the graph (the trap the pages warn of) and a
    rotary sign flip in the gradient oracle are each caught."""
    import torch
    cfg = tiny(window=4)
    real_attend = bptt._attend

    def attend_history_detached(q, K, V):
        if K.shape[0] > 1:
            K = torch.cat([K[:-1].detach(), K[-1:]])
            V = torch.cat([V[:-1].detach(), V[-1:]])
        return real_attend(q, K, V)

    monkeypatch.setattr(bptt, "_attend", attend_history_detached)
    assert "dec.0.wqkv" in fd_mismatches(cfg, 6, 0)
    monkeypatch.setattr(bptt, "_attend", real_attend)
    real_rope = bptt._rope
    monkeypatch.setattr(bptt, "_rope", lambda v, pos, dh, th: real_rope(v, -pos, dh, th))
    with pytest.raises(AssertionError):
        test_forward_matches_c_oracle(dict(), 0)


@pytest.mark.parametrize("kw", [dict(window=3), dict(window=5, ffn_kind=configs.SWIGLU,
                                                     mem_groups=2)])
def test_chunks_compose_into_full_gradient(kw):
    cfg = tiny(**kw)
    w = weights(cfg)
    T, k = 8, 5
    e, _, win0, G, _, _ = problem(cfg, T, 0)
    zero_win = np.zeros_like(win0)
    full = bptt.chunk_grads(cfg, w, e, w["sstar"], zero_win, 0, T, G)
    # the state at k from the forward of [0, k)
    import torch
    P = {n: torch.tensor(w[n]) for n in bptt.param_names(cfg)}
    _, s_k, win_k = bptt.chunk_forward(cfg, P, torch.tensor(e), torch.tensor(w["sstar"]),
                                       torch.tensor(zero_win), 0, k)
    late = bptt.chunk_grads(cfg, w, e, s_k.numpy(), win_k.numpy(), k, T, G[k:])
    early = bptt.chunk_grads(cfg, w, e, w["sstar"], zero_win, 0, k, G[:k],
                             late["s0"], late["win0"])
    for name in bptt.param_names(cfg):
        tot = early[name] + late[name]
        assert np.max(np.abs(tot - full[name])) <= 1e-11 * (1 + np.max(np.abs(full[name]))), name
    e_tot = late["e"].copy()
    e_tot[:k] += early["e"]
    assert np.max(np.abs(e_tot - full["e"])) <= 1e-11 * (1 + np.max(np.abs(full["e"])))


def test_alpha_zero_gives_no_gradient_to_gate_or_state():
    cfg = tiny(alpha=0.0, window=3)
    w = weights(cfg)
    T, t0 = 6, 2
    e, s0, win0, G, cs, cw = problem(cfg, T, t0)
    res = bptt.chunk_grads(cfg, w, e, s0, win0, t0, T, G, None, cw)
    assert not np.any(res["gate.w"]) and not np.any(res["gate.b"]) and not np.any(res["s0"])
    res0 = bptt.chunk_grads(cfg, w, e, s0, np.zeros_like(win0), 0, T, problem(cfg, T, 0)[3])
    assert not np.any(res0["sstar"])
    # the rest of the model still learns
    assert np.any(res["dec.0.wqkv"]) and np.any(res["mem.0.wk"])


def test_cache_paths_stay_open_when_only_s_is_detached():
    T, t0 = 3, 0
    for W, open_ in ((1, False), (2, True), (3, True)):
        cfg = tiny(window=W)
        w = weights(cfg)
        e, s0, win0, G, _, _ = problem(cfg, T, t0)
        G[:-1] = 0.0  # loss on the last output only
        full = bptt.chunk_grads(cfg, w, e, s0, np.zeros_like(win0), t0, T, G)
        cut = bptt.chunk_grads_s_detached(cfg, w, e, w["sstar"], np.zeros_like(win0), t0, T, G)
        assert np.linalg.norm(full["s0"]) > 0
        if open_:
            # s_0 still reaches the loss through the retained keys and values
            assert np.linalg.norm(cut["s0"]) > 1e-6 * np.linalg.norm(full["s0"])
            assert not np.allclose(cut["s0"], full["s0"])
        else:
            assert not np.any(cut["s0"])
