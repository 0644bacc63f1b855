"""Gradient oracle of the RLT recurrent decoder -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this module; the CUDA package never does.

What it computes: the gradient, by full backpropagation through time, of a
loss that is linear in the decoder outputs of one chunk of positions,

    L = sum_{t0 <= t < t1} <G_t, s_t>  +  <C_s, s_{t1-1}>  +  <C_win, win_{t1}>,

with respect to every decoder parameter, the memory projection, the encoder
outputs e_j, and the chunk's starting state H_{t0-1} = (s_{t0-1}, win_{t0}).
G_t is the upstream gradient dL/ds_t (e.g. from a next-token head and its
cross-entropy); C_s and C_win are the gradient of the state carried out of the
chunk, so chunks run backwards in order compose into the full-sequence
gradient exactly (truncation would have to name each detached tensor:
[RLT-96] "RLT Runs 96 Blocks Per Token With Recurrent State, No Resets"
(aimastery.page), "Training and serving implications" -- the state-to-state
Jacobian has cross-terms through the decoder's key/value cache, so detaching
s alone leaves paths open through it). The decoder is trained by full
backpropagation through time over the whole sequence ([RLT-PV] "Per-token
recurrence, no quality gain" (news.promtvault.app), body: a custom
reverse-traversal backward).

How: the forward transition restated with plain PyTorch CPU ops in float64
(same readings as the C oracle: gated merge, pre-RMSNorm, RoPE on the SWA's q
and k at the absolute position, the window of W positions including the
current one, cross-attention over memory rows 0..t, GELU-erf or SwiGLU FFN,
s_t = RMSNorm_f of the last residual), and reverse-mode differentiation of it
by torch.autograd (a library primitive). The memory rows are projected from
e inside the function (K^g_j = W_mk^g e_j, V^g_j = W_mv^g e_j) so the
gradient reaches e and the projection weights.

Pinned by ``tests/test_oracle_bptt.py``: the forward equals the C oracle's
step for step; every gradient equals central finite differences of the C
oracle's forward (float64); chunks composed through the carried gradient equal
one full pass; alpha = 0 gives exactly zero gradient to the gate and to s; a
window of one position with s detached cuts every path between steps, while
W >= 2 leaves the cache paths open.
"""
from __future__ import annotations

import math

import numpy as np
import torch

_PER_DEC = ("ln1", "wqkv", "wo", "ln2", "wqx", "wox", "ln3", "w1", "wb", "w2")


def param_names(cfg):
    """Names (the weight generator's) of the parameters the gradient covers."""
    swiglu = cfg.ffn_kind == 1
    names = ["gate.w", "gate.b", "sstar", "dec.lnf"]
    for l in range(cfg.n_dec):
        for k in _PER_DEC:
            if k == "w1" and swiglu:
                k = "wa"
            if k == "wb" and not swiglu:
                continue
            names.append(f"dec.{l}.{k}")
    for g in range(cfg.mem_groups):
        names += [f"mem.{g}.wk", f"mem.{g}.wv"]
    return names


def _rmsnorm(x, gamma, eps):
    return x / torch.sqrt(torch.mean(x * x) + eps) * gamma


def _rope(v, pos, dh, theta):
    half = dh // 2
    i = torch.arange(half, dtype=torch.float64)
    ang = pos * theta ** (-2.0 * i / dh)
    c, s = torch.cos(ang), torch.sin(ang)
    a, b = v[..., :half], v[..., half:]
    return torch.cat([a * c - b * s, b * c + a * s], dim=-1)


def _attend(q, K, V):
    """q [H][dh], K, V [n][H][dh] -> [H][dh]."""
    dh = q.shape[-1]
    sc = torch.einsum("hd,nhd->hn", q, K) / math.sqrt(dh)
    p = torch.softmax(sc, dim=-1)
    return torch.einsum("hn,nhd->hd", p, V)


def chunk_forward(cfg, P, e, s0, win0, t0, t1):
    """Steps t0..t1-1 of one sequence from the state (s0, win0).

    P: parameter name -> float64 tensor; e [>= t1][d]; s0 [d];
    win0 [L_D][2][W-1][d] (post-RoPE K and V of positions t0-W+1 .. t0-1,
    oldest first; entries of positions < 0 are never read).
    Returns (s_out [t1-t0][d], s_last, win_last).
    """
    d, H, dh, Ld, W = cfg.d, cfg.n_heads, cfg.head_dim, cfg.n_dec, cfg.window
    eps, theta, alpha = cfg.rms_eps, cfg.rope_theta, cfg.alpha
    swiglu = cfg.ffn_kind == 1
    mem = []
    for g in range(cfg.mem_groups):
        mem.append((e[:t1] @ P[f"mem.{g}.wk"].T, e[:t1] @ P[f"mem.{g}.wv"].T))
    # window as per-layer lists of (position, k, v), oldest first
    win = []
    for l in range(Ld):
        ent = []
        for i in range(W - 1):
            pos = t0 - (W - 1) + i
            ent.append((pos, win0[l, 0, i], win0[l, 1, i]))
        win.append(ent)
    s = s0
    outs = []
    for t in range(t0, t1):
        e_t = e[t]
        g = torch.sigmoid(P["gate.w"] @ torch.cat([e_t, s]) + P["gate.b"])
        h = e_t + alpha * g * s
        for l in range(Ld):
            pre = f"dec.{l}."
            u = _rmsnorm(h, P[pre + "ln1"], eps)
            qkv = P[pre + "wqkv"] @ u
            q = _rope(qkv[:d].reshape(H, dh), t, dh, theta)
            k = _rope(qkv[d:2 * d].reshape(H, dh), t, dh, theta)
            v = qkv[2 * d:].reshape(H, dh)
            keys = [(kk, vv) for (pos, kk, vv) in win[l] if pos >= 0 and pos > t - W]
            K = torch.stack([kk.reshape(H, dh) for kk, _ in keys] + [k])
            V = torch.stack([vv.reshape(H, dh) for _, vv in keys] + [v])
            a = _attend(q, K, V).reshape(d)
            h = h + P[pre + "wo"] @ a
            if W > 1:
                win[l] = win[l][1:] + [(t, k.reshape(d), v.reshape(d))]
            u = _rmsnorm(h, P[pre + "ln2"], eps)
            qx = (P[pre + "wqx"] @ u).reshape(H, dh)
            mk, mv = mem[0 if cfg.mem_groups == 1 else l]
            a = _attend(qx, mk[:t + 1].reshape(t + 1, H, dh),
                        mv[:t + 1].reshape(t + 1, H, dh)).reshape(d)
            h = h + P[pre + "wox"] @ a
            u = _rmsnorm(h, P[pre + "ln3"], eps)
            if swiglu:
                f = torch.nn.functional.silu(P[pre + "wa"] @ u) * (P[pre + "wb"] @ u)
            else:
                z = P[pre + "w1"] @ u
                f = 0.5 * z * (1.0 + torch.erf(z / math.sqrt(2.0)))
            h = h + P[pre + "w2"] @ f
        s = _rmsnorm(h, P["dec.lnf"], eps)
        outs.append(s)
    win_last = torch.zeros((Ld, 2, max(W - 1, 0), d), dtype=torch.float64)
    if W > 1:
        win_last = torch.stack([
            torch.stack([torch.stack([kk for (_, kk, _) in win[l]]),
                         torch.stack([vv for (_, _, vv) in win[l]])]) for l in range(Ld)])
    return torch.stack(outs) if outs else torch.zeros((0, d), dtype=torch.float64), s, win_last


def chunk_grads(cfg, weights, e, s0, win0, t0, t1, G, carry_s=None, carry_win=None):
    """Gradient of L (module docstring) over the chunk t0..t1-1 of one sequence.

    weights: name -> array (the generator's dict; bf16 models pass the bf16
    values); e [>= t1][d]; s0 [d]; win0 [L_D][2][W-1][d]; G [t1-t0][d];
    carry_s [d] and carry_win [L_D][2][W-1][d] optional.
    Returns a dict: each name of ``param_names`` -> gradient (numpy float64),
    "e" [t1][d], "s0" [d], "win0" [L_D][2][W-1][d], plus "loss".
    The entry "sstar" is the gradient through the parameter s*, which the chunk
    reads only when t0 = 0 (then s0 is s* and "s0" equals it).
    """
    names = param_names(cfg)
    P = {}
    for n in names:
        P[n] = torch.tensor(np.asarray(weights[n], np.float64), requires_grad=True)
    e_t = torch.tensor(np.asarray(e, np.float64)[:t1], requires_grad=True)
    s0_t = torch.tensor(np.asarray(s0, np.float64), requires_grad=True)
    if t0 == 0:
        s0_t = P["sstar"]
    w0 = torch.tensor(np.asarray(win0, np.float64).reshape(cfg.n_dec, 2, max(cfg.window - 1, 0),
                                                           cfg.d), requires_grad=True)
    out, s_last, win_last = chunk_forward(cfg, P, e_t, s0_t, w0, t0, t1)
    L = torch.sum(out * torch.tensor(np.asarray(G, np.float64).reshape(out.shape)))
    if carry_s is not None:
        L = L + torch.sum(s_last * torch.tensor(np.asarray(carry_s, np.float64)))
    if carry_win is not None and cfg.window > 1:
        cw = torch.tensor(np.asarray(carry_win, np.float64).reshape(win_last.shape))
        # retained entries of positions < 0 are constants outside the model
        pos = t1 - (cfg.window - 1) + np.arange(cfg.window - 1)
        mask = torch.tensor((pos >= 0).astype(np.float64)).reshape(1, 1, -1, 1)
        L = L + torch.sum(win_last * cw * mask)
    leaves = [P[n] for n in names] + [e_t, w0] + ([] if t0 == 0 else [s0_t])
    grads = torch.autograd.grad(L, leaves, allow_unused=True)
    res = {}
    for n, gr in zip(names, grads[:len(names)]):
        res[n] = np.zeros(P[n].shape) if gr is None else gr.detach().numpy()
    res["e"] = np.zeros(e_t.shape) if grads[len(names)] is None else grads[len(names)].numpy()
    gw = grads[len(names) + 1]
    res["win0"] = np.zeros(w0.shape) if gw is None else gw.numpy()
    if t0 == 0:
        res["s0"] = res["sstar"].copy()
    else:
        gs = grads[len(names) + 2]
        res["s0"] = np.zeros(cfg.d) if gs is None else gs.numpy()
    res["loss"] = float(L.detach())
    return res


def chunk_grads_s_detached(cfg, weights, e, s0, win0, t0, t1, G):
    """The same loss with s_{t-1} detached at every step's input (for t > t0):
    the truncation that keeps the cache paths ([RLT-96] "Training and serving
    implications"). Returns the gradient of s0 and of every parameter."""
    names = param_names(cfg)
    P = {n: torch.tensor(np.asarray(weights[n], np.float64), requires_grad=True) for n in names}
    e_t = torch.tensor(np.asarray(e, np.float64)[:t1])
    s0_t = torch.tensor(np.asarray(s0, np.float64), requires_grad=True)
    w0 = torch.tensor(np.asarray(win0, np.float64).reshape(cfg.n_dec, 2, max(cfg.window - 1, 0),
                                                           cfg.d))
    # run step by step, detaching s between steps but carrying the window
    s = s0_t
    win = w0
    L = torch.zeros((), dtype=torch.float64)
    for t in range(t0, t1):
        out, s_new, win = chunk_forward(cfg, P, e_t, s if t == t0 else s.detach(), win, t, t + 1)
        L = L + torch.sum(out[0] * torch.tensor(np.asarray(G, np.float64)[t - t0]))
        s = s_new
    grads = torch.autograd.grad(L, [s0_t] + [P[n] for n in names], allow_unused=True)
    res = {"s0": np.zeros(cfg.d) if grads[0] is None else grads[0].numpy()}
    for n, gr in zip(names, grads[1:]):
        res[n] = np.zeros(P[n].shape) if gr is None else gr.numpy()
    return res
