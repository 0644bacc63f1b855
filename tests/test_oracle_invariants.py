"""Pins of the whole oracle: closed forms, brute force and the invariants the
pages fix for the RLT recurrence. No GPU.

Closed forms (zeroed blocks reduce a sublayer to a routine with a plain
answer) pin the gated merge, the norm placement, the start state, the SWA
window range and the inclusive memory prefix. Brute force (full history with
an explicit mask) pins the retained-window bookkeeping. The invariants are
those the pages state: feedback off removes the dependence on s_{t-1}
("Per-token recurrence, no quality gain", body), the encoder is causal and the
memory prefix-restricted ("RLT Runs 96 Blocks ...", "Architecture"), the state
H_t carries everything (Proposition 3.1 in "Three design principles"), and a
standard parallel SWA decoder pass is not the recurrence (same section).
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from token_recurrent_decoding_b200 import configs, inputs

BASE = configs.TINY.replace(window=5)
T = 40


def _rms(x, g, eps):
    return x / np.sqrt(np.mean(x * x) + eps) * g


def _sig(x):
    return 1.0 / (1.0 + np.exp(-x))


def _weights(cfg, perturb=True, seed=0):
    return {k: v.astype(np.float64) for k, v in inputs.make_weights(cfg, seed, perturb).items()}


def _tokens(cfg, n=1, length=T, seed=1):
    return inputs.make_tokens(cfg.vocab, [length] * n, seed)


def _zero(w, names):
    for n in names:
        w[n] = np.zeros_like(w[n])


def _enc_block_names(cfg):
    out = []
    for l in range(cfg.n_enc):
        out += [f"enc.{l}.wqkv", f"enc.{l}.wo", f"enc.{l}.w1", f"enc.{l}.w2"]
    return out


# ------------------------------------------------------------ closed forms
@pytest.mark.parametrize("alpha", [1.0, 0.37])
def test_closed_form_merge_and_norms(alpha):
    """All block matrices zero: e_t = RMSNorm_E(E[tok_t]) and
    s_t = RMSNorm_f(e_t + alpha * sigmoid(W_g[e;s] + b) * s_{t-1}), s_{-1} = s*."""
    cfg = BASE.replace(alpha=alpha)
    w = _weights(cfg)
    blocks = _enc_block_names(cfg)
    for l in range(cfg.n_dec):
        blocks += [f"dec.{l}.wqkv", f"dec.{l}.wo", f"dec.{l}.wqx", f"dec.{l}.wox",
                   f"dec.{l}.w1", f"dec.{l}.w2"]
    _zero(w, blocks)
    tok = _tokens(cfg)[0]
    got, _, _ = oracle.Oracle(cfg, w).run(tok)
    s = w["sstar"]
    for t in range(T):
        e = _rms(w["embed"][tok[t]], w["enc.lnf"], cfg.rms_eps)
        g = _sig(w["gate.w"] @ np.concatenate([e, s]) + w["gate.b"])
        s = _rms(e + alpha * g * s, w["dec.lnf"], cfg.rms_eps)
        np.testing.assert_allclose(got[t], s, rtol=1e-12, atol=1e-12)


def test_closed_form_uniform_cross_attention_prefix_is_inclusive():
    """Zero cross-attention query: the sublayer adds W_ox mean_{j<=t} V_j."""
    cfg = BASE.replace(n_dec=1)
    w = _weights(cfg)
    _zero(w, _enc_block_names(cfg) + ["dec.0.wqkv", "dec.0.wo", "dec.0.wqx",
                                      "dec.0.w1", "dec.0.w2"])
    tok = _tokens(cfg)[0]
    got, _, _ = oracle.Oracle(cfg, w).run(tok)
    e = np.stack([_rms(w["embed"][k], w["enc.lnf"], cfg.rms_eps) for k in tok])
    V = e @ w["mem.0.wv"].T
    s = w["sstar"]
    for t in range(T):
        g = _sig(w["gate.w"] @ np.concatenate([e[t], s]) + w["gate.b"])
        x = e[t] + g * s
        h = x + w["dec.0.wox"] @ V[: t + 1].mean(0)
        s = _rms(h, w["dec.lnf"], cfg.rms_eps)
        np.testing.assert_allclose(got[t], s, rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("W", [1, 2, 5])
def test_closed_form_uniform_swa_window(W):
    """Zero SWA query rows: the sublayer adds W_o mean of v over positions
    max(0, t-W+1)..t (the window includes the current token); v carries no
    rotary encoding."""
    cfg = BASE.replace(n_dec=1, window=W)
    w = _weights(cfg)
    d = cfg.d
    w["dec.0.wqkv"] = w["dec.0.wqkv"].copy()
    w["dec.0.wqkv"][:d] = 0.0
    _zero(w, _enc_block_names(cfg) + ["dec.0.wqx", "dec.0.wox", "dec.0.w1", "dec.0.w2"])
    tok = _tokens(cfg)[0]
    got, _, _ = oracle.Oracle(cfg, w).run(tok)
    Wv = w["dec.0.wqkv"][2 * d:]
    s = w["sstar"]
    vs = []
    for t in range(T):
        e = _rms(w["embed"][tok[t]], w["enc.lnf"], cfg.rms_eps)
        g = _sig(w["gate.w"] @ np.concatenate([e, s]) + w["gate.b"])
        x = e + g * s
        vs.append(Wv @ _rms(x, w["dec.0.ln1"], cfg.rms_eps))
        h = x + w["dec.0.wo"] @ np.mean(vs[max(0, t - W + 1):], axis=0)
        s = _rms(h, w["dec.lnf"], cfg.rms_eps)
        np.testing.assert_allclose(got[t], s, rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("kind", [configs.GELU, configs.SWIGLU])
def test_closed_form_ffn(kind):
    """Attention outputs zeroed: each position adds W_2 act(W_1 RMSNorm_3(x))."""
    cfg = BASE.replace(n_dec=1, ffn_kind=kind)
    w = _weights(cfg)
    _zero(w, [n for n in w if n.startswith("enc.") and n.split(".")[-1]
              in ("wqkv", "wo", "w1", "wa", "wb", "w2")] + ["dec.0.wo", "dec.0.wox"])
    tok = _tokens(cfg)[0]
    got, _, _ = oracle.Oracle(cfg, w).run(tok)
    s = w["sstar"]
    for t in range(T):
        e = _rms(w["embed"][tok[t]], w["enc.lnf"], cfg.rms_eps)
        g = _sig(w["gate.w"] @ np.concatenate([e, s]) + w["gate.b"])
        x = e + g * s
        u = torch.tensor(_rms(x, w["dec.0.ln3"], cfg.rms_eps))
        if kind == configs.GELU:
            f = F.gelu(torch.tensor(w["dec.0.w1"]) @ u)
        else:
            f = F.silu(torch.tensor(w["dec.0.wa"]) @ u) * (torch.tensor(w["dec.0.wb"]) @ u)
        h = x + (torch.tensor(w["dec.0.w2"]) @ f).numpy()
        s = _rms(h, w["dec.lnf"], cfg.rms_eps)
        np.testing.assert_allclose(got[t], s, rtol=1e-11, atol=1e-11)


# ------------------------------------------------------------ brute force
@pytest.mark.parametrize("W", [1, 2, 3, 8])
def test_window_matches_bruteforce_masked_history(W):
    cfg = BASE.replace(window=W)
    o = oracle.Oracle(cfg, _weights(cfg))
    tok = _tokens(cfg)[0]
    got, _, _ = o.run(tok)
    e, mem = o.encode(tok)
    ref = o.decode_bruteforce(e, mem, T)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-13)


def test_short_sequence_equals_full_causal_attention():
    """T <= W: the window never drops an entry."""
    short = 12
    a = oracle.Oracle(BASE.replace(window=short), _weights(BASE))
    b = oracle.Oracle(BASE.replace(window=short + 9), _weights(BASE))
    tok = _tokens(BASE, length=short)[0]
    np.testing.assert_array_equal(a.run(tok)[0], b.run(tok)[0])
    e, mem = a.encode(tok)
    np.testing.assert_array_equal(a.run(tok)[0], b.decode_bruteforce(e, mem, short))


def test_window_one_keeps_only_current_token():
    """W = 1: SWA output is v_t whatever the queries and the history."""
    cfg = BASE.replace(window=1)
    w = _weights(cfg)
    w2 = dict(w)
    for l in range(cfg.n_dec):
        q = w[f"dec.{l}.wqkv"].copy()
        q[: cfg.d] = np.random.default_rng(l).standard_normal((cfg.d, cfg.d))
        w2[f"dec.{l}.wqkv"] = q
    tok = _tokens(cfg)[0]
    a = oracle.Oracle(cfg, w).run(tok)[0]
    b = oracle.Oracle(cfg, w2).run(tok)[0]
    np.testing.assert_array_equal(a, b)
    cfg2 = BASE.replace(window=2)
    c = oracle.Oracle(cfg2, w).run(tok)[0]
    d = oracle.Oracle(cfg2, w2).run(tok)[0]
    assert np.abs(c - d).max() > 1e-4


# ------------------------------------------------------------ invariants
def test_alpha_zero_removes_dependence_on_previous_output():
    cfg = BASE.replace(alpha=0.0)
    o = oracle.Oracle(cfg, _weights(cfg))
    tok = _tokens(cfg)[0]
    e, mem = o.encode(tok)
    s0, win0 = o.init_state()
    a, _, _ = o.decode(e, mem, 0, T, s0, win0)
    s_rand = np.random.default_rng(5).standard_normal(cfg.d) * 3
    b, _, _ = o.decode(e, mem, 0, T, s_rand, win0)
    np.testing.assert_array_equal(a, b)
    o1 = oracle.Oracle(BASE, _weights(BASE))
    a1, _, _ = o1.decode(e, mem, 0, T, s0, win0)
    b1, _, _ = o1.decode(e, mem, 0, T, s_rand, win0)
    assert np.abs(a1 - b1).max() > 1e-3


def test_alpha_zero_equals_parallel_pass_and_alpha_one_does_not():
    for alpha, equal in ((0.0, True), (1.0, False)):
        cfg = BASE.replace(alpha=alpha)
        o = oracle.Oracle(cfg, _weights(cfg))
        tok = _tokens(cfg)[0]
        rec, _, _ = o.run(tok)
        e, mem = o.encode(tok)
        par = o.decode_parallel_nofeedback(e, mem, T)
        if equal:
            np.testing.assert_allclose(rec, par, rtol=0, atol=1e-13)
        else:
            assert np.abs(rec - par).max() > 1e-2


def test_causality_future_tokens_do_not_change_the_past():
    o = oracle.Oracle(BASE, _weights(BASE))
    tok = _tokens(BASE)[0]
    tok2 = tok.copy()
    k = 23
    tok2[k + 1:] = (tok2[k + 1:] + 17) % BASE.vocab
    e1, m1 = o.encode(tok)
    e2, m2 = o.encode(tok2)
    np.testing.assert_array_equal(e1[: k + 1], e2[: k + 1])
    np.testing.assert_array_equal(m1[:, : k + 1], m2[:, : k + 1])
    s1 = o.run(tok)[0]
    s2 = o.run(tok2)[0]
    np.testing.assert_array_equal(s1[: k + 1], s2[: k + 1])
    assert np.abs(s1[k + 1:] - s2[k + 1:]).max() > 1e-3


@pytest.mark.parametrize("k", [1, 4, 5, 17])
def test_split_invariance_carried_state(k):
    """Proposition 3.1: moving the segment split changes nothing for a fixed
    history when H_t = (s_t, C_t) is carried across it."""
    o = oracle.Oracle(BASE, _weights(BASE))
    tok = _tokens(BASE)[0]
    e, mem = o.encode(tok)
    s0, w0 = o.init_state()
    whole, _, _ = o.decode(e, mem, 0, T, s0, w0)
    a, s_k, w_k = o.decode(e, mem, 0, k, s0, w0)
    # carry the state through plain arrays (a snapshot), then resume
    snap = (s_k.copy(), w_k.copy())
    b, _, _ = o.decode(e, mem, k, T, *snap)
    np.testing.assert_array_equal(whole, np.concatenate([a, b]))


def test_memory_groups_shared_equals_identical_per_layer():
    cfg1 = BASE.replace(mem_groups=1)
    cfgL = BASE.replace(mem_groups=BASE.n_dec)
    w1 = _weights(cfg1)
    wL = dict(w1)
    for g in range(cfgL.n_dec):
        wL[f"mem.{g}.wk"] = w1["mem.0.wk"]
        wL[f"mem.{g}.wv"] = w1["mem.0.wv"]
    tok = _tokens(BASE)[0]
    a = oracle.Oracle(cfg1, w1).run(tok)[0]
    b = oracle.Oracle(cfgL, wL).run(tok)[0]
    np.testing.assert_array_equal(a, b)
    wL2 = dict(wL)
    wL2["mem.1.wv"] = np.random.default_rng(9).standard_normal(w1["mem.0.wv"].shape) * 0.02
    c = oracle.Oracle(cfgL, wL2).run(tok)[0]
    assert np.abs(a - c).max() > 1e-4


@pytest.mark.parametrize("kind", [configs.GELU, configs.SWIGLU])
def test_tied_equals_untied_copy(kind):
    tied = BASE.replace(tied=True, ffn_kind=kind)
    untied = tied.replace(tied=False)
    wt = _weights(tied)
    wu = {k: v.copy() for k, v in wt.items()}  # decoder entries become copies
    tok = _tokens(BASE)[0]
    a = oracle.Oracle(tied, wt).run(tok)[0]
    b = oracle.Oracle(untied, wu).run(tok)[0]
    np.testing.assert_array_equal(a, b)


def test_fp32_build_agrees_with_fp64():
    cfg = configs.TINY
    w = inputs.make_weights(cfg)
    tok = inputs.make_tokens(cfg.vocab, [64])[0]
    a = oracle.Oracle(cfg, w, "f64").run(tok)[0]
    b = oracle.Oracle(cfg, w, "f32").run(tok)[0]
    rel = np.linalg.norm(a - b) / np.linalg.norm(a)
    assert rel <= 1e-6, rel


def test_batch_runner_equals_single_runs_ragged():
    o = oracle.Oracle(BASE, _weights(BASE))
    lengths = [7, 40, 1, 23]
    tok = inputs.make_tokens(BASE.vocab, lengths)
    got, used = o.run_batch(tok, lengths, n_threads=2)
    assert used >= 1
    for b, L in enumerate(lengths):
        np.testing.assert_array_equal(got[b], o.run(tok[b, :L])[1])


# ------------------------------------------- reductions to library attention
def _rot(x, pos, theta=1e4):
    """Rotary encoding as complex multiplication (independent of the oracle)."""
    dh = x.shape[-1]
    half = dh // 2
    z = x[..., :half] + 1j * x[..., half:]
    ang = pos[:, None] * theta ** (-2.0 * np.arange(half) / dh)
    z = z * np.exp(1j * ang)
    return np.concatenate([z.real, z.imag], -1)


def _mha(cfg, u, wqkv, mask):
    """Multi-head attention through torch SDPA with rotary q, k at 0..T-1."""
    d, H, dh = cfg.d, cfg.n_heads, cfg.head_dim
    n = u.shape[0]
    qkv = u @ wqkv.T
    pos = np.arange(n, dtype=np.float64)
    outs = []
    for h in range(H):
        q = _rot(qkv[:, h * dh:(h + 1) * dh], pos)
        k = _rot(qkv[:, d + h * dh:d + (h + 1) * dh], pos)
        v = qkv[:, 2 * d + h * dh:2 * d + (h + 1) * dh]
        o = F.scaled_dot_product_attention(torch.tensor(q)[None], torch.tensor(k)[None],
                                           torch.tensor(v)[None],
                                           attn_mask=torch.tensor(mask)[None])
        outs.append(o[0].numpy())
    return np.concatenate(outs, -1)


def test_encoder_layer_is_causal_rotary_attention():
    """One encoder block with its FFN zeroed is causal multi-head attention
    with rotary q/k at absolute positions; memory rows are W_mk e, W_mv e."""
    cfg = BASE.replace(n_enc=1)
    w = _weights(cfg)
    _zero(w, ["enc.0.w1", "enc.0.w2"])
    tok = _tokens(cfg)[0]
    e, mem = oracle.Oracle(cfg, w).encode(tok)
    x = w["embed"][tok]
    u = np.stack([_rms(r, w["enc.0.ln1"], cfg.rms_eps) for r in x])
    causal = np.tril(np.ones((T, T), dtype=bool))
    h = x + _mha(cfg, u, w["enc.0.wqkv"], causal) @ w["enc.0.wo"].T
    ref = np.stack([_rms(r, w["enc.lnf"], cfg.rms_eps) for r in h])
    np.testing.assert_allclose(e, ref, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(mem[0, :T, 0], ref @ w["mem.0.wk"].T, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(mem[0, :T, 1], ref @ w["mem.0.wv"].T, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("W", [1, 3, 8])
def test_decoder_swa_is_band_masked_rotary_attention(W):
    """alpha = 0, one decoder block with cross-attention and FFN zeroed: the
    recurrence is band-masked (t-W < j <= t) rotary attention over x_j = e_j."""
    cfg = BASE.replace(n_dec=1, window=W, alpha=0.0)
    w = _weights(cfg)
    _zero(w, ["dec.0.wox", "dec.0.w1", "dec.0.w2"])
    o = oracle.Oracle(cfg, w)
    tok = _tokens(cfg)[0]
    got, _, _ = o.run(tok)
    e, _ = o.encode(tok)
    u = np.stack([_rms(r, w["dec.0.ln1"], cfg.rms_eps) for r in e])
    i, j = np.arange(T)[:, None], np.arange(T)[None, :]
    band = (j <= i) & (j > i - W)
    h = e + _mha(cfg, u, w["dec.0.wqkv"], band) @ w["dec.0.wo"].T
    ref = np.stack([_rms(r, w["dec.lnf"], cfg.rms_eps) for r in h])
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-11)


# ---------------------------------------------- encoder FFN and layer stacking
def _enc_rows(cfg, w, x, l):
    """One encoder block with its attention output zeroed, through torch:
    x + W2 act(W1 RMSNorm_2(x)) per position (GELU or SwiGLU)."""
    u = torch.tensor(np.stack([_rms(r, w[f"enc.{l}.ln2"], cfg.rms_eps) for r in x]))
    if cfg.ffn_kind == configs.GELU:
        f = F.gelu(u @ torch.tensor(w[f"enc.{l}.w1"]).T)
    else:
        f = F.silu(u @ torch.tensor(w[f"enc.{l}.wa"]).T) * (u @ torch.tensor(w[f"enc.{l}.wb"]).T)
    return x + (f @ torch.tensor(w[f"enc.{l}.w2"]).T).numpy()


@pytest.mark.parametrize("kind", [configs.GELU, configs.SWIGLU])
def test_encoder_ffn_sublayer_closed_form(kind):
    """One encoder block whose attention writes nothing (W_o = 0): e_t =
    RMSNorm_E(x + W2 act(W1 RMSNorm_2(x))), x = E[tok_t]; memory rows are
    W_mk e, W_mv e."""
    cfg = BASE.replace(n_enc=1, ffn_kind=kind)
    w = _weights(cfg)
    _zero(w, ["enc.0.wo"])
    tok = _tokens(cfg)[0]
    e, mem = oracle.Oracle(cfg, w).encode(tok)
    h = _enc_rows(cfg, w, w["embed"][tok], 0)
    ref = np.stack([_rms(r, w["enc.lnf"], cfg.rms_eps) for r in h])
    np.testing.assert_allclose(e, ref, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(mem[0, :T, 1], ref @ w["mem.0.wv"].T, rtol=1e-11, atol=1e-12)


def _one_block_copy(w, src_layer, n_enc_names=True, prefix="enc"):
    """Weights of a one-block model whose block 0 is block `src_layer`."""
    out = {k: v for k, v in w.items() if not k.startswith(prefix + ".")
           or k == prefix + ".lnf"}
    for k, v in w.items():
        parts = k.split(".")
        if parts[0] == prefix and parts[1].isdigit() and int(parts[1]) == src_layer:
            out[f"{prefix}.0.{'.'.join(parts[2:])}"] = v
    return out


@pytest.mark.parametrize("zeroed,kept", [(1, 0), (0, 1)])
def test_encoder_blocks_stack_in_order(zeroed, kept):
    """A two-block encoder with one block's output matrices zeroed (the block
    is the identity) equals the one-block encoder made of the other block:
    every block uses its own matrices and norms, in layer order."""
    cfg2 = BASE.replace(n_enc=2)
    w = _weights(cfg2)
    _zero(w, [f"enc.{zeroed}.wo", f"enc.{zeroed}.w2"])
    tok = _tokens(cfg2)[0]
    e2, m2 = oracle.Oracle(cfg2, w).encode(tok)
    cfg1 = BASE.replace(n_enc=1)
    e1, m1 = oracle.Oracle(cfg1, _one_block_copy(w, kept)).encode(tok)
    np.testing.assert_array_equal(e2, e1)
    np.testing.assert_array_equal(m2, m1)
    # and the kept block is not the identity
    e0, _ = oracle.Oracle(BASE.replace(n_enc=0), w).encode(tok)
    assert np.abs(e2 - e0).max() > 1e-3


@pytest.mark.parametrize("G", ["shared", "per_layer"])
@pytest.mark.parametrize("zeroed,kept", [(0, 1), (1, 0)])
def test_decoder_layers_stack_in_order(zeroed, kept, G):
    """A two-layer decoder whose layer `zeroed` writes nothing (W_o, W_ox, W_2
    zero: the layer is the identity on the residual stream) equals the
    one-layer decoder made of layer `kept` -- its q/k/v, W_o, W_qx, W_ox, FFN,
    its three norms and (G = L_D) its own memory group. Pins the layer index
    of every decoder sublayer, which the brute-force twin shares."""
    groups = 2 if G == "per_layer" else 1
    cfg2 = BASE.replace(n_dec=2, mem_groups=groups)
    w = _weights(cfg2)
    _zero(w, [f"dec.{zeroed}.wo", f"dec.{zeroed}.wox", f"dec.{zeroed}.w2"])
    tok = _tokens(cfg2)[0]
    got2, _, _ = oracle.Oracle(cfg2, w).run(tok)
    cfg1 = BASE.replace(n_dec=1, mem_groups=1)
    w1 = _one_block_copy(w, kept, prefix="dec")
    w1 = {k: v for k, v in w1.items() if not k.startswith("mem.")}
    g = kept if groups > 1 else 0
    w1["mem.0.wk"], w1["mem.0.wv"] = w[f"mem.{g}.wk"], w[f"mem.{g}.wv"]
    got1, _, _ = oracle.Oracle(cfg1, w1).run(tok)
    np.testing.assert_array_equal(got2, got1)
