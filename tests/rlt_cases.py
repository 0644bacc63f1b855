"""Shared set-up for the GPU parity tests: small models with the shapes of the
five workloads, seeded inputs, and a prefilled device model."""
import numpy as np

from token_recurrent_decoding_b200 import configs, inputs

# Reduced shapes that keep each workload's structure (dtype, head size, G,
# tying, FFN form) but let the fp64 oracle finish in seconds.
SMALL = {
    "tiny_fp32": configs.TINY,
    "m50_like": configs.M50.replace(d=128, n_heads=2, n_enc=2, n_dec=2, ffn_dim=256,
                                    vocab=512, window=8),
    "m140_like": configs.M140.replace(d=128, n_heads=2, n_enc=2, n_dec=2, ffn_dim=256,
                                      vocab=512, window=16, mem_groups=2),
    "tied_like": configs.TIED.replace(d=256, n_heads=2, head_dim=128, n_enc=2, n_dec=2,
                                      ffn_dim=512, vocab=512, window=16),
    "ragged_like": configs.RAGGED_MODEL.replace(d=128, n_heads=2, n_enc=1, n_dec=2,
                                                ffn_dim=256, vocab=512, window=16),
    # FFN width 1536: the down projection (K = 1536) runs split-K
    "splitk_like": configs.M50.replace(d=128, n_heads=2, n_enc=1, n_dec=2, ffn_dim=1536,
                                       vocab=512, window=8),
}

# Parity tolerances: step-wise max|err| / RMS(s), trajectory rel-L2 of s.
STEP_TOL = {configs.F32: 1e-5, configs.BF16: 2e-2}
TRAJ_TOL = {configs.F32: 1e-4, configs.BF16: 5e-2}
# newest K/V entries written by one step (bf16: one storage rounding on top)
CACHE_TOL = {configs.F32: 1e-5, configs.BF16: 5e-2}


def rms(x):
    return float(np.sqrt(np.mean(np.square(x, dtype=np.float64))))


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def make_model(cfg, lengths, seed=0, perturb=True, max_seqs=None, max_len=None, prefill=True,
               **kw):
    import torch
    from token_recurrent_decoding_b200.rlt import Model
    w = inputs.make_weights(cfg, seed, perturb)
    tok = inputs.make_tokens(cfg.vocab, lengths)
    m = Model(cfg, w, max_seqs or len(lengths), max_len or max(lengths), **kw)
    if prefill:
        prefill_all(m, tok, lengths)
    return m, w, tok


def prefill_all(m, tok, lengths, ids=None):
    import torch
    lengths = list(lengths)
    flat = np.concatenate([tok[i, :L] for i, L in enumerate(lengths)]).astype(np.int32)
    offsets = np.concatenate([[0], np.cumsum(lengths)[:-1]]).astype(np.int32)
    ids = list(range(len(lengths))) if ids is None else ids
    m.prefill_encoder(torch.from_numpy(flat).cuda(), ids, offsets, lengths)


def to_np(t):
    import torch
    return t.detach().to(torch.float64).cpu().numpy()
