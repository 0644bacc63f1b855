"""rlt_attend_noalloc, the decode attention for callers that cannot allocate
device memory (for example a serving process whose memory pool already holds
the GPU, or a plugin handed only its input and output buffers). Its scratch is
an array compiled into the library. Through the C ABI this checks that two
calls in a row, both long enough to split every row into several 1024-row
chunks (so the second call runs after merge counters and partials the first
one used), give the output of rlt_attend with a caller workspace and of a
plain fp64 softmax attention on the CPU, and that a shape whose scratch does
not fit the array is refused before anything runs.

Collected last on purpose (file name), so a stop-at-first-failure run has run
every other test first; it also passes alone in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

from token_recurrent_decoding_b200 import rlt

pytestmark = pytest.mark.gpu

NOALLOC_BYTES = 8 << 20  # RLT_ATTEND_NOALLOC_BYTES in include/rlt.h


def _noalloc(q, kv, lengths, out):
    lib = rlt._lib()
    fn = lib.rlt_attend_noalloc
    fn.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 5 + [ctypes.c_void_p] * 2
    n, H, _, cap, dh = kv.shape
    lens = (ctypes.c_int32 * n)(*lengths)
    dtype = 1 if kv.dtype == torch.bfloat16 else 0
    stream = torch.cuda.current_stream().cuda_stream
    return fn(q.data_ptr(), kv.data_ptr(), ctypes.cast(lens, ctypes.c_void_p), n, H, dh, cap,
              dtype, out.data_ptr(), stream)


def _inputs(n, H, dh, cap, dtype, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    q = torch.randn((n, H, dh), generator=g)
    kv = torch.randn((n, H, 2, cap, dh), generator=g).to(dtype)
    return q, kv


def _softmax_attention_fp64(q, kv, lengths):
    """softmax(q . K^T / sqrt(dh)) V over the first lengths[i] rows, fp64 CPU."""
    n, H, _, _, dh = kv.shape
    qd, kvd = q.double(), kv.double()
    out = torch.empty((n, H, dh), dtype=torch.float64)
    for i, L in enumerate(lengths):
        K, V = kvd[i, :, 0, :L], kvd[i, :, 1, :L]
        p = torch.softmax(torch.einsum("hd,hld->hl", qd[i], K) / np.sqrt(dh), dim=-1)
        out[i] = torch.einsum("hl,hld->hd", p, V)
    return out


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_two_calls_match_the_workspace_entry_point(dtype):
    # two different multi-chunk shapes in a row: the second call must not see
    # stale scratch (merge counters, partials, positions) from the first
    cases = [(9, 2, 128 if dtype == torch.bfloat16 else 64, 2100,
              [2100, 1, 2099, 1025, 40, 1024, 2048, 600, 2049], 12),
             (13, 3, 64, 3000, [1, 3000, 1025, 2047, 2048, 3, 1500, 2999, 64, 1026, 700, 2,
                                2500], 11)]
    for n, H, dh, cap, lengths, seed in cases:
        assert rlt.attend_workspace_bytes(n, H, dh, cap) <= NOALLOC_BYTES
        q, kv = _inputs(n, H, dh, cap, dtype, seed)
        qd, kvd = q.cuda(), kv.cuda()
        ref = torch.empty((n, H, dh), dtype=dtype, device="cuda")
        ws = torch.empty(rlt.attend_workspace_bytes(n, H, dh, cap), dtype=torch.uint8,
                         device="cuda")
        rlt.attend(qd, kvd, lengths, ref, ws)
        got = torch.full((n, H, dh), float("nan"), dtype=dtype, device="cuda")
        assert _noalloc(qd, kvd, lengths, got) == 0
        torch.cuda.synchronize()
        assert torch.isfinite(got.float()).all()
        # bf16 output: one storage rounding (2^-9 relative); fp32: accumulation only
        tol = 1e-2 if dtype == torch.bfloat16 else 1e-5
        exact = _softmax_attention_fp64(q, kv, lengths)
        scale = exact.abs().max().item()
        assert (got.cpu().double() - exact).abs().max().item() <= tol * scale
        assert (got.float() - ref.float()).abs().max().item() <= tol * scale


def test_sizes_beyond_the_array_are_refused():
    # the smallest row count whose scratch exceeds the array, one head of 16,
    # rows of 1025 positions (two chunks); every buffer is sized for the shape
    H, dh, cap = 1, 16, 1025
    lo, hi = 1, 1 << 20
    while lo < hi:
        mid = (lo + hi) // 2
        if rlt.attend_workspace_bytes(mid, H, dh, cap) > NOALLOC_BYTES:
            hi = mid
        else:
            lo = mid + 1
    n = lo
    assert rlt.attend_workspace_bytes(n, H, dh, cap) > NOALLOC_BYTES
    assert rlt.attend_workspace_bytes(n - 1, H, dh, cap) <= NOALLOC_BYTES
    q = torch.zeros((n, H, dh), device="cuda")
    kv = torch.empty((n, H, 2, cap, dh), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((n, H, dh), dtype=torch.bfloat16, device="cuda")
    assert _noalloc(q, kv, [cap] * n, out) == 4  # RLT_ERR_CAPACITY
    del kv
    torch.cuda.empty_cache()
