"""rlt_attend_noalloc, the decode attention for callers that cannot allocate
device memory (for example a serving process whose memory pool already holds
the GPU, or a plugin handed only its input and output buffers). Its scratch is
an array compiled into the library; this checks, through the C ABI, that two
calls in a row give the output of rlt_attend with a caller workspace, and that
sizes beyond the array are refused.

Collected last on purpose (file name), so a stop-at-first-failure run has run
every other test first; it also passes alone in a fresh process."""
import ctypes

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
    q = torch.randn((n, H, dh), generator=g).cuda()
    kv = torch.randn((n, H, 2, cap, dh), generator=g).to(dtype).cuda()
    return q, kv


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_two_calls_match_the_workspace_entry_point(dtype):
    # two different shapes in a row: the second call must not see stale
    # scratch (merge counters, positions) from the first
    cases = [(13, 4, 64, 900, [1, 900, 255, 256, 257, 3, 512, 899, 64, 65, 700, 2, 511], 11),
             (9, 2, 128 if dtype == torch.bfloat16 else 64, 1300,
              [1300, 1, 1299, 513, 40, 1024, 7, 600, 300], 12)]
    for n, H, dh, cap, lengths, seed in cases:
        assert rlt.attend_workspace_bytes(n, H, dh, cap) <= NOALLOC_BYTES
        q, kv = _inputs(n, H, dh, cap, dtype, seed)
        ref = torch.empty((n, H, dh), dtype=dtype, device="cuda")
        ws = torch.empty(rlt.attend_workspace_bytes(n, H, dh, cap), dtype=torch.uint8,
                         device="cuda")
        rlt.attend(q, kv, lengths, ref, ws)
        got = torch.full((n, H, dh), float("nan"), dtype=dtype, device="cuda")
        assert _noalloc(q, kv, lengths, got) == 0
        torch.cuda.synchronize()
        tol = 1e-2 if dtype == torch.bfloat16 else 1e-5
        scale = ref.float().abs().max().item()
        assert torch.isfinite(got.float()).all()
        assert (got.float() - ref.float()).abs().max().item() <= tol * scale


def test_sizes_beyond_the_array_are_refused():
    n, H, dh, cap = 512, 16, 128, 4096
    assert rlt.attend_workspace_bytes(n, H, dh, cap) > NOALLOC_BYTES
    q = torch.zeros((1, 1, 1), device="cuda")  # never read: refused on the host
    lib = rlt._lib()
    fn = lib.rlt_attend_noalloc
    fn.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 5 + [ctypes.c_void_p] * 2
    lens = (ctypes.c_int32 * n)(*([cap] * n))
    rc = fn(q.data_ptr(), q.data_ptr(), ctypes.cast(lens, ctypes.c_void_p), n, H, dh, cap, 1,
            q.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 4  # RLT_ERR_CAPACITY
