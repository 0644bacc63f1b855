"""The decoder's cross-attention kernel through the standalone C-ABI call
rlt_attend, against the oracle's attention (fp64) row by row: ragged lengths
within one 1024-position chunk, lengths that split into several chunks merged
in chunk order (1025 .. 4096, with ragged tail chunks), one-row prefixes, both
storage types, and a full-size sample (256 rows x 12 heads x 1024)."""
import numpy as np
import pytest
import torch

import oracle
from token_recurrent_decoding_b200 import rlt

pytestmark = pytest.mark.gpu


def _case(n, H, dh, cap, lengths, dtype, seed=0):
    g = torch.Generator(device="cpu").manual_seed(seed)
    q = torch.randn((n, H, dh), generator=g, dtype=torch.float32)
    kv = torch.randn((n, H, 2, cap, dh), generator=g, dtype=torch.float32).to(dtype)
    qd, kvd = q.cuda(), kv.cuda()
    out = torch.empty((n, H, dh), dtype=dtype, device="cuda")
    ws = torch.empty(rlt.attend_workspace_bytes(n, H, dh, cap), dtype=torch.uint8, device="cuda")
    rlt.attend(qd, kvd, lengths, out, ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    return q.double().numpy(), kv.double().numpy(), out.double().cpu().numpy()


def _check(q, kv, out, lengths, rows, tol):
    """bf16 outputs (tol 1e-2): each element is one round-to-nearest-even of
    the fp32 result, so its error is bounded element by element, 2^-8 |ref|
    (twice the half-ulp bound), plus 1e-3 RMS for the fp32 accumulation; a
    bound relative to the row RMS alone fails long rows, whose average of
    many values has an RMS well below its largest element. fp32 outputs:
    accumulation only, tol x RMS."""
    for i in rows:
        L = lengths[i]
        for h in range(q.shape[1]):
            ref = oracle.attend(q[i, h], kv[i, h, 0, :L], kv[i, h, 1, :L])
            scale = max(np.sqrt(np.mean(ref ** 2)), 1e-3)
            if tol >= 1e-2:
                bound = 2.0 ** -8 * np.abs(ref) + 1e-3 * scale
            else:
                bound = tol * scale
            err = np.abs(out[i, h] - ref)
            assert (err <= bound).all(), (i, h, L, float(err.max()))


@pytest.mark.parametrize("dtype,dh", [(torch.bfloat16, 64), (torch.bfloat16, 128),
                                      (torch.float32, 16), (torch.float32, 64)])
def test_attend_matches_oracle_ragged(dtype, dh):
    lengths = [1, 2, 255, 256, 257, 511, 700, 64, 3, 700, 129]
    n, H, cap = len(lengths), 3, 700
    q, kv, out = _case(n, H, dh, cap, lengths, dtype)
    # bf16 output: one storage rounding (2^-9 relative); fp32: accumulation only
    _check(q, kv, out, lengths, range(n), 1e-2 if dtype == torch.bfloat16 else 1e-5)


@pytest.mark.parametrize("dtype,dh", [(torch.bfloat16, 64), (torch.bfloat16, 128),
                                      (torch.float32, 32)])
def test_attend_split_kv_chunks_match_oracle(dtype, dh):
    """Rows longer than one 1024-position chunk: partials of every chunk,
    merged by the row's last finishing unit in chunk order."""
    lengths = [1025, 2047, 2048, 3000, 4096, 1, 1024, 2049, 4095, 1500]
    n, H, cap = len(lengths), 2, 4096
    q, kv, out = _case(n, H, dh, cap, lengths, dtype, seed=5)
    _check(q, kv, out, lengths, range(n), 1e-2 if dtype == torch.bfloat16 else 1e-5)
    # a second call agrees bitwise: a row's result depends on its own length only
    q2, kv2, out2 = _case(n, H, dh, cap, lengths, dtype, seed=5)
    np.testing.assert_array_equal(out, out2)


def test_attend_full_size_sampled():
    n, H, dh, cap = 256, 12, 64, 1024
    lengths = [1024] * n
    q, kv, out = _case(n, H, dh, cap, lengths, torch.bfloat16, seed=3)
    _check(q, kv, out, lengths, [0, 77, 128, 255], 1e-2)


def test_attend_rejects_bad_arguments():
    n, H, dh, cap = 2, 1, 64, 8
    q = torch.zeros((n, H, dh), device="cuda")
    kv = torch.zeros((n, H, 2, cap, dh), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((n, H, dh), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(rlt.attend_workspace_bytes(n, H, dh, cap), dtype=torch.uint8, device="cuda")
    with pytest.raises(rlt.RLTError) as e:
        rlt.attend(q, kv, [0, 3], out, ws)
    assert e.value.status == 1
    with pytest.raises(rlt.RLTError) as e:
        rlt.attend(q, kv, [9, 3], out, ws)
    assert e.value.status == 1
    with pytest.raises(rlt.RLTError) as e:
        rlt.attend(q, kv, [2, 3], out, ws[:64])
    assert e.value.status == 4
