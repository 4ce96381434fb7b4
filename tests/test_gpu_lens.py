"""Right-padded ragged batches through nys_attn_forward_lens, against the
oracle's reading (nystrom_forward_lens: each element is the method on its own
first L tokens; its padding rows are zero).  The lengths cut segments, 128-row
output tiles and 128-key chunks; every segment keeps at least one token."""
import numpy as np
import pytest

import nystr_self_attention_segment_b200 as nys
from nystr_self_attention_segment_b200.inputs import BF16, F32, make_custom
from oracle import nystrom as orc
from tests.gpu_util import TOL, normwise, run, to_dev, torch

pytestmark = pytest.mark.gpu

CASES = [
    # (B, H, n, d, m, dtype, conv_k, lens)
    (3, 2, 1000, 64, 32, BF16, 33, [1000, 777, 530]),
    (2, 2, 4096, 64, 64, BF16, 33, [4096, 2100]),
    (2, 1, 2048, 64, 128, BF16, 33, [2048, 1400]),
    (2, 1, 640, 64, 64, BF16, 0, [640, 320]),       # no conv: rows only
    (3, 2, 70, 32, 8, F32, 5, [70, 64, 50]),
    (2, 1, 24, 8, 3, F32, 3, [24, 7]),
]


def _valid(L, m):
    return (m - 1) * (-(-L // m)) < L


@pytest.mark.parametrize("dummy", [0])
def test_case_lengths_keep_every_segment(dummy):
    for B, H, n, d, m, dtype, conv_k, lens in CASES:
        assert all(m <= L <= n and _valid(L, m) for L in lens), (n, m, lens)


def _lens(x):
    t = torch()
    return t.tensor(x, dtype=t.int32, device="cuda")


@pytest.mark.parametrize("B,H,n,d,m,dtype,conv_k,lens", CASES)
def test_ragged_batch_against_oracle(B, H, n, d, m, dtype, conv_k, lens):
    x = make_custom((B, H, n, d), dtype, seed=13 * n + m, conv_k=conv_k)
    Q, K, V = (to_dev(x[k], dtype) for k in ("Q", "K", "V"))
    t = torch()
    cw = t.from_numpy(x["conv_w"]).cuda() if conv_k else None
    ws = nys.Workspace(Q, m)
    out = t.full_like(Q, 3.0)
    nys.nys_attn_forward_lens(Q, K, V, m, _lens(lens), 6, cw, out=out, workspace=ws)
    t.cuda.synchronize()
    nys.nys_attn_check_error(ws)
    got = out.float().cpu().numpy().astype(np.float64)
    want = orc.nystrom_forward_lens(x["Q"], x["K"], x["V"], m, lens, 6,
                                    x["conv_w"] if conv_k else None)
    for b in range(B):
        L = lens[b]
        assert np.all(got[b, :, L:] == 0.0), b
        for h in range(H):
            assert normwise(got[b, h, :L], want[b, h, :L]) <= TOL[dtype], (b, h)


@pytest.mark.parametrize("dtype,m", [(BF16, 64), (F32, 8)])
def test_full_lengths_equal_the_plain_forward(dtype, m):
    shape = (2, 2, 640, 64) if dtype == BF16 else (2, 2, 64, 32)
    x = make_custom(shape, dtype, seed=21, conv_k=33 if dtype == BF16 else 3)
    want, _, (Q, K, V, cw) = run(x, dtype, m)
    out = nys.nys_attn_forward_lens(Q, K, V, m, _lens([shape[2]] * shape[0]), 6, cw)
    torch().cuda.synchronize()
    assert np.array_equal(out.float().cpu().numpy().astype(np.float64), want)


def test_invalid_length_is_reported_and_zeroes_only_its_element():
    t = torch()
    B, H, n, d, m = 2, 2, 1000, 64, 32
    x = make_custom((B, H, n, d), BF16, seed=5, conv_k=33)
    Q, K, V = (to_dev(x[k], BF16) for k in ("Q", "K", "V"))
    cw = t.from_numpy(x["conv_w"]).cuda()
    ws = nys.Workspace(Q, m)
    out = t.full_like(Q, 3.0)
    nys.nys_attn_forward_lens(Q, K, V, m, _lens([900, 20]), 6, cw, out=out, workspace=ws)
    with pytest.raises(nys.NysError) as e:
        nys.nys_attn_check_error(ws)
    assert e.value.name == "NYS_ERR_INVALID_ARG"
    got = out.float().cpu().numpy().astype(np.float64)
    assert np.all(got[1] == 0.0)
    want = orc.nystrom_forward_lens(x["Q"][:1], x["K"][:1], x["V"][:1], m, [900], 6, x["conv_w"])
    for h in range(H):
        assert normwise(got[0, h, :900], want[0, h, :900]) <= TOL[BF16]
    assert np.all(got[0, :, 900:] == 0.0)
