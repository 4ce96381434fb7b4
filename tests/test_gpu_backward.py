"""Backward pass on the GPU (nys_attn_backward) against the oracle's
fp64 chain rule (nystrom_backward, itself pinned by finite differences).

Normwise error per head and per gradient, max|gpu - oracle| / max|oracle|:
the gradients are computed in fp32 on the CUDA cores from the same rounded
inputs, so the fp32 path is held to 1e-3 (the six Lemma 1 steps are
differentiated in fp32: their products amplify rounding by the conditioning
of A) and the bf16 path to 2e-2 (bf16 rounding of the gradients, dQ and dK
twice)."""
import numpy as np
import pytest

import nystr_self_attention_segment_b200 as nys
from nystr_self_attention_segment_b200.inputs import BF16, F32, make_custom
from oracle import nystrom as orc
from tests.gpu_util import normwise, to_dev, torch

pytestmark = pytest.mark.gpu

BWD_TOL = {F32: 1e-3, BF16: 2e-2}

CASES = [
    # (B, H, n, d, m, dtype, conv_k, iters)
    (1, 2, 64, 32, 8, F32, 5, 6),
    (1, 1, 70, 32, 8, F32, 3, 6),        # m does not divide n
    (2, 1, 96, 16, 12, F32, 0, 3),
    (1, 1, 64, 32, 64, F32, 0, 6),       # m = n
    (1, 2, 512, 64, 64, BF16, 33, 6),
    (1, 2, 1000, 64, 32, BF16, 33, 6),   # m does not divide n
    (1, 1, 1024, 64, 128, BF16, 33, 6),
]


@pytest.mark.parametrize("B,H,n,d,m,dtype,conv_k,iters", CASES)
def test_backward_against_oracle(B, H, n, d, m, dtype, conv_k, iters):
    t = torch()
    x = make_custom((B, H, n, d), dtype, seed=17 * n + m, conv_k=conv_k)
    rng = np.random.default_rng(n + m)
    G = rng.standard_normal((B, H, n, d))
    dtd = t.bfloat16 if dtype == BF16 else t.float32
    Gd = t.from_numpy(G.astype(np.float32)).cuda().to(dtd)
    Gr = Gd.float().cpu().numpy().astype(np.float64)      # the rounded dO both sides see
    Q, K, V = (to_dev(x[k], dtype) for k in ("Q", "K", "V"))
    cw = t.from_numpy(x["conv_w"]).cuda() if conv_k else None
    dQ, dK, dV, dcw = nys.nys_attn_backward(Q, K, V, m, Gd, iters, cw)
    t.cuda.synchronize()
    want = orc.nystrom_backward(x["Q"], x["K"], x["V"], m, Gr, iters,
                                x["conv_w"] if conv_k else None)
    for name, got in (("dQ", dQ), ("dK", dK), ("dV", dV)):
        g = got.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(g).all(), name
        for b in range(B):
            for h in range(H):
                e = normwise(g[b, h], want[name][b, h])
                assert e <= BWD_TOL[dtype], (name, b, h, e)
    if conv_k:
        e = normwise(dcw.cpu().numpy().astype(np.float64), want["dconv"])
        assert e <= BWD_TOL[dtype], ("dconv", e)
    else:
        assert dcw is None


def test_backward_is_deterministic_and_takes_a_workspace():
    t = torch()
    x = make_custom((1, 2, 512, 64), BF16, seed=3, conv_k=33)
    Q, K, V = (to_dev(x[k], BF16) for k in ("Q", "K", "V"))
    cw = t.from_numpy(x["conv_w"]).cuda()
    G = to_dev(np.random.default_rng(1).standard_normal((1, 2, 512, 64)), BF16)
    a = nys.nys_attn_backward(Q, K, V, 64, G, 6, cw)
    nb = nys._lib.nys_attn_backward_workspace_size(nys.desc_of(Q), 64, 6, 33)
    ws = t.empty(nb + 256, dtype=t.uint8, device="cuda")
    b = nys.nys_attn_backward(Q, K, V, 64, G, 6, cw, workspace=ws)
    t.cuda.synchronize()
    for u, v in zip(a, b):
        assert t.equal(u, v)


@pytest.mark.parametrize("name", ["headline_n8192_m64", "headline_n8192_m32"])
def test_backward_at_full_size_against_oracle(name):
    # The workload's full batch (B = 2, H = 12, n = 8192, the low-rank values
    # of its recipe, conv k = 33) through the same entry point and launch
    # configuration that bench.py --backward times; every head's gradients
    # against the oracle's fp64 chain rule (about 0.2 s per head on the host).
    from nystr_self_attention_segment_b200.inputs import WORKLOADS, make_inputs
    t = torch()
    wl = WORKLOADS[name]
    x = make_inputs(wl)
    shape = x["Q"].shape
    G = np.random.default_rng(7).standard_normal(shape)
    Gd = to_dev(G, BF16)
    Gr = Gd.float().cpu().numpy().astype(np.float64)
    Q, K, V = (to_dev(x[k], BF16) for k in ("Q", "K", "V"))
    cw = t.from_numpy(np.ascontiguousarray(x["conv_w"], dtype=np.float32)).cuda()
    dQ, dK, dV, dcw = nys.nys_attn_backward(Q, K, V, wl.landmarks, Gd, 6, cw)
    t.cuda.synchronize()
    got = {n: g.float().cpu().numpy().astype(np.float64)
           for n, g in (("dQ", dQ), ("dK", dK), ("dV", dV))}
    want = orc.nystrom_backward(x["Q"], x["K"], x["V"], wl.landmarks, Gr, 6, x["conv_w"])
    for n in ("dQ", "dK", "dV"):
        for b in range(shape[0]):
            for h in range(shape[1]):
                e = normwise(got[n][b, h], want[n][b, h])
                assert e <= BWD_TOL[BF16], (n, b, h, e)
    e = normwise(dcw.cpu().numpy().astype(np.float64), want["dconv"])
    assert e <= BWD_TOL[BF16], ("dconv", e)
