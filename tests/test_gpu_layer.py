"""The attention layer (nys_attn_layer_forward: tensor-core QKV projection,
the forward, tensor-core output projection) against the oracle's layer
(nystrom_layer_forward, fp64, pinned by identity projections and the head
split / concat), and the projections alone against X W^T."""
import numpy as np
import pytest

import nystr_self_attention_segment_b200 as nys
from nystr_self_attention_segment_b200.inputs import BF16, round_to_bf16_as_f32
from oracle import nystrom as orc
from tests.gpu_util import TOL, normwise, torch

pytestmark = pytest.mark.gpu


def _inputs(B, n, H, seed):
    rng = np.random.default_rng(seed)
    D = H * 64
    X = round_to_bf16_as_f32(rng.standard_normal((B, n, D)))
    Wqkv = round_to_bf16_as_f32(rng.standard_normal((3 * D, D)) / np.sqrt(D))
    Wo = round_to_bf16_as_f32(rng.standard_normal((D, D)) / np.sqrt(D))
    cw = (0.02 * rng.standard_normal((H, 33))).astype(np.float32)
    return X, Wqkv, Wo, cw


def _dev(a):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda().to(t.bfloat16)


@pytest.mark.parametrize("B,n,H,m", [(2, 640, 2, 64), (1, 1000, 3, 32), (1, 512, 2, 128)])
def test_layer_against_oracle(B, n, H, m):
    t = torch()
    X, Wqkv, Wo, cw = _inputs(B, n, H, 7 * n + H)
    Y, ws = nys.nys_attn_layer_forward(_dev(X), _dev(Wqkv), _dev(Wo), H, m, 6,
                                       t.from_numpy(cw).cuda())
    nys.nys_attn_layer_check_error(ws, H, B, n, m)
    got = Y.float().cpu().numpy().astype(np.float64)
    want = orc.nystrom_layer_forward(X, Wqkv, Wo, H, m, 6, cw)
    for b in range(B):
        assert normwise(got[b], want[b]) <= TOL[BF16], b
    # the projections alone: Q, K, V at the start of the workspace, [B, H, n, 64] bf16
    D = H * 64
    T = B * H * n * 64 * 2
    for i in range(3):
        start = i * ((T + 255) // 256 * 256)
        got_p = ws[start:start + T].view(t.bfloat16).view(B, H, n, 64).float().cpu().numpy()
        want_p = (X @ Wqkv[i * D:(i + 1) * D].T).reshape(B, n, H, 64).transpose(0, 2, 1, 3)
        assert normwise(got_p.astype(np.float64), want_p) <= 5e-3, i
