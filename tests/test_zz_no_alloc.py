"""nys_attn_forward_static (the entry point that allocates nothing) against
nys_attn_forward, through the C ABI.

The file name sorts last so that it runs after every other test as well as
alone in a fresh process: the first call on the device is the one that looks
up the fixed scratch array's address."""
import ctypes

import numpy as np
import pytest

import nystr_self_attention_segment_b200 as nys
from nystr_self_attention_segment_b200 import _lib
from nystr_self_attention_segment_b200.inputs import WORKLOADS, make_inputs
from tests.gpu_util import TOL, normwise, run, to_dev, torch

pytestmark = pytest.mark.gpu


def ptr(x):
    return ctypes.c_void_p(x.data_ptr()) if x is not None else None


def static_forward(Q, K, V, m, iters, cw):
    t = torch()
    out = t.empty_like(Q)
    dt = _lib.NYS_BF16 if Q.dtype == t.bfloat16 else _lib.NYS_F32
    desc = _lib.make_desc(dt, *Q.shape)
    stream = ctypes.c_void_p(t.cuda.current_stream().cuda_stream)
    st = _lib.raw_forward_static(ptr(Q), ptr(K), ptr(V), desc, m, iters, ptr(cw),
                                 cw.shape[1] if cw is not None else 0, ptr(out), stream)
    _lib.check(st, "nys_attn_forward_static")
    t.cuda.synchronize()
    return out


@pytest.mark.parametrize("name", ["tiny_f32_m8", "headline_n8192_m64", "long_n4096_m64"])
def test_static_matches_forward_on_two_calls_in_a_row(name):
    wl = WORKLOADS[name]
    x = make_inputs(wl)
    want, _, (Q, K, V, cw) = run(x, wl.dtype, wl.landmarks, wl.pinv_iters)
    for _ in range(2):
        got = static_forward(Q, K, V, wl.landmarks, wl.pinv_iters, cw)
        got = got.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(got).all()
        assert normwise(got, want) <= TOL[wl.dtype]


def test_static_rejects_a_problem_larger_than_the_array():
    t = torch()
    wl = WORKLOADS["bert_n512_m64"]        # needs about 9 MiB of scratch
    desc = _lib.make_desc(_lib.NYS_BF16, wl.batch, wl.heads, wl.seq_len, wl.head_dim)
    assert nys._lib.nys_attn_workspace_size(desc, wl.landmarks) > _lib.NYS_STATIC_SCRATCH_BYTES
    shape = (wl.batch, wl.heads, wl.seq_len, wl.head_dim)
    Q = t.zeros(shape, dtype=t.bfloat16, device="cuda")
    out = t.full(shape, 7.0, dtype=t.bfloat16, device="cuda")
    stream = ctypes.c_void_p(t.cuda.current_stream().cuda_stream)
    st = _lib.raw_forward_static(ptr(Q), ptr(Q), ptr(Q), desc, wl.landmarks, 6, None, 0,
                                 ptr(out), stream)
    assert _lib.STATUS_NAMES[st] == "NYS_ERR_WORKSPACE"
    t.cuda.synchronize()
    assert bool((out == 7.0).all())
