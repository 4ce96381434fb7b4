"""nys_attn_forward_static (the entry point that allocates nothing) against
nys_attn_forward, through the C ABI.

Some callers cannot allocate device memory at call time: a host that owns the
device's memory pool, a path that cannot take cudaMalloc's implicit
synchronisation, a process held to a memory budget fixed at start-up.  The
static entry point keeps its scratch in one fixed device array of the
library instead.

Every call shares that array, so each call must clear what starts at zero
(the error word, the per-head counters) and leave nothing of the previous
call in its result: the second call of each pair runs on different inputs
from the first, and both are checked against nys_attn_forward on the same
inputs.  The file name sorts last so that the tests run after every other
test as well as alone in a fresh process."""
import ctypes

import numpy as np
import pytest

import nystr_self_attention_segment_b200 as nys
from nystr_self_attention_segment_b200 import _lib
from nystr_self_attention_segment_b200.inputs import WORKLOADS, make_inputs
from tests.gpu_util import TOL, normwise, run, torch

pytestmark = pytest.mark.gpu


def ptr(x):
    return ctypes.c_void_p(x.data_ptr()) if x is not None else None


def _desc(Q):
    t = torch()
    dt = _lib.NYS_BF16 if Q.dtype == t.bfloat16 else _lib.NYS_F32
    return _lib.make_desc(dt, *Q.shape)


def _stream():
    return ctypes.c_void_p(torch().cuda.current_stream().cuda_stream)


def static_forward(Q, K, V, m, iters, cw):
    t = torch()
    out = t.empty_like(Q)
    st = _lib.raw_forward_static(ptr(Q), ptr(K), ptr(V), _desc(Q), m, iters, ptr(cw),
                                 cw.shape[1] if cw is not None else 0, ptr(out), _stream())
    _lib.check(st, "nys_attn_forward_static")
    _lib.check(_lib.raw_check_error_static(_desc(Q), m, _stream()),
               "nys_attn_check_error_static")
    t.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64)


def _other_inputs(x):
    """A second input set of the same workload: values negated and permuted
    along the sequence, so that every landmark, B~ V partial and W differs."""
    y = dict(x)
    for k in ("Q", "K", "V"):
        y[k] = -np.ascontiguousarray(x[k][:, :, ::-1])
    return y


# m = 64 and m = 32 (power-form pseudoinverse, split products), m = 128
# (power form at full width), fp32
NAMES = ["tiny_f32_m8", "headline_n8192_m64", "headline_n8192_m32", "long_n4096_m64",
         "sweep_n4096_m128"]


@pytest.mark.parametrize("name", NAMES)
def test_static_matches_forward_on_two_calls_in_a_row(name):
    wl = WORKLOADS[name]
    desc = _lib.make_desc(_lib.NYS_BF16 if wl.dtype == "bf16" else _lib.NYS_F32, wl.batch,
                          wl.heads, wl.seq_len, wl.head_dim)
    assert _lib.nys_attn_workspace_size(desc, wl.landmarks) <= _lib.NYS_STATIC_SCRATCH_BYTES
    x1 = make_inputs(wl)
    for x in (x1, _other_inputs(x1)):
        want, _, (Q, K, V, cw) = run(x, wl.dtype, wl.landmarks, wl.pinv_iters)
        got = static_forward(Q, K, V, wl.landmarks, wl.pinv_iters, cw)
        assert np.isfinite(got).all()
        assert normwise(got, want) <= TOL[wl.dtype]


def test_static_rejects_a_problem_larger_than_the_array():
    t = torch()
    wl = WORKLOADS["bert_n512_m64"]        # needs about 9.8 MiB of scratch
    desc = _lib.make_desc(_lib.NYS_BF16, wl.batch, wl.heads, wl.seq_len, wl.head_dim)
    assert nys._lib.nys_attn_workspace_size(desc, wl.landmarks) > _lib.NYS_STATIC_SCRATCH_BYTES
    shape = (wl.batch, wl.heads, wl.seq_len, wl.head_dim)
    Q = t.zeros(shape, dtype=t.bfloat16, device="cuda")
    out = t.full(shape, 7.0, dtype=t.bfloat16, device="cuda")
    st = _lib.raw_forward_static(ptr(Q), ptr(Q), ptr(Q), desc, wl.landmarks, 6, None, 0,
                                 ptr(out), _stream())
    assert _lib.STATUS_NAMES[st] == "NYS_ERR_WORKSPACE"
    st = _lib.raw_check_error_static(desc, wl.landmarks, _stream())
    assert _lib.STATUS_NAMES[st] == "NYS_ERR_WORKSPACE"
    t.cuda.synchronize()
    assert bool((out == 7.0).all())
