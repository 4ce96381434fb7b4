"""Error paths of the C ABI on the GPU, through the test build of the library
(libnys_attn_test.so: the same sources with test-only entry points).

- A launch that the runtime refuses (one launch of the call asks for more
  dynamic shared memory than a block may have) returns NYS_ERR_CUDA at once:
  no later kernel of the call runs, so the output is left untouched, and the
  next call works.
- A bounded device wait that runs out (an mbarrier nothing completes, with a
  short limit, no copy or MMA in flight) records NYS_ERR_TIMEOUT in the
  workspace error word; nys_attn_check_error reports it once and clears it.
- The backward's key blocks wait (bounded) on a flag of the per-head kernel;
  with the flag held back the wait gives up, NYS_ERR_TIMEOUT lands in the
  backward workspace's first word, and the next call recovers.

Nothing here faults or hangs the GPU: the refused launch never starts, and
the waits give up after about a millisecond (the probe) or 0.2 s (the key
blocks)."""
import ctypes

import numpy as np
import pytest

import nystr_self_attention_segment_b200 as nys
from nystr_self_attention_segment_b200 import _lib
from nystr_self_attention_segment_b200 import build as nys_build
from nystr_self_attention_segment_b200.inputs import BF16, F32, make_custom
from tests.gpu_util import TOL, normwise, run, torch

TEST_LIB = nys_build.VARIANTS["test"][0]


def _test_lib():
    nys_build.build(variant="test")
    lib = ctypes.CDLL(TEST_LIB)
    P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    D = ctypes.POINTER(_lib.nys_desc)
    lib.nys_attn_forward.restype = I
    lib.nys_attn_forward.argtypes = [P, P, P, D, I, I, P, I, P, P, S, P]
    lib.nys_attn_workspace_size.restype = I
    lib.nys_attn_workspace_size.argtypes = [D, I, ctypes.POINTER(S)]
    lib.nys_attn_check_error.restype = I
    lib.nys_attn_check_error.argtypes = [P, D, I, P]
    lib.nys_attn_launch_count.restype = I
    lib.nys_attn_launch_count.argtypes = [D, I, I, ctypes.POINTER(I)]
    lib.nys_test_fail_launch.restype = None
    lib.nys_test_fail_launch.argtypes = [I]
    lib.nys_test_timeout_probe.restype = I
    lib.nys_test_timeout_probe.argtypes = [P, D, I, ctypes.c_longlong, P]
    return lib


def test_hooks_exist_only_in_the_test_build():
    lib = _test_lib()
    prod = nys.load()
    for name in ("nys_test_fail_launch", "nys_test_timeout_probe", "nys_test_hold_head_flag"):
        assert hasattr(lib, name)
        assert not hasattr(prod, name)


def _stream():
    t = torch()
    return ctypes.c_void_p(t.cuda.current_stream().cuda_stream)


def _forward(lib, Q, K, V, m, cw, out, ws, ws_bytes):
    t = torch()
    dt = _lib.NYS_BF16 if Q.dtype == t.bfloat16 else _lib.NYS_F32
    desc = _lib.make_desc(dt, *Q.shape)
    return lib.nys_attn_forward(Q.data_ptr(), K.data_ptr(), V.data_ptr(), ctypes.byref(desc), m,
                                6, cw.data_ptr() if cw is not None else None,
                                cw.shape[1] if cw is not None else 0, out.data_ptr(),
                                ctypes.c_void_p(ws), ctypes.c_size_t(ws_bytes), _stream())


CASES = [((1, 2, 1000, 64), 32, BF16, 33), ((1, 1, 70, 32), 8, F32, 5)]


@pytest.mark.gpu
@pytest.mark.parametrize("shape,m,dtype,conv_k", CASES)
def test_refused_launch_returns_cuda_error_and_runs_nothing_after_it(shape, m, dtype, conv_k):
    t = torch()
    lib = _test_lib()
    x = make_custom(shape, dtype, seed=11, conv_k=conv_k)
    want, _, (Q, K, V, cw) = run(x, dtype, m)
    desc = _lib.make_desc(_lib.NYS_BF16 if dtype == BF16 else _lib.NYS_F32, *shape)
    nl = ctypes.c_int(0)
    assert lib.nys_attn_launch_count(ctypes.byref(desc), m, conv_k, ctypes.byref(nl)) == 0
    wsb = ctypes.c_size_t(0)
    assert lib.nys_attn_workspace_size(ctypes.byref(desc), m, ctypes.byref(wsb)) == 0
    buf = t.zeros(wsb.value + 256, dtype=t.uint8, device="cuda")
    ws = buf.data_ptr() + (-buf.data_ptr()) % 256
    for idx in range(nl.value):
        out = t.full_like(Q, 7.0)
        lib.nys_test_fail_launch(idx)
        st = _forward(lib, Q, K, V, m, cw, out, ws, wsb.value)
        assert _lib.STATUS_NAMES[st] == "NYS_ERR_CUDA", idx
        t.cuda.synchronize()
        # the output kernel is the last launch: it never ran
        assert bool((out == 7.0).all()), idx
        # the next call is unaffected and matches the product library
        st = _forward(lib, Q, K, V, m, cw, out, ws, wsb.value)
        assert st == 0
        assert lib.nys_attn_check_error(ctypes.c_void_p(ws), ctypes.byref(desc), m, _stream()) == 0
        got = out.float().cpu().numpy().astype(np.float64)
        assert normwise(got, want) <= TOL[dtype]


@pytest.mark.gpu
def test_bounded_wait_that_runs_out_reports_timeout_once():
    t = torch()
    lib = _test_lib()
    shape, m = (1, 2, 512, 64), 64
    desc = _lib.make_desc(_lib.NYS_BF16, *shape)
    wsb = ctypes.c_size_t(0)
    assert lib.nys_attn_workspace_size(ctypes.byref(desc), m, ctypes.byref(wsb)) == 0
    buf = t.zeros(wsb.value + 256, dtype=t.uint8, device="cuda")
    ws = ctypes.c_void_p(buf.data_ptr() + (-buf.data_ptr()) % 256)
    # about a millisecond of SM cycles, then the wait gives up
    assert lib.nys_test_timeout_probe(ws, ctypes.byref(desc), m, 2_000_000, _stream()) == 0
    st = lib.nys_attn_check_error(ws, ctypes.byref(desc), m, _stream())
    assert _lib.STATUS_NAMES[st] == "NYS_ERR_TIMEOUT"
    assert lib.nys_attn_check_error(ws, ctypes.byref(desc), m, _stream()) == 0   # cleared
    # and the same workspace serves a normal forward afterwards
    x = make_custom(shape, BF16, seed=3, conv_k=33)
    want, _, (Q, K, V, cw) = run(x, BF16, m)
    out = t.empty_like(Q)
    assert _forward(lib, Q, K, V, m, cw, out, ws.value, wsb.value) == 0
    assert lib.nys_attn_check_error(ws, ctypes.byref(desc), m, _stream()) == 0
    assert normwise(out.float().cpu().numpy().astype(np.float64), want) <= TOL[BF16]


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["bert_n512_m64", "headline_n8192_m32", "sweep_n1024_m128"])
def test_w_is_the_same_whichever_block_forms_it(name):
    # W = Z Y is formed by the second of {the pseudoinverse block, the block
    # that merges Y} to finish.  The test build delays one side or the other
    # (a bounded busy delay), so each hand-off runs; both run the same
    # function on the same inputs and must give the same bits.
    from nystr_self_attention_segment_b200.inputs import WORKLOADS, make_inputs
    t = torch()
    lib = _test_lib()
    lib.nys_test_w_order.restype = ctypes.c_int
    lib.nys_test_w_order.argtypes = [ctypes.c_int]
    wl = WORKLOADS[name]
    x = make_inputs(wl, batch=1, heads=min(wl.heads, 4))
    want, _, (Q, K, V, cw) = run(x, BF16, wl.landmarks)
    desc = _lib.make_desc(_lib.NYS_BF16, *Q.shape)
    wsb = ctypes.c_size_t(0)
    assert lib.nys_attn_workspace_size(ctypes.byref(desc), wl.landmarks, ctypes.byref(wsb)) == 0
    buf = t.zeros(wsb.value + 256, dtype=t.uint8, device="cuda")
    ws = buf.data_ptr() + (-buf.data_ptr()) % 256
    outs = []
    try:
        for mode in (1, 2, 0):
            assert lib.nys_test_w_order(mode) == 0
            out = t.empty_like(Q)
            assert _forward(lib, Q, K, V, wl.landmarks, cw, out, ws, wsb.value) == 0
            assert lib.nys_attn_check_error(ctypes.c_void_p(ws), ctypes.byref(desc),
                                            wl.landmarks, _stream()) == 0
            outs.append(out.float().cpu().numpy().astype(np.float64))
    finally:
        lib.nys_test_w_order(0)
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[1], outs[2])
    assert np.array_equal(outs[2], want)


@pytest.mark.gpu
def test_backward_key_wait_that_runs_out_reports_timeout_and_next_call_recovers():
    # The backward's key-tile kernel starts beside the per-head kernel and
    # waits (bounded, about 0.2 s) for the head's dY / D flag.  The test build
    # can hold that flag back: every key block's wait then gives up, records
    # NYS_ERR_TIMEOUT in the workspace's first word and leaves.  The next call
    # (flag published again) must clear the word and give the same gradients
    # as before, bit for bit.
    t = torch()
    lib = _test_lib()
    lib.nys_test_hold_head_flag.restype = None
    lib.nys_test_hold_head_flag.argtypes = [ctypes.c_int]
    P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    D = ctypes.POINTER(_lib.nys_desc)
    lib.nys_attn_backward_workspace_size.restype = I
    lib.nys_attn_backward_workspace_size.argtypes = [D, I, I, I, ctypes.POINTER(S)]
    lib.nys_attn_backward.restype = I
    lib.nys_attn_backward.argtypes = [P, P, P, D, I, I, P, I, P, P, P, P, P, P, S, P]
    shape, m, ck = (1, 2, 512, 64), 64, 33
    x = make_custom(shape, BF16, seed=5, conv_k=ck)
    _, _, (Q, K, V, cw) = run(x, BF16, m)
    G = t.randn(shape, device="cuda", generator=t.Generator(device="cuda").manual_seed(5))
    G = G.to(t.bfloat16)
    desc = _lib.make_desc(_lib.NYS_BF16, *shape)
    wsb = ctypes.c_size_t(0)
    assert lib.nys_attn_backward_workspace_size(ctypes.byref(desc), m, 6, ck,
                                                ctypes.byref(wsb)) == 0
    buf = t.zeros(wsb.value + 256, dtype=t.uint8, device="cuda")
    off = (-buf.data_ptr()) % 256
    ws = buf.data_ptr() + off

    def backward():
        dQ, dK, dV = t.empty_like(Q), t.empty_like(Q), t.empty_like(Q)
        dcw = t.empty_like(cw)
        st = lib.nys_attn_backward(Q.data_ptr(), K.data_ptr(), V.data_ptr(), ctypes.byref(desc),
                                   m, 6, cw.data_ptr(), ck, G.data_ptr(), dQ.data_ptr(),
                                   dK.data_ptr(), dV.data_ptr(), dcw.data_ptr(),
                                   ctypes.c_void_p(ws), ctypes.c_size_t(wsb.value), _stream())
        t.cuda.synchronize()
        word = int(buf[off:off + 4].cpu().numpy().view(np.uint32)[0])
        return st, word, (dQ, dK, dV, dcw)

    st, word, want = backward()
    assert st == 0 and word == 0
    try:
        lib.nys_test_hold_head_flag(1)
        st, word, _ = backward()
    finally:
        lib.nys_test_hold_head_flag(0)
    assert st == 0
    assert _lib.STATUS_NAMES[word] == "NYS_ERR_TIMEOUT"
    st, word, got = backward()
    assert st == 0 and word == 0
    for a, b in zip(got, want):
        assert t.equal(a, b)
