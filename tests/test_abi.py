"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point the header declares, sizes workspaces, and rejects invalid
calls before anything is enqueued."""
import ctypes
import os
import re

import pytest

import nystr_self_attention_segment_b200 as nys
from nystr_self_attention_segment_b200 import _lib
from nystr_self_attention_segment_b200.inputs import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nys_attn.h")


def header_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"NYS_ATTN_API\s+[\w\s\*]*?\b(nys_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = nys.load()
    declared = header_functions()
    assert declared, "no declarations found"
    assert sorted(_lib.EXPORTS) == declared
    for name in declared:
        assert hasattr(lib, name), name


def test_status_strings_and_version():
    for code, name in _lib.STATUS_NAMES.items():
        assert nys.nys_status_string(code).startswith(name)
    assert nys.nys_version() >= 100


def desc(dtype=nys.NYS_BF16, b=2, h=12, n=8192, d=64):
    return nys.make_desc(dtype, b, h, n, d)


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_workspace_sizes_for_every_workload(name):
    wl = WORKLOADS[name]
    dt = nys.NYS_BF16 if wl.dtype == "bf16" else nys.NYS_F32
    ds = nys.make_desc(dt, wl.batch, wl.heads, wl.seq_len, wl.head_dim)
    ws = nys.nys_attn_workspace_size(ds, wl.landmarks)
    lay = nys.nys_attn_intermediates(ds, wl.landmarks)
    bh, m, d = wl.bh, wl.landmarks, wl.head_dim
    assert lay["total"] == ws
    regions = [(lay["q_landmarks"], bh * m * d * 4), (lay["k_landmarks"], bh * m * d * 4),
               (lay["z"], bh * m * m * 4), (lay["y"], bh * m * d * 4), (lay["w"], bh * m * d * 4),
               (lay["error_word"], 4)]
    for off, size in regions:
        assert off % 256 == 0 and off + size <= ws
    regions.sort()
    for (a, sa), (b, _) in zip(regions, regions[1:]):
        assert a + sa <= b
    hb = nys.nys_attn_host_buffer_size(ds, wl.landmarks, wl.conv_k)
    assert hb >= ws + 4 * bh * wl.seq_len * d * (2 if wl.dtype == "bf16" else 4)
    assert nys.nys_attn_launch_count(ds, wl.landmarks, wl.conv_k) >= 1


FAKE = 1 << 40       # never dereferenced: every call below fails validation


def forward_status(ds, m=64, iters=6, conv=None, conv_k=0, q=FAKE, k=FAKE + (1 << 32),
                   v=FAKE + (2 << 32), out=FAKE + (3 << 32), ws=None, ws_bytes=0):
    return _lib.raw_forward(q, k, v, ds, m, iters, conv, conv_k, out, ws, ws_bytes, None)


S = _lib.STATUS


def test_rejects_invalid_calls_without_launching():
    assert forward_status(desc(n=100), m=64) == S["NYS_ERR_NOT_DIVISIBLE"]   # 64 segments of 2
    assert forward_status(desc(d=32)) == S["NYS_ERR_UNSUPPORTED"]
    assert forward_status(desc(n=6144), m=48) == S["NYS_ERR_UNSUPPORTED"]
    assert forward_status(desc(nys.NYS_F32, n=8192), m=128) == S["NYS_ERR_UNSUPPORTED"]
    assert forward_status(desc(nys.NYS_F32, d=65, n=64), m=8) == S["NYS_ERR_UNSUPPORTED"]
    assert forward_status(desc(), m=0) == S["NYS_ERR_INVALID_ARG"]
    assert forward_status(desc(n=64), m=128) == S["NYS_ERR_INVALID_ARG"]
    assert forward_status(desc(), iters=-1) == S["NYS_ERR_INVALID_ARG"]
    assert forward_status(desc(), iters=65) == S["NYS_ERR_UNSUPPORTED"]
    assert forward_status(desc(), conv=FAKE + (5 << 32), conv_k=32) == S["NYS_ERR_INVALID_ARG"]
    assert forward_status(desc(), conv=FAKE + (5 << 32), conv_k=0) == S["NYS_ERR_INVALID_ARG"]
    assert forward_status(desc(), conv=FAKE + (5 << 32), conv_k=65) == S["NYS_ERR_UNSUPPORTED"]
    assert forward_status(desc(), q=None) == S["NYS_ERR_INVALID_ARG"]
    assert forward_status(desc(), out=None) == S["NYS_ERR_INVALID_ARG"]
    assert forward_status(nys.make_desc(7, 1, 1, 64, 64)) == S["NYS_ERR_INVALID_ARG"]
    assert forward_status(desc(b=-1)) == S["NYS_ERR_INVALID_ARG"]
    # output aliasing an input, or partly overlapping one
    assert forward_status(desc(), out=FAKE) == S["NYS_ERR_ALIAS"]
    assert forward_status(desc(), out=FAKE + (2 << 32) + 4096) == S["NYS_ERR_ALIAS"]
    # misaligned operands: 16 bytes for bf16, 4 for fp32 and the conv weights
    assert forward_status(desc(), q=FAKE + 8) == S["NYS_ERR_INVALID_ARG"]
    assert forward_status(desc(), out=FAKE + (3 << 32) + 2) == S["NYS_ERR_INVALID_ARG"]
    f32 = desc(nys.NYS_F32, b=1, h=1, n=64, d=32)
    assert forward_status(f32, m=8, k=FAKE + (1 << 32) + 2) == S["NYS_ERR_INVALID_ARG"]
    assert forward_status(desc(), conv=FAKE + (5 << 32) + 2, conv_k=33) == S["NYS_ERR_INVALID_ARG"]
    # workspace too small or misaligned
    ds = desc()
    need = nys.nys_attn_workspace_size(ds, 64)
    assert forward_status(ds, ws=FAKE + (8 << 32), ws_bytes=need - 1) == S["NYS_ERR_WORKSPACE"]
    assert forward_status(ds, ws=FAKE + (8 << 32) + 16, ws_bytes=need) == S["NYS_ERR_INVALID_ARG"]
    # workspace overlapping the output
    assert forward_status(ds, ws=FAKE + (3 << 32), ws_bytes=need) == S["NYS_ERR_ALIAS"]


def test_empty_problems_are_no_ops():
    # nothing is enqueued, so even null tensors are accepted
    for ds in (desc(b=0), desc(h=0), desc(n=0)):
        assert forward_status(ds, q=None, k=None, v=None, out=None) == S["NYS_OK"]
        assert nys.nys_attn_workspace_size(ds, 64) == 0
        assert nys.nys_attn_launch_count(ds, 64, 33) == 0


def test_ragged_segments_validate_when_none_is_empty():
    # segments of ceil(n/m) tokens: valid while (m - 1) * ceil(n/m) < n
    for n, m in ((8100, 64), (4090, 128), (1000, 32), (127, 64), (8192 + 1, 64)):
        assert nys.nys_attn_workspace_size(desc(n=n), m) > 0, (n, m)
    for n, m in ((126, 64), (100, 64), (65, 64), (4000, 128)):
        with pytest.raises(nys.NysError) as e:
            nys.nys_attn_workspace_size(desc(n=n), m)
        assert e.value.name == "NYS_ERR_NOT_DIVISIBLE", (n, m)


def test_size_queries_validate_too():
    with pytest.raises(nys.NysError) as e:
        nys.nys_attn_workspace_size(desc(n=100), 64)
    assert e.value.name == "NYS_ERR_NOT_DIVISIBLE"
    with pytest.raises(nys.NysError):
        nys.nys_attn_intermediates(desc(d=16), 64)
    lib = nys.load()
    assert lib.nys_attn_workspace_size(ctypes.byref(desc()), 64, None) == S["NYS_ERR_INVALID_ARG"]
    assert lib.nys_attn_workspace_size(None, 64, ctypes.byref(ctypes.c_size_t())) == \
        S["NYS_ERR_INVALID_ARG"]


# ------------------------------------------------------------------ layout property

from hypothesis import given, settings, strategies as st   # noqa: E402


def _valid_n(n, m):
    seg = -(-n // m)
    return (m - 1) * seg < n


@settings(max_examples=300, deadline=None)
@given(b=st.integers(1, 8), h=st.integers(1, 24), m=st.sampled_from([32, 64, 128]),
       n=st.integers(32, 70000))
def test_bf16_layout_holds_every_region(b, h, m, n):
    # Every region the kernels write, for any valid shape: the five exported
    # intermediates 256-byte aligned and disjoint inside the total, and room
    # in the total for the split partial states (S splits of m x (64 + 2)
    # floats per head) and the bf16 W operand the merge and the output
    # kernel use.
    if n < m or not _valid_n(n, m):
        with pytest.raises(nys.NysError):
            nys.nys_attn_workspace_size(desc(b=b, h=h, n=n), m)
        return
    ds = desc(b=b, h=h, n=n)
    ws = nys.nys_attn_workspace_size(ds, m)
    lay = nys.nys_attn_intermediates(ds, m)
    bh = b * h
    regions = [(lay["q_landmarks"], bh * m * 64 * 4), (lay["k_landmarks"], bh * m * 64 * 4),
               (lay["z"], bh * m * m * 4), (lay["y"], bh * m * 64 * 4),
               (lay["w"], bh * m * 64 * 4), (lay["error_word"], 256)]
    for off, size in regions:
        assert off % 256 == 0 and off + size <= ws
    regions.sort()
    for (a, sa), (c, _) in zip(regions, regions[1:]):
        assert a + sa <= c
    chunks = -(-n // 128)
    splits = max(1, min((148 - bh) // bh, chunks, 16))
    partials = bh * splits * m * (64 + 2) * 4
    assert ws >= sum(sz for _, sz in regions) + partials + bh * m * 128


@settings(max_examples=200, deadline=None)
@given(m=st.integers(1, 64), d=st.integers(1, 64), n=st.integers(1, 3000))
def test_f32_shapes_validate_by_the_segment_rule(m, d, n):
    ds = desc(nys.NYS_F32, b=1, h=2, n=n, d=d)
    if m > n:
        with pytest.raises(nys.NysError):
            nys.nys_attn_workspace_size(ds, m)
    elif not _valid_n(n, m):
        with pytest.raises(nys.NysError) as e:
            nys.nys_attn_workspace_size(ds, m)
        assert e.value.name == "NYS_ERR_NOT_DIVISIBLE"
    else:
        assert nys.nys_attn_workspace_size(ds, m) > 0
