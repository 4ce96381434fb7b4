"""B200 (sm_100a) Nystromformer attention forward behind a C ABI.

Python side of the library: argument marshalling from torch tensors to the
C entry points of include/nys_attn.h (same names).  Every step of the forward
pass runs in the CUDA kernels of libnys_attn.so; torch only supplies device
memory and streams.  There is no CPU path: without the built library every
call raises.
"""

from . import _lib
from ._lib import (NYS_BF16, NYS_F32, NysError, EXPORTS, load, make_desc,  # noqa: F401
                   nys_attn_host_buffer_size, nys_attn_intermediates, nys_attn_launch_count,
                   nys_attn_launch_names,
                   nys_attn_workspace_size, nys_status_string, nys_version)

__all__ = [
    "NYS_F32", "NYS_BF16", "NysError", "load", "desc_of", "nys_attn_forward",
    "nys_attn_forward_host", "nys_attn_workspace_size", "nys_attn_intermediates",
    "nys_attn_host_buffer_size", "nys_attn_check_error", "nys_attn_launch_count",
    "nys_status_string", "nys_version", "Workspace", "nys_attn_launch_names",
    "nys_attn_forward_timed", "nys_attn_forward_lens", "nys_attn_backward",
    "nys_attn_layer_forward",
]


def _torch():
    import torch
    return torch


def _dtype_code(t):
    torch = _torch()
    if t.dtype == torch.float32:
        return NYS_F32
    if t.dtype == torch.bfloat16:
        return NYS_BF16
    raise TypeError("Q/K/V must be float32 or bfloat16, got %s" % t.dtype)


def desc_of(Q):
    """nys_desc of a [batch, heads, n, d] tensor."""
    if Q.dim() != 4:
        raise ValueError("expected [batch, heads, seq_len, head_dim], got %s" % (tuple(Q.shape),))
    b, h, n, d = Q.shape
    return make_desc(_dtype_code(Q), b, h, n, d)


def _check_operands(Q, K, V, out, conv_w, on_cuda=True):
    """Q, K, V and out: contiguous tensors of one shape and dtype on one
    device (CUDA, or CPU for the host-buffer entry point); conv_w: None or a
    contiguous float32 [heads, k] tensor on that device.  The kernels size
    every access from Q's descriptor, so a mismatch caught here would
    otherwise be an out-of-bounds access on the device."""
    torch = _torch()
    where = "CUDA" if on_cuda else "CPU"
    for name, t in (("Q", Q), ("K", K), ("V", V), ("out", out)):
        if bool(t.is_cuda) != on_cuda or not t.is_contiguous():
            raise ValueError("%s must be a contiguous %s tensor" % (name, where))
        if tuple(t.shape) != tuple(Q.shape) or t.dtype != Q.dtype or t.device != Q.device:
            raise ValueError("%s must match Q in shape, dtype and device" % name)
    if conv_w is not None:
        if (conv_w.dtype != torch.float32 or bool(conv_w.is_cuda) != on_cuda
                or not conv_w.is_contiguous() or conv_w.device != Q.device):
            raise ValueError("conv_w must be a contiguous float32 %s tensor [heads, k] on "
                             "the device of Q" % where)
        if conv_w.dim() != 2 or conv_w.shape[0] != Q.shape[1]:
            raise ValueError("conv_w must be [heads, k]")


def _on_device(dev):
    """The current-device context for a CUDA device (nothing to do when it
    is already current, which keeps graph capture untouched)."""
    import contextlib
    torch = _torch()
    if dev.index is None or dev.index == torch.cuda.current_device():
        return contextlib.nullcontext()
    return torch.cuda.device(dev)


def _stream_ptr(stream):
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


class Workspace:
    """A device workspace sized for one shape, reusable across calls."""

    def __init__(self, Q, num_landmarks):
        torch = _torch()
        self.desc = desc_of(Q)
        self.num_landmarks = int(num_landmarks)
        self.nbytes = nys_attn_workspace_size(self.desc, num_landmarks)
        # +256 so that the start can be rounded up to a 256-byte boundary
        self.buf = torch.empty(max(self.nbytes, 1) + 256, dtype=torch.uint8, device=Q.device)
        base = self.buf.data_ptr()
        self.offset = (-base) % 256
        self.ptr = base + self.offset

    def region(self, name, shape):
        """A float32 view of one intermediate (see nys_attn_intermediates)."""
        torch = _torch()
        lay = nys_attn_intermediates(self.desc, self.num_landmarks)
        count = 1
        for s in shape:
            count *= s
        start = self.offset + lay[name]
        return self.buf[start:start + 4 * count].view(torch.float32).view(*shape)


def nys_attn_forward(Q, K, V, num_landmarks, pinv_iters=6, conv_w=None, out=None,
                     workspace=None, stream=None):
    """out = F~ (Z (B~ V)) + DConv(V) for [batch, heads, n, d] CUDA tensors
    (float32 or bfloat16, contiguous).  conv_w: [heads, k] float32 CUDA tensor
    or None.  workspace: a Workspace for this shape, or None (the library then
    allocates one stream-ordered per call).  Asynchronous on `stream`."""
    torch = _torch()
    if out is None and getattr(Q, "is_cuda", False):
        out = torch.empty_like(Q)
    _check_operands(Q, K, V, Q if out is None else out, conv_w)
    desc = desc_of(Q)
    conv_ptr, conv_k = None, 0
    if conv_w is not None:
        conv_ptr, conv_k = conv_w.data_ptr(), conv_w.shape[1]
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = workspace.ptr, workspace.nbytes
    with _on_device(Q.device):
        st = _lib.raw_forward(Q.data_ptr(), K.data_ptr(), V.data_ptr(), desc, num_landmarks,
                              pinv_iters, conv_ptr, conv_k, out.data_ptr(), ws_ptr, ws_bytes,
                              _stream_ptr(stream))
    _lib.check(st, "nys_attn_forward")
    return out


def nys_attn_layer_forward(X, Wqkv, Wo, heads, num_landmarks, pinv_iters=6, conv_w=None,
                           workspace=None, stream=None):
    """The attention layer: Y = concat_h(forward(X Wq_h^T, X Wk_h^T, X Wv_h^T)) Wo^T for
    X [batch, n, D] bf16 (D = heads * 64), Wqkv [3D, D], Wo [D, D] bf16 CUDA tensors.
    workspace: a CUDA uint8 tensor of at least nys_attn_layer_workspace_size bytes
    (+256 for alignment), or None (allocated here).  Returns (Y, workspace_view): the
    view holds Q, K, V and the attention output (bf16, [batch, heads, n, 64] each) at
    its start."""
    torch = _torch()
    if X.dim() != 3 or X.dtype != torch.bfloat16 or not X.is_cuda or not X.is_contiguous():
        raise ValueError("X must be a contiguous bfloat16 CUDA tensor [batch, n, D]")
    B, n, D = X.shape
    if D != heads * 64:
        raise ValueError("D must be heads * 64")
    for name, w, shape in (("Wqkv", Wqkv, (3 * D, D)), ("Wo", Wo, (D, D))):
        if (tuple(w.shape) != shape or w.dtype != torch.bfloat16 or w.device != X.device
                or not w.is_contiguous()):
            raise ValueError("%s must be a contiguous bfloat16 tensor %s on X's device"
                             % (name, shape))
    if conv_w is not None:
        if (conv_w.dtype != torch.float32 or conv_w.device != X.device or conv_w.dim() != 2
                or conv_w.shape[0] != heads or not conv_w.is_contiguous()):
            raise ValueError("conv_w must be a contiguous float32 [heads, k] tensor on X's device")
    desc = make_desc(NYS_BF16, B, heads, n, 64)
    nb = _lib.nys_attn_layer_workspace_size(desc, num_landmarks)
    if workspace is None:
        workspace = torch.empty(nb + 256, dtype=torch.uint8, device=X.device)
    base = workspace.data_ptr()
    off = (-base) % 256
    if workspace.numel() - off < nb or workspace.device != X.device:
        raise ValueError("workspace too small or on another device")
    Y = torch.empty_like(X)
    conv_ptr, conv_k = (None, 0) if conv_w is None else (conv_w.data_ptr(), conv_w.shape[1])
    with _on_device(X.device):
        st = _lib.raw_layer_forward(X.data_ptr(), Wqkv.data_ptr(), Wo.data_ptr(), desc,
                                    num_landmarks, pinv_iters, conv_ptr, conv_k, Y.data_ptr(),
                                    base + off, nb, _stream_ptr(stream))
    _lib.check(st, "nys_attn_layer_forward")
    return Y, workspace[off:off + nb]


def nys_attn_layer_check_error(workspace_view, heads, batch, n, num_landmarks, stream=None):
    """Synchronises and raises if a layer kernel recorded an error."""
    desc = make_desc(NYS_BF16, batch, heads, n, 64)
    st = _lib.raw_layer_check_error(workspace_view.data_ptr(), desc, num_landmarks,
                                    _stream_ptr(stream))
    _lib.check(st, "nys_attn_layer_check_error")


def nys_attn_backward(Q, K, V, num_landmarks, dO, pinv_iters=6, conv_w=None, workspace=None,
                      stream=None):
    """Gradients of the forward with respect to Q, K, V (and conv_w) given
    dO = dL/dout: returns (dQ, dK, dV, dconv) with dconv None without the
    conv skip.  workspace: a CUDA uint8 tensor of at least
    nys_attn_backward_workspace_size bytes, or None (the library allocates
    one stream-ordered per call)."""
    torch = _torch()
    _check_operands(Q, K, V, dO, conv_w)
    desc = desc_of(Q)
    dQ, dK, dV = torch.empty_like(Q), torch.empty_like(Q), torch.empty_like(Q)
    conv_ptr, conv_k, dconv = None, 0, None
    if conv_w is not None:
        conv_ptr, conv_k = conv_w.data_ptr(), conv_w.shape[1]
        dconv = torch.empty_like(conv_w)
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        if not workspace.is_cuda or workspace.device != Q.device:
            raise ValueError("workspace must be a CUDA tensor on Q's device")
        ws_ptr = workspace.data_ptr() + (-workspace.data_ptr()) % 256
        ws_bytes = workspace.numel() * workspace.element_size() - (ws_ptr - workspace.data_ptr())
    with _on_device(Q.device):
        st = _lib.raw_backward(Q.data_ptr(), K.data_ptr(), V.data_ptr(), desc, num_landmarks,
                               pinv_iters, conv_ptr, conv_k, dO.data_ptr(), dQ.data_ptr(),
                               dK.data_ptr(), dV.data_ptr(),
                               dconv.data_ptr() if dconv is not None else None, ws_ptr,
                               ws_bytes, _stream_ptr(stream))
    _lib.check(st, "nys_attn_backward")
    return dQ, dK, dV, dconv


def nys_attn_forward_lens(Q, K, V, num_landmarks, lens, pinv_iters=6, conv_w=None, out=None,
                          workspace=None, stream=None):
    """nys_attn_forward on right-padded ragged batches: element b holds
    lens[b] real tokens (lens: int32 CUDA tensor [batch]); its output rows
    from lens[b] on are zero.  See nys_attn_forward_lens in the header."""
    torch = _torch()
    if out is None and getattr(Q, "is_cuda", False):
        out = torch.empty_like(Q)
    _check_operands(Q, K, V, Q if out is None else out, conv_w)
    if (not lens.is_cuda or lens.dtype != torch.int32 or not lens.is_contiguous()
            or lens.dim() != 1 or lens.shape[0] != Q.shape[0] or lens.device != Q.device):
        raise ValueError("lens must be a contiguous int32 CUDA tensor [batch] on Q's device")
    desc = desc_of(Q)
    conv_ptr, conv_k = (None, 0) if conv_w is None else (conv_w.data_ptr(), conv_w.shape[1])
    ws_ptr, ws_bytes = (None, 0) if workspace is None else (workspace.ptr, workspace.nbytes)
    with _on_device(Q.device):
        st = _lib.raw_forward_lens(Q.data_ptr(), K.data_ptr(), V.data_ptr(), desc,
                                   num_landmarks, pinv_iters, conv_ptr, conv_k, lens.data_ptr(),
                                   out.data_ptr(), ws_ptr, ws_bytes, _stream_ptr(stream))
    _lib.check(st, "nys_attn_forward_lens")
    return out


def nys_attn_forward_timed(Q, K, V, num_landmarks, pinv_iters, conv_w, out, workspace, events,
                           stream=None):
    """nys_attn_forward recording events[0] before the first kernel and
    events[i + 1] after kernel i (torch.cuda.Event objects with timing)."""
    _check_operands(Q, K, V, out, conv_w)
    desc = desc_of(Q)
    conv_ptr, conv_k = (None, 0) if conv_w is None else (conv_w.data_ptr(), conv_w.shape[1])
    for e in events:
        if not e.cuda_event:          # torch creates the CUDA event on first record
            e.record()
    with _on_device(Q.device):
        st = _lib.raw_forward_timed(Q.data_ptr(), K.data_ptr(), V.data_ptr(), desc,
                                    num_landmarks, pinv_iters, conv_ptr, conv_k, out.data_ptr(),
                                    workspace.ptr, workspace.nbytes, _stream_ptr(stream),
                                    [e.cuda_event for e in events])
    _lib.check(st, "nys_attn_forward_timed")
    return out


def nys_attn_check_error(workspace, stream=None):
    """Synchronises the stream and raises if a kernel recorded an error."""
    st = _lib.raw_check_error(workspace.ptr, workspace.desc, workspace.num_landmarks,
                              _stream_ptr(stream))
    _lib.check(st, "nys_attn_check_error")


def nys_attn_forward_host(Qh, Kh, Vh, num_landmarks, pinv_iters, conv_w_host, out_host,
                          device_buf, stream=None):
    """End-to-end call on HOST tensors (CPU, contiguous, ideally pinned):
    host->device copies, the forward, and the device->host copy of the output,
    all enqueued on `stream`.  device_buf: a CUDA uint8 tensor of at least
    nys_attn_host_buffer_size bytes (256-byte aligned).  Returns out_host;
    synchronise the stream before reading it."""
    _check_operands(Qh, Kh, Vh, out_host, conv_w_host, on_cuda=False)
    if not device_buf.is_cuda or not device_buf.is_contiguous():
        raise ValueError("device_buf must be a contiguous CUDA tensor")
    desc = desc_of(Qh)
    conv_ptr, conv_k = None, 0
    if conv_w_host is not None:
        conv_ptr, conv_k = conv_w_host.data_ptr(), conv_w_host.shape[1]
    with _on_device(device_buf.device):
        st = _lib.raw_forward_host(Qh.data_ptr(), Kh.data_ptr(), Vh.data_ptr(), desc,
                                   num_landmarks, pinv_iters, conv_ptr, conv_k,
                                   out_host.data_ptr(), device_buf.data_ptr(),
                                   device_buf.numel() * device_buf.element_size(),
                                   _stream_ptr(stream))
    _lib.check(st, "nys_attn_forward_host")
    return out_host
