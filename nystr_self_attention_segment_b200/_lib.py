"""ctypes binding of the C ABI in include/nys_attn.h.

Argument marshalling only: every step of the forward pass runs in the CUDA
kernels of libnys_attn.so.  There is no fallback: if the library is missing,
every call raises."""

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libnys_attn.so")

NYS_F32 = 0
NYS_BF16 = 1

STATUS_NAMES = {
    0: "NYS_OK",
    1: "NYS_ERR_INVALID_ARG",
    2: "NYS_ERR_UNSUPPORTED",
    3: "NYS_ERR_NOT_DIVISIBLE",
    4: "NYS_ERR_ALIAS",
    5: "NYS_ERR_WORKSPACE",
    6: "NYS_ERR_CUDA",
    7: "NYS_ERR_TIMEOUT",
}
STATUS = {v: k for k, v in STATUS_NAMES.items()}

# Every entry point include/nys_attn.h declares.
EXPORTS = (
    "nys_status_string",
    "nys_version",
    "nys_attn_workspace_size",
    "nys_attn_forward",
    "nys_attn_intermediates",
    "nys_attn_check_error",
    "nys_attn_host_buffer_size",
    "nys_attn_forward_host",
    "nys_attn_launch_count",
    "nys_attn_forward_timed",
    "nys_attn_launch_names",
    "nys_attn_forward_static",
    "nys_attn_check_error_static",
    "nys_attn_forward_lens",
    "nys_attn_backward_workspace_size",
    "nys_attn_backward",
    "nys_attn_layer_workspace_size",
    "nys_attn_layer_forward",
    "nys_attn_layer_check_error",
)

# Size of the fixed scratch array of nys_attn_forward_static (see the header).
NYS_STATIC_SCRATCH_BYTES = 8 << 20


class NysError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        self.name = STATUS_NAMES.get(status, "status %d" % status)
        msg = _LIB.nys_status_string(status).decode() if _LIB is not None else self.name
        super().__init__("%s: %s" % (where, msg))


class nys_desc(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("batch", ctypes.c_int), ("heads", ctypes.c_int),
                ("seq_len", ctypes.c_int), ("head_dim", ctypes.c_int)]


class nys_intermediates(ctypes.Structure):
    _fields_ = [("q_landmarks", ctypes.c_size_t), ("k_landmarks", ctypes.c_size_t),
                ("z", ctypes.c_size_t), ("y", ctypes.c_size_t), ("w", ctypes.c_size_t),
                ("error_word", ctypes.c_size_t), ("total", ctypes.c_size_t)]


_LIB = None


def load():
    """Loads libnys_attn.so (once).  Raises if it has not been built."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libnys_attn.so is not built (python -m "
                           "nystr_self_attention_segment_b200.build); there is no fallback")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    D = ctypes.POINTER(nys_desc)
    lib.nys_status_string.restype = ctypes.c_char_p
    lib.nys_status_string.argtypes = [I]
    lib.nys_version.restype = I
    lib.nys_version.argtypes = []
    lib.nys_attn_workspace_size.restype = I
    lib.nys_attn_workspace_size.argtypes = [D, I, ctypes.POINTER(S)]
    lib.nys_attn_forward.restype = I
    lib.nys_attn_forward.argtypes = [P, P, P, D, I, I, P, I, P, P, S, P]
    lib.nys_attn_intermediates.restype = I
    lib.nys_attn_intermediates.argtypes = [D, I, ctypes.POINTER(nys_intermediates)]
    lib.nys_attn_check_error.restype = I
    lib.nys_attn_check_error.argtypes = [P, D, I, P]
    lib.nys_attn_host_buffer_size.restype = I
    lib.nys_attn_host_buffer_size.argtypes = [D, I, I, ctypes.POINTER(S)]
    lib.nys_attn_forward_host.restype = I
    lib.nys_attn_forward_host.argtypes = [P, P, P, D, I, I, P, I, P, P, S, P]
    lib.nys_attn_launch_count.restype = I
    lib.nys_attn_launch_count.argtypes = [D, I, I, ctypes.POINTER(I)]
    lib.nys_attn_forward_timed.restype = I
    lib.nys_attn_forward_timed.argtypes = [P, P, P, D, I, I, P, I, P, P, S, P,
                                           ctypes.POINTER(P), I]
    lib.nys_attn_launch_names.restype = I
    lib.nys_attn_launch_names.argtypes = [D, I, ctypes.c_char_p, S]
    lib.nys_attn_forward_static.restype = I
    lib.nys_attn_forward_static.argtypes = [P, P, P, D, I, I, P, I, P, P]
    lib.nys_attn_check_error_static.restype = I
    lib.nys_attn_check_error_static.argtypes = [D, I, P]
    lib.nys_attn_backward_workspace_size.restype = I
    lib.nys_attn_backward_workspace_size.argtypes = [D, I, I, I, ctypes.POINTER(S)]
    lib.nys_attn_backward.restype = I
    lib.nys_attn_backward.argtypes = [P, P, P, D, I, I, P, I, P, P, P, P, P, P, S, P]
    lib.nys_attn_layer_workspace_size.restype = I
    lib.nys_attn_layer_workspace_size.argtypes = [D, I, ctypes.POINTER(S)]
    lib.nys_attn_layer_forward.restype = I
    lib.nys_attn_layer_forward.argtypes = [P, P, P, D, I, I, P, I, P, P, S, P]
    lib.nys_attn_layer_check_error.restype = I
    lib.nys_attn_layer_check_error.argtypes = [P, D, I, P]
    lib.nys_attn_forward_lens.restype = I
    lib.nys_attn_forward_lens.argtypes = [P, P, P, D, I, I, P, I, P, P, P, S, P]
    _LIB = lib
    return lib


def make_desc(dtype, batch, heads, seq_len, head_dim):
    return nys_desc(int(dtype), int(batch), int(heads), int(seq_len), int(head_dim))


def check(status, where):
    if status != 0:
        raise NysError(status, where)


def nys_status_string(status):
    return load().nys_status_string(int(status)).decode()


def nys_version():
    return load().nys_version()


def nys_attn_workspace_size(desc, num_landmarks):
    out = ctypes.c_size_t(0)
    check(load().nys_attn_workspace_size(ctypes.byref(desc), int(num_landmarks),
                                         ctypes.byref(out)), "nys_attn_workspace_size")
    return out.value


def nys_attn_intermediates(desc, num_landmarks):
    out = nys_intermediates()
    check(load().nys_attn_intermediates(ctypes.byref(desc), int(num_landmarks),
                                        ctypes.byref(out)), "nys_attn_intermediates")
    return {f: getattr(out, f) for f, _ in nys_intermediates._fields_}


def nys_attn_host_buffer_size(desc, num_landmarks, conv_k):
    out = ctypes.c_size_t(0)
    check(load().nys_attn_host_buffer_size(ctypes.byref(desc), int(num_landmarks), int(conv_k),
                                           ctypes.byref(out)), "nys_attn_host_buffer_size")
    return out.value


def nys_attn_launch_count(desc, num_landmarks, conv_k):
    out = ctypes.c_int(0)
    check(load().nys_attn_launch_count(ctypes.byref(desc), int(num_landmarks), int(conv_k),
                                       ctypes.byref(out)), "nys_attn_launch_count")
    return out.value


def raw_forward(q_ptr, k_ptr, v_ptr, desc, num_landmarks, pinv_iters, conv_ptr, conv_k,
                out_ptr, ws_ptr, ws_bytes, stream_ptr):
    """nys_attn_forward on raw addresses; returns the status code."""
    return load().nys_attn_forward(q_ptr, k_ptr, v_ptr, ctypes.byref(desc), int(num_landmarks),
                                   int(pinv_iters), conv_ptr, int(conv_k), out_ptr, ws_ptr,
                                   ctypes.c_size_t(ws_bytes), stream_ptr)


def nys_attn_launch_names(desc, num_landmarks):
    buf = ctypes.create_string_buffer(512)
    check(load().nys_attn_launch_names(ctypes.byref(desc), int(num_landmarks), buf, 512),
          "nys_attn_launch_names")
    return [s for s in buf.value.decode().split(",") if s]


def raw_forward_timed(q_ptr, k_ptr, v_ptr, desc, num_landmarks, pinv_iters, conv_ptr, conv_k,
                      out_ptr, ws_ptr, ws_bytes, stream_ptr, event_handles):
    """nys_attn_forward_timed; event_handles: list of cudaEvent_t addresses."""
    arr = (ctypes.c_void_p * len(event_handles))(*event_handles)
    return load().nys_attn_forward_timed(q_ptr, k_ptr, v_ptr, ctypes.byref(desc),
                                         int(num_landmarks), int(pinv_iters), conv_ptr,
                                         int(conv_k), out_ptr, ws_ptr, ctypes.c_size_t(ws_bytes),
                                         stream_ptr, arr, len(event_handles))


def raw_forward_host(q_ptr, k_ptr, v_ptr, desc, num_landmarks, pinv_iters, conv_ptr, conv_k,
                     out_ptr, dbuf_ptr, dbuf_bytes, stream_ptr):
    return load().nys_attn_forward_host(q_ptr, k_ptr, v_ptr, ctypes.byref(desc),
                                        int(num_landmarks), int(pinv_iters), conv_ptr,
                                        int(conv_k), out_ptr, dbuf_ptr,
                                        ctypes.c_size_t(dbuf_bytes), stream_ptr)


def raw_forward_static(q_ptr, k_ptr, v_ptr, desc, num_landmarks, pinv_iters, conv_ptr, conv_k,
                       out_ptr, stream_ptr):
    """nys_attn_forward_static: no workspace, no allocation."""
    return load().nys_attn_forward_static(q_ptr, k_ptr, v_ptr, ctypes.byref(desc),
                                          int(num_landmarks), int(pinv_iters), conv_ptr,
                                          int(conv_k), out_ptr, stream_ptr)


def raw_forward_lens(q_ptr, k_ptr, v_ptr, desc, num_landmarks, pinv_iters, conv_ptr, conv_k,
                     lens_ptr, out_ptr, ws_ptr, ws_bytes, stream_ptr):
    """nys_attn_forward_lens on raw addresses (lens_ptr: device int32 [batch])."""
    return load().nys_attn_forward_lens(q_ptr, k_ptr, v_ptr, ctypes.byref(desc),
                                        int(num_landmarks), int(pinv_iters), conv_ptr,
                                        int(conv_k), lens_ptr, out_ptr, ws_ptr,
                                        ctypes.c_size_t(ws_bytes), stream_ptr)


def nys_attn_backward_workspace_size(desc, num_landmarks, pinv_iters, conv_k):
    out = ctypes.c_size_t(0)
    check(load().nys_attn_backward_workspace_size(ctypes.byref(desc), int(num_landmarks),
                                                  int(pinv_iters), int(conv_k),
                                                  ctypes.byref(out)),
          "nys_attn_backward_workspace_size")
    return out.value


def raw_backward(q_ptr, k_ptr, v_ptr, desc, num_landmarks, pinv_iters, conv_ptr, conv_k, do_ptr,
                 dq_ptr, dk_ptr, dv_ptr, dconv_ptr, ws_ptr, ws_bytes, stream_ptr):
    """nys_attn_backward on raw addresses; returns the status code."""
    return load().nys_attn_backward(q_ptr, k_ptr, v_ptr, ctypes.byref(desc), int(num_landmarks),
                                    int(pinv_iters), conv_ptr, int(conv_k), do_ptr, dq_ptr,
                                    dk_ptr, dv_ptr, dconv_ptr, ws_ptr, ctypes.c_size_t(ws_bytes),
                                    stream_ptr)


def nys_attn_layer_workspace_size(desc, num_landmarks):
    out = ctypes.c_size_t(0)
    check(load().nys_attn_layer_workspace_size(ctypes.byref(desc), int(num_landmarks),
                                               ctypes.byref(out)), "nys_attn_layer_workspace_size")
    return out.value


def raw_layer_forward(x_ptr, wqkv_ptr, wo_ptr, desc, num_landmarks, pinv_iters, conv_ptr, conv_k,
                      y_ptr, ws_ptr, ws_bytes, stream_ptr):
    return load().nys_attn_layer_forward(x_ptr, wqkv_ptr, wo_ptr, ctypes.byref(desc),
                                         int(num_landmarks), int(pinv_iters), conv_ptr,
                                         int(conv_k), y_ptr, ws_ptr, ctypes.c_size_t(ws_bytes),
                                         stream_ptr)


def raw_layer_check_error(ws_ptr, desc, num_landmarks, stream_ptr):
    return load().nys_attn_layer_check_error(ws_ptr, ctypes.byref(desc), int(num_landmarks),
                                             stream_ptr)


def raw_check_error_static(desc, num_landmarks, stream_ptr):
    return load().nys_attn_check_error_static(ctypes.byref(desc), int(num_landmarks), stream_ptr)


def raw_check_error(ws_ptr, desc, num_landmarks, stream_ptr):
    return load().nys_attn_check_error(ws_ptr, ctypes.byref(desc), int(num_landmarks),
                                       stream_ptr)
