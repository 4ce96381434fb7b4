/*
 * nys_attn.h -- C ABI of the B200 (sm_100a) Nystromformer attention forward.
 *
 * The library computes, for every (batch, head) pair of [B, H, n, d] inputs,
 *
 *     out = F~ (Z (B~ V)) + DConv(V)
 *
 * where (notation of "Nystromformer: A Nystrom-Based Algorithm for
 * Approximating Self-Attention", section 3.4, and of the blog post
 * "Approximating self-attention in linear time and memory via the Nystrom
 * method"):
 *   Q~, K~  segment means of Q, K over l = ceil(n/m) contiguous tokens
 *           (Eq. 16, with the page's own divide-by-l correction; blog "How do
 *           we select landmarks?").  When m does not divide n the sequence
 *           reads as padded to m*l tokens ("can be ensured by padding"): the
 *           last segment is shorter and each landmark is the mean over the
 *           real tokens of its segment, so no pad value enters,
 *   F~      = softmax(Q K~^T / sqrt(d)), n x m, softmax over the m landmarks,
 *   A       = softmax(Q~ K~^T / sqrt(d)), m x m, row-wise,
 *   Z       = pinv_iters steps of Lemma 1 from Z0 = A^T / (||A||_1 ||A||_inf)
 *             ("Moore-Penrose Pseudoinverse Computation"),
 *   B~      = softmax(Q~ K^T / sqrt(d)), m x n, softmax over the n keys,
 *   DConv   depthwise 1-D cross-correlation of V along the sequence with one
 *           odd-length kernel per head, shared by the d features, zero "same"
 *           padding (Figure 4 "DConv k x 1"; blog "DConv box"),
 * and the n x n attention matrix is never formed (Eq. 17 / Algorithm 1).
 *
 * Conventions for every entry point:
 *  - Tensors Q, K, V, out are [batch][heads][seq_len][head_dim], contiguous,
 *    row-major, all of the dtype in the descriptor; out has the same dtype.
 *  - Pointers named *_dev are CUDA device pointers; *_host are host pointers.
 *    The caller owns every buffer and the library never frees caller memory.
 *    The only global mutable state is the fixed scratch array of
 *    nys_attn_forward_static (used by that entry point alone).
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and never synchronise the device.  Arguments are validated on the
 *    host before anything is enqueued: an invalid call returns a status and
 *    launches nothing.  Each launch is checked as it is made: a launch that
 *    the runtime refuses returns NYS_ERR_CUDA at once and no later kernel of
 *    the call is enqueued (kernels enqueued before it stay enqueued).
 *  - Results are bitwise reproducible run to run (fixed-order reductions, no
 *    floating-point atomics).
 *  - batch * heads * seq_len == 0 is valid and enqueues nothing.
 *
 * Supported shapes:
 *  - NYS_F32:  1 <= head_dim <= 64, 1 <= m <= 64, m <= seq_len.
 *  - NYS_BF16: head_dim == 64, m in {32, 64, 128}, m <= seq_len.
 *  - Every segment holds at least one token: (m - 1) * ceil(seq_len / m) <
 *    seq_len (always true when m divides seq_len or seq_len >= m * m).
 *  - conv_k odd, 1 <= conv_k <= 63 (or conv_w == NULL / conv_k == 0: no skip).
 *  - 0 <= pinv_iters <= 64.
 *  - batch * heads <= 65535, seq_len <= 2^24 (else NYS_ERR_UNSUPPORTED).
 */
#ifndef NYS_ATTN_H
#define NYS_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define NYS_ATTN_API __attribute__((visibility("default")))

typedef enum {
  NYS_OK = 0,
  NYS_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad enum value      */
  NYS_ERR_UNSUPPORTED = 2,   /* valid request without a kernel (d, m, dtype, k)  */
  NYS_ERR_NOT_DIVISIBLE = 3, /* a segment of ceil(seq_len/m) tokens would be empty */
  NYS_ERR_ALIAS = 4,         /* out overlaps Q, K, V or the workspace            */
  NYS_ERR_WORKSPACE = 5,     /* workspace smaller than nys_attn_workspace_size   */
  NYS_ERR_CUDA = 6,          /* a CUDA runtime call or kernel launch failed      */
  NYS_ERR_TIMEOUT = 7        /* a bounded on-device wait gave up (see below)     */
} nys_status;

typedef enum { NYS_F32 = 0, NYS_BF16 = 1 } nys_dtype;

/* Shape of the [batch][heads][seq_len][head_dim] inputs. */
typedef struct {
  int dtype; /* nys_dtype */
  int batch;
  int heads;
  int seq_len;
  int head_dim;
} nys_desc;

/* A cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st *nys_stream_t;

/* Human-readable name of a status code (static string, never NULL). */
NYS_ATTN_API const char *nys_status_string(nys_status status);

/* Library version as 10000*major + 100*minor + patch. */
NYS_ATTN_API int nys_version(void);

/* Bytes of device workspace nys_attn_forward needs for this shape.  Writes
 * *bytes; returns the same validation status nys_attn_forward would for the
 * shape part of its arguments. */
NYS_ATTN_API nys_status nys_attn_workspace_size(const nys_desc *desc, int num_landmarks,
                                                size_t *bytes);

/* The forward pass (Eq. 17 / Algorithm 1 with the Figure 4 DConv skip of the
 * paper summary).
 *   Q_dev, K_dev, V_dev  inputs, layout above; 16-byte aligned for NYS_BF16,
 *                        4-byte aligned for NYS_F32 (else NYS_ERR_INVALID_ARG).
 *   num_landmarks        m; segments of ceil(seq_len / m) tokens, the last one
 *                        possibly shorter, none empty (see Supported shapes).
 *   pinv_iters           steps of Lemma 1 (the paper uses 6).
 *   conv_w_dev           [heads][conv_k] fp32 kernel of the DConv skip, 4-byte
 *                        aligned, or NULL for no skip (then conv_k is ignored).
 *   out_dev              output, same dtype, layout and alignment as Q; must
 *                        not overlap any input or the workspace.
 *   workspace_dev        device scratch of at least nys_attn_workspace_size
 *                        bytes, 256-byte aligned, or NULL: then the call
 *                        allocates and frees it stream-ordered
 *                        (cudaMallocAsync / cudaFreeAsync on `stream`).
 * The workspace holds the per-head intermediates afterwards (see
 * nys_attn_intermediates) until the next call reuses it.
 * NYS_ERR_TIMEOUT is reserved for kernels that wait on other blocks of the
 * same launch; every such wait is bounded and reports through the workspace
 * error word, read back by nys_attn_check_error. */
NYS_ATTN_API nys_status nys_attn_forward(const void *Q_dev, const void *K_dev, const void *V_dev,
                                         const nys_desc *desc, int num_landmarks, int pinv_iters,
                                         const float *conv_w_dev, int conv_k, void *out_dev,
                                         void *workspace_dev, size_t workspace_bytes,
                                         nys_stream_t stream);

/* nys_attn_forward on right-padded ragged batches: element b holds
 * lens_dev[b] real tokens followed by padding, and is computed as the method
 * on its first lens_dev[b] tokens alone.  The pages describe no mask (every
 * token attends to every token) and make divisibility a matter of padding
 * ("Landmark Selection: Segment-Means"); this is that reading for a caller
 * with ragged batches:
 *   - landmarks are the segment means over the element's L = lens_dev[b]
 *     tokens (segments of ceil(L / m) tokens, the last one possibly shorter),
 *   - B~'s softmax runs over its L keys and F~ over its L queries,
 *   - the DConv skip pads with zeros from row L on,
 *   - output rows L .. seq_len - 1 are zero.
 *   lens_dev   device array of `batch` int32, 4-byte aligned; each
 *              m <= L <= seq_len with no empty segment ((m - 1) * ceil(L/m) <
 *              L).  A length that breaks this records NYS_ERR_INVALID_ARG in
 *              the workspace error word (nys_attn_check_error) and its
 *              element's output is all zero; the other elements are computed.
 * Every other argument, the workspace size and the error behaviour are those
 * of nys_attn_forward; lens_dev == NULL (with a non-empty problem) is
 * NYS_ERR_INVALID_ARG.  With every L = seq_len the result equals
 * nys_attn_forward's. */
NYS_ATTN_API nys_status nys_attn_forward_lens(const void *Q_dev, const void *K_dev,
                                              const void *V_dev, const nys_desc *desc,
                                              int num_landmarks, int pinv_iters,
                                              const float *conv_w_dev, int conv_k,
                                              const int *lens_dev, void *out_dev,
                                              void *workspace_dev, size_t workspace_bytes,
                                              nys_stream_t stream);

/* The attention layer around the forward: the projections of "Standard
 * Self-Attention: The Mathematical Baseline" (Q = X W_Q, K = X W_K,
 * V = X W_V) and an output projection, with the forward in between
 * (Figure 4 takes the layer input X):
 *   Y = concat_h( forward(Q_h, K_h, V_h) ) Wo^T
 * NYS_BF16 and head_dim 64 only; D = heads * 64.
 *   X_dev     [batch][seq_len][D] bf16, the layer input;
 *   Wqkv_dev  [3 D][D] bf16: rows 0 .. D-1 give Q, D .. 2D-1 K, 2D .. 3D-1 V
 *             (nn.Linear weight layout: output feature, input feature), head
 *             h takes features h*64 .. h*64 + 63 of each;
 *   Wo_dev    [D][D] bf16; Y_dev [batch][seq_len][D] bf16 (must not overlap
 *             X, the weights or the workspace);
 *   workspace_dev  nys_attn_layer_workspace_size bytes, 256-byte aligned
 *             (required): Q, K, V and the attention output in bf16, then the
 *             forward's workspace;
 * all pointers 16-byte aligned.  The projections are tensor-core GEMMs (fp32
 * accumulation, bf16 results); Q, K, V and the attention output are rounded
 * to bf16 between the steps.  A status a kernel records on the device is read
 * with nys_attn_layer_check_error.  (The pages' layer wraps the attention in
 * these projections; the library measures the attention itself.) */
NYS_ATTN_API nys_status nys_attn_layer_workspace_size(const nys_desc *desc, int num_landmarks,
                                                      size_t *bytes);
NYS_ATTN_API nys_status nys_attn_layer_forward(const void *X_dev, const void *Wqkv_dev,
                                               const void *Wo_dev, const nys_desc *desc,
                                               int num_landmarks, int pinv_iters,
                                               const float *conv_w_dev, int conv_k, void *Y_dev,
                                               void *workspace_dev, size_t workspace_bytes,
                                               nys_stream_t stream);
NYS_ATTN_API nys_status nys_attn_layer_check_error(void *workspace_dev, const nys_desc *desc,
                                                   int num_landmarks, nys_stream_t stream);

/* Backward pass ("Moore-Penrose Pseudoinverse Computation": gradients flow
 * through the iteration's matrix products like through any other layer):
 * given dO = dL/dout of the forward with the same arguments, writes
 *   dQ_dev, dK_dev, dV_dev   dL/dQ, dL/dK, dL/dV, same dtype, layout and
 *                            alignment as Q; must not overlap each other, the
 *                            inputs, dO or the workspace,
 *   dconv_w_dev              dL/dconv_w, [heads][conv_k] fp32 (summed over
 *                            the batch), non-NULL exactly when conv_w_dev is.
 * The forward's landmark steps are recomputed (A, every iterate of Lemma 1
 * and B~'s normaliser are kept in the workspace); the chain rule then runs
 * through the conv, F~ W, Z Y, B~ V, the three softmaxes (row-softmax
 * backward), each Lemma 1 step's products in reverse, Z0's norms (the
 * gradient goes to the maximising column and row) and the segment means.
 * Arithmetic is fp32 on the CUDA cores; for NYS_BF16 the gradients are
 * rounded to bf16 (dQ and dK twice: their first part, then the landmark
 * part added).
 *   workspace_dev            at least nys_attn_backward_workspace_size
 *                            bytes, 256-byte aligned, or NULL (allocated and
 *                            freed stream-ordered).
 * Shapes, validation, errors and determinism as for nys_attn_forward.  The
 * key-tile kernel runs beside the per-head kernel and waits, bounded, for
 * its dY; a wait that gives up writes NYS_ERR_TIMEOUT to the first 4 bytes
 * of the workspace (uint32, cleared by every call).  Ragged batches
 * (nys_attn_forward_lens) have no backward here. */
NYS_ATTN_API nys_status nys_attn_backward_workspace_size(const nys_desc *desc, int num_landmarks,
                                                         int pinv_iters, int conv_k,
                                                         size_t *bytes);
NYS_ATTN_API nys_status nys_attn_backward(const void *Q_dev, const void *K_dev,
                                          const void *V_dev, const nys_desc *desc,
                                          int num_landmarks, int pinv_iters,
                                          const float *conv_w_dev, int conv_k,
                                          const void *dO_dev, void *dQ_dev, void *dK_dev,
                                          void *dV_dev, float *dconv_w_dev,
                                          void *workspace_dev, size_t workspace_bytes,
                                          nys_stream_t stream);

/* Offsets (in bytes from the start of the workspace) of the fp32
 * intermediates a forward leaves there, for parity checks:
 *   q_landmarks, k_landmarks  [batch*heads][m][head_dim]   Q~, K~
 *   z                          [batch*heads][m][m]          Z after pinv_iters
 *   y                          [batch*heads][m][head_dim]   B~ V
 *   w                          [batch*heads][m][head_dim]   Z (B~ V)
 *   error_word                 one uint32: 0, or a nys_status a kernel set. */
typedef struct {
  size_t q_landmarks;
  size_t k_landmarks;
  size_t z;
  size_t y;
  size_t w;
  size_t error_word;
  size_t total;
} nys_intermediates;

NYS_ATTN_API nys_status nys_attn_intermediates(const nys_desc *desc, int num_landmarks,
                                               nys_intermediates *layout);

/* Synchronises `stream`, reads the workspace error word and clears it.
 * Returns NYS_OK or the status a kernel recorded (e.g. NYS_ERR_TIMEOUT). */
NYS_ATTN_API nys_status nys_attn_check_error(void *workspace_dev, const nys_desc *desc,
                                             int num_landmarks, nys_stream_t stream);

/* End-to-end variant on HOST buffers: copies Q, K, V (and conv_w) from host
 * memory into `device_buf`, runs the forward and copies the output back into
 * out_host, all enqueued on `stream` (asynchronous: synchronise the stream
 * before reading out_host; pinned host memory makes the copies truly async).
 *   Q_host, K_host, V_host  [batch][heads][seq_len][head_dim] of desc->dtype.
 *   conv_w_host             [heads][conv_k] fp32 or NULL.
 *   device_buf              device memory of at least
 *                           nys_attn_host_buffer_size bytes, 256-byte aligned,
 *                           owned by the caller (staging for the inputs,
 *                           output, conv weights and the workspace).
 * Bytes moved per call: 3*T in, T out (+ heads*conv_k*4 in), T = tensor size. */
NYS_ATTN_API nys_status nys_attn_host_buffer_size(const nys_desc *desc, int num_landmarks,
                                                  int conv_k, size_t *bytes);
NYS_ATTN_API nys_status nys_attn_forward_host(const void *Q_host, const void *K_host,
                                              const void *V_host, const nys_desc *desc,
                                              int num_landmarks, int pinv_iters,
                                              const float *conv_w_host, int conv_k,
                                              void *out_host, void *device_buf,
                                              size_t device_buf_bytes, nys_stream_t stream);

/* nys_attn_forward with per-kernel CUDA events for live timing: records
 * events[0] on `stream` before the first kernel and events[i + 1] right after
 * kernel i, for the nys_attn_launch_count kernels the call enqueues.  events
 * are caller-created cudaEvent_t handles (timing enabled); n_events must be
 * at least launches + 1, else NYS_ERR_INVALID_ARG.  Same results as
 * nys_attn_forward. */
NYS_ATTN_API nys_status nys_attn_forward_timed(const void *Q_dev, const void *K_dev,
                                               const void *V_dev, const nys_desc *desc,
                                               int num_landmarks, int pinv_iters,
                                               const float *conv_w_dev, int conv_k,
                                               void *out_dev, void *workspace_dev,
                                               size_t workspace_bytes, nys_stream_t stream,
                                               void *const *events, int n_events);

/* Size of the fixed device scratch array nys_attn_forward_static uses. */
#define NYS_STATIC_SCRATCH_BYTES (8u << 20)

/* nys_attn_forward without any device allocation: for callers that cannot
 * allocate device memory -- hosts that own the whole device memory pool and
 * forbid side allocations, paths where cudaMalloc's implicit device
 * synchronisation is not acceptable, code held to a memory budget fixed at
 * start-up.  (The paper has no counterpart; this is a deployment variant.)
 *
 * The scratch the forward needs (landmarks, Z, B~ V partials, W, error word
 * and counters) lives in one file-scope __device__ array of
 * NYS_STATIC_SCRATCH_BYTES in this library; every device that loads the
 * library holds it until the process exits.  The caller still passes the
 * inputs and the output (same arguments and layout as nys_attn_forward,
 * without the workspace).
 *  - A problem whose workspace (nys_attn_workspace_size) exceeds
 *    NYS_STATIC_SCRATCH_BYTES is rejected with NYS_ERR_WORKSPACE before
 *    anything is enqueued.
 *  - The array's device address is looked up (cudaGetSymbolAddress) with
 *    the device current on every call made outside stream capture, and
 *    remembered per CUDA context; a call made while `stream` is capturing
 *    uses the address remembered for the current context, so the first call
 *    in a context must come before any stream capture (else NYS_ERR_CUDA).
 *  - Every call on a device shares the one array, which keeps the last
 *    call's contents (the intermediates of nys_attn_intermediates, at the
 *    same offsets); what must start at zero is cleared by each call.  Calls
 *    that overlap on the GPU (different streams, or host threads without
 *    ordering) race on the array: order them.
 *  - A status a kernel records on the device (NYS_ERR_TIMEOUT) is read with
 *    nys_attn_check_error_static, before the next call clears it.
 *  - Never calls cudaMalloc, cudaFree or any allocating routine. */
NYS_ATTN_API nys_status nys_attn_forward_static(const void *Q_dev, const void *K_dev,
                                                const void *V_dev, const nys_desc *desc,
                                                int num_landmarks, int pinv_iters,
                                                const float *conv_w_dev, int conv_k,
                                                void *out_dev, nys_stream_t stream);

/* nys_attn_check_error for the scratch array of nys_attn_forward_static:
 * synchronises `stream`, reads the error word the last static call left for
 * this shape and clears it.  Returns NYS_OK or the recorded status;
 * NYS_ERR_WORKSPACE for a shape the array cannot hold.  Allocates nothing.
 * (No counterpart in the paper; it belongs to the deployment variant above.) */
NYS_ATTN_API nys_status nys_attn_check_error_static(const nys_desc *desc, int num_landmarks,
                                                    nys_stream_t stream);

/* Number of kernel launches one nys_attn_forward call enqueues for this
 * shape (0 for an empty problem), and a short name for each launch in
 * order, written as a comma-separated list into names (may be NULL). */
NYS_ATTN_API nys_status nys_attn_launch_count(const nys_desc *desc, int num_landmarks,
                                              int conv_k, int *launches);
NYS_ATTN_API nys_status nys_attn_launch_names(const nys_desc *desc, int num_landmarks,
                                              char *names, size_t names_bytes);

#ifdef __cplusplus
}
#endif

#endif /* NYS_ATTN_H */
