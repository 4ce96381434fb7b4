"""Plain fp64 CPU oracle of the Nystromformer attention forward pass.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or run
this module: only the tests, the smoke check and the CPU-baseline leg of the
benchmark do.  It shares no code with the CUDA kernels.

Every step is written in the order and notation of the pages it follows, one
(b, h) attention head at a time, with numpy fp64 arrays and numpy's matmul as
the only library primitive.  There is no blocking, fusion or reordering beyond
what the definitions state.

Sources (page title, then section / equation):
  [P1] "Approximating self-attention in linear time and memory via the Nystrom
       method" (blog post): "How can we adapt the Nystrom method to approximate
       self-attention?" (the three softmax matrices F~, A~, B~),
       "How do we select landmarks?" (segment means, DConv skip),
       "How is Nystromformer implemented?" (library excerpt: landmarks by
       reshape + mean, kernel_1/2/3, product order).
  [P5] "Nystromformer: A Nystrom-Based Algorithm for Approximating
       Self-Attention" (paper summary), section 3.4:
       "Moore-Penrose Pseudoinverse Computation" (Lemma 1, Z0 initialisation),
       "Landmark Selection: Segment-Means" (Eq. 16 and its normalisation note),
       "Putting It Together" (Eq. 17, Algorithm 1, Figure 4 with the DConv skip),
       "Theoretical Analysis" (Lemma 2), and section 3.2 (the five stages).

Readings where the pages are silent or inconsistent (each also listed in the
design notes):
  * Eq. 16 prints a divide-by-m; the page itself calls that a typo.  Landmark j
    is the mean of the l = n/m contiguous tokens [j*l, (j+1)*l).
  * When m does not divide n ("can be ensured by padding", no pad value given)
    the sequence is read as padded to m*ceil(n/m) tokens and each landmark is
    the mean over the real tokens of its segment of l = ceil(n/m); a shape
    with an empty segment is rejected.
  * Masks are not on the pages (every token attends to every token).  For
    right-padded ragged batches (nystrom_forward_lens) an element with L real
    tokens is the method on those L tokens alone, and its padding rows of
    the output are zero.
  * The 1/sqrt(d) scale is applied inside all three softmaxes (P1 definitions,
    P5 Algorithm 1); the library excerpt omits it for brevity.
  * B~ is a softmax over the n keys for every landmark row (P1 definitions,
    library excerpt softmax over the last axis).
  * The DConv skip is a depthwise 1-D cross-correlation along the sequence with
    one odd-length kernel w[h, :] per head, shared by the d features of that
    head, zero "same" padding, no bias.
  * The output uses Z after `iters` iterations, never the exact pseudoinverse.
  * Product order F~ (Z (B~ V)); equal in exact arithmetic to the pages' other
    orders.

Parity is pinned (see tests/test_oracle_pins.py) by: brute-force loops on tiny
inputs, the mean-of-landmarks invariant, softmax row sums, the SVD
pseudoinverse (numpy/LAPACK) at convergence, the closed-form one-step residual
of Lemma 1's recurrence, the exact fixed point for a uniform kernel, Lemma 2
(m = n) and the exactness on segment-constant Q/K against brute-force n x n
softmax attention, and numpy.correlate for the convolution.
"""

import numpy as np

__all__ = [
    "segment_means",
    "softmax_rows",
    "kernel_F",
    "kernel_A",
    "kernel_B",
    "pinv_init",
    "pinv_step",
    "iterative_pinv",
    "depthwise_conv",
    "nystrom_head",
    "nystrom_forward",
    "nystrom_forward_lens",
    "nystrom_head_backward",
    "nystrom_backward",
    "nystrom_layer_forward",
    "exact_attention_head",
    "exact_attention",
    "algorithmic_flops",
    "algorithmic_bytes",
]


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def segment_means(X, m):
    """Landmarks by segment means ([P5] "Landmark Selection: Segment-Means",
    Eq. 16 with the page's own 1/l correction; [P1] "How do we select
    landmarks?").

    X: [n, d].  Returns [m, d]: row j is the mean of the tokens of segment j,
    rows j*l .. min(j*l + l, n) - 1 with l = ceil(n / m).  When m divides n
    every segment holds l = n / m tokens, as on the pages.  Otherwise the
    sequence is read as padded to m * l tokens ("can be ensured by padding")
    and each landmark is the mean over the real tokens of its segment, so
    the pad value never enters.  Raises ValueError when a segment would hold
    no real token ((m - 1) * l >= n)."""
    X = _f64(X)
    n, d = X.shape
    if m < 1 or m > n:
        raise ValueError("segment_means needs 1 <= m <= n (n=%d, m=%d)" % (n, m))
    seg = -(-n // m)
    if (m - 1) * seg >= n:
        raise ValueError("segment_means: a segment of %d tokens would be empty (n=%d, m=%d)"
                         % (seg, n, m))
    out = np.empty((m, d), dtype=np.float64)
    for j in range(m):
        rows = X[j * seg:min((j + 1) * seg, n)]
        out[j] = rows.sum(axis=0) / rows.shape[0]
    return out


def softmax_rows(S):
    """Row-wise softmax.  The row maximum is subtracted first; that changes
    nothing mathematically and keeps exp() finite for peaky logits."""
    S = _f64(S)
    E = np.exp(S - S.max(axis=1, keepdims=True))
    return E / E.sum(axis=1, keepdims=True)


def kernel_F(Q, Kt, scale):
    """F~ = softmax(Q K~^T / sqrt(d)), n x m, softmax over the m landmarks
    ([P1] definitions of F~; [P5] Algorithm 1)."""
    return softmax_rows(_f64(Q) @ _f64(Kt).T * scale)


def kernel_A(Qt, Kt, scale):
    """softmax(Q~ K~^T / sqrt(d)), m x m, row-wise ([P1] definitions; [P5]
    section 3.2 stage 2a).  Its pseudoinverse is taken by iterative_pinv."""
    return softmax_rows(_f64(Qt) @ _f64(Kt).T * scale)


def kernel_B(Qt, K, scale):
    """B~ = softmax(Q~ K^T / sqrt(d)), m x n, softmax over the n keys of every
    landmark row ([P1] definitions; [P5] Algorithm 1)."""
    return softmax_rows(_f64(Qt) @ _f64(K).T * scale)


def pinv_init(A):
    """Z0 = A^T / (||A||_1 ||A||_inf) ([P5] "Moore-Penrose Pseudoinverse
    Computation", initialisation scheme).  ||A||_1 is the largest absolute
    column sum, ||A||_inf the largest absolute row sum."""
    A = _f64(A)
    norm_1 = np.abs(A).sum(axis=0).max()
    norm_inf = np.abs(A).sum(axis=1).max()
    return A.T / (norm_1 * norm_inf)


def pinv_step(A, Z):
    """One step of Lemma 1 ([P5] "Moore-Penrose Pseudoinverse Computation"):
    Z <- 1/4 Z (13 I - A Z (15 I - A Z (7 I - A Z)))."""
    A = _f64(A)
    Z = _f64(Z)
    I = np.eye(A.shape[0])
    AZ = A @ Z
    return 0.25 * (Z @ (13.0 * I - AZ @ (15.0 * I - AZ @ (7.0 * I - AZ))))


def iterative_pinv(A, iters, return_all=False):
    """Z after `iters` steps of Lemma 1 from Z0 ([P5] section 3.2 stage 3: six
    iterations in the paper's runs).  With return_all, the list Z0..Z_iters."""
    Z = pinv_init(A)
    allz = [Z]
    for _ in range(iters):
        Z = pinv_step(A, Z)
        allz.append(Z)
    return allz if return_all else Z


def depthwise_conv(V, w):
    """DConv skip on the values ([P1] "How do we select landmarks?" DConv box;
    [P5] Figure 4 "DConv k x 1").  V: [n, d]; w: [k], k odd, shared by the d
    features.  C[i, c] = sum_t w[t] V[i + t - (k-1)/2, c], V = 0 outside
    [0, n)."""
    V = _f64(V)
    w = _f64(w).reshape(-1)
    k = w.shape[0]
    if k % 2 != 1:
        raise ValueError("conv kernel length must be odd")
    n, d = V.shape
    half = (k - 1) // 2
    C = np.zeros((n, d), dtype=np.float64)
    for t in range(k):
        off = t - half                      # source row = i + off
        lo = max(0, -off)
        hi = min(n, n - off)
        if hi > lo:
            C[lo:hi] += w[t] * V[lo + off:hi + off]
    return C


def nystrom_head(Q, K, V, m, iters=6, w=None, scale=None):
    """One attention head of the Nystrom forward pass ([P5] Eq. 17 / Algorithm
    1 with the Figure 4 skip).  Returns a dict of every intermediate:
    Qt, Kt (landmarks), F (n x m), A (m x m), Z (after `iters` steps),
    B (m x n), Y = B V, W = Z Y, O = F W, C (conv skip or zeros), out = O + C."""
    Q = _f64(Q)
    K = _f64(K)
    V = _f64(V)
    n, d = Q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    Qt = segment_means(Q, m)
    Kt = segment_means(K, m)
    F = kernel_F(Q, Kt, scale)
    A = kernel_A(Qt, Kt, scale)
    Z = iterative_pinv(A, iters)
    B = kernel_B(Qt, K, scale)
    Y = B @ V
    W = Z @ Y
    O = F @ W
    C = depthwise_conv(V, w) if w is not None else np.zeros_like(V)
    return {"Qt": Qt, "Kt": Kt, "F": F, "A": A, "Z": Z, "B": B,
            "Y": Y, "W": W, "O": O, "C": C, "out": O + C}


def nystrom_forward(Q, K, V, m, iters=6, conv_w=None, keep=()):
    """Batched forward over [B, H, n, d] inputs, head by head.  conv_w is
    [H, k] (one kernel per head) or None for no skip.  Returns out [B, H, n, d]
    fp64 and, for each name in `keep`, that intermediate stacked to
    [B, H, ...]."""
    Q = _f64(Q)
    K = _f64(K)
    V = _f64(V)
    Bn, H, n, d = Q.shape
    out = np.empty((Bn, H, n, d), dtype=np.float64)
    kept = {name: [] for name in keep}
    for b in range(Bn):
        for h in range(H):
            w = None if conv_w is None else _f64(conv_w)[h]
            r = nystrom_head(Q[b, h], K[b, h], V[b, h], m, iters, w)
            out[b, h] = r["out"]
            for name in keep:
                kept[name].append(r[name])
    extra = {name: np.stack(v).reshape((Bn, H) + v[0].shape) for name, v in kept.items()}
    return (out, extra) if keep else out


def nystrom_forward_lens(Q, K, V, m, lens, iters=6, conv_w=None):
    """Forward over right-padded ragged batches: element b holds lens[b] real
    tokens followed by padding.  Each element is the method on its first
    lens[b] tokens alone (landmarks, the softmax over keys, the queries and
    the conv's zero padding all end at lens[b]); the padding rows of the
    output are zero.  Q, K, V: [B, H, n, d]; lens: B ints, m <= lens[b] <= n.
    Masks are not on the pages: this is the plainest reading for a caller
    with ragged batches."""
    Q = _f64(Q)
    K = _f64(K)
    V = _f64(V)
    Bn, H, n, d = Q.shape
    lens = [int(x) for x in lens]
    if len(lens) != Bn or any(L < m or L > n for L in lens):
        raise ValueError("lens must hold B values in [m, n]")
    out = np.zeros((Bn, H, n, d), dtype=np.float64)
    for b in range(Bn):
        L = lens[b]
        for h in range(H):
            w = None if conv_w is None else _f64(conv_w)[h]
            r = nystrom_head(Q[b, h, :L], K[b, h, :L], V[b, h, :L], m, iters, w)
            out[b, h, :L] = r["out"]
    return out


# ----------------------------------------------------------------- backward
#
# Gradients of one head's output with respect to Q, K, V and the conv kernel
# ([P5] "Moore-Penrose Pseudoinverse Computation", gradient computation:
# backpropagation runs through the iteration's matrix products like any other
# layer).  Each step below is the chain rule of one forward step, taken in
# reverse order.  Readings (not on the pages):
#   * softmax rows: dS = P * (dP - rowsum(dP * P)) (P the softmax, dP its
#     upstream gradient), times the 1/sqrt(d) scale for the logits' inputs;
#   * the two norms of Z0 are maxima of absolute sums: the gradient flows to
#     the maximising column / row (numpy.argmax order at ties), d|a|/da =
#     sign(a).  A row-softmax has every row sum 1, so the infinity-norm term
#     vanishes after the softmax backward whichever row is chosen.


def _softmax_rows_backward(P, dP):
    return P * (dP - (dP * P).sum(axis=1, keepdims=True))


def _segment_means_backward(dXt, n, m):
    """Gradient of segment_means: every token of segment j receives
    dXt[j] / (tokens of segment j)."""
    seg = -(-n // m)
    dX = np.zeros((n, dXt.shape[1]), dtype=np.float64)
    for j in range(m):
        lo, hi = j * seg, min((j + 1) * seg, n)
        dX[lo:hi] = dXt[j] / (hi - lo)
    return dX


def _pinv_backward(A, Zs, dZ):
    """Gradient with respect to A of Z = iterative_pinv(A, len(Zs) - 1), given
    the iterates Zs = [Z0, .., ZT] and dZ = dL/dZT."""
    A = _f64(A)
    m = A.shape[0]
    I = np.eye(m)
    dA = np.zeros_like(A)
    for j in range(len(Zs) - 2, -1, -1):
        Z = Zs[j]
        P = A @ Z
        T1 = 7.0 * I - P
        T2 = 15.0 * I - P @ T1
        T3 = 13.0 * I - P @ T2
        # Z' = 1/4 Z T3
        dT3 = 0.25 * Z.T @ dZ
        dZ_prev = 0.25 * dZ @ T3.T
        # T3 = 13 I - P T2
        dP = -dT3 @ T2.T
        dT2 = -P.T @ dT3
        # T2 = 15 I - P T1
        dP += -dT2 @ T1.T
        dT1 = -P.T @ dT2
        # T1 = 7 I - P
        dP += -dT1
        # P = A Z
        dA += dP @ Z.T
        dZ_prev += A.T @ dP
        dZ = dZ_prev
    # Z0 = A^T c, c = 1 / (||A||_1 ||A||_inf)
    col = np.abs(A).sum(axis=0)
    row = np.abs(A).sum(axis=1)
    n1, ninf = col.max(), row.max()
    c = 1.0 / (n1 * ninf)
    dA += c * dZ.T
    dc = float((dZ * A.T).sum())
    jc, ir = int(np.argmax(col)), int(np.argmax(row))
    dA[:, jc] += (-dc * c / n1) * np.sign(A[:, jc])
    dA[ir, :] += (-dc * c / ninf) * np.sign(A[ir, :])
    return dA


def nystrom_head_backward(Q, K, V, m, dout, iters=6, w=None, scale=None):
    """Gradients of sum(dout * nystrom_head(Q, K, V, m, iters, w)["out"])
    with respect to Q, K, V and w.  Returns a dict dQ, dK, dV ([n, d]) and
    dw ([k], or None without the conv skip)."""
    Q = _f64(Q)
    K = _f64(K)
    V = _f64(V)
    G = _f64(dout)
    n, d = Q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    # forward, keeping every intermediate the chain rule needs
    Qt = segment_means(Q, m)
    Kt = segment_means(K, m)
    F = kernel_F(Q, Kt, scale)
    A = kernel_A(Qt, Kt, scale)
    Zs = iterative_pinv(A, iters, return_all=True)
    Z = Zs[-1]
    B = kernel_B(Qt, K, scale)
    Y = B @ V
    W = Z @ Y
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    dw = None
    # out = O + C, C = DConv(V): C[i] = sum_t w[t] V[i + t - half]
    if w is not None:
        w = _f64(w).reshape(-1)
        k = w.shape[0]
        half = (k - 1) // 2
        dw = np.zeros(k, dtype=np.float64)
        for t in range(k):
            off = t - half
            lo, hi = max(0, -off), min(n, n - off)
            if hi > lo:
                dV[lo + off:hi + off] += w[t] * G[lo:hi]
                dw[t] = float((G[lo:hi] * V[lo + off:hi + off]).sum())
    # O = F W
    dF = G @ W.T
    dW = F.T @ G
    # W = Z Y
    dZ = dW @ Y.T
    dY = Z.T @ dW
    # Y = B V
    dB = dY @ V.T
    dV += B.T @ dY
    # B = softmax(s Qt K^T)
    dSB = _softmax_rows_backward(B, dB)
    dQt = scale * dSB @ K
    dK += scale * dSB.T @ Qt
    # F = softmax(s Q Kt^T)
    dSF = _softmax_rows_backward(F, dF)
    dQ += scale * dSF @ Kt
    dKt = scale * dSF.T @ Q
    # Z = iterative_pinv(A), A = softmax(s Qt Kt^T)
    dA = _pinv_backward(A, Zs, dZ)
    dSA = _softmax_rows_backward(A, dA)
    dQt += scale * dSA @ Kt
    dKt += scale * dSA.T @ Qt
    # Qt, Kt = segment means
    dQ += _segment_means_backward(dQt, n, m)
    dK += _segment_means_backward(dKt, n, m)
    return {"dQ": dQ, "dK": dK, "dV": dV, "dw": dw}


def nystrom_backward(Q, K, V, m, dout, iters=6, conv_w=None):
    """Batched backward over [B, H, n, d]: dQ, dK, dV [B, H, n, d] and dconv
    [H, k] (summed over the batch) or None."""
    Q = _f64(Q)
    Bn, H, n, d = Q.shape
    dQ = np.empty_like(Q)
    dK = np.empty_like(Q)
    dV = np.empty_like(Q)
    dconv = None if conv_w is None else np.zeros(_f64(conv_w).shape, dtype=np.float64)
    for b in range(Bn):
        for h in range(H):
            w = None if conv_w is None else _f64(conv_w)[h]
            g = nystrom_head_backward(Q[b, h], K[b, h], V[b, h], m, dout[b, h], iters, w)
            dQ[b, h], dK[b, h], dV[b, h] = g["dQ"], g["dK"], g["dV"]
            if dconv is not None:
                dconv[h] += g["dw"]
    return {"dQ": dQ, "dK": dK, "dV": dV, "dconv": dconv}


def nystrom_layer_forward(X, Wqkv, Wo, heads, m, iters=6, conv_w=None):
    """The attention layer around the method ([P5] "Standard Self-Attention:
    The Mathematical Baseline": Q = X W_Q, K = X W_K, V = X W_V; Figure 4
    takes the layer input X): per-head Nystrom attention of the projections,
    heads concatenated, then an output projection.
    X: [B, n, D]; Wqkv: [3D, D] (rows 0..D-1 give Q, D..2D-1 K, 2D..3D-1 V,
    head h the features h*d .. h*d + d - 1 of each, d = D / heads); Wo:
    [D, D] (nn.Linear layout: Y = concat(O) Wo^T).  Returns Y [B, n, D]."""
    X = _f64(X)
    Wqkv = _f64(Wqkv)
    Wo = _f64(Wo)
    Bn, n, D = X.shape
    d = D // heads

    def split(M):   # [B, n, D] -> [B, H, n, d]
        return M.reshape(Bn, n, heads, d).transpose(0, 2, 1, 3)

    Q = split(X @ Wqkv[:D].T)
    K = split(X @ Wqkv[D:2 * D].T)
    V = split(X @ Wqkv[2 * D:].T)
    O = nystrom_forward(Q, K, V, m, iters, conv_w)
    return O.transpose(0, 2, 1, 3).reshape(Bn, n, D) @ Wo.T


def exact_attention_head(Q, K, V, scale=None):
    """Standard softmax attention softmax(Q K^T / sqrt(d)) V ([P5] section 3.4,
    "Standard Self-Attention"), forming the n x n matrix.  Used for Lemma 2
    and for the approximation-error report only."""
    Q = _f64(Q)
    K = _f64(K)
    V = _f64(V)
    if scale is None:
        scale = 1.0 / np.sqrt(Q.shape[1])
    return softmax_rows(Q @ K.T * scale) @ V


def exact_attention(Q, K, V):
    Q = _f64(Q)
    Bn, H, n, d = Q.shape
    out = np.empty((Bn, H, n, V.shape[-1]), dtype=np.float64)
    for b in range(Bn):
        for h in range(H):
            out[b, h] = exact_attention_head(Q[b, h], K[b, h], V[b, h])
    return out


def algorithmic_flops(Bn, H, n, d, m, iters=6):
    """Dense-contraction flops of one forward: per head 2nmd each for Q K~^T,
    Q~ K^T, B~ V and F~ W, 2m^2 d each for Q~ K~^T and Z Y, and 8 m^3 per
    pinv step (four m x m products)."""
    per_head = 8 * n * m * d + 4 * m * m * d + iters * 8 * m ** 3
    return Bn * H * per_head


def algorithmic_bytes(Bn, H, n, d, elem_bytes):
    """Q, K, V read once and the output written once."""
    return 4 * Bn * H * n * d * elem_bytes
