"""Pins of the fp64 oracle to facts outside itself.

Each test checks the oracle against something it does not compute the same
way: brute-force loops on tiny inputs, invariants the definitions imply,
numpy/LAPACK routines (SVD pseudoinverse, matrix norms, correlate), closed
forms derived by hand, Lemma 2 of the paper summary ("Theoretical Analysis")
and brute-force n x n softmax attention.  A plausible slip anywhere in the
oracle (a dropped term, a wrong coefficient, a softmax over the wrong axis, a
transposed operand, dividing a segment sum by m instead of l) fails one of
them.
"""

import math

import numpy as np
import pytest

from oracle import nystrom as orc


def _rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- segment means

def test_segment_means_bruteforce_loops():
    # Plain Python loops over a tiny input (n=12, m=3, l=4).
    rng = _rng(1)
    n, m, d = 12, 3, 2
    X = rng.standard_normal((n, d))
    got = orc.segment_means(X, m)
    seg = n // m
    for j in range(m):
        for c in range(d):
            acc = 0.0
            for t in range(seg):
                acc += float(X[j * seg + t, c])
            assert abs(got[j, c] - acc / seg) < 1e-15


def test_segment_means_m_equals_n_is_identity():
    X = _rng(2).standard_normal((16, 5))
    assert np.array_equal(orc.segment_means(X, 16), X)


def test_segment_means_preserve_global_mean():
    # mean over landmarks == mean over tokens; with m != l a divide-by-m
    # (the printed typo of Eq. 16) would scale this by l/m.
    X = _rng(3).standard_normal((64, 7))
    for m in (2, 4, 8, 16):
        L = orc.segment_means(X, m)
        np.testing.assert_allclose(L.mean(axis=0), X.mean(axis=0), rtol=0, atol=1e-14)


def test_segment_means_constant_segments():
    vals = _rng(4).standard_normal((4, 3))
    X = np.repeat(vals, 5, axis=0)          # n=20, four segments of 5
    np.testing.assert_allclose(orc.segment_means(X, 4), vals, rtol=0, atol=1e-15)


def test_segment_means_ragged_bruteforce_loops():
    # m does not divide n: segments of ceil(n/m) tokens, the last one short,
    # each averaged over its own tokens (n=14, m=4: 4, 4, 4 and 2 tokens).
    rng = _rng(41)
    n, m, d = 14, 4, 3
    X = rng.standard_normal((n, d))
    got = orc.segment_means(X, m)
    bounds = [(0, 4), (4, 8), (8, 12), (12, 14)]
    for j, (a, b) in enumerate(bounds):
        for c in range(d):
            acc = 0.0
            for t in range(a, b):
                acc += float(X[t, c])
            assert abs(got[j, c] - acc / (b - a)) < 1e-15


def test_segment_means_ragged_is_zero_padding_over_true_counts():
    # The padded reading: pad with zeros to m * ceil(n/m) tokens, sum each
    # segment of the padded sequence, divide by the number of real tokens in
    # it.  Any pad value other than zero would show up here.
    rng = _rng(42)
    n, m, d = 70, 8, 5
    seg = -(-n // m)
    X = rng.standard_normal((n, d))
    P = np.zeros((m * seg, d))
    P[:n] = X
    sums = P.reshape(m, seg, d).sum(axis=1)
    counts = np.minimum(seg, n - np.arange(m) * seg)
    np.testing.assert_allclose(orc.segment_means(X, m), sums / counts[:, None], rtol=0,
                               atol=1e-14)


def test_segment_means_ragged_weighted_mean_and_constants():
    # sum_j count_j * landmark_j == sum of all tokens, and a segment of equal
    # rows keeps that row, the short last one included.
    rng = _rng(43)
    n, m = 4090, 128                       # 127 segments of 32, the last of 26
    X = rng.standard_normal((n, 4))
    L = orc.segment_means(X, m)
    counts = np.array([32] * 127 + [26], dtype=np.float64)
    np.testing.assert_allclose((counts[:, None] * L).sum(axis=0), X.sum(axis=0), rtol=0,
                               atol=1e-10)
    vals = rng.standard_normal((5, 2))
    Y = np.repeat(vals, [4, 4, 4, 4, 1], axis=0)   # n=17, m=5: segments of 4, the last of 1
    np.testing.assert_allclose(orc.segment_means(Y, 5), vals, rtol=0, atol=1e-15)


def test_segment_means_rejects_empty_segments():
    # n=5, m=4: segments of 2 tokens would leave the fourth one empty.
    with pytest.raises(ValueError):
        orc.segment_means(np.zeros((5, 2)), 4)
    with pytest.raises(ValueError):
        orc.segment_means(np.zeros((65, 2)), 64)
    orc.segment_means(np.zeros((10, 2)), 3)        # 4, 4, 2: all non-empty


# ---------------------------------------------------------------- softmax kernels

def test_softmax_kernels_row_sums_and_axes():
    rng = _rng(5)
    n, m, d = 48, 6, 8
    Q = rng.standard_normal((n, d)) * 3
    K = rng.standard_normal((n, d)) * 3
    Qt, Kt = orc.segment_means(Q, m), orc.segment_means(K, m)
    s = 1 / math.sqrt(d)
    F = orc.kernel_F(Q, Kt, s)
    A = orc.kernel_A(Qt, Kt, s)
    B = orc.kernel_B(Qt, K, s)
    assert F.shape == (n, m) and A.shape == (m, m) and B.shape == (m, n)
    for M in (F, A, B):
        assert np.all(M > 0)
        np.testing.assert_allclose(M.sum(axis=1), 1.0, rtol=0, atol=1e-15)
    # B is normalised over the n keys: its columns do not sum to one.
    assert abs(B.sum(axis=0) - 1).max() > 1e-3
    # entries against the textbook softmax written with exp / sum per entry
    i, j = 7, 3
    z = [math.exp(s * float(Q[i] @ Kt[t])) for t in range(m)]
    assert abs(F[i, j] - z[j] / sum(z)) < 1e-14
    z = [math.exp(s * float(Qt[j] @ K[t])) for t in range(n)]
    assert abs(B[j, i] - z[i] / sum(z)) < 1e-14


def test_softmax_is_shift_invariant_and_handles_peaky_logits():
    S = _rng(6).standard_normal((5, 9)) * 400.0      # exp would overflow unshifted
    P = orc.softmax_rows(S)
    assert np.all(np.isfinite(P))
    np.testing.assert_allclose(P, orc.softmax_rows(S + 123.0), rtol=0, atol=1e-15)


# ---------------------------------------------------------------- pseudoinverse

def test_pinv_init_uses_the_matrix_norms():
    A = _rng(7).random((6, 6))
    Z0 = orc.pinv_init(A)
    c = np.linalg.norm(A, 1) * np.linalg.norm(A, np.inf)   # LAPACK-side norms
    np.testing.assert_allclose(Z0 * c, A.T, rtol=1e-15, atol=0)
    # a row-stochastic kernel has ||A||_inf = 1 exactly
    S = orc.kernel_A(_rng(8).standard_normal((6, 4)), _rng(9).standard_normal((6, 4)), 0.5)
    assert abs(np.linalg.norm(S, np.inf) - 1.0) < 1e-15


def test_pinv_one_step_residual_closed_form():
    # With E = I - A Z, one step of Lemma 1 gives exactly
    # I - A Z' = E^3 (3I + E) / 4 (expand x(13 - 15x + 7x^2 - x^3)/4 at
    # x = 1 - e).  A wrong coefficient or a dropped product breaks it.
    rng = _rng(10)
    for m in (3, 8, 17):
        A = rng.standard_normal((m, m))
        Z = rng.standard_normal((m, m)) * 0.3
        I = np.eye(m)
        E = I - A @ Z
        E_next = I - A @ orc.pinv_step(A, Z)
        want = E @ E @ E @ (3 * I + E) / 4
        np.testing.assert_allclose(E_next, want, rtol=1e-10, atol=1e-10 * np.abs(want).max())


def test_pinv_converges_to_svd_pseudoinverse():
    rng = _rng(11)
    for m in (4, 8, 16):
        Qt = rng.standard_normal((m, 8)) * 0.7
        Kt = rng.standard_normal((m, 8)) * 0.7
        A = orc.kernel_A(Qt, Kt, 1 / math.sqrt(8))
        Z = orc.iterative_pinv(A, 40)
        ref = np.linalg.pinv(A)                # SVD route
        assert np.abs(Z - ref).max() <= 1e-10 * np.abs(ref).max()


def test_pinv_of_singular_kernel_matches_svd():
    # two identical landmark queries give two identical rows: rank m-1
    rng = _rng(12)
    m = 6
    Qt = rng.standard_normal((m, 4)) * 0.5
    Qt[3] = Qt[1]
    Kt = rng.standard_normal((m, 4)) * 0.5
    A = orc.kernel_A(Qt, Kt, 0.5)
    assert np.linalg.matrix_rank(A) == m - 1
    # Z0 ~ A^T keeps Z off the null space in exact arithmetic; rounding noise
    # there grows by 13/4 per step once converged, so stop soon after.
    Z = orc.iterative_pinv(A, 13)
    ref = np.linalg.pinv(A, rcond=1e-12)
    assert np.abs(Z - ref).max() <= 1e-12 * np.abs(ref).max()


def test_pinv_uniform_kernel_is_a_fixed_point():
    # Q~ = 0 makes A = J/m; then Z0 = J/m = A^+ and every step keeps it.
    for m in (1, 5, 64):
        A = orc.kernel_A(np.zeros((m, 3)), _rng(13).standard_normal((m, 3)), 1.0)
        J = np.full((m, m), 1.0 / m)
        np.testing.assert_allclose(A, J, rtol=0, atol=1e-16)
        for Z in orc.iterative_pinv(A, 6, return_all=True):
            np.testing.assert_allclose(Z, J, rtol=0, atol=1e-15)


def test_pinv_zero_iterations_is_the_initialisation():
    A = _rng(14).random((5, 5))
    np.testing.assert_array_equal(orc.iterative_pinv(A, 0), orc.pinv_init(A))


# ---------------------------------------------------------------- conv skip

def test_conv_matches_numpy_correlate():
    rng = _rng(15)
    for n, k in ((40, 33), (10, 33), (7, 3), (5, 1)):
        V = rng.standard_normal((n, 3))
        w = rng.standard_normal(k)
        C = orc.depthwise_conv(V, w)
        for c in range(3):
            # full cross-correlation, then the centred n samples
            full = np.correlate(np.pad(V[:, c], (k - 1) // 2), w, mode="valid")
            np.testing.assert_allclose(C[:, c], full, rtol=0, atol=1e-13)


def test_conv_kernel_one_is_a_scale():
    V = _rng(16).standard_normal((9, 4))
    np.testing.assert_allclose(orc.depthwise_conv(V, [0.37]), 0.37 * V, rtol=0, atol=1e-16)


def test_conv_rejects_even_kernel():
    with pytest.raises(ValueError):
        orc.depthwise_conv(np.zeros((4, 2)), [1.0, 2.0])


# ---------------------------------------------------------------- whole method

def test_lemma2_m_equals_n_gives_exact_attention():
    # Lemma 2 ("Theoretical Analysis"): landmarks equal to every token make
    # the approximation exact once the pseudoinverse has converged.
    rng = _rng(17)
    n, d = 16, 8
    Q = rng.standard_normal((n, d)) * 0.8
    K = rng.standard_normal((n, d)) * 0.8
    V = rng.standard_normal((n, d))
    got = orc.nystrom_head(Q, K, V, m=n, iters=40)["out"]
    want = orc.exact_attention_head(Q, K, V)
    assert np.abs(got - want).max() <= 1e-10 * np.abs(want).max()


def test_segment_constant_inputs_are_reproduced_exactly():
    # If Q and K are constant inside every segment, F~ = A rows, B~ = A
    # columns / l, so F~ A^+ B~ equals the exact softmax matrix for any
    # m | n (converged pseudoinverse).  Exercises segment means, all three
    # softmax axes and the product chain with m < n.
    rng = _rng(18)
    n, m, d = 24, 4, 8
    seg = n // m
    Q = np.repeat(rng.standard_normal((m, d)), seg, axis=0)
    K = np.repeat(rng.standard_normal((m, d)), seg, axis=0)
    V = rng.standard_normal((n, d))                    # V is not constant
    got = orc.nystrom_head(Q, K, V, m=m, iters=40)["out"]
    want = orc.exact_attention_head(Q, K, V)
    assert np.abs(got - want).max() <= 1e-10 * np.abs(want).max()


def test_zero_queries_average_the_values():
    # Q = 0: F~ uniform over m, A = J/m (fixed point), B~ uniform over n,
    # so every output row is the mean of V (plus the conv skip), at any
    # number of iterations and any m.
    rng = _rng(19)
    n, d = 32, 4
    K = rng.standard_normal((n, d)) * 2
    V = rng.standard_normal((n, d))
    w = rng.standard_normal(5)
    for m in (1, 4, 32):
        r = orc.nystrom_head(np.zeros((n, d)), K, V, m=m, iters=6, w=w)
        want = np.tile(V.mean(axis=0), (n, 1)) + orc.depthwise_conv(V, w)
        np.testing.assert_allclose(r["out"], want, rtol=0, atol=1e-13)


def test_single_landmark_closed_form():
    # m = 1: A = [1], Z = 1 at every step, F~ = 1, and each output row is the
    # softmax-weighted mean of V with weights exp(s q~ . k_i).
    rng = _rng(20)
    n, d = 10, 3
    Q = rng.standard_normal((n, d))
    K = rng.standard_normal((n, d))
    V = rng.standard_normal((n, d))
    s = 1 / math.sqrt(d)
    qbar = [sum(float(Q[i, c]) for i in range(n)) / n for c in range(d)]
    wts = [math.exp(s * sum(qbar[c] * float(K[i, c]) for c in range(d))) for i in range(n)]
    tot = sum(wts)
    row = [sum(wts[i] * float(V[i, c]) for i in range(n)) / tot for c in range(d)]
    out = orc.nystrom_head(Q, K, V, m=1, iters=6)["out"]
    np.testing.assert_allclose(out, np.tile(row, (n, 1)), rtol=0, atol=1e-14)


def test_linear_in_values_and_heads_independent():
    rng = _rng(21)
    Bn, H, n, d, m = 1, 3, 16, 4, 4
    Q = rng.standard_normal((Bn, H, n, d))
    K = rng.standard_normal((Bn, H, n, d))
    V1 = rng.standard_normal((Bn, H, n, d))
    V2 = rng.standard_normal((Bn, H, n, d))
    o1 = orc.nystrom_forward(Q, K, V1, m)
    o2 = orc.nystrom_forward(Q, K, V2, m)
    o12 = orc.nystrom_forward(Q, K, 2 * V1 - V2, m)
    np.testing.assert_allclose(o12, 2 * o1 - o2, rtol=0, atol=1e-10 * np.abs(o12).max())
    perm = [2, 0, 1]
    op = orc.nystrom_forward(Q[:, perm], K[:, perm], V1[:, perm], m)
    np.testing.assert_allclose(op, o1[:, perm], rtol=0, atol=1e-15)


def test_flop_and_byte_counts():
    # 8nmd + 4m^2 d + 48 m^3 per head at six iterations; 4 n d e bytes
    assert orc.algorithmic_flops(1, 1, 8192, 64, 64) == 8 * 8192 * 64 * 64 + 4 * 64 * 64 * 64 + 48 * 64 ** 3
    assert orc.algorithmic_bytes(2, 12, 8192, 64, 2) == 2 * 12 * 8192 * 64 * 2 * 4


# ---------------------------------------------------------------- ragged batches

def _ragged_inputs(seed, Bn=3, H=2, n=40, d=8):
    rng = _rng(seed)
    return (rng.standard_normal((Bn, H, n, d)), rng.standard_normal((Bn, H, n, d)),
            rng.standard_normal((Bn, H, n, d)), 0.2 * rng.standard_normal((H, 5)))


def test_lens_padding_content_never_enters():
    # Garbage in the padding changes nothing, and padding rows come out zero.
    Q, K, V, w = _ragged_inputs(51)
    lens = [40, 29, 16]                     # 29: segments of 4, the last of 1
    ref = orc.nystrom_forward_lens(Q, K, V, 8, lens, 6, w)
    rng = _rng(52)
    Q2, K2, V2 = Q.copy(), K.copy(), V.copy()
    for b, L in enumerate(lens):
        for X in (Q2, K2, V2):
            X[b, :, L:] = 1e3 * rng.standard_normal(X[b, :, L:].shape)
    got = orc.nystrom_forward_lens(Q2, K2, V2, 8, lens, 6, w)
    np.testing.assert_array_equal(got, ref)
    for b, L in enumerate(lens):
        assert not got[b, :, L:].any()


def test_lens_equal_to_n_is_the_plain_forward():
    Q, K, V, w = _ragged_inputs(53)
    np.testing.assert_array_equal(orc.nystrom_forward_lens(Q, K, V, 8, [40] * 3, 6, w),
                                  orc.nystrom_forward(Q, K, V, 8, 6, w))


def test_lens_lemma2_exact_attention_over_real_tokens():
    # m = L real tokens with a converged pseudoinverse: exact softmax
    # attention over those L tokens only (brute force on the truncated
    # sequence); a softmax that let the padding in would miss this.
    Q, K, V, _ = _ragged_inputs(54, Bn=2, H=1, n=24, d=6)
    Q *= 0.3
    K *= 0.3
    lens = [20, 10]
    got = orc.nystrom_forward_lens(Q, K, V, 10, lens, 60, None)
    for b, L in enumerate(lens):
        if L != 10:
            continue
        want = orc.exact_attention_head(Q[b, 0, :L], K[b, 0, :L], V[b, 0, :L])
        np.testing.assert_allclose(got[b, 0, :L], want, rtol=0, atol=1e-9)


def test_lens_uniform_queries_closed_form_with_boundary_conv():
    # Q = 0: every softmax is uniform and Z0 = J/m is a fixed point, so each
    # real row is the mean of the real V rows, plus the conv of the real rows
    # with zeros past L (numpy.correlate).
    Q, K, V, w = _ragged_inputs(55, Bn=2, H=2, n=30, d=4)
    Q[:] = 0.0
    lens = [30, 21]                         # 21: segments of 4, the last of 1
    got = orc.nystrom_forward_lens(Q, K, V, 6, lens, 6, w)
    for b, L in enumerate(lens):
        for h in range(2):
            mean = V[b, h, :L].mean(axis=0)
            for c in range(4):
                conv = np.correlate(np.pad(V[b, h, :L, c], 2), w[h], mode="valid")
                np.testing.assert_allclose(got[b, h, :L, c], mean[c] + conv, rtol=0, atol=1e-12)


# ------------------------------------------------------------------ layer

def test_layer_with_identity_projections_is_the_attention():
    # one head, D = d, W_Q = W_K = W_V = W_O = I: the layer is the method on
    # Q = K = V = X
    rng = np.random.default_rng(31)
    B, n, d, m = 2, 24, 8, 4
    X = rng.standard_normal((B, n, d))
    I = np.eye(d)
    Y = orc.nystrom_layer_forward(X, np.vstack([I, I, I]), I, 1, m)
    want = orc.nystrom_forward(X[:, None], X[:, None], X[:, None], m)[:, 0]
    assert np.allclose(Y, want, rtol=0, atol=1e-13)


def test_layer_head_split_and_concat_follow_the_features():
    # the layer equals the per-head attention of the head's feature slices,
    # placed at the head's columns before Wo; swapping two heads' slices in
    # W_Q, W_K, W_V and the matching columns of Wo leaves Y unchanged
    rng = np.random.default_rng(32)
    B, n, H, d, m = 1, 16, 2, 4, 4
    D = H * d
    X = rng.standard_normal((B, n, D))
    W = rng.standard_normal((3 * D, D)) / np.sqrt(D)
    Wo = rng.standard_normal((D, D)) / np.sqrt(D)
    cw = 0.1 * rng.standard_normal((H, 3))
    Y = orc.nystrom_layer_forward(X, W, Wo, H, m, 6, cw)
    O = np.zeros((B, n, D))
    for h in range(H):
        sl = slice(h * d, (h + 1) * d)
        q = X @ W[:D][sl].T
        k = X @ W[D:2 * D][sl].T
        v = X @ W[2 * D:][sl].T
        O[:, :, sl] = orc.nystrom_forward(q[:, None], k[:, None], v[:, None], m, 6,
                                          cw[h:h + 1])[:, 0]
    assert np.allclose(Y, O @ Wo.T, rtol=0, atol=1e-12)
    perm = np.r_[np.arange(d, 2 * d), np.arange(0, d)]
    Wp = np.vstack([W[:D][perm], W[D:2 * D][perm], W[2 * D:][perm]])
    Yp = orc.nystrom_layer_forward(X, Wp, Wo[:, perm], H, m, 6, cw[::-1])
    assert np.allclose(Y, Yp, rtol=0, atol=1e-12)
