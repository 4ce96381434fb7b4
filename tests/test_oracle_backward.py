"""Pins of the oracle's backward pass (gradients of the Nystrom forward with
respect to Q, K, V and the conv kernel), against things other than itself:

- central finite differences of the oracle's forward in fp64, entry by entry,
  on tiny shapes (m dividing n or not, 0 to 6 pinv steps, with and without
  the conv skip): a dropped term, a wrong sign or a transposed product in any
  step of the chain rule shows up here;
- closed forms: m = 1 (F~ = 1, A = [1] and Z = 1 at every step, so the output
  is softmax(s mean(Q) K^T) V plus the conv) and Q = 0 (the output is the
  mean of V plus the conv, linear in V)."""
import numpy as np
import pytest

from oracle import nystrom as orc


def _fd(f, X, h=1e-6):
    g = np.zeros_like(X)
    it = np.nditer(X, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        x0 = X[i]
        X[i] = x0 + h
        fp = f()
        X[i] = x0 - h
        fm = f()
        X[i] = x0
        g[i] = (fp - fm) / (2 * h)
    return g


CASES = [
    # n, d, m, iters, conv k
    (12, 4, 3, 2, 3),
    (10, 3, 4, 6, 5),     # m does not divide n: segments of 3, the last of 1
    (16, 4, 4, 6, 0),
    (9, 2, 9, 3, 3),      # m = n
    (11, 3, 2, 0, 1),     # Z = Z0
]


@pytest.mark.parametrize("n,d,m,iters,k", CASES)
def test_backward_matches_finite_differences(n, d, m, iters, k):
    rng = np.random.default_rng(100 * n + m)
    Q, K, V = rng.standard_normal((3, n, d))
    G = rng.standard_normal((n, d))
    w = rng.standard_normal(k) if k else None
    g = orc.nystrom_head_backward(Q, K, V, m, G, iters, w)

    def loss():
        return float((G * orc.nystrom_head(Q, K, V, m, iters, w)["out"]).sum())

    for name, X in (("dQ", Q), ("dK", K), ("dV", V)):
        num = _fd(loss, X)
        assert np.abs(num - g[name]).max() <= 1e-6 * np.abs(num).max(), name
    if w is not None:
        num = _fd(loss, w)
        assert np.abs(num - g["dw"]).max() <= 1e-6 * np.abs(num).max()
    else:
        assert g["dw"] is None


def test_single_landmark_closed_form():
    # m = 1: out = b V + C with b = softmax(s qbar K^T), qbar = mean(Q)
    rng = np.random.default_rng(5)
    n, d, k = 13, 4, 3
    Q, K, V = rng.standard_normal((3, n, d))
    G = rng.standard_normal((n, d))
    w = rng.standard_normal(k)
    s = 1 / np.sqrt(d)
    qbar = Q.mean(axis=0)
    logits = s * K @ qbar
    b = np.exp(logits - logits.max())
    b /= b.sum()
    gsum = G.sum(axis=0)
    # conv part: dV[j] = sum_t w[t] G[j - t + half]
    half = (k - 1) // 2
    dv_conv = np.zeros_like(V)
    for j in range(n):
        for t in range(k):
            i = j - t + half
            if 0 <= i < n:
                dv_conv[j] += w[t] * G[i]
    dV = np.outer(b, gsum) + dv_conv
    e = V @ gsum                        # d loss / d b_k
    dlog = b * (e - (b * e).sum())      # softmax backward
    dK = s * np.outer(dlog, qbar)
    dqbar = s * dlog @ K
    dQ = np.tile(dqbar / n, (n, 1))
    g = orc.nystrom_head_backward(Q, K, V, 1, G, 6, w)
    assert np.allclose(g["dV"], dV, rtol=0, atol=1e-12)
    assert np.allclose(g["dK"], dK, rtol=0, atol=1e-12)
    assert np.allclose(g["dQ"], dQ, rtol=0, atol=1e-12)


def test_zero_queries_value_gradient_is_the_mean():
    # Q = 0: F~ and B~ are uniform and Z = J/m is a fixed point, so out is the
    # mean of V in every row (plus the conv): dV = sum_i G_i / n in every row
    rng = np.random.default_rng(6)
    n, d, m = 16, 4, 4
    Q = np.zeros((n, d))
    K, V = rng.standard_normal((2, n, d))
    G = rng.standard_normal((n, d))
    g = orc.nystrom_head_backward(Q, K, V, m, G, 6, None)
    assert np.allclose(g["dV"], np.tile(G.sum(axis=0) / n, (n, 1)), rtol=0, atol=1e-12)


def test_batched_backward_sums_conv_gradient_over_the_batch():
    rng = np.random.default_rng(7)
    Bn, H, n, d, m, k = 2, 2, 8, 3, 2, 3
    Q, K, V, G = rng.standard_normal((4, Bn, H, n, d))
    cw = rng.standard_normal((H, k))
    out = orc.nystrom_backward(Q, K, V, m, G, 6, cw)
    for h in range(H):
        tot = np.zeros(k)
        for b in range(Bn):
            g = orc.nystrom_head_backward(Q[b, h], K[b, h], V[b, h], m, G[b, h], 6, cw[h])
            assert np.array_equal(out["dQ"][b, h], g["dQ"])
            assert np.array_equal(out["dV"][b, h], g["dV"])
            tot += g["dw"]
        assert np.allclose(out["dconv"][h], tot, rtol=1e-14, atol=0)
