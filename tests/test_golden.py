"""The stored tiny-workload fixtures (written by tests/golden/make_golden.py
from the fp64 oracle) still match the generator and the oracle."""
import numpy as np
import pytest

from oracle import nystrom as orc
from nystr_self_attention_segment_b200.inputs import WORKLOADS, make_inputs
from tests.golden.make_golden import read


@pytest.mark.parametrize("name", ["tiny_f32_m8", "tiny_f32_m64", "tiny_f32_n70_m8"])
def test_golden_fixture_matches_oracle(name):
    wl = WORKLOADS[name]
    x = make_inputs(wl)
    sums, data = read(name)
    got_sums = [float(x[t].astype(np.float64).sum()) for t in ("Q", "K", "V")]
    np.testing.assert_allclose(got_sums, sums, rtol=0, atol=1e-12)
    out, extra = orc.nystrom_forward(x["Q"], x["K"], x["V"], wl.landmarks, wl.pinv_iters,
                                     x["conv_w"], keep=("Z",))
    np.testing.assert_allclose(out.reshape(-1), data["out"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(extra["Z"].reshape(-1), data["Z"], rtol=0, atol=1e-12)


def test_tiny_m_equals_n_against_exact_attention():
    # Lemma 2 on the tiny workload: with m = n the error to exact attention
    # falls to rounding once the pseudoinverse has converged; six steps leave
    # a visible gap (the truncated iteration is part of the method).
    wl = WORKLOADS["tiny_f32_m64"]
    x = make_inputs(wl)
    exact = orc.exact_attention(x["Q"], x["K"], x["V"])
    conv = orc.nystrom_forward(x["Q"], x["K"], x["V"], 64, 40)
    six = orc.nystrom_forward(x["Q"], x["K"], x["V"], 64, 6)
    scale = np.abs(exact).max()
    assert np.abs(conv - exact).max() <= 1e-9 * scale
    assert np.abs(six - exact).max() > 1e-4 * scale
