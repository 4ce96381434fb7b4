"""Writes the stored expected values under tests/golden/ by calling the fp64
oracle only (never the CUDA path).

  python tests/golden/make_golden.py

tiny_f32_m8.txt / tiny_f32_m64.txt: the tiny fp32 workload (batch 1, heads 1,
n = 64, d = 32, iid N(0,1) inputs from the seeded generator, six pseudoinverse
steps, no conv skip) with m = 8 and m = n = 64 landmarks.  Method: Eq. 17 /
Algorithm 1 of "Nystromformer: A Nystrom-Based Algorithm for Approximating
Self-Attention" (section 3.4) with the Lemma 1 pseudoinverse and segment-mean
landmarks (Eq. 16, mean over l = n/m tokens).

tiny_f32_n70_m8.txt: the same method with m = 8 not dividing n = 70 (batch 1,
heads 1, d = 32, its own seeds): segments of ceil(70 / 8) = 9 tokens, the
last one of 7, each landmark the mean over its segment's real tokens (the
"Landmark Selection: Segment-Means" section's padding, read with true
counts).
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import nystrom as orc                                  # noqa: E402
from nystr_self_attention_segment_b200.inputs import WORKLOADS, make_inputs  # noqa: E402


def write(name):
    wl = WORKLOADS[name]
    x = make_inputs(wl)
    out, extra = orc.nystrom_forward(x["Q"], x["K"], x["V"], wl.landmarks, wl.pinv_iters,
                                     x["conv_w"], keep=("Z",))
    path = os.path.join(HERE, name + ".txt")
    with open(path, "w") as f:
        f.write("# workload %s: B=%d H=%d n=%d d=%d m=%d iters=%d dtype=%s conv=none\n"
                % (name, wl.batch, wl.heads, wl.seq_len, wl.head_dim, wl.landmarks,
                   wl.pinv_iters, wl.dtype))
        f.write("# source: fp64 oracle (Eq. 17 / Algorithm 1, Lemma 1 pseudoinverse,\n"
                "# Eq. 16 segment means) on the seeded generator's inputs\n")
        f.write("# input checksums (sum of Q, K, V): %.17g %.17g %.17g\n"
                % (x["Q"].astype(np.float64).sum(), x["K"].astype(np.float64).sum(),
                   x["V"].astype(np.float64).sum()))
        f.write("out %d\n" % out.size)
        for v in out.reshape(-1):
            f.write("%.17g\n" % v)
        Z = extra["Z"]
        f.write("Z %d\n" % Z.size)
        for v in Z.reshape(-1):
            f.write("%.17g\n" % v)


def read(name):
    """Returns (checksums, {'out': array, 'Z': array}) of a stored fixture."""
    path = os.path.join(HERE, name + ".txt")
    lines = open(path).read().split("\n")
    sums = None
    data = {}
    i = 0
    while i < len(lines):
        ln = lines[i]
        if ln.startswith("# input checksums"):
            sums = [float(t) for t in ln.split(":")[1].split()]
        elif ln and not ln.startswith("#"):
            key, cnt = ln.split()
            cnt = int(cnt)
            data[key] = np.array([float(t) for t in lines[i + 1:i + 1 + cnt]])
            i += cnt
        i += 1
    return sums, data


if __name__ == "__main__":
    for nm in ("tiny_f32_m8", "tiny_f32_m64", "tiny_f32_n70_m8"):
        write(nm)
        print("wrote", nm)
