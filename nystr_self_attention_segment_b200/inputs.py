"""Seeded synthetic inputs for the Nystrom attention forward.

This module holds no part of the method's arithmetic: it only draws random
tensors and rounds them to the device dtype.  Both the CUDA path and the CPU
oracle are fed from here, so that they see the SAME rounded values (input
quantisation is never counted as error).

Recipe: numpy default_rng(seed), draws in fp64, then rounding to the device
dtype (fp32 round-to-nearest-even, then bf16 round-to-nearest-even of that
fp32 value).  Seeds are 1000 * workload id + tensor id with Q=1, K=2, V=3,
conv=4 and the low-rank factors U_Q=5, W_Q=6, U_K=7, W_K=8; the sequence
length sweep adds 100 * log2(n / 1024).  Layout is [batch, heads, n, d]
contiguous; conv weights are [heads, k].

The workloads follow the shapes the pages time (Table 1 of the paper summary:
n = 512 ... 8192, 32 or 64 landmarks, random inputs) and the two larger
structured cases (low-rank peaky Q/K; a sequence-length sweep with 128
landmarks).
"""

import math
from dataclasses import dataclass, field

import numpy as np

F32 = "f32"
BF16 = "bf16"


@dataclass(frozen=True)
class Workload:
    name: str
    wid: int                 # workload id, used in the seeds
    batch: int
    heads: int
    seq_len: int
    head_dim: int
    landmarks: int
    dtype: str               # "f32" or "bf16"
    conv_k: int              # 0 = no conv skip
    pinv_iters: int = 6
    values: str = "iid"      # "iid", "iid_scaled" (N(0,1)/sqrt(d)) or "lowrank16"
    seed_extra: int = 0

    @property
    def bh(self):
        return self.batch * self.heads

    @property
    def tokens(self):
        return self.batch * self.heads * self.seq_len

    def with_landmarks(self, m):
        return Workload(self.name, self.wid, self.batch, self.heads, self.seq_len,
                        self.head_dim, m, self.dtype, self.conv_k, self.pinv_iters,
                        self.values, self.seed_extra)


def _sweep(n):
    return Workload("sweep_n%d_m128" % n, 5, 1, 16, n, 64, 128, BF16, 33,
                    values="iid", seed_extra=100 * int(round(math.log2(n / 1024))))


WORKLOADS = {
    # tiny fp32 correctness case, and the same inputs with m = n
    "tiny_f32_m8": Workload("tiny_f32_m8", 1, 1, 1, 64, 32, 8, F32, 0),
    "tiny_f32_m64": Workload("tiny_f32_m64", 1, 1, 1, 64, 32, 64, F32, 0),
    # tiny fp32 with m not dividing n: segments of 9 tokens, the last of 7
    "tiny_f32_n70_m8": Workload("tiny_f32_n70_m8", 7, 1, 1, 70, 32, 8, F32, 0),
    # BERT-base shape, inputs scaled by 1/sqrt(d)
    "bert_n512_m64": Workload("bert_n512_m64", 2, 8, 12, 512, 64, 64, BF16, 33,
                              values="iid_scaled"),
    # long context, also the approximation-error report case
    "long_n4096_m64": Workload("long_n4096_m64", 3, 4, 12, 4096, 64, 64, BF16, 33),
    # headline length, low-rank peaky Q/K
    "headline_n8192_m64": Workload("headline_n8192_m64", 4, 2, 12, 8192, 64, 64, BF16, 33,
                                   values="lowrank16"),
    "headline_n8192_m32": Workload("headline_n8192_m32", 4, 2, 12, 8192, 64, 32, BF16, 33,
                                   values="lowrank16"),
    # m does not divide n: segments of ceil(n/m) tokens, the last one shorter
    "ragged_n8100_m64": Workload("ragged_n8100_m64", 6, 1, 2, 8100, 64, 64, BF16, 33),
}
for _n in (1024, 2048, 4096, 8192, 16384, 32768, 65536):
    WORKLOADS["sweep_n%d_m128" % _n] = _sweep(_n)


def round_to_f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def round_to_bf16_as_f32(x):
    """Round to bf16 (round-to-nearest-even on the fp32 bit pattern); returns
    the bf16 values held in an fp32 array."""
    f = round_to_f32(x)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = (u + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)
    return u.astype(np.uint32).view(np.float32)


def bf16_bits(x_f32):
    """The upper 16 bits of fp32 values that are exactly bf16."""
    return (np.asarray(x_f32, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _rng(wl, tensor_id):
    return np.random.default_rng(1000 * wl.wid + wl.seed_extra + tensor_id)


def make_inputs(wl, batch=None, heads=None):
    """Draw Q, K, V (and conv weights) for a workload.  Returns a dict with
    fp32 arrays 'Q', 'K', 'V' holding values exactly representable in the
    device dtype, 'conv_w' ([H, k] fp32 or None) and the workload.  batch /
    heads override the workload's (used for bounded samples)."""
    Bn = wl.batch if batch is None else batch
    H = wl.heads if heads is None else heads
    n, d = wl.seq_len, wl.head_dim
    shape = (Bn, H, n, d)
    if wl.values == "lowrank16":
        r = 16
        def lowrank(u_id, w_id, e_id):
            U = _rng(wl, u_id).standard_normal((Bn, H, n, r))
            Wf = _rng(wl, w_id).standard_normal((Bn, H, r, d))
            E = _rng(wl, e_id).standard_normal(shape)
            return np.matmul(U, Wf) + 0.1 * E
        Q = lowrank(5, 6, 1)
        K = lowrank(7, 8, 2)
    else:
        Q = _rng(wl, 1).standard_normal(shape)
        K = _rng(wl, 2).standard_normal(shape)
        if wl.values == "iid_scaled":
            Q = Q / math.sqrt(d)
            K = K / math.sqrt(d)
    V = _rng(wl, 3).standard_normal(shape)
    if wl.values == "iid_scaled":
        V = V / math.sqrt(d)
    conv_w = None
    if wl.conv_k > 0:
        conv_w = round_to_f32(0.02 * _rng(wl, 4).standard_normal((H, wl.conv_k)))
    rnd = round_to_bf16_as_f32 if wl.dtype == BF16 else round_to_f32
    return {"Q": rnd(Q), "K": rnd(K), "V": rnd(V), "conv_w": conv_w, "workload": wl}


def make_custom(shape, dtype, seed, scale=1.0, conv_k=0):
    """Generic iid N(0, scale^2) inputs of a given [B, H, n, d] shape (edge-case
    tests).  Same rounding rule as make_inputs."""
    rng = np.random.default_rng(seed)
    Q = scale * rng.standard_normal(shape)
    K = scale * rng.standard_normal(shape)
    V = rng.standard_normal(shape)
    rnd = round_to_bf16_as_f32 if dtype == BF16 else round_to_f32
    conv_w = None
    if conv_k > 0:
        conv_w = round_to_f32(0.02 * rng.standard_normal((shape[1], conv_k)))
    return {"Q": rnd(Q), "K": rnd(K), "V": rnd(V), "conv_w": conv_w}
