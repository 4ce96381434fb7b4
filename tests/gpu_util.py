"""Helpers for the GPU parity tests: upload seeded inputs, run the CUDA path
through the C ABI, and compare with the fp64 oracle."""
import numpy as np

import nystr_self_attention_segment_b200 as nys

TOL = {"f32": 1e-4, "bf16": 2e-2}     # max |gpu - oracle| / max |oracle|


def torch():
    import torch as t
    return t


def to_dev(x, dtype):
    t = torch()
    td = t.bfloat16 if dtype == "bf16" else t.float32
    return t.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to("cuda").to(td).contiguous()


def run(x, dtype, m, iters=6, conv=True, workspace=True):
    """Runs the CUDA forward on the inputs dict x; returns (out fp64 numpy,
    workspace or None, device tensors)."""
    t = torch()
    Q, K, V = (to_dev(x[k], dtype) for k in ("Q", "K", "V"))
    cw = None
    if conv and x.get("conv_w") is not None:
        cw = t.from_numpy(np.ascontiguousarray(x["conv_w"], dtype=np.float32)).cuda()
    ws = nys.Workspace(Q, m) if workspace else None
    out = nys.nys_attn_forward(Q, K, V, m, iters, cw, workspace=ws)
    t.cuda.synchronize()
    if ws is not None:
        nys.nys_attn_check_error(ws)
    return out.float().cpu().numpy().astype(np.float64), ws, (Q, K, V, cw)


def normwise(got, want):
    return float(np.abs(got - want).max() / max(np.abs(want).max(), 1e-300))


def per_head_worst(got, want):
    Bn, H = want.shape[:2]
    return max(normwise(got[b, h], want[b, h]) for b in range(Bn) for h in range(H))
