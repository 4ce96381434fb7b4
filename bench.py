"""Throughput benchmark of the B200 Nystrom attention forward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

One step = one forward pass (segment means, landmark kernel + pseudoinverse,
B~ V, Z (B~ V), F~ W + DConv skip) over one batch of the workload, through the
C ABI.  Prints ONE JSON line on rank 0.  Metric: tokens/s (batch x heads x n)
over all ranks; every rank runs its own full batch (weak scaling, no data-path
collective: heads are independent).

Timing: W untimed warm-up steps, then exactly K steps bracketed by a barrier
and a device synchronisation, timed with CUDA events on the launching stream,
max over ranks.  The step inputs rotate over enough copies that every step
reads inputs last touched more than one L2 (126 MB) of traffic ago, so they
come from HBM.  Per-kernel CUDA events inside the same timed region give the
dominant kernel's duration for the roofline.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Nyström attention fwd tokens/sec (b×h×n) at n=8192,m=64,d=64; % roofline"
L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="headline_n8192_m64")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass (nys_attn_backward) instead of the forward")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ----------------------------------------------------------------- traffic

# Sources of each kernel of the bf16 path: a DRAM traffic figure recorded
# from an ncu capture holds only while these files are unchanged.
KERNEL_SOURCES = {
    "mid_tc": ["common.cuh", "sm100.cuh", "trace.cuh", "pinv_pow.cuh", "pinv_pow128.cuh",
               "mid_tc.cuh"],
    "out_tc": ["common.cuh", "sm100.cuh", "trace.cuh", "out_tc.cuh"],
    "seg_means": ["common.cuh", "sm100.cuh", "trace.cuh", "stream_bf16.cuh"],
}


def code_tokens(text):
    """C++ source without comments, whitespace runs collapsed: what the
    compiler sees, so that comment edits keep a recorded profile valid."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def source_digest(kernel, read=None):
    """Digest of the code (comments excluded) of a kernel's source files."""
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES.get(kernel, []):
        if read is None:
            with open(os.path.join(ROOT, "nystr_self_attention_segment_b200", "csrc", f)) as fh:
                text = fh.read()
        else:
            text = read(f)
        h.update(code_tokens(text).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes (read + write) per launch from the committed ncu summary
    profiles/<kernel>_<workload>.md ("traffic_bytes:" and "source_digest:"
    lines), or None when absent or when the code of the kernel sources has
    changed since (comments and whitespace do not count)."""
    p = os.path.join(ROOT, "profiles", "%s_%s.md" % (kernel, workload))
    if not os.path.exists(p):
        return None
    vals = {}
    for line in open(p):
        if ":" in line and line.split(":", 1)[0].strip() in ("traffic_bytes", "source_digest"):
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    if vals.get("source_digest") != source_digest(kernel) or "traffic_bytes" not in vals:
        return None
    return int(float(vals["traffic_bytes"]))


# ----------------------------------------------------------------- config

def workload_config(wl, world):
    """The `config` object of the JSON line: the workload alone, identical for
    both arms."""
    return {"workload": wl.name, "batch": wl.batch, "heads": wl.heads,
            "seq_len": wl.seq_len, "head_dim": wl.head_dim, "landmarks": wl.landmarks,
            "pinv_iters": wl.pinv_iters, "conv_k": wl.conv_k, "values": wl.values,
            "dtype": wl.dtype,
            "parallelism": "dp%d (independent batches per GPU)" % world}


# ----------------------------------------------------------------- ranks

def max_over_ranks(x, world, device):
    """The max of a per-rank float over all ranks: one all-reduce, outside any
    timed region (identity for a single process)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank, world, ms_per_step):
    """Whole-job tokens/s: every rank processes its own batch (weak scaling),
    and the step takes as long as the slowest rank."""
    return tokens_per_rank * world / (ms_per_step / 1e3)


# ----------------------------------------------------------------- CPU oracle

def cpu_baseline(wl, seconds):
    """The fp64 oracle as it stands, on a bounded sample: whole heads of the
    workload, as many as fit in about `seconds`."""
    from oracle import nystrom as orc
    from nystr_self_attention_segment_b200.inputs import make_inputs
    x = make_inputs(wl, batch=1, heads=min(wl.heads, 4))
    heads = 0
    t0 = time.perf_counter()
    while True:
        h = heads % x["Q"].shape[1]
        orc.nystrom_head(x["Q"][0, h], x["K"][0, h], x["V"][0, h], wl.landmarks,
                         wl.pinv_iters, None if x["conv_w"] is None else x["conv_w"][h])
        heads += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    threads = None
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        pass
    return {"value": heads * wl.seq_len / el, "unit": "tokens/s",
            "cores": threads or os.cpu_count(), "host_cpus": os.cpu_count(), "kind": "oracle",
            "sample": "%d whole heads (n=%d, m=%d, d=%d, conv k=%d) of the workload in %.1f s, "
                      "fp64 numpy" % (heads, wl.seq_len, wl.landmarks, wl.head_dim, wl.conv_k, el)}


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """Polls the SM clock, its maximum, the power draw and the active clock
    event reasons through NVML (read-only queries) from a host thread, about
    once per millisecond, with host timestamps, so that samples can be
    assigned to the timed region.  Records nothing when NVML is unavailable.
    Changes no setting of the GPU."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "sw_power_cap": 0x4}

    def __init__(self, uuid, index, period_s=0.001):
        self.uuid = uuid
        self.index = index
        self.period = period_s
        self.samples = []          # (t, sm_mhz, max_mhz, reasons bitmask, power W)
        self.thread = None
        self.stop_flag = False
        self.source = None

    def start(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            try:
                h = pynvml.nvmlDeviceGetHandleByUUID(self.uuid)
            except Exception:
                h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.source = "nvml"
        except Exception:
            return

        def poll():
            smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            while not self.stop_flag:
                t = time.perf_counter()
                try:
                    sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                    rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    pw = pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0
                except Exception:
                    break
                self.samples.append((t, sm, smax, rs, pw))
                time.sleep(self.period)

        self.thread = threading.Thread(target=poll, daemon=True)
        self.thread.start()

    def stop(self):
        if self.thread is None:
            return
        self.stop_flag = True
        self.thread.join(timeout=5)

    def summary(self, windows):
        """Clock record over the samples that fall inside the given host-time
        windows [(t0, t1), ...]."""
        sel = [x for x in self.samples if any(a <= x[0] <= b for a, b in windows)]
        if not sel:
            return None
        reasons = sorted({nm for x in sel for nm, bit in self.REASONS.items() if x[3] & bit})
        return {"sm_mhz": statistics.median(x[1] for x in sel),
                "sm_min_mhz": min(x[1] for x in sel), "sm_max_mhz": max(x[2] for x in sel),
                "power_w_median": round(statistics.median(x[4] for x in sel), 1),
                "samples": len(sel), "reasons": reasons, "source": self.source}


# ----------------------------------------------------------------- backward

FP32_FMA_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12   # CUDA-core fp32 FMA, max clock


def backward_flops(wl):
    """fp32 flops of one backward step: per head the two streaming passes
    (rows: S, dF, dQ, dW, dK~; keys: S, dB, dK, dV, dQ~; 2 n m d each), the
    recomputed B~ V (4 n m d), the pseudoinverse forward and backward (8 m^3
    and about 28 m^3 per step) and the conv (4 n k d)."""
    n, m, d, k, it = wl.seq_len, wl.landmarks, wl.head_dim, wl.conv_k, wl.pinv_iters
    per_head = 24 * n * m * d + it * 36 * m ** 3 + 4 * n * k * d
    return wl.bh * per_head


def run_backward(args, rank, world):
    import torch
    import nystr_self_attention_segment_b200 as nys
    from nystr_self_attention_segment_b200.inputs import WORKLOADS, make_inputs
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    wl = WORKLOADS[args.workload]
    x = make_inputs(wl)
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    Q, K, V = (torch.from_numpy(x[k]).to(dev).to(tdt) for k in ("Q", "K", "V"))
    G = torch.randn(Q.shape, device=dev).to(tdt)
    cw = torch.from_numpy(x["conv_w"]).to(dev) if x["conv_w"] is not None else None
    nb = nys._lib.nys_attn_backward_workspace_size(nys.desc_of(Q), wl.landmarks, wl.pinv_iters,
                                                   wl.conv_k)
    ws = torch.empty(nb + 256, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        nys.nys_attn_backward(Q, K, V, wl.landmarks, G, wl.pinv_iters, cw, workspace=ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        nys.nys_attn_backward(Q, K, V, wl.landmarks, G, wl.pinv_iters, cw, workspace=ws)
    e1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    if rank != 0:
        return None
    fl = backward_flops(wl)
    ach = fl / (ms / 1e3) / 1e12
    return {"metric": "Nyström attention bwd tokens/sec (b×h×n)", "value": wl.tokens * world / (ms / 1e3),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32 arithmetic, %s tensors" % wl.dtype, "data": "synthetic",
            "config": workload_config(wl, world),
            "roofline": {"bound": "alu", "achieved": round(ach, 2), "peak": round(FP32_FMA_PEAK_TFLOPS, 1),
                         "unit": "TFLOP/s", "frac": round(ach / FP32_FMA_PEAK_TFLOPS, 4),
                         "traffic": None, "algorithmic_flops": fl,
                         "peak_source": "148 SMs x 128 fp32 FMA lanes x 2 x 1.965 GHz"}}


# ----------------------------------------------------------------- our arm

def run_ours(args, rank, world):
    import numpy as np
    import torch
    import torch.distributed as dist
    import nystr_self_attention_segment_b200 as nys
    from nystr_self_attention_segment_b200.inputs import WORKLOADS, make_inputs

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    wl = WORKLOADS[args.workload]
    m, iters = wl.landmarks, wl.pinv_iters
    x = make_inputs(wl)
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    host = {k: torch.from_numpy(x[k]).to(tdt).contiguous() for k in ("Q", "K", "V")}
    conv = torch.from_numpy(x["conv_w"]).to(dev) if x["conv_w"] is not None else None
    tensor_bytes = host["Q"].numel() * host["Q"].element_size()
    step_bytes = 4 * tensor_bytes
    rot = max(2, -(-2 * L2_BYTES // step_bytes) + 1)        # rotations: > 2 L2 between reuses
    sets = []
    for _ in range(rot):
        s = {k: v.to(dev) for k, v in host.items()}
        s["out"] = torch.empty_like(s["Q"])
        sets.append(s)
    ws = nys.Workspace(sets[0]["Q"], m)
    desc = nys.desc_of(sets[0]["Q"])
    nl = nys.nys_attn_launch_count(desc, m, wl.conv_k)
    names = nys.nys_attn_launch_names(desc, m)
    stream = torch.cuda.current_stream()

    def step(i, events=None):
        s = sets[i % rot]
        if events is None:
            nys.nys_attn_forward(s["Q"], s["K"], s["V"], m, iters, conv, s["out"], ws)
        else:
            nys.nys_attn_forward_timed(s["Q"], s["K"], s["V"], m, iters, conv, s["out"], ws,
                                       events)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    nys.nys_attn_check_error(ws)

    K = args.steps
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(nl + 1)] for _ in range(rot)]
    for evs in kev:                     # create the CUDA events before capture
        for e in evs:
            e.record()
    torch.cuda.synchronize()
    # CUDA graphs of the forward's launches (replays take the host launch cost
    # out of the device timeline): one graph of `rot` forwards, one per input
    # set in turn, and one single-forward graph per input set.  The timed
    # region replays the rot-forward graph K // rot times and then the first
    # K % rot single graphs: exactly K forwards, inputs rotating.  A second
    # set of single graphs with an event after each kernel gives the kernel
    # breakdown, outside the timed region (an event between two kernels
    # would serialise their programmatic overlap).
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    g_all = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_all, stream=cap):
        for i in range(rot):
            step(i)
    singles, tgraphs = [], []
    for i in range(rot):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            step(i)
        singles.append(g)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            step(i, kev[i])
        tgraphs.append(g)
    torch.cuda.synchronize()

    def replay(k):
        for _ in range(k // rot):
            g_all.replay()
        for i in range(k % rot):
            singles[i].replay()

    replay(max(args.warmup, rot))
    torch.cuda.synchronize()
    nys.nys_attn_check_error(ws)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid, dev.index if dev.index is not None else 0)
    clocks.start()
    time.sleep(0.05)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    h0 = time.perf_counter()
    t_start.record(stream)
    replay(K)
    t_end.record(stream)
    torch.cuda.synchronize()
    h1 = time.perf_counter()
    if world > 1:
        dist.barrier()
    total_ms = t_start.elapsed_time(t_end)
    # the same replays, untimed, for about 0.3 s: the clock record under
    # sustained load (the timed region itself is short at the default K)
    sus_steps = max(rot, int(0.3 / max(total_ms / K / 1e3, 1e-6)))
    h2 = time.perf_counter()
    replay(sus_steps)
    torch.cuda.synchronize()
    h3 = time.perf_counter()
    clocks.stop()
    nys.nys_attn_check_error(ws)
    clk = clocks.summary([(h0, h1), (h2, h3)])
    in_timed = clocks.summary([(h0, h1)])
    if clk is not None:
        clk["samples_in_timed_region"] = in_timed["samples"] if in_timed else 0
        clk["window"] = ("NVML samples at about 1 kHz during the timed region (%.1f ms) and "
                         "during %d more untimed replays of the same graphs right after it "
                         "(%.0f ms)" % ((h1 - h0) * 1e3, sus_steps, (h3 - h2) * 1e3))
    # per-kernel breakdown (not timed above): the evented single graphs
    reps = 3
    per_kernel = [0.0] * nl
    for _ in range(reps):
        for i in range(rot):
            tgraphs[i].replay()
            torch.cuda.synchronize()
            for j in range(nl):
                per_kernel[j] += kev[i][j].elapsed_time(kev[i][j + 1]) / (reps * rot)
    nys.nys_attn_check_error(ws)
    total_ms = max_over_ranks(total_ms, world, dev)

    # end to end through the host-buffer entry point (copies in the timed region)
    hb = nys.nys_attn_host_buffer_size(desc, m, wl.conv_k)
    dbuf = torch.empty(hb + 256, dtype=torch.uint8, device=dev)
    off = (-dbuf.data_ptr()) % 256
    dview = dbuf[off:off + hb]
    hp = {k: v.pin_memory() for k, v in host.items()}
    outh = torch.empty_like(hp["Q"]).pin_memory()
    convh = torch.from_numpy(x["conv_w"]).contiguous() if x["conv_w"] is not None else None
    for _ in range(2):
        nys.nys_attn_forward_host(hp["Q"], hp["K"], hp["V"], m, iters, convh, outh, dview)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    e0.record(stream)
    for _ in range(args.e2e_steps):
        nys.nys_attn_forward_host(hp["Q"], hp["K"], hp["V"], m, iters, convh, outh, dview)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / args.e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, world, dev)

    if rank != 0:
        return None
    pk = peaks()
    ms = total_ms / K
    tokens = wl.tokens * world
    value = job_throughput(wl.tokens, world, ms)
    # per-kernel algorithmic bytes (inputs read once + outputs written once)
    T = tensor_bytes
    kbytes = {"seg_means": 2 * T, "bv_partial": 2 * T, "out": 3 * T,
              "mid_tc": 2 * T, "out_tc": 3 * T, "fused": 4 * T}
    dom = max(range(nl), key=lambda j: per_kernel[j])
    dname = names[dom] if dom < len(names) else "kernel%d" % dom
    dbytes = kbytes.get(dname)
    roof = None
    if dbytes:
        ach = dbytes / (per_kernel[dom] / 1e3) / 1e9
        roof = {"bound": "hbm", "kernel": dname, "achieved": round(ach, 1),
                "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": round(ach / pk["hbm_gbs"], 4),
                "traffic": recorded_traffic(dname, wl.name), "algorithmic_bytes": dbytes,
                "avg_ms": round(per_kernel[dom], 5), "peak_source": pk["source"]}
    step_ach = step_bytes / (ms / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
        "config": workload_config(wl, world),
        "timing": {"launch": "CUDA graphs of the library's launches (chained by programmatic "
                             "dependent launch), replayed: K forwards in the timed region; "
                             "kernel times from separate replays with an event after each "
                             "kernel",
                   "l2": "inputs rotate over %d copies (%.0f MB per step set, above 2x L2); "
                         "no L2 flush" % (rot, step_bytes / 1e6)},
        "roofline": roof,
        "roofline_step": {"bound": "hbm", "achieved": round(step_ach, 1),
                          "peak": pk["hbm_gbs"], "unit": "GB/s",
                          "frac": round(step_ach / pk["hbm_gbs"], 4),
                          "algorithmic_bytes": step_bytes},
        "kernels_ms": {names[j] if j < len(names) else str(j): round(per_kernel[j], 5)
                       for j in range(nl)},
        "gpu_launches": nl * K,
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": 3 * T + (x["conv_w"].nbytes if x["conv_w"] is not None else 0),
                "d2h_bytes_per_step": T, "ms_per_step": e2e_ms},
        "clocks": clk,
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds)
    return line


def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle on the host cores (rank 0 only),
    each step a bounded sample (one head) of the workload."""
    if rank != 0:
        return None
    from oracle import nystrom as orc
    from nystr_self_attention_segment_b200.inputs import WORKLOADS, make_inputs
    wl = WORKLOADS[args.workload]
    x = make_inputs(wl, batch=1, heads=1)
    w = None if x["conv_w"] is None else x["conv_w"][0]

    def one():
        orc.nystrom_head(x["Q"][0, 0], x["K"][0, 0], x["V"][0, 0], wl.landmarks,
                         wl.pinv_iters, w)
    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    el = time.perf_counter() - t0
    ms = el / args.steps * 1e3
    value = wl.seq_len / (ms / 1e3)
    threads = os.cpu_count()
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [threads])
    except Exception:
        pass
    sample = "one head (n=%d, m=%d, d=%d) of %s per step, fp64 numpy oracle" % (
        wl.seq_len, wl.landmarks, wl.head_dim, wl.name)
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def launch_ranks(args):
    """`--gpus N` without a launcher: start N ranks on this node with
    torch.distributed.run (127.0.0.1 rendezvous) and return their status."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           "--nproc-per-node=%d" % args.gpus, "--master-addr", "127.0.0.1",
           "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.gpus != world:
        if "WORLD_SIZE" not in os.environ and args.gpus > 1:
            sys.exit(launch_ranks(args))
        sys.exit("bench.py: --gpus %d but WORLD_SIZE is %d; launch one process per GPU "
                 "(torch.distributed.run --nproc-per-node %d) or drop --gpus"
                 % (args.gpus, world, args.gpus))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    import datetime
    import torch.distributed as dist
    if world > 1:
        import torch
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        line = run_backward(args, rank, world) if args.backward else run_ours(args, rank, world)
    finally:
        if world > 1:
            dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
