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
    "mid_tc": ["common.cuh", "sm100.cuh", "pinv_pow.cuh", "pinv_tc.cuh", "mid_tc.cuh"],
    "out_tc": ["common.cuh", "sm100.cuh", "out_tc.cuh"],
    "seg_means": ["common.cuh", "sm100.cuh", "stream_bf16.cuh"],
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
    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.path = os.path.join("/tmp", "nys_clocks_%d.csv" % os.getpid())

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [c.strip() for c in line.split(",")]
            if len(f) < 10 or (self.uuid and f[1] != self.uuid):
                continue
            try:
                sm.append(float(f[2]))
                smax.append(float(f[3]))
            except ValueError:
                continue
            for nm, v in zip(names, f[6:10]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "samples": len(sm), "reasons": sorted(reasons)}


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
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(nl + 1)] for _ in range(K)]
    for evs in kev:                     # create the CUDA events before capture
        for e in evs:
            e.record()
    torch.cuda.synchronize()
    # One CUDA graph per timed step (the forward's launches, with its own
    # timing events as graph nodes), input sets rotating as above.  Replaying
    # graphs takes the host launch cost out of the device timeline.
    # The timed graphs hold plain forwards (an event between two kernels
    # would serialise their programmatic overlap); a second set with
    # per-kernel events gives the kernel breakdown, outside the timed region.
    graphs, tgraphs = [], []
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    for i in range(K):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            step(args.warmup + i)
        graphs.append(g)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            step(args.warmup + i, kev[i])
        tgraphs.append(g)
    torch.cuda.synchronize()
    for i in range(min(args.warmup, K)):
        graphs[i].replay()
    torch.cuda.synchronize()
    nys.nys_attn_check_error(ws)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_start.record(stream)
    for i in range(K):
        graphs[i].replay()
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    nys.nys_attn_check_error(ws)
    total_ms = t_start.elapsed_time(t_end)
    for i in range(K):            # per-kernel breakdown (not timed above)
        tgraphs[i].replay()
    torch.cuda.synchronize()
    nys.nys_attn_check_error(ws)
    per_kernel = [sum(kev[i][j].elapsed_time(kev[i][j + 1]) for i in range(K)) / K
                  for j in range(nl)]
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
        "config": {"workload": wl.name, "batch": wl.batch, "heads": wl.heads,
                   "seq_len": wl.seq_len, "head_dim": wl.head_dim, "landmarks": m,
                   "pinv_iters": iters, "conv_k": wl.conv_k, "values": wl.values,
                   "parallelism": "dp%d (independent batches per GPU)" % world,
                   "launch": "one CUDA graph per step (the library's launches, chained by "
                             "programmatic dependent launch), replayed; kernel times from a "
                             "separate replay with an event after each kernel",
                   "l2": "inputs rotate over %d copies (%.0f MB per step set); no L2 flush"
                         % (rot, step_bytes / 1e6)},
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


def run_reference(args, rank):
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
            "config": {"workload": wl.name, "batch": wl.batch, "heads": wl.heads,
                       "seq_len": wl.seq_len, "head_dim": wl.head_dim,
                       "landmarks": wl.landmarks},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank)
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
        line = run_ours(args, rank, world)
    finally:
        if world > 1:
            dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
