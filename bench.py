"""Benchmark of the EFLA forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl efla|reference]

One step = one efla_chunk_fwd call over the 1.3B-layer workload (B=4, H=16, T=2048,
d_k=d_v=128, chunk 64, bf16 in / fp32 state): the gate, the intra-chunk UT transform and
the inter-chunk state propagation, fused.  Multi-GPU (torchrun, one rank per GPU) is data
parallel over independent (b, h) streams: every rank runs its own batch with no data-path
collective (weak scaling); the timing is the max over ranks.  The single-token decode step
(N=256, H=16, d=128, fp32 state, in place) and the backward pass on the forward's workload
are measured in the same run and reported under "decode" and "backward".  Rank 0 prints
one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

WORKLOAD = workloads.CHUNK_WORKLOADS["lm1p3b_bf16"]
DECODE = workloads.DECODE_WORKLOAD
METRIC = "EFLA fwd tokens/s (B4 H16 T2048 d128 bf16)"
N_ROTATE = 4            # rotating input sets: 4 x 139 MB > 126 MB L2, so no set is L2-resident


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, "fallback"


def chunk_alg(w):
    """Algorithmic bytes and flops of one forward call.

    Bytes: read q, k, v, beta and write o (2 bytes each) plus S_T (fp32) and S0 if given.
    Flops per (stream, chunk): KK^T, QK^T, TK, TV, P Delta (5 x 2 C^2 d) and WS, QS, K^T Delta
    (3 x 2 C d^2), with C = 64, d = d_k = d_v.
    """
    es = 2 if w.dtype == torch.bfloat16 else 4
    BH, T, d = w.B * w.H, w.T, w.dk
    nbytes = BH * T * (3 * d * es + es + d * es) + BH * d * d * 4
    if w.s0_std is not None:
        nbytes += BH * d * d * 4
    chunks = (T + 63) // 64
    flops = BH * chunks * (5 * 2 * 64 * 64 * d + 3 * 2 * 64 * d * d)
    return nbytes, flops


def decode_alg(w):
    """One decode step: read + write the fp32 state, read q, k, v, beta, write o."""
    NH, d = w.N * w.H, w.dk
    return NH * (2 * d * d * 4 + (3 * d + 1 + d) * 4), NH * 6 * d * d


# The sources each entry point's kernels are compiled from (the C-ABI glue and the other
# entry points' files excluded): a traffic figure stays valid while these are unchanged.
KERNEL_SOURCES = {
    "efla_chunk_fwd": ["efla_chunk_tc.cu", "efla_ut.cu", "efla_ut_tf32.cuh", "efla_ut_solve.cuh",
                       "efla_chunk_simt.cu", "efla_common.cuh", "efla_tma.cuh", "sm100.cuh"],
    "efla_recurrent_step": ["efla_decode.cu", "efla_common.cuh"],
    "efla_backward": ["efla_bwd.cu", "efla_bwd_chunk.cu", "efla_chunk_tc.cu", "efla_ut.cu",
                      "efla_ut_tf32.cuh", "efla_common.cuh", "efla_tma.cuh", "sm100.cuh"],
    "efla_backward_saved": ["efla_bwd_chunk.cu", "efla_common.cuh", "efla_tma.cuh", "sm100.cuh"],
}


def backward_alg(w):
    """One backward call, counted for the method's chunked form (not for the kernel as built).

    Bytes: read q, k, v, dO, beta (w.dtype), write dq, dk, dv, dbeta (fp32) and dS0 (fp32).
    Flops per (stream, chunk): the forward's chunk products recomputed (5 x 2 C^2 d +
    3 x 2 C d^2) and their transposed products for the gradients, two per forward product
    (dA = dC B^T, dB = A^T dC): 3 x the forward's count.
    """
    es = 2 if w.dtype == torch.bfloat16 else 4
    BH, T, d = w.B * w.H, w.T, w.dk
    nbytes = BH * T * (4 * d * es + es + 3 * d * 4 + 4) + BH * d * d * 4
    chunks = (T + 63) // 64
    flops = 3 * BH * chunks * (5 * 2 * 64 * 64 * d + 3 * 2 * 64 * d * d)
    return nbytes, flops


def roofline_record(nbytes, flops, seconds, hbm, tc, peak_kind):
    """Roofline of one call from its algorithmic bytes and flops and its measured time: the
    bound is whichever of bytes / HBM bandwidth and flops / tensor peak takes longer, and
    frac = that time / the measured time."""
    t_hbm, t_tc = nbytes / (hbm * 1e9), flops / (tc * 1e12)
    if t_hbm >= t_tc:
        rec = {"bound": "hbm", "achieved": nbytes / seconds / 1e9, "peak": hbm, "unit": "GB/s",
               "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"}
    else:
        rec = {"bound": "tensor", "achieved": flops / seconds / 1e12, "peak": tc, "unit": "TFLOP/s",
               "peak_source": f"{peak_kind} cuBLAS bf16 burst (MEASURED_PEAKS.json bf16_tflops)"}
    rec["frac"] = max(t_hbm, t_tc) / seconds
    rec.update({"alg_bytes_per_launch": nbytes, "alg_flops_per_launch": flops,
                "tensor_tflops": flops / seconds / 1e12, "hbm_gbs": nbytes / seconds / 1e9,
                "roofline_time_us": max(t_hbm, t_tc) * 1e6})
    return rec


def kernel_source_hash(entry=None):
    """sha256 prefix over the kernel sources of one entry point (all of csrc/ for None)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "delta_rule_linear_02_b200", "csrc")
    names = sorted(os.listdir(csrc)) if entry is None else sorted(KERNEL_SOURCES[entry])
    for name in names:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


TRAFFIC_JSON = os.path.join(ROOT, "profiles", "traffic.json")
# the kernels each entry point launches (ncu kernel-name prefixes)
ENTRY_KERNELS = {
    "efla_chunk_fwd": ("ut_kernel", "chunk_tc_kernel"),
    "efla_recurrent_step": ("decode_kernel",),
    "efla_backward": ("ut_kernel", "chunk_tc_kernel", "bwd_chain_kernel", "bwd_tile_kernel"),
    "efla_backward_saved": ("bwd_chain_kernel", "bwd_tile_kernel"),
}


def ncu_traffic(entry: str):
    """DRAM bytes (read + write) per call of an entry point, from profiles/traffic.json as
    written by --traffic-from; None unless it was recorded for the current kernel sources."""
    try:
        with open(TRAFFIC_JSON) as f:
            rec = json.load(f).get(entry)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("kernel_source") != kernel_source_hash(entry):
        return None
    return int(rec["bytes_per_call"])


def traffic_from_csv(csv_path: str, entry: str, calls: int):
    """Write profiles/traffic.json's record for `entry` from an ncu --csv log of
    dram__bytes_read.sum and dram__bytes_write.sum: the last `calls` calls' launches of the
    entry point's kernels, summed and divided by `calls`."""
    import csv
    rows = []
    with open(csv_path) as f:
        lines = [ln for ln in f if ln.startswith('"')]
    def bare(name):      # "void efla::<unnamed>::decode_kernel<float, 128, 0>(...)" -> "decode_kernel"
        head = name.replace("(anonymous namespace)", "anon").split("(")[0].strip()
        if head.endswith(">"):                       # drop the trailing template arguments
            depth, i = 0, len(head) - 1
            while i >= 0:
                depth += {">": 1, "<": -1}.get(head[i], 0)
                if depth == 0:
                    break
                i -= 1
            head = head[:i]
        return head.split("::")[-1].split(" ")[-1].strip()

    for r in csv.DictReader(lines):
        name = bare(r.get("Kernel Name", ""))
        if name in ENTRY_KERNELS[entry] and r.get("Metric Name", "").startswith("dram__bytes_"):
            unit = r.get("Metric Unit", "byte")
            scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "KB": 1e3, "MB": 1e6, "GB": 1e9}.get(unit, 1)
            rows.append((int(r["ID"]), name, r["Metric Name"], float(r["Metric Value"].replace(",", "")) * scale))
    ids = sorted({i for i, _, _, _ in rows})
    per_call = len(ENTRY_KERNELS[entry])
    keep = set(ids[-calls * per_call:])
    total = sum(v for i, _, _, v in rows if i in keep)
    rec = {"bytes_per_call": int(round(total / calls)), "calls": calls,
           "launches": len(keep), "kernel_source": kernel_source_hash(entry),
           "kernels": sorted({n for i, n, _, _ in rows if i in keep}),
           "from": os.path.basename(csv_path)}
    try:
        with open(TRAFFIC_JSON) as f:
            data = json.load(f)
    except (OSError, ValueError):
        data = {}
    data[entry] = rec
    with open(TRAFFIC_JSON, "w") as f:
        json.dump(data, f, indent=1, sort_keys=True)
        f.write("\n")
    return rec


class Clocks:
    """SM clock and throttle-reason sampler (NVML, a background thread polling every ~2 ms)
    running during the timed region."""
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.max_mhz = None
        self._stop = None

    def __enter__(self):
        try:
            import threading
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self._stop = threading.Event()

            def run():
                while not self._stop.is_set():
                    try:
                        mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                        rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((mhz, rs))
                    except Exception:  # pragma: no cover
                        pass
                    time.sleep(0.002)

            self._thread = threading.Thread(target=run, daemon=True)
            self._thread.start()
            time.sleep(0.02)
        except Exception:
            self._stop = None
        return self

    def __exit__(self, *exc):
        if self._stop is not None:
            self._stop.set()
            self._thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return None
        reasons = sorted({n for _, rs in self.samples for n, bit in self.REASONS.items() if rs & bit})
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples), "source": "NVML, ~2 ms polling"}


def dist_setup(backend: str = "nccl"):
    """Rank, world size and local rank from the torchrun environment; joins the process
    group when there is more than one rank (NCCL on GPUs, gloo for host-only use)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return rank, world, local


def barrier(world):
    if torch.cuda.is_available():
        torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """The largest of the ranks' values (every rank gets it): device times are reported
    as the slowest rank's."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_seed(rank: int) -> int:
    """Each rank draws its own independent batch of streams (weak scaling)."""
    return WORKLOAD.seed + 1000 * rank


def rank_workload(rank: int, world: int):
    """The rank's share of the job and the job's total tokens per step: every rank runs a
    full bench workload of its own streams (weak scaling; streams never interact, so no
    data-path collective exists)."""
    w = WORKLOAD.replace(seed=shard_seed(rank))
    return w, w.tokens * world


def cpu_baseline(w, cpu_seconds: float = 12.0):
    """The fp64 oracle, as it stands, on the workload's streams: whole passes over all
    B*H streams, repeated until about `cpu_seconds` of CPU work (wall x threads) is done;
    and the same oracle on one thread over a sample of 4 streams."""
    import oracle
    inp = workloads.make_chunk_inputs(w)
    threads = oracle.default_threads()
    passes, t0 = 0, time.perf_counter()
    while True:
        oracle.fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["S0"], threads=threads)
        passes += 1
        dt = time.perf_counter() - t0
        if dt * threads >= cpu_seconds or dt >= 60.0:
            break
    tokens = passes * w.B * w.T                 # a token spans all H heads
    n1 = 4
    one = {k: (None if v is None else v[0, :n1].unsqueeze(0).contiguous()) for k, v in inp.items()}
    t1 = time.perf_counter()
    oracle.fwd(one["q"], one["k"], one["v"], one["beta"], one["S0"], threads=1)
    dt1 = time.perf_counter() - t1
    return {"value": tokens / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{passes} full pass(es) over all {w.B * w.H} (b,h) streams of the workload "
                      f"(T={w.T}), {dt:.1f} s wall on {threads} threads",
            "single_thread": {"value": n1 * w.T / w.H / dt1, "unit": "tokens/s", "cores": 1,
                              "sample": f"{n1} of {w.B * w.H} (b,h) streams at T={w.T} on 1 thread, "
                                        f"{dt1:.2f} s; tokens counted as streams x T / H"}}


def run_reference(args):
    """The oracle as the reference arm: rank 0 only, each step a bounded sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    w = WORKLOAD
    streams = 8
    inp = workloads.make_chunk_inputs(w.replace(B=1, H=streams))
    threads = oracle.default_threads()
    for _ in range(args.warmup):
        oracle.fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["S0"], threads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["S0"], threads=threads)
    dt = (time.perf_counter() - t0) / args.steps
    tokens = streams * w.T / w.H
    value = tokens / dt
    sample = f"{streams} of {w.B * w.H} (b,h) streams at full T={w.T} per step"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "d_k": w.dk, "d_v": w.dv,
                   "chunk": w.chunk, "parallelism": f"dp{args.gpus}"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def profile_call(args):
    """warm-up + steps calls of one entry point on its bench workload and nothing else, so
    that an ncu capture (-s warm-up launches, -c launches) sees only those launches."""
    import delta_rule_linear_02_b200 as efla
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    if args.profile_call == "decode":
        S = workloads.make_decode_state(DECODE, device=dev)
        n = args.warmup + args.steps
        st = workloads.make_decode_steps(DECODE, steps=n, device=dev)
        o = torch.empty(DECODE.N, DECODE.H, DECODE.dv, device=dev)
        calls = [lambda i=i: efla.efla_recurrent_step(st["q"][i], st["k"][i], st["v"][i], st["beta"][i], S,
                                                       o=o, stream=stream) for i in range(n)]
    else:
        w = workloads.CHUNK_WORKLOADS["longctx_bf16"] if args.profile_call.startswith("long") else WORKLOAD
        x = {k: (None if v is None else v.to(dev)) for k, v in workloads.make_chunk_inputs(w).items()}
        B, H, T, d = w.B, w.H, w.T, w.dk
        if args.profile_call == "longseg":
            n = efla.lib.efla_chunk_fwd_segmented_workspace_bytes(B, H, T, d, d, 64, 1, 0, 0)
            ws = torch.zeros(n, dtype=torch.uint8, device=dev)
            one = lambda: efla.efla_chunk_fwd_segmented(x["q"], x["k"], x["v"], x["beta"], x["S0"], workspace=ws,
                                                        stream=stream)
        elif args.profile_call == "gated":
            gd = workloads.make_log_decay((B, H, T), w.seed + 7).to(dev)
            one = lambda: efla.efla_chunk_fwd_gated(x["q"], x["k"], x["v"], x["beta"], gd, x["S0"], stream=stream)
        elif args.profile_call in ("fwd", "long"):
            ws = efla.new_workspace(B, H, T, d, d, 64, w.dtype, dev)
            o = torch.empty(B, H, T, d, dtype=w.dtype, device=dev)
            ST = torch.empty(B, H, d, d, dtype=torch.float32, device=dev)
            # --profile-rotate N: N input sets taken in turn, as in the timed region (so that an
            # ncu capture with --cache-control none sees the L2 state the timed calls see)
            xs = [x] + [{k: (None if v is None else v.to(dev))
                         for k, v in workloads.make_chunk_inputs(w.replace(seed=w.seed + 1 + r)).items()}
                        for r in range(max(1, args.profile_rotate) - 1)]
            calls = [lambda xi=xs[i % len(xs)]: efla.efla_chunk_fwd(xi["q"], xi["k"], xi["v"], xi["beta"], xi["S0"],
                                                                    o=o, S_T=ST, workspace=ws, stream=stream)
                     for i in range(args.warmup + args.steps)]
            one = None
        else:
            dO = workloads.make_cotangents(w, with_state_grad=False)["dO"].to(dev)
            f32 = dict(device=dev, dtype=torch.float32)
            g = (torch.empty(B, H, T, d, **f32), torch.empty(B, H, T, d, **f32), torch.empty(B, H, T, d, **f32),
                 torch.empty(B, H, T, **f32), torch.empty(B, H, d, d, **f32))
            if args.profile_call == "bwd":
                wsb = torch.zeros(efla.efla_backward_workspace_bytes(B, H, T, d, d, w.dtype), dtype=torch.uint8,
                                  device=dev)
                one = lambda: efla.efla_backward(x["q"], x["k"], x["v"], x["beta"], dO, grads=g, workspace=wsb,
                                                 stream=stream)
            else:       # the backward from saved residuals; the forward that saves them runs once first
                ob = torch.empty(B, H, T, d, dtype=w.dtype, device=dev)
                _, _, saved = efla.efla_chunk_fwd_save(x["q"], x["k"], x["v"], x["beta"], o=ob, want_state=False,
                                                       stream=stream)
                wss = torch.zeros(efla.lib.efla_backward_saved_workspace_bytes(B, H, T, d, d, efla.EFLA_DTYPE_BF16),
                                  dtype=torch.uint8, device=dev)
                one = lambda: efla.efla_backward_saved(x["q"], x["k"], x["v"], x["beta"], dO, saved, grads=g,
                                                       workspace=wss, stream=stream)
        if one is not None:
            calls = [one] * (args.warmup + args.steps)
    for c in calls:
        c()
    torch.cuda.synchronize(dev)
    print(json.dumps({"profile_call": args.profile_call, "calls": len(calls)}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="efla", choices=["efla", "reference"])
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--bwd-steps", type=int, default=5,
                    help="backward calls timed on the forward's workload (0: skip)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--other-steps", type=int, default=10,
                    help="forwards timed on each of the long-context and stiff workloads (0: skip)")
    ap.add_argument("--profile-call", choices=["fwd", "decode", "bwd", "bwd_saved", "long", "longseg", "gated"],
                    help="only run warm-up + steps calls of one entry point (for an ncu capture)")
    ap.add_argument("--profile-rotate", type=int, default=1,
                    help="with --profile-call fwd: input sets taken in turn (the timed region uses %d)" % N_ROTATE)
    ap.add_argument("--traffic-from", metavar="CSV",
                    help="write profiles/traffic.json's record from an ncu --csv log of "
                         "dram__bytes_read.sum and dram__bytes_write.sum, then exit")
    ap.add_argument("--traffic-entry", default="efla_chunk_fwd", choices=sorted(ENTRY_KERNELS))
    ap.add_argument("--traffic-calls", type=int, default=1,
                    help="calls of the entry point at the end of the CSV that the record averages")
    args = ap.parse_args()
    if args.traffic_from:
        print(json.dumps(traffic_from_csv(args.traffic_from, args.traffic_entry, args.traffic_calls)))
        return
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        run_reference(args)
        return
    if args.profile_call:
        profile_call(args)
        return

    import delta_rule_linear_02_b200 as efla
    rank, world, local = dist_setup("nccl")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    w, tokens = rank_workload(rank, world)
    hbm, tc, peak_kind = peaks()

    # ---- device-resident inputs: N_ROTATE independent sets, so every step misses L2
    sets = []
    for i in range(N_ROTATE):
        inp = workloads.make_chunk_inputs(w.replace(seed=w.seed + 97 * i))
        sets.append({k: (None if v is None else v.to(dev)) for k, v in inp.items()})
    B, H, T, d = w.B, w.H, w.T, w.dk
    ws = efla.new_workspace(B, H, T, d, d, 64, w.dtype, dev)
    outs = [(torch.empty(B, H, T, d, dtype=w.dtype, device=dev),
             torch.empty(B, H, d, d, dtype=torch.float32, device=dev)) for _ in range(N_ROTATE)]

    def step(i):
        s, (o, ST) = sets[i % N_ROTATE], outs[i % N_ROTATE]
        efla.efla_chunk_fwd(s["q"], s["k"], s["v"], s["beta"], s["S0"], o=o, S_T=ST,
                            workspace=ws, stream=stream)

    for i in range(args.warmup):
        step(i)
    barrier(world)
    # the timed region holds exactly the K calls; the per-call events are taken in a second,
    # untimed pass of the same calls (recording them between the calls would add to the time)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * args.steps + 2)]
    with Clocks(local) as clk:
        ev[0].record(stream)
        for i in range(args.steps):
            step(i)
        ev[1].record(stream)
        barrier(world)
    total_ms = max_over_ranks(ev[0].elapsed_time(ev[1]), world)
    for i in range(args.steps):
        ev[2 + 2 * i].record(stream)
        step(i)
        ev[3 + 2 * i].record(stream)
    torch.cuda.synchronize(dev)
    launch_ms = statistics.mean(ev[2 + 2 * i].elapsed_time(ev[3 + 2 * i]) for i in range(args.steps))
    launch_ms = max_over_ranks(launch_ms, world)
    status = efla.efla_workspace_status(ws, clear=True, stream=stream)
    if status != efla.EFLA_OK:
        raise SystemExit(f"device reported {efla.efla_status_string(status)}")
    ms_per_step = total_ms / args.steps
    value = tokens / (ms_per_step * 1e-3)

    nbytes, flops = chunk_alg(w)
    # the same timed region as `value`: whole-region time / steps
    roofline = roofline_record(nbytes, flops, ms_per_step * 1e-3, hbm, tc, peak_kind)
    roofline.update({"traffic": ncu_traffic("efla_chunk_fwd"), "timed": "whole timed region / steps",
                     "call_events_mean_us": launch_ms * 1e3})

    # ---- end to end through the public API with host buffers (pinned), copies timed.
    # Every step copies its inputs from pinned host memory and reads its result (o and
    # S_T) back; steps are pipelined two deep on three streams, as a serving loop would
    # run them: the upload of step i+1 and the download of step i-1 overlap the forward of
    # step i (PCIe is full duplex).
    host = {k: (None if v is None else v.cpu().pin_memory()) for k, v in sets[0].items()}
    o_h = [torch.empty(B, H, T, d, dtype=w.dtype).pin_memory() for _ in range(2)]
    ST_h = [torch.empty(B, H, d, d, dtype=torch.float32).pin_memory() for _ in range(2)]
    dbuf = [{k: (None if v is None else torch.empty_like(v, device=dev)) for k, v in host.items()}
            for _ in range(2)]
    outd = [outs[0], outs[1]]
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = o_h[0].numel() * o_h[0].element_size() + ST_h[0].numel() * ST_h[0].element_size()
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    up_done = [torch.cuda.Event() for _ in range(2)]
    fw_done = [torch.cuda.Event() for _ in range(2)]
    down_done = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        b = i % 2
        with torch.cuda.stream(s_up):
            if i >= 2:
                s_up.wait_event(fw_done[b])             # the forward of step i-2 has read dbuf[b]
            for k, v in host.items():
                if v is not None:
                    dbuf[b][k].copy_(v, non_blocking=True)
            up_done[b].record(s_up)
        stream.wait_event(up_done[b])
        if i >= 2:
            stream.wait_event(down_done[b])             # step i-2's results have left outd[b]
        efla.efla_chunk_fwd(dbuf[b]["q"], dbuf[b]["k"], dbuf[b]["v"], dbuf[b]["beta"], dbuf[b]["S0"],
                            o=outd[b][0], S_T=outd[b][1], workspace=ws, stream=stream)
        fw_done[b].record(stream)
        with torch.cuda.stream(s_down):
            s_down.wait_event(fw_done[b])
            o_h[b].copy_(outd[b][0], non_blocking=True)
            ST_h[b].copy_(outd[b][1], non_blocking=True)
            down_done[b].record(s_down)

    e2e_steps = max(4, min(args.steps, 20))
    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    for i in range(e2e_steps):
        e2e_step(i)
    e1.record(s_down)                                   # after the last download
    torch.cuda.synchronize(dev)
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / e2e_steps
    e2e = {"value": tokens / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
           "pipeline": "2 steps in flight: upload, forward and download on three streams"}
    del sets, outs, dbuf, o_h, ST_h

    # ---- decode step (N=256, H=16, d=128, fp32 state updated in place)
    dec = None
    if args.decode_steps > 0:
        wd = DECODE.replace(seed=DECODE.seed + 1000 * rank)
        S = workloads.make_decode_state(wd, device=dev)
        nd = args.decode_steps
        st = workloads.make_decode_steps(wd, steps=nd + args.warmup, device=dev)
        o_dec = torch.empty(wd.N, wd.H, wd.dv, device=dev)
        for i in range(args.warmup):
            efla.efla_recurrent_step(st["q"][i], st["k"][i], st["v"][i], st["beta"][i], S, o=o_dec,
                                     stream=stream)
        barrier(world)
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        d0.record(stream)
        for i in range(args.warmup, args.warmup + nd):
            efla.efla_recurrent_step(st["q"][i], st["k"][i], st["v"][i], st["beta"][i], S, o=o_dec,
                                     stream=stream)
        d1.record(stream)
        barrier(world)
        dms = max_over_ranks(d0.elapsed_time(d1), world) / nd
        dbytes, dflops = decode_alg(wd)
        dach = dbytes / (dms * 1e-3) / 1e9
        dec = {"metric": "EFLA decode tokens/s (N256 H16 d128 fp32 state, in place)",
               "value": wd.N * world / (dms * 1e-3), "unit": "tokens/s", "us_per_step": dms * 1e3,
               "steps": nd, "dtype": "f32",
               "roofline": {"bound": "hbm", "achieved": dach, "peak": hbm, "unit": "GB/s",
                            "frac": dach / hbm, "traffic": ncu_traffic("efla_recurrent_step"),
                            "alg_bytes_per_launch": dbytes, "alg_flops_per_launch": dflops},
               "gpu_launches": nd}
        del S, st

    # ---- backward (training) pass on the forward's workload: dq, dk, dv, dbeta, dS0 from dO
    bwd = None
    if args.bwd_steps > 0:
        wb = w.replace(seed=w.seed + 500)
        xb = {k_: v_.to(dev) for k_, v_ in workloads.make_chunk_inputs(wb).items() if v_ is not None}
        cb = workloads.make_cotangents(wb, with_state_grad=False)
        dOb = cb["dO"].to(dev)
        f32 = dict(device=dev, dtype=torch.float32)
        gb = (torch.empty(B, H, T, d, **f32), torch.empty(B, H, T, d, **f32), torch.empty(B, H, T, d, **f32),
              torch.empty(B, H, T, **f32), torch.empty(B, H, d, d, **f32))
        wsb = torch.zeros(efla.efla_backward_workspace_bytes(B, H, T, d, d, wb.dtype), dtype=torch.uint8, device=dev)
        callb = lambda: efla.efla_backward(xb["q"], xb["k"], xb["v"], xb["beta"], dOb, grads=gb, workspace=wsb,
                                           stream=stream)
        for _ in range(args.warmup):
            callb()
        barrier(world)
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b0.record(stream)
        for _ in range(args.bwd_steps):
            callb()
        b1.record(stream)
        barrier(world)
        bms = max_over_ranks(b0.elapsed_time(b1), world) / args.bwd_steps
        bbytes, bflops = backward_alg(wb)
        brf = roofline_record(bbytes, bflops, bms * 1e-3, hbm, tc, peak_kind)
        brf["traffic"] = ncu_traffic("efla_backward")
        bwd = {"metric": "EFLA backward tokens/s (B4 H16 T2048 d128 bf16 in, fp32 state and gradients)",
               "value": wb.tokens * world / (bms * 1e-3), "unit": "tokens/s", "ms_per_step": bms,
               "steps": args.bwd_steps, "dtype": "bf16", "grad_dtype": "f32",
               "roofline": brf, "roofline_basis": "the method's chunked form: bytes at HBM, 3x forward flops at tensor peak",
               # bf16, d = 128: the UT kernel, the forward chain storing states, the reverse chain and
               # the per-chunk gradient kernel per call
               "gpu_launches": 4 * args.bwd_steps}
        # training with saved residuals: the forward keeps T and every chunk's entering state
        # (efla_chunk_fwd_save) and the backward reads them instead of recomputing them
        ob = torch.empty(B, H, T, d, device=dev, dtype=wb.dtype)
        _, _, saved = efla.efla_chunk_fwd_save(xb["q"], xb["k"], xb["v"], xb["beta"], o=ob, want_state=False,
                                               stream=stream)
        wss = torch.zeros(efla.lib.efla_backward_saved_workspace_bytes(B, H, T, d, d, efla.EFLA_DTYPE_BF16),
                          dtype=torch.uint8, device=dev)
        call_fs = lambda: efla.efla_chunk_fwd_save(xb["q"], xb["k"], xb["v"], xb["beta"], o=ob, want_state=False,
                                                   saved=saved, stream=stream)
        call_bs = lambda: efla.efla_backward_saved(xb["q"], xb["k"], xb["v"], xb["beta"], dOb, saved, grads=gb,
                                                   workspace=wss, stream=stream)

        def timed(fn, steps):
            for _ in range(args.warmup):
                fn()
            barrier(world)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(steps):
                fn()
            e1.record(stream)
            barrier(world)
            return max_over_ranks(e0.elapsed_time(e1), world) / steps

        bs_ms = timed(call_bs, args.bwd_steps)
        ts_ms = timed(lambda: (call_fs(), call_bs()), args.bwd_steps)
        bsrf = roofline_record(bbytes, bflops, bs_ms * 1e-3, hbm, tc, peak_kind)
        bsrf["traffic"] = ncu_traffic("efla_backward_saved")
        bwd["saved_residuals"] = {
            "what": "efla_backward_saved: the same gradients from T and the chunk states that "
                    "efla_chunk_fwd_save kept (no forward recompute)",
            "ms_per_step": bs_ms, "value": wb.tokens * world / (bs_ms * 1e-3), "unit": "tokens/s",
            "roofline": bsrf, "gpu_launches": 2 * args.bwd_steps}
        bwd["train_step"] = {
            "what": "efla_chunk_fwd_save then efla_backward_saved, one training step of the layer's recurrence",
            "ms_per_step": ts_ms, "value": wb.tokens * world / (ts_ms * 1e-3), "unit": "tokens/s",
            "gpu_launches": 4 * args.bwd_steps}
        del xb, dOb, gb, wsb, ob, saved, wss

    # ---- the other forward workloads (long context, stiff keys): tokens/s and roofline
    # fraction of a few forwards each, inputs resident in HBM, CUDA events around the calls
    others = {}
    for name in ([] if args.other_steps <= 0 else ["longctx_bf16", "longctx_bf16_segmented", "stiff_bf16",
                                                    "lm1p3b_bf16_gated"]):
        gated = name.endswith("_gated")
        segmented = name.endswith("_segmented")
        wo = workloads.CHUNK_WORKLOADS[name.removesuffix("_gated").removesuffix("_segmented")]
        wo = wo.replace(seed=wo.seed + 1000 * rank)
        xo = {k_: (None if v_ is None else v_.to(dev)) for k_, v_ in workloads.make_chunk_inputs(wo).items()}
        oo = torch.empty(wo.B, wo.H, wo.T, wo.dv, dtype=wo.dtype, device=dev)
        So = torch.empty(wo.B, wo.H, wo.dk, wo.dv, dtype=torch.float32, device=dev)
        if gated:   # Gated EFLA: the same shape with a per-token log-decay
            go = workloads.make_log_decay((wo.B, wo.H, wo.T), wo.seed + 7).to(dev)
            wso = torch.zeros(efla.lib.efla_chunk_fwd_gated_workspace_bytes(wo.B, wo.H, wo.T, wo.dk, wo.dv, 64, 1),
                              dtype=torch.uint8, device=dev)
            call = lambda: efla.efla_chunk_fwd_gated(xo["q"], xo["k"], xo["v"], xo["beta"], go, xo["S0"], o=oo,
                                                     S_T=So, workspace=wso, stream=stream)
        elif segmented:   # long streams as a segmented scan, the library's segment count
            wso = torch.zeros(efla.lib.efla_chunk_fwd_segmented_workspace_bytes(wo.B, wo.H, wo.T, wo.dk, wo.dv, 64, 1,
                                                                                 0, 0), dtype=torch.uint8, device=dev)
            call = lambda: efla.efla_chunk_fwd_segmented(xo["q"], xo["k"], xo["v"], xo["beta"], xo["S0"], o=oo,
                                                         S_T=So, workspace=wso, stream=stream)
        else:
            wso = efla.new_workspace(wo.B, wo.H, wo.T, wo.dk, wo.dv, 64, wo.dtype, dev)
            call = lambda: efla.efla_chunk_fwd(xo["q"], xo["k"], xo["v"], xo["beta"], xo["S0"], o=oo, S_T=So,
                                               workspace=wso, stream=stream)
        for _ in range(args.warmup):
            call()
        barrier(world)
        o0, o1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        o0.record(stream)
        for _ in range(args.other_steps):
            call()
        o1.record(stream)
        barrier(world)
        oms = max_over_ranks(o0.elapsed_time(o1), world) / args.other_steps
        if efla.efla_workspace_status(wso, clear=True, stream=stream) != efla.EFLA_OK:
            raise SystemExit(f"device reported a timeout on {name}")
        ob, of = chunk_alg(wo)
        if gated:
            ob += wo.B * wo.H * wo.T * 4          # the fp32 log-decay is read too
        others[name] = {"value": wo.tokens * world / (oms * 1e-3), "unit": "tokens/s", "ms_per_step": oms,
                        "steps": args.other_steps,
                        "config": {"B": wo.B, "H": wo.H, "T": wo.T, "d_k": wo.dk, "d_v": wo.dv, "chunk": 64},
                        "roofline": roofline_record(ob, of, oms * 1e-3, hbm, tc, peak_kind),
                        "gpu_launches": (4 if segmented else 2) * args.other_steps}
        del xo, wso, oo, So

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(WORKLOAD)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; q,k unit direction x LogNormal(0,0.5) norm, v~N(0,1), beta=sigmoid(N(0,1)))",
            "config": {"workload": w.name, "B": B, "H": H, "T": T, "d_k": d, "d_v": d, "chunk": 64,
                       "global_batch": B * world, "seq_len": T, "parallelism": f"dp{world}",
                       "l2": f"{N_ROTATE} rotating input sets ({N_ROTATE * nbytes / 1e6:.0f} MB) > 126 MB L2"},
            "roofline": roofline, "e2e": e2e,
            # bf16, d = 128: each efla_chunk_fwd launches the UT kernel and the chain kernel
            "gpu_launches": 2 * args.steps,
            "clocks": clk.summary(), "decode": dec, "backward": bwd, "other_workloads": others, "cpu_baseline": cpu,
            "kernel_source": {e: kernel_source_hash(e) for e in KERNEL_SOURCES},
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
