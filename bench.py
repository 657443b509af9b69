#!/usr/bin/env python
"""Benchmark of the fused LM-head linear + softcapped cross-entropy, forward + backward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl flce|reference]

One step = one fused forward that forms loss, lse, dX and dW (flce_forward with
want_grads=1) plus the backward call that applies the upstream gradient (a device
scalar equal to 1, the autograd default for a scalar loss), on one batch of the
3.8B model's head: N = 16384 tokens (batch 16 x context 1024), d = 3072,
V = 50257 -> 50304, softcap 15.  Credited work: 6*N*d*Vpad FLOP per step.

Multi-GPU (torchrun): every rank holds W and its own batch (weak scaling) and runs the
data-parallel step -- loss normalised by the count of rows in the loss over all ranks, dW
accumulated over --accum-steps micro-batches with each loss divided by their number, and
all-reduced after the last in --buckets vocabulary buckets that overlap the last gradient
launches; --no-allreduce gives independent replicas.  The time is the max over ranks.
``--impl reference`` times the fp64 CPU oracle on a bounded sample of rows of the
same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused linear-CE fwd+bwd tokens/sec and TFLOP/s (% bf16 peak) at d=3072,V=50304"
UNIT = "tokens/s"
DATASHEET_BF16_TFLOPS = 2250.0
FP8_OVER_BF16 = 2.0      # nominal dense fp8 / bf16 tensor rate (4.5 / 2.25 PFLOP/s)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# rows per chunk the library picks when chunk_rows = 0, and the most rows one logits launch
# covers (used to label the JSON line and to match recorded DRAM traffic to launch sizes)
AUTO_CHUNK_ROWS = 8192
LOGITS_LAUNCH_ROWS = 4096

def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["flce", "reference"], default="flce")
    ap.add_argument("--config", default="3.8b")
    ap.add_argument("--chunk-rows", type=int, default=0)
    ap.add_argument("--rows", type=int, default=0,
                    help="override the token count N (small profiling cases)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-unfused", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--graph", action="store_true",
                    help="device-timed steps replay one captured CUDA graph of the step")
    ap.add_argument("--accum-steps", type=int, default=7,
                    help="N>1: micro-batches per optimizer step; dW is accumulated over them and "
                         "all-reduced after the last (the write-ups: 7)")
    ap.add_argument("--no-allreduce", action="store_true",
                    help="N>1: independent replicas with no collective (weak-scaling floor)")
    ap.add_argument("--grad-fp8", action="store_true",
                    help="fp8 workload: the gradient contractions in FP8 too (e5m2 gradient x "
                         "e4m3 operands) instead of bf16")
    ap.add_argument("--buckets", type=int, default=4,
                    help="N>1: vocabulary buckets of the dW all-reduce, each exchanged as soon "
                         "as the last chunk's gradient launch for it is done (1: one all-reduce "
                         "after the step)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--ref-rows", type=int, default=128,
                    help="rows per step of the --impl reference arm")
    ap.add_argument("--norm", action="store_true",
                    help="time the final-RMSNorm kernels (forward, backward) on the workload's "
                         "shape against the measured HBM copy bandwidth")
    ap.add_argument("--compare-cublas", action="store_true",
                    help="per-contraction efficiency at the operating clock next to cuBLAS "
                         "(torch.matmul) on the same shapes, with NVML clock/power sampling")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_desc(c, chunk):
    return {
        "workload": f"{c.name}: fused linear-CE fwd+bwd, N={c.N} tokens, d={c.d}, "
                    f"Vreal={c.Vreal} padded to Vpad={c.Vpad}, softcap={c.cap:g}",
        "N": c.N, "d": c.d, "Vreal": c.Vreal, "Vpad": c.Vpad, "cap": c.cap,
        "ignore_index": c.ignore_index, "ignored_rows": c.ignore_count,
        "targets": "Zipf(1.1)" if c.target_dist == "zipf" else c.target_dist,
        "x": c.x_dist, "w_std": c.w_std, "chunk_rows": chunk,
        "l2": f"inputs larger than L2: X {c.N * c.d * 2 / 1e6:.1f} MB + W "
              f"{c.Vpad * c.d * 2 / 1e6:.1f} MB > 126 MB L2 (no flush)",
    }


def arm_config(c, chunk, world, dp, accum_steps, buckets=1):
    """The ``config`` object of the JSON line; both arms print the same one for the same
    arguments."""
    return dict(workload_desc(c, chunk),
                parallelism=(f"data parallel x{world}: global-count loss, dW all-reduce every "
                             f"{accum_steps} micro-batches in {buckets} vocabulary buckets "
                             f"overlapping the last gradient launches" if dp else
                             f"replicas x{world}" if world > 1 else "single GPU"))


# ----------------------------------------------------------------------------------- CPU oracle
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_step(inp, r0: int, rows: int):
    """Oracle forward + backward on rows [r0, r0+rows) of the workload (all Vpad, all d)."""
    import oracle
    import synth
    c = inp["cfg"]
    X = synth.bf16_to_f64(inp["X"][r0:r0 + rows])
    W = inp.get("_W64")
    if W is None:
        W = inp["_W64"] = synth.bf16_to_f64(inp["W"])
    t = inp["targets"][r0:r0 + rows]
    return oracle.forward_backward(X, W, t, c.Vreal, c.cap, c.ignore_index)


def cpu_baseline(inp, target_s: float):
    """Time the oracle as it stands on a contiguous row slice sized for ~target_s seconds (the
    whole workload, repeated, when it takes less than that)."""
    c = inp["cfg"]
    probe = min(32, c.N)
    oracle_step(inp, 0, probe)                   # warm-up: the fp64 copy of W, BLAS threads
    t0 = time.perf_counter()
    oracle_step(inp, 0, probe)
    dt = max(time.perf_counter() - t0, 1e-4)
    per_row = dt / probe
    for _ in range(3):                            # refine the size: small slices run faster per row
        want = int(target_s / per_row)
        rows = max(probe, min(c.N, (want // 32) * 32 if want >= 32 else want))
        reps = max(1, int(want // rows)) if rows == c.N else 1
        t0 = time.perf_counter()
        for _ in range(reps):
            oracle_step(inp, 0, rows)
        dt = time.perf_counter() - t0
        per_row = dt / (rows * reps)
        if dt >= 0.5 * target_s:
            break
    what = (f"the whole {c.name} workload ({rows} rows) {reps} times" if reps > 1 else
            f"rows [0, {rows}) of the {c.name} workload")
    return {"value": rows * reps / dt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{what}: fp64 forward + backward over all Vpad={c.Vpad} columns and "
                      f"d={c.d} (that slice's dW contribution included); {dt:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    import synth
    inp = synth.make_inputs(args.config, N=args.rows or None)
    c = inp["cfg"]
    rows = max(1, min(args.ref_rows, c.N))
    times = []
    for s in range(args.warmup + args.steps):
        r0 = (s * rows) % max(1, c.N - rows + 1)
        t0 = time.perf_counter()
        oracle_step(inp, r0, rows)
        if s >= args.warmup:
            times.append(time.perf_counter() - t0)
    step_s = sum(times) / len(times)
    value = rows / step_s
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": arm_config(c, args.chunk_rows or min(c.N, AUTO_CHUNK_ROWS), world,
                             world > 1 and not args.no_allreduce and args.config != "fp8",
                             args.accum_steps, args.buckets),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"{rows} contiguous rows per step (fp64 forward + backward "
                                   f"over all Vpad and d, dW contribution included)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.proc = None
        self.path = None
        self.gpu_id = gpu_id

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", "50"]
            if self.gpu_id:
                cmd += ["-i", self.gpu_id]
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), max=float(parts[2]),
                                 power=float(parts[3]) if parts[3] not in ("[N/A]", "") else 0.0,
                                 hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in rows),
                "sm_max_mhz": max(r["max"] for r in rows),
                "power_w_max": max(r["power"] for r in rows),
                "samples": len(rows), "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------------- GPU arm
def main_gpu(args):
    import torch
    import torch.distributed as dist
    import lm_head_linear_gemm_b200 as flce
    import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (B200); the CPU oracle arm is --impl reference")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    cfg = synth.CONFIGS[args.config]
    fp8 = args.config == "fp8"
    if fp8:
        inp = synth.make_fp8_inputs(cfg, seed=cfg.seed + rank, N=args.rows or None)
    else:
        inp = synth.make_inputs(cfg, seed=cfg.seed + rank, N=args.rows or None)
    c = inp["cfg"]
    N, d, Vp, Vr = c.N, c.d, c.Vpad, c.Vreal

    def host_bf16(a):
        import numpy as np
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)

    X_h = host_bf16(inp["X"]).pin_memory()
    t_h = torch.from_numpy(inp["targets"]).pin_memory()
    W = host_bf16(inp["W"]).to(dev)
    X = X_h.to(dev)
    t = t_h.to(dev)
    torch.cuda.synchronize()
    mem_inputs = torch.cuda.memory_allocated(dev)
    g_one = torch.ones((), dtype=torch.float32, device=dev)
    dX = torch.empty_like(X)
    dW = torch.empty((Vp, d), dtype=torch.float32, device=dev)
    shape = flce.make_shape(N, d, Vp, Vr, c.cap, c.ignore_index, args.chunk_rows)
    ws = flce.alloc_workspace(shape, True, dev)
    stream = torch.cuda.current_stream()

    if fp8:
        X8 = torch.from_numpy(inp["X8"]).to(dev)
        W8 = torch.from_numpy(inp["W8"]).to(dev)
        sX = torch.tensor(float(inp["sX"]), dtype=torch.float32, device=dev)
        sW = torch.tensor(float(inp["sW"]), dtype=torch.float32, device=dev)

    dp = world > 1 and not args.no_allreduce and not fp8
    micro = [0]
    # each micro-batch's loss is divided by the number of micro-batches
    g_accum = torch.tensor(1.0 / max(1, args.accum_steps), dtype=torch.float32, device=dev)
    dp_ops = flce.data_parallel.LibraryOps() if dp else None

    def step(Xd=None, td=None):
        Xd = X if Xd is None else Xd
        td = t if td is None else td
        if dp:
            # data-parallel micro-batch: global-count normalisation; dW accumulated over
            # --accum-steps micro-batches and all-reduced after the last one
            k = micro[0] % max(1, args.accum_steps)
            micro[0] += 1
            loss, _, _, _, _ = flce.dp_step(
                Xd, W, td, Vr, c.cap, c.ignore_index, dW=dW, accumulate_dW=k > 0,
                allreduce_dW=k == max(1, args.accum_steps) - 1, workspace=ws,
                chunk_rows=args.chunk_rows, grad_scale=g_accum, buckets=args.buckets,
                ops=dp_ops)
            return loss
        if fp8:
            loss, lse, _, _, _ = flce.forward_fp8(X8, W8, sX, sW, Xd, W, td, Vr, c.cap,
                                                  c.ignore_index, True, dX=dX, dW=dW,
                                                  workspace=ws, chunk_rows=args.chunk_rows,
                                                  grad_fp8=args.grad_fp8)
        else:
            loss, lse, _, _, _ = flce.forward(Xd, W, td, Vr, c.cap, c.ignore_index, True, dX=dX,
                                              dW=dW, workspace=ws, chunk_rows=args.chunk_rows)
        flce.backward(Xd, W, td, lse, Vr, c.cap, c.ignore_index, grad_out=g_one, dX=dX, dW=dW,
                      grads_precomputed=True)
        return loss

    # ---- device-resident timing
    torch.cuda.reset_peak_memory_stats(dev)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    timed_step = step
    launches_per_graph_step = None
    if args.graph and world == 1:
        flce.instrument(True)
        step()
        launches_per_graph_step = flce.instrument_read()["launches_total"]
        flce.instrument(False)
        # one step captured into a CUDA graph (same buffers, so replays redo the whole step)
        cap_stream = torch.cuda.Stream(device=dev)
        cap_stream.wait_stream(torch.cuda.current_stream())
        graph = torch.cuda.CUDAGraph()
        holder = {}
        with torch.cuda.graph(graph, stream=cap_stream):
            holder["loss"] = step()
        graph.replay()
        torch.cuda.synchronize()

        def timed_step():
            graph.replay()
            return holder["loss"]
    status, nv = flce.read_status(ws)
    # everything the fused step holds beyond its inputs: dX, dW, workspace, lse, loss
    peak_fused = torch.cuda.max_memory_allocated(dev) - mem_inputs
    barrier()
    gpu_id = None
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    clocks = ClockSampler(gpu_id)
    clocks.start()
    nvml = None
    try:
        nvml = NvmlSampler(dev).__enter__()
    except Exception:
        nvml = None
    flce.instrument(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    # one event pair per step as well (median / min / max of the same steps); recording an
    # event adds no work to the stream
    step_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(args.steps)]
    e0.record(stream)
    for a, b in step_evs:
        a.record(stream)
        loss = timed_step()
        b.record(stream)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    elapsed_ms = e0.elapsed_time(e1)
    per = [a.elapsed_time(b) for a, b in step_evs]
    spread = {"median": statistics.median(per), "min": min(per), "max": max(per)}
    kstats = flce.instrument_read()
    flce.instrument(False)
    clk = clocks.stop()
    nvml_clk = None
    if nvml is not None:
        nvml.__exit__(None, None, None)
        nvml_clk = nvml.summary()
    if world > 1:
        tt = torch.tensor([elapsed_ms], device=dev, dtype=torch.float64)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        elapsed_ms = float(tt.item())
    ms_per_step = elapsed_ms / args.steps
    value = world * N / (ms_per_step / 1e3)
    credited = 6.0 * N * d * Vp
    tflops = credited / (ms_per_step / 1e3) / 1e12 * world

    # ---- end-to-end through the public API with host buffers: every step copies its X and
    # targets from pinned host memory and reads its loss back.  The copy for step i+2 runs on a
    # side stream into the buffer step i has finished with, so copies overlap compute.
    e2e = None
    if not args.no_e2e:
        loss_h = torch.empty((), dtype=torch.float32).pin_memory()
        Xb = [X, torch.empty_like(X)]
        tb = [t, torch.empty_like(t)]
        copy_stream = torch.cuda.Stream(device=dev)
        copied = [torch.cuda.Event(), torch.cuda.Event()]
        used = [torch.cuda.Event(), torch.cuda.Event()]

        def issue_copy(b, first=False):
            with torch.cuda.stream(copy_stream):
                if not first:
                    copy_stream.wait_event(used[b])
                Xb[b].copy_(X_h, non_blocking=True)
                tb[b].copy_(t_h, non_blocking=True)
                copied[b].record(copy_stream)

        def e2e_run(nsteps):
            issue_copy(0, True)
            if nsteps > 1:
                issue_copy(1, True)
            for i in range(nsteps):
                b = i % 2
                stream.wait_event(copied[b])
                loss = step(Xb[b], tb[b])
                used[b].record(stream)
                loss_h.copy_(loss, non_blocking=True)
                if i + 2 < nsteps:
                    issue_copy(b)

        e2e_run(max(2, args.warmup))
        torch.cuda.synchronize()
        barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        copy_stream.wait_event(f0)
        e2e_run(args.steps)
        f1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = f0.elapsed_time(f1)
        if world > 1:
            tt = torch.tensor([e2e_ms], device=dev, dtype=torch.float64)
            dist.all_reduce(tt, op=dist.ReduceOp.MAX)
            e2e_ms = float(tt.item())
        e2e = {"value": world * N / (e2e_ms / args.steps / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": X.numel() * 2 + t.numel() * 8, "d2h_bytes_per_step": 4,
               "ms_per_step": e2e_ms / args.steps,
               "what": "pinned-host X and targets copied in and the loss copied out every step "
                       "(copies on a side stream, double-buffered, overlapping the previous "
                       "step); W and dW stay resident (the head's parameter and its gradient), "
                       "and dX stays on the device, where the backward of the layer below "
                       "consumes it"}

    peaks, peaks_src = load_peaks()
    sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    # algorithmic FLOPs of the gradient launches: they run over each chunk's rows in the loss
    # only (compaction), 4 * rows_in_loss * d * Vpad per chunk
    import numpy as np
    tv = np.asarray(inp["targets"])
    in_loss = (tv != c.ignore_index) & (tv >= 0) & (tv < Vr)
    grad_flop_step = 4.0 * d * Vp * float(in_loss.sum())
    # 8-bit contractions are measured against the bf16 peak times the nominal fp8/bf16 ratio
    fp8_kinds = ({"logits"} | ({"dX+dW"} if args.grad_fp8 else set())) if fp8 else set()
    kinds = {}
    for name, k in kstats["gemm"].items():
        if k["launches"]:
            flop = k["flop"]
            if name == "dX+dW":
                flop = grad_flop_step * args.steps      # every timed step's gradient launches
            kinds[name] = {"launches": k["launches"], "ms_per_launch": k["ms"] / k["launches"],
                           "tflops": flop / (k["ms"] / 1e3) / 1e12,
                           "dtype": "fp8" if name in fp8_kinds else "bf16",
                           "share_of_step": k["ms"] / elapsed_ms if elapsed_ms else None}
    dom = max(kinds, key=lambda n: kstats["gemm"][n]["ms"]) if kinds else None
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if dom and os.path.exists(tpath):
        tj = json.load(open(tpath))
        ent = tj.get(dom)
        chunk = min(N, shape.chunk_rows or AUTO_CHUNK_ROWS)
        launch_rows = {"dX+dW": chunk, "logits": min(chunk, LOGITS_LAUNCH_ROWS)}.get(dom)
        if (ent and ent.get("kernel_rev") == kernel_rev() and ent.get("config") == c.name
                and ent.get("rows_per_launch") == launch_rows):
            traffic = ent.get("bytes_per_launch")
    roofline = None
    if dom:
        ach = kinds[dom]["tflops"]
        is8 = kinds[dom]["dtype"] == "fp8"
        peak = sustained * (FP8_OVER_BF16 if is8 else 1.0)
        roofline = {"bound": "tensor", "kernel": dom, "achieved": ach, "peak": peak,
                    "unit": "TFLOP/s", "frac": ach / peak, "traffic": traffic,
                    "peak_source": f"bf16_tflops_sustained ({peaks_src} MEASURED_PEAKS.json; "
                                   "the kernel runs inside a long step)" +
                                   (f" x {FP8_OVER_BF16:g}, the nominal fp8/bf16 dense ratio "
                                    "(4.5 / 2.25 PFLOP/s)" if is8 else ""),
                    "algorithmic": "logits: 2*rows*Vpad*d FLOP per launch; dX+dW: "
                                   "4*(rows in the loss)*Vpad*d per launch (the gradient "
                                   "contractions skip rows outside the loss)"}

    # After the timed region (the GPU already at its power cap): the recompute path -- a forward
    # without gradients, then a backward that recomputes the logits with lse known (8 N d Vpad
    # executed FLOPs against 6).
    recompute = None
    if world == 1:
        if not fp8:
            ws_fwd = flce.alloc_workspace(shape, False, dev)

            def rec_step():
                _, lse_r, _, _, _ = flce.forward(X, W, t, Vr, c.cap, c.ignore_index, False,
                                                 workspace=ws_fwd, chunk_rows=args.chunk_rows)
                flce.backward(X, W, t, lse_r, Vr, c.cap, c.ignore_index, grad_out=g_one, dX=dX,
                              dW=dW, workspace=ws, chunk_rows=args.chunk_rows)

            for _ in range(max(2, args.warmup)):
                rec_step()
            torch.cuda.synchronize()
            r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            r0.record(stream)
            for _ in range(args.steps):
                rec_step()
            r1.record(stream)
            torch.cuda.synchronize()
            rms = r0.elapsed_time(r1) / args.steps
            recompute = {"ms_per_step": rms, "tokens_per_s": N / (rms / 1e3),
                         "credited_tflops": credited / (rms / 1e3) / 1e12,
                         "executed_tflops": (4.0 * N * d * Vp + grad_flop_step) / (rms / 1e3) / 1e12,
                         "what": "flce_forward(want_grads=0), then flce_backward recomputing the "
                                 "logits with lse known, timed after the fused steps; executed = "
                                 "two logits passes + the gradient contractions over the rows in "
                                 "the loss"}

    unfused = None
    cpu = None
    if rank == 0 and world == 1 and not args.no_unfused:
        unfused = unfused_torch_baseline(X, W, t, c, args)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(inp, args.cpu_seconds)

    if rank == 0:
        if roofline is not None:
            roofline["kernel_rev"] = kernel_rev()
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": ("e4m3 logits + e5m2 x e4m3 gradients" if fp8 and args.grad_fp8 else
                      "e4m3 logits + bf16 gradients" if fp8 else "bf16"), "data": "synthetic",
            "config": arm_config(c, shape.chunk_rows or min(N, AUTO_CHUNK_ROWS), world, dp,
                                 args.accum_steps, args.buckets),
            "tflops": tflops,
            "pct_of_bf16_datasheet_2250": tflops / world / DATASHEET_BF16_TFLOPS,
            "pct_of_measured_bf16_burst": tflops / world / burst,
            "pct_of_measured_bf16_sustained": tflops / world / sustained,
            "credited_flop_per_step": credited,
            "algorithmic_flop_per_step": 2.0 * N * d * Vp + grad_flop_step,
            "roofline": roofline, "kernels": kinds, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": kstats["launches_total"] if launches_per_graph_step is None else
                            launches_per_graph_step * args.steps,
            "graph_replay": bool(args.graph and world == 1),
            "gpu_launches_per_step": kstats["launches_total"] / args.steps,
            "clocks": clk,
            "clocks_nvml_10ms": nvml_clk,
            "mcycles_per_step": (ms_per_step * nvml_clk["sm_mhz"] / 1e3) if nvml_clk else None,
            "peak_mem_MiB": {"fused_step": peak_fused / 2**20,
                             "workspace": ws.numel() / 2**20,
                             "unfused_torch": unfused["peak_MiB"] if unfused else None},
            "per_step_ms": spread, "recompute_path": recompute,
            "unfused_torch": unfused, "device_status": status, "n_valid": nv,
            "loss": float(loss.item()),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def kernel_rev() -> str:
    """Hash of the kernel sources; DRAM traffic recorded for another hash is stale."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "lm_head_linear_gemm_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.endswith((".cu", ".cuh")):
            h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def unfused_torch_baseline(X, W, t, c, args):
    """Comparator only (not the product path): materialised bf16 logits, fp32 softcap,
    torch cross_entropy and autograd, as a plain PyTorch training loss would do."""
    import torch
    dev = X.device
    Xg = X.detach().clone().requires_grad_(True)
    Wg = W.detach().clone().requires_grad_(True)

    def step():
        z = Xg @ Wg.T
        s = c.cap * torch.tanh(z.float() / c.cap)
        loss = torch.nn.functional.cross_entropy(s[:, :c.Vreal], t, ignore_index=c.ignore_index)
        loss.backward()
        Xg.grad = None
        Wg.grad = None
        return loss

    try:
        torch.cuda.synchronize()
        torch.cuda.reset_peak_memory_stats(dev)
        base = torch.cuda.memory_allocated(dev)   # beyond its (cloned) inputs: logits, grads
        for _ in range(2):
            step()
        torch.cuda.synchronize()
        peak = torch.cuda.max_memory_allocated(dev) - base
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n = max(3, min(args.steps, 10))
        e0.record()
        for _ in range(n):
            step()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / n
        return {"tokens_per_s": c.N / (ms / 1e3), "ms_per_step": ms, "peak_MiB": peak / 2**20,
                "what": "torch: bf16 X@W.T, fp32 cap*tanh, F.cross_entropy, autograd"}
    except torch.cuda.OutOfMemoryError:
        return {"error": "out of memory"}


class NvmlSampler:
    """SM clock, power and clock-event reasons every 10 ms while a loop runs (NVML)."""

    def __init__(self, torch_device):
        import threading
        import pynvml
        self.nv = pynvml
        pynvml.nvmlInit()
        self.h = pynvml.nvmlDeviceGetHandleByIndex(0)
        uuid = str(getattr(__import__("torch").cuda.get_device_properties(torch_device), "uuid", ""))
        for i in range(pynvml.nvmlDeviceGetCount()):
            hh = pynvml.nvmlDeviceGetHandleByIndex(i)
            u = pynvml.nvmlDeviceGetUUID(hh)
            u = u.decode() if isinstance(u, bytes) else u
            if uuid and uuid in u:
                self.h = hh
        self.threading = threading

    def __enter__(self):
        self.samples, self.stop = [], False

        def run():
            nv = self.nv
            while not self.stop:
                self.samples.append((nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0,
                                     nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)))
                time.sleep(0.01)
        self.t = self.threading.Thread(target=run)
        self.t.start()
        return self

    def __exit__(self, *exc):
        self.stop = True
        self.t.join()

    def summary(self):
        c = [x[0] for x in self.samples] or [0]
        p = [x[1] for x in self.samples] or [0]
        return {"sm_mhz": statistics.median(c), "power_w": statistics.median(p),
                "samples": len(self.samples),
                "power_capped": any(x[2] & 0x4 for x in self.samples)}


def compare_cublas(args):
    """Each contraction of one chunk (Nc rows) next to torch.matmul (cuBLAS) on the same shape,
    each looped for ~2 s; efficiency = achieved FLOP/s / (8192 FLOP/clk/SM x SMs x median clock)."""
    import numpy as np
    import torch
    import lm_head_linear_gemm_b200 as flce
    import synth
    dev = torch.device("cuda", 0)
    cfg = synth.CONFIGS[args.config]
    Nc = args.rows or AUTO_CHUNK_ROWS
    inp = synth.make_inputs(cfg, N=Nc)
    c = inp["cfg"]
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    flop = 2.0 * Nc * c.d * c.Vpad

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    X, W = bf(inp["X"]), bf(inp["W"])
    t = torch.from_numpy(inp["targets"]).to(dev)
    Ap = (torch.randn(Nc, c.Vpad, device=dev) * 1e-3).to(torch.bfloat16)

    def loop(fn, seconds=2.0):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n, t0 = 0, time.time()
        with NvmlSampler(dev) as smp:
            e0.record()
            while time.time() - t0 < seconds:
                fn()
                n += 1
                if n % 4 == 0:
                    torch.cuda.synchronize()
            e1.record()
            torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n, smp.summary()

    def row(ms, smp):
        tf = flop / (ms * 1e-3) / 1e12
        peak = 8192 * sms * smp["sm_mhz"] * 1e6 / 1e12
        return {"ms": ms, "tflops": tf, "pct_of_clock_peak": 100 * tf / peak, **smp}

    out = {}
    for name, fn in (("cublas_logits_shape", lambda: torch.matmul(X, W.T)),
                     ("cublas_dX_shape", lambda: torch.matmul(Ap, W)),
                     ("cublas_dW_shape", lambda: torch.matmul(Ap.T, X))):
        out[name] = row(*loop(fn))
    dX = torch.empty_like(X)
    dW = torch.empty((c.Vpad, c.d), dtype=torch.float32, device=dev)
    ws = flce.alloc_workspace(flce.make_shape(Nc, c.d, c.Vpad, c.Vreal, c.cap), True, dev)
    flce.instrument(True)
    ms, smp = loop(lambda: flce.forward(X, W, t, c.Vreal, c.cap, c.ignore_index, True, dX=dX,
                                        dW=dW, workspace=ws), 3.0)
    st = flce.instrument_read()
    flce.instrument(False)
    for k, v in st["gemm"].items():
        if v["launches"]:
            r = row(v["ms"] / v["launches"], smp)
            r["tflops"] = v["flop"] / (v["ms"] * 1e-3) / 1e12       # the dX+dW launch does 2 shapes
            r["pct_of_clock_peak"] = 100 * r["tflops"] / (8192 * sms * smp["sm_mhz"] * 1e6 / 1e12)
            out["flce_" + k] = r
    out["flce_chunk_step_ms"] = ms
    print(json.dumps({"compare_cublas": out, "rows": Nc, "config": c.name}), flush=True)
    return 0


def norm_bench(args):
    """The model's final RMSNorm on the workload's shape, two ways:
    * its row kernels alone (forward, backward), HBM-bound: achieved GB/s of the algorithmic
      bytes against the measured copy bandwidth;
    * a training step of the norm and the head (loss and the gradients of H, gamma and W, on the
      workload's W and targets): the head alone (for reference), the norm's row kernels around
      the head, and one flce_forward_rmsnorm call, whose dX epilogue writes dH directly (the
      norm's backward folded into the dX contraction).  CUDA-event timed, interleaved."""
    import torch
    import lm_head_linear_gemm_b200 as flce
    import synth
    cfg = synth.CONFIGS[args.config]
    inp = synth.make_rmsnorm_inputs(cfg, N=args.rows or None)
    c = inp["cfg"]
    N, d = c.N, c.d
    dev = torch.device("cuda", 0)

    def D(a):
        import numpy as np
        a = np.ascontiguousarray(a)
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(a).to(dev)

    H, gamma, W, t = D(inp["H"]), D(inp["gamma"]), D(inp["W"]), D(inp["targets"])
    g = torch.Generator(device=dev).manual_seed(0)
    dXr = (torch.randn(N, d, device=dev, generator=g) * 1e-3).to(torch.bfloat16)
    X, rstd = flce.rmsnorm_forward(H, gamma)
    dH, dgamma = flce.rmsnorm_backward(H, gamma, rstd, dXr)
    peaks, src = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))

    def timed(fn, reps):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    out = {}
    for name, fn, nbytes in (
            ("forward", lambda: flce.rmsnorm_forward(H, gamma, X=X, rstd=rstd), 4 * N * d + 4 * N),
            ("backward", lambda: flce.rmsnorm_backward(H, gamma, rstd, dXr, dH=dH, dgamma=dgamma),
             10 * N * d + 8 * N)):
        ms = timed(fn, 50)
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[name] = {"ms": ms, "algorithmic_bytes": nbytes, "GB/s": gbs, "frac_of_hbm": gbs / hbm}

    # a training step of the norm and the head
    g_one = torch.ones((), dtype=torch.float32, device=dev)
    dX = torch.empty_like(H)
    dW = torch.empty(W.shape, dtype=torch.float32, device=dev)
    shape = flce.make_shape(N, d, c.Vpad, c.Vreal, c.cap, c.ignore_index, args.chunk_rows)
    ws = flce.alloc_workspace(shape, True, dev)
    import ctypes
    ws_r = torch.empty(int(flce.lib().flce_workspace_bytes_rmsnorm(ctypes.byref(shape), 1)),
                       dtype=torch.uint8, device=dev)

    def head():
        _, lse, _, _, _ = flce.forward(X, W, t, c.Vreal, c.cap, c.ignore_index, True, dX=dX,
                                       dW=dW, workspace=ws, chunk_rows=args.chunk_rows)
        flce.backward(X, W, t, lse, c.Vreal, c.cap, c.ignore_index, grad_out=g_one, dX=dX,
                      dW=dW, grads_precomputed=True)

    def separate():
        flce.rmsnorm_forward(H, gamma, X=X, rstd=rstd)
        head()
        flce.rmsnorm_backward(H, gamma, rstd, dX, dH=dH, dgamma=dgamma)

    def fused():
        flce.forward_rmsnorm(H, gamma, W, t, c.Vreal, c.cap, c.ignore_index, 1e-6, True, dH=dH,
                             dgamma=dgamma, dW=dW, workspace=ws_r, chunk_rows=args.chunk_rows)
        flce.scale_grads_rmsnorm(g_one, dH, dgamma, dW, c.Vreal, c.cap, c.ignore_index)

    steps = {}
    for _ in range(2):
        for name, fn in (("head alone", head), ("norm kernels around the head", separate),
                         ("one call, norm backward folded into dX", fused)):
            steps.setdefault(name, []).append(timed(fn, args.steps))
    print(json.dumps({"rmsnorm": out, "N": N, "d": d, "Vpad": c.Vpad, "hbm_peak_gbs": hbm,
                      "peak_source": src,
                      "bytes": "forward: read h, write x (2+2 B per element) + rstd; backward: "
                               "dH pass reads h, dX, writes dH (6 B), dgamma pass re-reads h, "
                               "dX (4 B)",
                      "step_ms": steps,
                      "step": f"{c.name}: loss and the gradients of H, gamma and W; "
                              f"{args.steps} steps per timing, two interleaved rounds"}),
          flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.compare_cublas:
        return compare_cublas(args)
    if args.norm:
        return norm_bench(args)
    return main_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
