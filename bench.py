"""Benchmark of the tensor-parallel MLP over t virtual shards on one B200 (N GPUs = N replicas).

One step = one full pass of the hot path on the Llama-3-8B-shaped SwiGLU MLP, t=8 virtual shards:
  column-parallel GEMM + SwiGLU epilogue (Z_r = SiLU(X G_r) * X U_r)
  -> row-parallel GEMM with its ring ReduceScatter along tokens and the AllGather fused into the
     epilogue (tp_row_linear_reduce, TP_OUT_RS_AG): the partials U_r = Z_r W_down[r] are summed in
     ring order inside the kernel and each reduced tile is written to every shard.
The standalone ring ReduceScatter (the second half of the metric) is timed in its own loop on the
same data volume: 8 fp32 partials [4096, 4096].
X [4096, 4096] bf16 ~N(0,1); fused gate|up [4096, 2*14336] and W_down [14336, 4096] ~N(0, 0.02), drawn
on the device from a seeded generator, sharded once by the library's layout kernels (not timed).

Output: one JSON line (rank 0). value = whole-job TFLOP/s (algorithmic FLOPs 2*N*h*F*2 + 2*N*F*h per
step per replica, summed over replicas / max-over-ranks time). Per-kernel CUDA-event times inside the
timed region give the roofline of the dominant kernel (the column GEMM, tensor-bound); the standalone
ReduceScatter loop gives the HBM roofline (algorithmic bytes (t+1)*M). `e2e` repeats the step through tp_mlp_fwd with
X copied in from pinned host memory and the result copied back, every step. `cpu_baseline` times the
oracle, single-threaded, on bounded row samples of the same workload on this host. On one GPU the line
also carries `workloads`: the TP+SP forward, the 70B layer, every sharded-matmul strategy and ring
collective points, each timed with CUDA events under one clock record.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Multi-GPU: launched by torchrun, one process per GPU, each an independent replica (no collective
between GPUs: the path's collectives are among virtual shards inside one GPU).
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "TP-MLP fwd TFLOP/s (% BF16 peak); shard reduce-scatter GB/s (% HBM peak)"
N_TOK, H, F, T = 4096, 4096, 14336, 8
FLOPS_COL = 2.0 * N_TOK * H * (2 * F)           # gate and up GEMMs
FLOPS_ROW = 2.0 * N_TOK * F * H                 # down GEMM
FLOPS_STEP = FLOPS_COL + FLOPS_ROW              # 1443.1 GFLOP
M_PARTIAL = N_TOK * H * 4                       # one fp32 partial, 64 MiB
RS_BYTES = (T + 1) * M_PARTIAL                  # read t*M, write M
AG_BYTES = T * M_PARTIAL                        # in place: read M once, write the t-1 other copies
WORKLOAD = ("llama3-8b SwiGLU TP-MLP forward, t=8 virtual shards, 4096 tokens x h=4096, F=14336; "
            "column GEMM+SwiGLU -> row GEMM fused with ring ReduceScatter(tokens) + AllGather")
ORACLE_ROWS = 128          # token rows per oracle sample (the reference arm's step and cpu_baseline alike)
CPU_BASELINE_SAMPLES = 8   # cpu_baseline: this many samples of ORACLE_ROWS rows each

def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), d.get("bf16_tflops_sustained", 1400.0), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def _traffic(kernel_key: str, source_file: str):
    """dram bytes per launch from the committed ncu summary, or None when absent or stale."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel_key)
    if not e:
        return None
    src = os.path.join(ROOT, "tensor_sharded_matmul_b200", "csrc", source_file)
    if e.get("code_sha") != code_sha(open(src, encoding="utf-8").read()):
        return None
    return e.get("bytes_per_launch")


def code_sha(source: str) -> str:
    """First 16 hex digits of the sha256 of a C++/CUDA source with its comments and blank space
    removed, so that editing a comment does not retire counters taken from unchanged code."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", source, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    text = " ".join(text.split())
    return hashlib.sha256(text.encode("utf-8")).hexdigest()[:16]


class ClockSampler:
    """nvidia-smi clocks/throttle sampling while the GPU works."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str | None):
        self.bus_id = bus_id
        self.proc = None

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.bus_id:
            cmd += ["-i", self.bus_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        loaded = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons), "samples": len(sm)}


def _dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def _emit(obj):
    print(json.dumps(obj), flush=True)


def max_over_ranks(values, dist=None, device=None):
    """Element-wise maximum over all ranks of a list of per-rank timings (identity for one process).
    Every rank must call it with the same number of values, at the same point."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def whole_job_rate(work_per_step: float, steps: int, n_ranks: int, max_ms: float) -> float:
    """Throughput of the whole job: every rank processes `work_per_step` per step (weak scaling), the
    job lasts as long as its slowest rank."""
    return n_ranks * work_per_step * steps / (max_ms * 1e-3)


# ------------------------------------------------------------------------------ CPU oracle timing
def _oracle_sample(rows: int, seed: int = 0):
    """Oracle inputs for a row sample: X rows and the sharded weights (fp32 copies of bf16, exact)."""
    import synthetic as S
    from oracle import layouts as OL
    X, Wgu, Wd = S.llama8b_mlp(seed=seed, device="cpu")
    Xs = X[:rows].double().numpy()
    Wg = Wgu[:, :F].float().numpy()
    Wu = Wgu[:, F:].float().numpy()
    shards_in = list(OL.shard_gate_up(Wg, Wu, T))
    shards_down = list(OL.shard_rows(Wd.float().numpy(), T))
    return Xs, shards_in, shards_down


def _oracle_step(Xs, shards_in, shards_down):
    """The oracle's TP MLP on a row sample: per-shard fp64 GEMMs, then the ring RS + AG of the partials."""
    import numpy as np
    from oracle import collectives as OC
    from oracle import mlp as OM
    U = OM.mlp_partials(Xs, shards_in, shards_down, "swiglu")
    rs = OC.reduce_scatter([u.astype(np.float32) for u in U], axis=0)
    return OC.all_gather(rs, axis=0)


def _single_thread():
    """Context that holds numpy's BLAS to one thread: the oracle is timed as the plain single-threaded
    program it is meant to be, whatever BLAS the host's numpy links."""
    from threadpoolctl import threadpool_limits
    return threadpool_limits(limits=1, user_api="blas")


def _blas_threads() -> int:
    """Threads numpy's BLAS would use right now (1 inside _single_thread())."""
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def _oracle_rates(steps: int, warmup: int):
    """Times the oracle on `steps` row samples of ORACLE_ROWS rows (after `warmup` untimed ones),
    single-threaded. Returns (seconds per sample, BLAS threads used)."""
    Xs_all, si, sd = _oracle_sample(ORACLE_ROWS * 4)
    times = []
    with _single_thread():
        threads = _blas_threads()
        for i in range(warmup + steps):
            r0 = (i % 4) * ORACLE_ROWS
            t0 = time.perf_counter()
            _oracle_step(Xs_all[r0:r0 + ORACLE_ROWS], si, sd)
            if i >= warmup:
                times.append(time.perf_counter() - t0)
    return sum(times) / len(times), threads


def _oracle_sample_text(n: int, per: float) -> str:
    return (f"{n} samples of {ORACLE_ROWS} of {N_TOK} token rows of the same MLP (all 8 shards' fp64 GEMMs + "
            f"binary32 ring RS/AG), {per:.2f} s each, single-threaded; value = sample FLOPs / time")


def cpu_baseline() -> dict:
    per, threads = _oracle_rates(CPU_BASELINE_SAMPLES, 1)
    flops = FLOPS_STEP * ORACLE_ROWS / N_TOK
    return {"value": flops / per / 1e12, "unit": "TFLOP/s", "cores": threads, "host_cpus": os.cpu_count(),
            "blas_threads": threads, "kind": "oracle", "sample": _oracle_sample_text(CPU_BASELINE_SAMPLES, per)}


def run_reference(args) -> int:
    ws, rank, _ = _dist_env()
    if rank != 0:
        return 0
    per_step, threads = _oracle_rates(args.steps, args.warmup)
    flops = FLOPS_STEP * ORACLE_ROWS / N_TOK
    value = flops / per_step / 1e12
    _emit({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample_rows_per_step": ORACLE_ROWS},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "host_cpus": os.cpu_count(),
                         "blas_threads": threads, "kind": "oracle",
                         "sample": _oracle_sample_text(args.steps, per_step)},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    })
    return 0


# ------------------------------------------------------------------------------ GPU arm
def run_gpu(args) -> int:
    import torch
    ws, rank, local = _dist_env()
    if args.gpus > 1 and ws != args.gpus:
        print("bench.py --gpus N>1 must be launched by torchrun with N processes", file=sys.stderr)
        return 2
    torch.cuda.set_device(local)
    dist = None
    if ws > 1:
        import datetime
        import torch.distributed as dist_mod
        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        dist = dist_mod

    import synthetic as S
    import tensor_sharded_matmul_b200 as tp

    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    X, Wgu, Wd = S.llama8b_mlp(seed=rank, device=dev)
    f = F // T
    w_in = torch.empty((T, H, 2 * f), dtype=torch.bfloat16, device=dev)
    w_down = torch.empty((T, f, H), dtype=torch.bfloat16, device=dev)
    tp.tp_shard_gate_up(Wgu, 2 * F, Wgu.data_ptr() + 2 * F, 2 * F, H, F, T, w_in)
    tp.tp_shard_rows(Wd, H, F, H, T, w_down)
    del Wgu, Wd
    z = torch.empty((T, N_TOK, f), dtype=torch.bfloat16, device=dev)
    out = [torch.empty((N_TOK, H), device=dev) for _ in range(T)]

    def step(ev=None):
        # exactly tp_mlp_fwd(..., TP_OUT_RS_AG), split at its kernel boundary so each launch is timed
        if ev is not None:
            ev[0].record(stream)
        tp.tp_column_linear(X, N_TOK, H, F, T, tp.TP_ACT_SWIGLU, w_in, z)
        if ev is not None:
            ev[1].record(stream)
        tp.tp_row_linear_reduce(z, N_TOK, F, H, T, w_down, tp.TP_OUT_RS_AG, 0, out)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st, site = tp.tp_device_status(1)
    if st != tp.TP_OK:
        print(f"device wait ran out at site {site}", file=sys.stderr)
        return 3

    bus = None
    try:
        pci = torch.cuda.get_device_properties(dev)
        bus = f"{pci.pci_domain_id:08X}:{pci.pci_bus_id:02X}:{pci.pci_device_id:02X}.0"
    except Exception:
        bus = None
    clocks = ClockSampler(bus if rank == 0 else None)
    if rank == 0:
        clocks.start()
        time.sleep(0.3)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    stop.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clk = clocks.stop() if rank == 0 else None
    total_ms = start.elapsed_time(stop)
    st, site = tp.tp_device_status(1)
    if st != tp.TP_OK:
        print(f"device wait ran out at site {site}", file=sys.stderr)
        return 3
    per = [[evs[i][k].elapsed_time(evs[i][k + 1]) for i in range(args.steps)] for k in range(2)]
    avg = [sum(p) / len(p) for p in per]      # ms: column GEMM, fused row GEMM + RS + AG

    # ---- the standalone ring ReduceScatter on the same volume (8 fp32 partials [4096, 4096]) -----
    partials = [torch.empty((N_TOK, H), device=dev).normal_() for _ in range(T)]
    chunk = N_TOK // T
    rs_out = [torch.empty((chunk, H), device=dev) for _ in range(T)]
    for _ in range(3):
        tp.tp_reduce_scatter(partials, rs_out, N_TOK, H, 0, tp.TP_F32, T)
    rs_start, rs_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    rs_iters = max(args.steps, 20)
    torch.cuda.synchronize()
    rs_start.record(stream)
    for _ in range(rs_iters):
        tp.tp_reduce_scatter(partials, rs_out, N_TOK, H, 0, tp.TP_F32, T)
    rs_stop.record(stream)
    torch.cuda.synchronize()
    rs_ms = rs_start.elapsed_time(rs_stop) / rs_iters
    del partials, rs_out

    # ---- end to end through tp_mlp_fwd with host buffers --------------------------------------
    # Every step copies its input X from pinned host memory and reads its result back (one replica
    # of the reduced output). As a serving loop would, the copies run on their own streams and overlap
    # the neighbouring steps' compute: copy-in of step i+1 || tp_mlp_fwd of step i || copy-out of step
    # i-1, with NB buffer sets and events guarding every reuse. The copy-out (64 MiB over PCIe) takes
    # longer than the device step, so three sets keep it streaming back to back: with two, step i's
    # compute waited for step i-2's copy-out to finish.
    NB = 3
    x_host = X.cpu().pin_memory()
    y_host = [torch.empty((N_TOK, H), dtype=torch.float32).pin_memory() for _ in range(NB)]
    x_dev = [torch.empty_like(X) for _ in range(NB)]
    outs = [out] + [[torch.empty((N_TOK, H), device=dev) for _ in range(T)] for _ in range(NB - 1)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(NB)]
    ev_comp = [torch.cuda.Event() for _ in range(NB)]
    ev_out = [torch.cuda.Event() for _ in range(NB)]
    for e in ev_comp + ev_out:
        e.record(stream)

    def e2e_steps(n):
        for i in range(n):
            b = i % NB
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_comp[b])                  # step i-NB no longer reads x_dev[b]
                x_dev[b].copy_(x_host, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])                     # step i-NB's result has been read back
            tp.tp_mlp_fwd(x_dev[b], N_TOK, H, F, T, tp.TP_ACT_SWIGLU, w_in, w_down, z, None, tp.TP_OUT_RS_AG,
                          outs[b], stream)
            ev_comp[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[b])
                y_host[b].copy_(outs[b][0], non_blocking=True)
                ev_out[b].record(s_out)

    e2e_steps(max(NB, min(args.warmup, 4)))
    torch.cuda.synchronize()
    e_start, e_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e_start.record(s_in)
    stream.wait_event(e_start)
    s_out.wait_event(e_start)
    e2e_steps(args.steps)
    for e in ev_out:
        stream.wait_event(e)
    e_stop.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e_start.elapsed_time(e_stop)

    # the copy-out alone (one 64 MiB replica to pinned host memory), for the e2e bound
    d_start, d_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d_iters = 10
    with torch.cuda.stream(s_out):
        d_start.record(s_out)
        for _ in range(d_iters):
            y_host[0].copy_(outs[0][0], non_blocking=True)
        d_stop.record(s_out)
    torch.cuda.synchronize()
    d2h_gbs = d_iters * N_TOK * H * 4 / (d_start.elapsed_time(d_stop) * 1e-3) / 1e9

    # ---- the other workloads (one GPU only: the scaling runs time the headline step alone) ---------
    extra = None
    if ws == 1 and not args.no_workloads:
        del outs, x_dev, y_host, x_host
        torch.cuda.empty_cache()
        extra = workloads(X, w_in, w_down, z)

    # ---- max over ranks ------------------------------------------------------------------------
    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dist, dev)
    n = ws
    per_step_ms = total_ms / args.steps
    value = whole_job_rate(FLOPS_STEP, args.steps, n, total_ms) / 1e12
    e2e_value = whole_job_rate(FLOPS_STEP, args.steps, n, e2e_ms) / 1e12

    if rank == 0:
        hbm, bf16_burst, bf16_sust, src = _peaks()
        long_region = total_ms > 1000.0
        gemm_peak = bf16_sust if long_region else bf16_burst
        col_tflops = FLOPS_COL / (avg[0] * 1e-3) / 1e12
        rs_gbs = RS_BYTES / (rs_ms * 1e-3) / 1e9
        roofline = {"bound": "tensor", "kernel": "gemm_pair_kernel<SwiGLU> (column-parallel gate|up GEMM, CTA pairs)",
                    "achieved": col_tflops, "peak": gemm_peak, "unit": "TFLOP/s", "frac": col_tflops / gemm_peak,
                    "peak_source": f"{src} bf16 {'sustained' if long_region else 'burst'}",
                    "frac_of_sustained": col_tflops / bf16_sust,
                    "flops_per_launch": FLOPS_COL, "avg_launch_ms": avg[0],
                    "traffic": _traffic("gemm_swiglu_8b", "gemm.cu")}
        roofline_rs = {"bound": "hbm", "kernel": "ring_reduce_kernel<f32,t=8> (standalone ReduceScatter along tokens)",
                       "achieved": rs_gbs, "peak": hbm, "unit": "GB/s", "frac": rs_gbs / hbm,
                       "peak_source": f"{src} hbm copy", "bytes_per_launch": RS_BYTES, "avg_launch_ms": rs_ms,
                       "bus_bw_gbs": (T - 1) / T * M_PARTIAL / (rs_ms * 1e-3) / 1e9,
                       "traffic": _traffic("ring_rs_f32_t8", "collectives.cu")}
        row_tflops = FLOPS_ROW / (avg[1] * 1e-3) / 1e12
        fused_roof = {"bound": "tensor", "kernel": "gemm_ring_pair_kernel<f32,AR> (row GEMM + ring RS + AG, CTA pairs)",
                      "achieved": row_tflops, "peak": gemm_peak, "unit": "TFLOP/s", "frac": row_tflops / gemm_peak,
                      "frac_of_sustained": row_tflops / bf16_sust,
                      "flops_per_launch": FLOPS_ROW, "avg_launch_ms": avg[1],
                      "bytes_written_per_launch": T * M_PARTIAL,
                      "traffic": _traffic("gemm_ring_8b", "gemm.cu")}
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": n, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": per_step_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD, "tokens": N_TOK, "h": H, "F": F, "t": T,
                       "parallelism": f"{T} virtual TP shards per GPU; {n} independent replica(s)",
                       "l2": "no flush: each step touches ~1 GB (weights 336 MiB, Z 112 MiB, 8 output replicas 512 MiB) > 126 MB L2"},
            "frac_of_peak_bf16": value / n / gemm_peak,
            "reduce_scatter": {"value": rs_gbs, "unit": "GB/s", "frac_hbm": rs_gbs / hbm},
            "kernels_ms": {"column_gemm_swiglu": avg[0], "row_gemm_rs_ag_fused": avg[1],
                           "standalone_reduce_scatter": rs_ms},
            "kernels_rate": {"column_gemm_tflops": col_tflops, "row_gemm_fused_tflops": row_tflops,
                             "reduce_scatter_gbs": rs_gbs},
            "roofline": roofline, "roofline_fused_row_reduce": fused_roof, "roofline_reduce_scatter": roofline_rs,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": X.numel() * 2,
                    "d2h_bytes_per_step": N_TOK * H * 4, "ms_per_step": e2e_ms / args.steps,
                    "d2h_alone_gbs": d2h_gbs,
                    "how": "tp_mlp_fwd per step; pinned H2D of X and D2H of one reduced replica on separate "
                           "streams, three buffer sets, overlapping the neighbouring steps"},
            "gpu_launches": 2 * args.steps,
            "clocks": clk,
        }
        if extra is not None:
            line["workloads"] = extra
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline()
        _emit(line)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ------------------------------------------------------------------------------ other workloads
def _time_ms(fn, iters: int, warmup: int = 3) -> float:
    """Average device time of fn() over `iters` back-to-back calls (CUDA events, current stream)."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(iters):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters


def _time_graph_ms(fn, per_graph: int, replays: int = 5) -> float:
    """Average device time of one fn() call, measured by replaying a CUDA graph that holds `per_graph`
    back-to-back calls (CUDA events around the replays, after one warm-up replay). The host's per-call
    cost (argument marshalling, launch) stays out of the measurement, which matters for payloads
    whose kernels run for a few microseconds."""
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(3):
            fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(per_graph):
            fn()
    graph.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(replays):
        graph.replay()
    b.record()
    torch.cuda.synchronize()
    del graph
    return a.elapsed_time(b) / (replays * per_graph)


def _iters_for(expected_ms: float, budget_ms: float = 60.0, lo: int = 5, hi: int = 200) -> int:
    return max(lo, min(hi, int(budget_ms / max(expected_ms, 1e-3))))


L2_BYTES = 126 * 2**20   # B200 L2


def collective_point(t: int, dt: str, mib: int, op: str) -> dict:
    """One point of the collective sweep: ReduceScatter / AllGather / AllReduce in ring order over t
    shard buffers resident in HBM. M = each shard's full buffer for RS/AR, the gathered tensor for AG.
    GB/s = algorithmic bytes / time: RS and AG (t+1)M, AR 2tM; ring_bus_gbs is the NCCL-style
    (t-1)/t M (x2 for AR) over the same time. Each point replays a CUDA graph of back-to-back calls
    (the host's per-call cost stays out), and the calls cycle through enough independent buffer sets
    that about twice the L2's size streams between two uses of a set: small payloads are timed from
    HBM, not from L2."""
    import torch
    import tensor_sharded_matmul_b200 as tp
    es = 4 if dt == "f32" else 2
    tdt = torch.float32 if dt == "f32" else torch.bfloat16
    code = tp.TP_F32 if dt == "f32" else tp.TP_BF16
    elems = mib * (1 << 20) // es
    cols = 4096 if elems >= 4096 * 64 else 256
    rows = elems // cols
    M = mib * (1 << 20)
    footprint = {"RS": (t + 1) * M, "AG": (t + 1) * M, "AR": 2 * t * M}[op]
    nsets = max(1, min(128, -(-2 * L2_BYTES // footprint)))
    sets = []
    for _ in range(nsets):
        if op == "AG":
            ins = [torch.empty((rows // t, cols), dtype=tdt, device="cuda").normal_() for _ in range(t)]
            outs = [torch.empty((rows, cols), dtype=tdt, device="cuda") for _ in range(t)]
        else:
            ins = [torch.empty((rows, cols), dtype=tdt, device="cuda").normal_() for _ in range(t)]
            shape = (rows // t, cols) if op == "RS" else (rows, cols)
            outs = [torch.empty(shape, dtype=tdt, device="cuda") for _ in range(t)]
        sets.append((ins, outs))
    nbytes = footprint
    calls = {"RS": lambda i, o: tp.tp_reduce_scatter(i, o, rows, cols, 0, code, t),
             "AG": lambda i, o: tp.tp_all_gather(i, o, rows, cols, 0, code, t),
             "AR": lambda i, o: tp.tp_all_reduce(i, o, rows, cols, code, t)}[op]
    state = {"k": 0}

    def fn():
        i, o = sets[state["k"] % nsets]
        state["k"] += 1
        calls(i, o)

    per_graph = max(2, min(128, int(20e-3 / max(nbytes / 6.0e12, 1e-6))))   # about 20 ms of work per replay
    per_graph = nsets * max(1, -(-per_graph // nsets))                       # every set equally often
    ms = _time_graph_ms(fn, per_graph)
    del sets
    torch.cuda.empty_cache()
    gbs = nbytes / (ms * 1e-3) / 1e9
    bus = (t - 1) / t * M * (2 if op == "AR" else 1) / (ms * 1e-3) / 1e9
    return {"ms": ms, "gbs": gbs, "frac_hbm": gbs / _peaks()[0], "ring_bus_gbs": bus, "bytes": nbytes,
            "buffer_sets": nsets}


CASE_NAMES = {(1, 0): "local", (2, 0): "allgather", (2, 1): "allreduce", (3, 0): "allreduce", (3, 1): "rs_b",
              (3, 2): "rs_f", (4, 0): "gather_x", (4, 1): "gather_w"}


def sharded_matmul_cases(which=None, iters=None):
    """The four sharded-matmul cases of C[B,F] = X[B,D] W[D,F] at B=D=8192, F=28672 over t=4 shards
    (`which`: the (case, strategy) pairs to time, default all). TFLOP/s counts the FLOPs executed
    (case 2 AllGather computes C on every shard). Yields (case, strategy, name, ms, tflops, ws_bytes)."""
    import torch
    import synthetic as S
    import tensor_sharded_matmul_b200 as tp
    B, D, F, t = 8192, 8192, 28672, 4
    X, W = S.case_operands(seed=0, device="cuda")
    shard = {1: (list(X.chunk(t, 0)), [W] * t), 2: (list(X.chunk(t, 1)), [W] * t),
             3: (list(X.chunk(t, 1)), list(W.chunk(t, 0))), 4: (list(X.chunk(t, 0)), list(W.chunk(t, 1)))}
    shapes = {(1, 0): (B // t, F), (2, 0): (B, F), (2, 1): (B, F), (3, 0): (B, F), (3, 1): (B // t, F),
              (3, 2): (B, F // t), (4, 0): (B, F // t), (4, 1): (B // t, F)}
    for (case_id, strategy), name in CASE_NAMES.items():
        if which is not None and (case_id, strategy) not in which:
            continue
        xs, ws = shard[case_id]
        xs = [x.contiguous() for x in xs]
        ws = [w.contiguous() for w in ws] if case_id in (3, 4) else ws
        c = [torch.empty(shapes[(case_id, strategy)], device="cuda") for _ in range(t)]
        nbytes = tp.tp_sharded_matmul_ws_bytes(case_id, strategy, B, D, F, t)
        wsb = torch.empty(max(nbytes, 256), dtype=torch.uint8, device="cuda")
        fn = lambda: tp.tp_sharded_matmul(case_id, strategy, xs, ws, B, D, F, t, c, tp.TP_F32, wsb, nbytes)  # noqa: E731
        flops = 2.0 * B * D * F * (t if (case_id, strategy) == (2, 0) else 1)
        ms = _time_ms(fn, iters if iters else _iters_for(flops / 1.2e12, 60.0, lo=5, hi=50))
        yield case_id, strategy, name, ms, flops / (ms * 1e-3) / 1e12, nbytes
        del c, wsb, xs, ws
        torch.cuda.empty_cache()


def layer70b():
    """One Llama-3-70B-shaped TP=8 layer on 2048 tokens without its attention core (QKV column GEMM,
    W_O row GEMM + AllReduce + residual, SwiGLU MLP + AllReduce + residual). Returns (ms, GFLOP)."""
    import torch
    import synthetic as S
    import tensor_sharded_matmul_b200 as tp
    N, h, n_h, n_kv, d_h, F, t = 2048, 8192, 64, 8, 128, 28672, 8
    L = S.llama70b_layer(seed=0, device="cuda")
    qkv_w = (n_h // t + 2 * (n_kv // t)) * d_h
    w_qkv = torch.empty((t, h, qkv_w), dtype=torch.bfloat16, device="cuda")
    w_o = torch.empty((t, n_h * d_h // t, h), dtype=torch.bfloat16, device="cuda")
    w_gu = torch.empty((t, h, 2 * F // t), dtype=torch.bfloat16, device="cuda")
    w_down = torch.empty((t, F // t, h), dtype=torch.bfloat16, device="cuda")
    tp.tp_shard_qkv(L["Wq"], n_h * d_h, L["Wk"], n_kv * d_h, L["Wv"], n_kv * d_h, h, n_h, n_kv, d_h, t, w_qkv)
    tp.tp_shard_rows(L["Wo"], h, n_h * d_h, h, t, w_o)
    tp.tp_shard_gate_up(L["Wg"], F, L["Wu"], F, h, F, t, w_gu)
    tp.tp_shard_rows(L["Wd"], h, F, h, t, w_down)
    o = [L["O"][:, r * n_h * d_h // t:(r + 1) * n_h * d_h // t].contiguous() for r in range(t)]
    X = L["X"]
    del L
    qkv = torch.empty((t, N, qkv_w), dtype=torch.bfloat16, device="cuda")
    h1 = [torch.empty((N, h), device="cuda") for _ in range(t)]
    h1b = torch.empty((N, h), dtype=torch.bfloat16, device="cuda")
    z = torch.empty((t, N, F // t), dtype=torch.bfloat16, device="cuda")
    y = [torch.empty((N, h), device="cuda") for _ in range(t)]
    fn = lambda: tp.tp_layer_fwd(X, o, N, h, n_h, n_kv, d_h, F, t, w_qkv, w_o, w_gu, w_down, qkv, h1, h1b, z,  # noqa: E731
                                 None, y)
    flops = 2.0 * N * (h * qkv_w * t + n_h * d_h * h + h * 2 * F + F * h)
    ms = _time_ms(fn, 30)
    del w_qkv, w_o, w_gu, w_down, o, X, qkv, h1, h1b, z, y
    torch.cuda.empty_cache()
    return ms, flops / 1e9


def mlp_backward_ms(X, w_in, w_down, z, iters: int) -> float:
    """CUDA-event ms per call of the Llama-3-8B TP-MLP backward (t=8, SwiGLU) from the forward's own
    bf16 intermediates (H recomputed here, Z into z): dZ, dW_down, the SwiGLU backward, dW_in, and dX
    with its ring AllReduce fused into the GEMM."""
    import torch
    import synthetic as S
    import tensor_sharded_matmul_b200 as tp
    t, N, h, f = T, N_TOK, H, F // T
    bf16 = torch.bfloat16
    dY = S.Draw(1, "cuda").normal((N, h), 1.0)
    h_pre = torch.empty((t, N, 2 * f), dtype=bf16, device="cuda")
    tp.tp_column_linear(X, N, h, 2 * F, t, tp.TP_ACT_NONE, w_in, h_pre)
    tp.tp_column_linear(X, N, h, F, t, tp.TP_ACT_SWIGLU, w_in, z)
    dz = torch.empty((t, N, f), dtype=bf16, device="cuda")
    dh = torch.empty((t, N, 2 * f), dtype=bf16, device="cuda")
    g_in = torch.empty((t, h, 2 * f), device="cuda")
    g_down = torch.empty((t, f, h), device="cuda")
    gx = [torch.empty((N, h), device="cuda") for _ in range(t)]
    ms = _time_ms(lambda: tp.tp_mlp_bwd(X, dY, N, h, F, t, tp.TP_ACT_SWIGLU, w_in, w_down, h_pre, z, dz, dh, g_in,
                                        g_down, gx), iters)
    st, site = tp.tp_device_status(1)
    if st != tp.TP_OK:
        raise RuntimeError(f"device wait ran out at site {site}")
    del h_pre, dz, dh, g_in, g_down, gx, dY
    torch.cuda.empty_cache()
    return ms


def all_to_all_ms(iters: int) -> tuple[float, int]:
    """CUDA-event ms per AllToAll over 8 fp32 [4096, 4096] shard buffers (split rows, concatenate
    columns), and the bytes a bit copy must move (read t*M, write t*M)."""
    import torch
    import tensor_sharded_matmul_b200 as tp
    t, N, h = T, N_TOK, H
    ins = [torch.empty((N, h), device="cuda").normal_() for _ in range(t)]
    outs = [torch.empty((N // t, t * h), device="cuda") for _ in range(t)]
    ms = _time_ms(lambda: tp.tp_all_to_all(ins, outs, N, h, 0, 1, tp.TP_F32, t), iters)
    del ins, outs
    torch.cuda.empty_cache()
    return ms, 2 * t * M_PARTIAL


def workloads(X, w_in, w_down, z) -> dict:
    """The other workloads, each timed with CUDA events on the current stream after warm-up, under one
    nvidia-smi clock record: the TP+SP MLP forward, the MLP backward and AllToAll on the 8B shape
    (reusing the headline step's weights), the 70B layer, every sharded-matmul strategy and the ring
    collectives at t in {2, 8}, fp32/bf16, 64 MiB and 1 GiB. Fractions are of the measured burst peaks (each kernel is timed in a short loop)."""
    import torch
    import tensor_sharded_matmul_b200 as tp
    hbm, burst, _, src = _peaks()
    out = {"peak_source": f"{src} (bf16 burst, hbm copy)"}
    clocks = ClockSampler(None)
    clocks.start()
    time.sleep(0.2)
    t0 = time.perf_counter()
    # the TP + SP MLP forward (AllGather along tokens fused into the column GEMM's operand loads,
    # ReduceScatter fused into the row GEMM), on the headline step's weights
    t, N, h = T, N_TOK, H
    x_shards = [X[r * N // t:(r + 1) * N // t].contiguous() for r in range(t)]
    out_sp = [torch.empty((N // t, h), device="cuda") for _ in range(t)]
    ms = _time_ms(lambda: tp.tp_mlp_fwd_sp(x_shards, N, h, F, t, tp.TP_ACT_SWIGLU, w_in, w_down, z, out_sp), 50)
    rate = FLOPS_STEP / (ms * 1e-3) / 1e12
    out["tp_sp_mlp_fwd_llama8b"] = {"ms": ms, "tflops": rate, "frac_bf16_peak": rate / burst}
    del x_shards, out_sp
    ms = mlp_backward_ms(X, w_in, w_down, z, 20)
    rate = 2 * FLOPS_STEP / (ms * 1e-3) / 1e12
    out["mlp_bwd_llama8b"] = {"ms": ms, "tflops": rate, "frac_bf16_peak": rate / burst}
    ms, nbytes = all_to_all_ms(50)
    out["all_to_all_t8_f32_64MiB"] = {"ms": ms, "gbs": nbytes / (ms * 1e-3) / 1e9,
                                      "frac_hbm": nbytes / (ms * 1e-3) / 1e9 / hbm}
    ms, gflop = layer70b()
    rate = gflop / ms
    out["llama70b_tp8_layer"] = {"ms": ms, "tflops": rate, "frac_bf16_peak": rate / burst, "gflop": gflop}
    for case_id, strategy, name, ms, rate, nbytes in sharded_matmul_cases():
        out[f"case{case_id}_{name}"] = {"ms": ms, "tflops": rate, "frac_bf16_peak": rate / burst,
                                        "workspace_bytes": nbytes}
    coll = {}
    for t_ in (2, 8):
        for dt in ("f32", "bf16"):
            for mib in (64, 1024):
                for op in ("RS", "AG", "AR"):
                    r = collective_point(t_, dt, mib, op)
                    coll[f"{op}_t{t_}_{dt}_{mib}MiB"] = {k: r[k] for k in ("ms", "gbs", "frac_hbm")}
    out["collectives"] = coll
    out["wall_s"] = time.perf_counter() - t0
    out["clocks"] = clocks.stop()
    st, site = tp.tp_device_status(1)
    if st != tp.TP_OK:
        raise RuntimeError(f"device wait ran out at site {site}")
    return out


def run_sweep(args) -> int:
    """The collective sweep: ReduceScatter, AllGather and AllReduce in ring order over t in {2,4,8} shard
    buffers, fp32 and bf16, payload M = 1 MiB .. 1 GiB in powers of 4 (M = each shard's full buffer for
    RS/AR, the gathered tensor for AG). GB/s = algorithmic bytes / time: RS and AG (t+1)M, AR 2tM."""
    import torch
    torch.cuda.set_device(0)
    for t in (2, 4, 8):
        for dt in ("f32", "bf16"):
            for mib in (1, 4, 16, 64, 256, 1024):
                for op in ("RS", "AG", "AR"):
                    r = collective_point(t, dt, mib, op)
                    _emit({"config": "collective_sweep", "op": op, "t": t, "dtype": dt, "payload_mib": mib,
                           **{k: r[k] for k in ("ms", "gbs", "frac_hbm", "ring_bus_gbs")}})
    return 0


def run_cases(args) -> int:
    """The four sharded-matmul cases at B=D=8192, F=28672 over t=4 shards, every strategy."""
    import torch
    torch.cuda.set_device(0)
    peak = _peaks()[1]
    which = None
    if args.case:
        c, st = (int(v) for v in args.case.split("."))
        which = {(c, st)}
    iters = args.steps if args.steps < 500 else None
    import tensor_sharded_matmul_b200 as tp
    for case_id, strategy, name, ms, rate, nbytes in sharded_matmul_cases(which, iters):
        # the strategy the pages' byte rule would pick on t devices (case 3: the output sharding decides)
        rule = tp.tp_sharded_matmul_choose(case_id, 8192, 8192, 28672, 4) if case_id != 3 else None
        _emit({"config": "sharded_matmul", "case": case_id, "strategy": name, "ms": ms, "tflops_executed": rate,
               "frac_bf16_peak": rate / peak, "workspace_bytes": nbytes,
               "cost_rule_choice": None if rule is None else rule == strategy})
    return 0


def run_layer70b(args) -> int:
    """One Llama-3-70B-shaped TP=8 layer on 2048 tokens without its attention core."""
    import torch
    torch.cuda.set_device(0)
    ms, gflop = layer70b()
    _emit({"config": "llama70b_tp8_layer", "tokens": 2048, "ms": ms, "gflop": gflop,
           "tflops": gflop / ms, "frac_bf16_peak": gflop / ms / _peaks()[1]})
    return 0


ROW_REDUCE_SHAPES = {
    # name: (t, tokens, k (the full contraction), n, reduce mode) of tp_row_linear_reduce
    "8b_rs_ag": (8, 4096, 14336, 4096, "RS_AG"),     # Llama-3-8B down projection, RS along tokens + AG
    "8b_rs": (8, 4096, 14336, 4096, "RS"),           # the same, ReduceScatter only (TP+SP exit)
    "70b_wo_ar": (8, 2048, 8192, 8192, "AR"),        # Llama-3-70B attention output projection + AR
    "70b_down_ar": (8, 2048, 28672, 8192, "AR"),     # Llama-3-70B down projection + AR
}
# chunk axis of each shape's ReduceScatter: the 70B layer's AllReduces scatter along h (columns)
ROW_REDUCE_AXIS = {"8b_rs_ag": 0, "8b_rs": 0, "70b_wo_ar": 1, "70b_down_ar": 1}


def run_rowreduce(args) -> int:
    """The row-parallel GEMM fused with its ring collective (tp_row_linear_reduce) on the Llama-3 8B
    and 70B shapes, one JSON line per shape: x bf16 [t][N][k/t] ~N(0,1), w bf16 [t][k/t][n] ~N(0,0.02).
    TFLOP/s counts 2*N*k*n; the fraction is of the measured bf16 burst peak."""
    import torch
    import synthetic as S
    import tensor_sharded_matmul_b200 as tp
    torch.cuda.set_device(0)
    burst = _peaks()[1]
    modes = {"RS": tp.TP_OUT_RS, "AR": tp.TP_OUT_AR, "RS_AG": tp.TP_OUT_RS_AG}
    names = [args.shape] if args.shape else list(ROW_REDUCE_SHAPES)
    for name in names:
        t, N, k, n, mode = ROW_REDUCE_SHAPES[name]
        d = S.Draw(7, "cuda")
        x = d.normal((t, N, k // t), 1.0)
        w = d.normal((t, k // t, n), 0.02)
        rows = N // t if mode == "RS" else N
        out = [torch.empty((rows, n), device="cuda") for _ in range(t)]
        axis = ROW_REDUCE_AXIS[name] if args.axis is None else args.axis
        fn = lambda: tp.tp_row_linear_reduce(x, N, k, n, t, w, modes[mode], axis, out)  # noqa: E731
        ms = _time_ms(fn, args.steps if args.steps < 500 else 50)
        rate = 2.0 * N * k * n / (ms * 1e-3) / 1e12
        _emit({"config": "rowreduce", "shape": name, "t": t, "tokens": N, "k": k, "n": n, "mode": mode, "axis": axis,
               "ms": ms,
               "tflops": rate, "frac_bf16_peak": rate / burst,
               "bytes_written": t * rows * n * 4})
        del x, w, out
        torch.cuda.empty_cache()
    st, site = tp.tp_device_status(1)
    if st != tp.TP_OK:
        print(f"device wait ran out at site {site}", file=sys.stderr)
        return 3
    return 0


def run_next(args) -> int:
    """The rows beyond the forward MLP, on the Llama-3-8B shape (4096 tokens, h=4096, F=14336, t=8):
    the TP+SP MLP forward (AllGather along tokens fused into the column GEMM's operand loads,
    ReduceScatter fused into the row GEMM), the MLP's backward pass (dZ, dW_down, activation
    backward, dW_in, dX with its ring AllReduce), and AllToAll over the 8 fp32 [4096,4096] shard
    buffers. TFLOP/s counts algorithmic FLOPs (forward 6*N*h*F, backward 12*N*h*F); GB/s counts the
    bytes a bit copy must move (read t*M, write t*M)."""
    import torch
    import synthetic as S
    import tensor_sharded_matmul_b200 as tp
    torch.cuda.set_device(0)
    hbm, burst, sust, _ = _peaks()
    t, N, h, f = T, N_TOK, H, F // T
    bf16 = torch.bfloat16
    X, Wgu, Wd = S.llama8b_mlp(seed=0, device="cuda")
    w_in = torch.empty((t, h, 2 * f), dtype=bf16, device="cuda")
    w_down = torch.empty((t, f, h), dtype=bf16, device="cuda")
    tp.tp_shard_gate_up(Wgu, 2 * F, Wgu.data_ptr() + 2 * F, 2 * F, h, F, t, w_in)
    tp.tp_shard_rows(Wd, h, F, h, t, w_down)
    del Wgu, Wd
    z = torch.empty((t, N, f), dtype=bf16, device="cuda")

    def tensor_line(row, ms, flops):
        rate = flops / (ms * 1e-3) / 1e12
        _emit({"config": "next", "row": row, "ms": ms, "tflops": rate, "frac_bf16_peak": rate / burst,
               "frac_of_sustained": rate / sust, "flops": flops})

    # f1: TP + SP forward
    x_shards = [X[r * N // t:(r + 1) * N // t].contiguous() for r in range(t)]
    out_sp = [torch.empty((N // t, h), device="cuda") for _ in range(t)]
    ms = _time_ms(lambda: tp.tp_mlp_fwd_sp(x_shards, N, h, F, t, tp.TP_ACT_SWIGLU, w_in, w_down, z, out_sp), 50)
    tensor_line("f1 TP+SP MLP forward (AG fused into the column GEMM, RS fused into the row GEMM)", ms, FLOPS_STEP)
    del out_sp, x_shards

    # f3: backward, from the forward's own intermediates
    ms = mlp_backward_ms(X, w_in, w_down, z, 20)
    tensor_line("f3 MLP backward (dZ, dW_down, SwiGLU backward, dW_in, dX + ring AllReduce)", ms, 2 * FLOPS_STEP)

    # f4: AllToAll, split rows / concatenate columns
    ms, nbytes = all_to_all_ms(50)
    gbs = nbytes / (ms * 1e-3) / 1e9
    _emit({"config": "next", "row": "f4 AllToAll, 8 x fp32 [4096,4096], split rows / concat columns", "ms": ms,
           "gbs": gbs, "frac_hbm": gbs / hbm, "bytes": nbytes})
    return 0


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing (profiling runs)")
    ap.add_argument("--no-workloads", action="store_true",
                    help="time the headline step only (profiling runs; multi-GPU runs always do)")
    ap.add_argument("--config", choices=["mlp8b", "sweep", "cases", "layer70b", "next", "rowreduce"], default="mlp8b",
                    help="mlp8b: the headline step (one JSON line); the others print one line per measurement")
    ap.add_argument("--axis", type=int, choices=[0, 1], default=None,
                    help="--config rowreduce: chunk axis of the ReduceScatter (default: the shape's own)")
    ap.add_argument("--case", default=None, help="--config cases: one strategy only, as CASE.STRATEGY (e.g. 4.1)")
    ap.add_argument("--shape", choices=sorted(ROW_REDUCE_SHAPES), default=None,
                    help="--config rowreduce: one shape only (default: all)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.config == "sweep":
        return run_sweep(args)
    if args.config == "cases":
        return run_cases(args)
    if args.config == "layer70b":
        return run_layer70b(args)
    if args.config == "next":
        return run_next(args)
    if args.config == "rowreduce":
        return run_rowreduce(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
