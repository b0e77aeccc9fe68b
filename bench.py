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
oracle on a bounded row sample of the same workload on this host.

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
CPU_SAMPLE_ROWS = 512
REF_ROWS_PER_STEP = 64


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
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if e.get("source_sha") != sha:
        return None
    return e.get("bytes_per_launch")


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


def _blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def cpu_baseline(rows: int = CPU_SAMPLE_ROWS) -> dict:
    Xs, si, sd = _oracle_sample(rows)
    t0 = time.perf_counter()
    _oracle_step(Xs, si, sd)
    dt = time.perf_counter() - t0
    flops = FLOPS_STEP * rows / N_TOK
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{rows} of {N_TOK} token rows of the same MLP (all 8 shards' fp64 GEMMs + fp32 ring RS/AG), "
                      f"{dt:.2f} s; value = sample FLOPs / time"}


def run_reference(args) -> int:
    ws, rank, _ = _dist_env()
    if rank != 0:
        return 0
    Xs_all, si, sd = _oracle_sample(REF_ROWS_PER_STEP * 4)
    times = []
    for i in range(args.warmup + args.steps):
        r0 = (i % 4) * REF_ROWS_PER_STEP
        Xs = Xs_all[r0:r0 + REF_ROWS_PER_STEP]
        t0 = time.perf_counter()
        _oracle_step(Xs, si, sd)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    per_step = sum(times) / len(times)
    flops = FLOPS_STEP * REF_ROWS_PER_STEP / N_TOK
    value = flops / per_step / 1e12
    cores = _blas_threads()
    _emit({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample_rows_per_step": REF_ROWS_PER_STEP},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"{REF_ROWS_PER_STEP} of {N_TOK} token rows per step"},
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
    x_host = X.cpu().pin_memory()
    y_host = torch.empty((N_TOK, H), dtype=torch.float32).pin_memory()
    x_dev = torch.empty_like(X)
    for _ in range(max(1, min(args.warmup, 3))):
        x_dev.copy_(x_host, non_blocking=True)
        tp.tp_mlp_fwd(x_dev, N_TOK, H, F, T, tp.TP_ACT_SWIGLU, w_in, w_down, z, None, tp.TP_OUT_RS_AG, out)
        y_host.copy_(out[0], non_blocking=True)
    e_start, e_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e_start.record(stream)
    for _ in range(args.steps):
        x_dev.copy_(x_host, non_blocking=True)
        tp.tp_mlp_fwd(x_dev, N_TOK, H, F, T, tp.TP_ACT_SWIGLU, w_in, w_down, z, None, tp.TP_OUT_RS_AG, out)
        y_host.copy_(out[0], non_blocking=True)
    e_stop.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e_start.elapsed_time(e_stop)

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
        roofline = {"bound": "tensor", "kernel": "gemm_tcgen05_kernel<SwiGLU> (column-parallel gate|up GEMM)",
                    "achieved": col_tflops, "peak": gemm_peak, "unit": "TFLOP/s", "frac": col_tflops / gemm_peak,
                    "peak_source": f"{src} bf16 {'sustained' if long_region else 'burst'}",
                    "flops_per_launch": FLOPS_COL, "avg_launch_ms": avg[0],
                    "traffic": _traffic("gemm_swiglu_8b", "gemm.cu")}
        roofline_rs = {"bound": "hbm", "kernel": "ring_reduce_kernel<f32,t=8> (standalone ReduceScatter along tokens)",
                       "achieved": rs_gbs, "peak": hbm, "unit": "GB/s", "frac": rs_gbs / hbm,
                       "peak_source": f"{src} hbm copy", "bytes_per_launch": RS_BYTES, "avg_launch_ms": rs_ms,
                       "bus_bw_gbs": (T - 1) / T * M_PARTIAL / (rs_ms * 1e-3) / 1e9,
                       "traffic": _traffic("ring_rs_f32_t8", "collectives.cu")}
        row_tflops = FLOPS_ROW / (avg[1] * 1e-3) / 1e12
        fused_roof = {"bound": "tensor", "kernel": "gemm_ring_kernel<f32,AR> (row GEMM + ring RS + AG)",
                      "achieved": row_tflops, "peak": gemm_peak, "unit": "TFLOP/s", "frac": row_tflops / gemm_peak,
                      "flops_per_launch": FLOPS_ROW, "avg_launch_ms": avg[1],
                      "bytes_written_per_launch": T * M_PARTIAL,
                      "traffic": _traffic("gemm_ring_8b", "gemm.cu")}
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": n, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": per_step_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD, "model": "llama3-8b-mlp", "tokens": N_TOK, "h": H, "F": F, "t": T,
                       "parallelism": f"{T} virtual TP shards per GPU; {n} independent replica(s)",
                       "l2": "no flush: each step touches ~1.5 GB (weights 336 MiB, partials and outputs 1 GiB) > 126 MB L2"},
            "frac_of_peak_bf16": value / n / gemm_peak,
            "reduce_scatter": {"value": rs_gbs, "unit": "GB/s", "frac_hbm": rs_gbs / hbm},
            "kernels_ms": {"column_gemm_swiglu": avg[0], "row_gemm_rs_ag_fused": avg[1],
                           "standalone_reduce_scatter": rs_ms},
            "kernels_rate": {"column_gemm_tflops": col_tflops, "row_gemm_fused_tflops": row_tflops,
                             "reduce_scatter_gbs": rs_gbs},
            "roofline": roofline, "roofline_fused_row_reduce": fused_roof, "roofline_reduce_scatter": roofline_rs,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": X.numel() * 2,
                    "d2h_bytes_per_step": N_TOK * H * 4},
            "gpu_launches": 2 * args.steps,
            "clocks": clk,
        }
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline()
        _emit(line)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing (profiling runs)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
