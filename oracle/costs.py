"""Closed-form sizes and costs the pages state (test infrastructure; pinned to the pages' printed numbers).

Sources:
  * "Scaling Book 入门第 6 章", §6.1 (per-device memory of a sharded array, Pop Quiz), §6.5 (roofline of
    case 3: T_math = 2BDF/(N*C), T_comms = 4BF/W), §6.9 Problem 1 (replication ratio).
  * "张量并行与序列并行", §预备 (ring bytes per rank: AllGather and ReduceScatter (t-1)/t*M, AllReduce
    2(t-1)/t*M), §精确的通信量 (Llama-3 70B example), §为什么 TP 留在节点内 (TP bound F*W/C),
    §GQA (Llama-3 70B per-shard weight shapes and parameter counts).
  * "Scaling Book 入门第 5 章", §5.3 AllToAll (unidirectional ring traffic V(N-1)/(2N) vs AllGather V(N-1)/N).
"""
from __future__ import annotations

from math import prod

MiB = 1 << 20
GiB = 1 << 30


def local_shape(shape, split_axes, mesh: dict):
    """Local shape of an array whose dimension d is split over the mesh axes split_axes[d] (a tuple
    of axis names, possibly empty); a mesh axis may be used at most once."""
    used = [a for axes in split_axes for a in axes]
    if len(used) != len(set(used)):
        raise ValueError("a mesh axis cannot shard two dimensions")
    out = []
    for n, axes in zip(shape, split_axes):
        k = prod(mesh[a] for a in axes) if axes else 1
        if n % k:
            raise ValueError("dimension not divisible by its mesh axes")
        out.append(n // k)
    return tuple(out)


def per_device_bytes(shape, split_axes, mesh: dict, itemsize: int) -> int:
    return prod(local_shape(shape, split_axes, mesh)) * itemsize


def total_bytes(shape, split_axes, mesh: dict, itemsize: int) -> int:
    """Bytes over all devices of the mesh (every device holds one local block)."""
    return per_device_bytes(shape, split_axes, mesh, itemsize) * prod(mesh.values())


def replication_ratio(split_axes, mesh: dict) -> int:
    """Total bytes over all devices divided by the size of one copy = product of unused axes."""
    used = {a for axes in split_axes for a in axes}
    return prod(n for a, n in mesh.items() if a not in used)


def ring_bytes_per_rank(op: str, M: float, t: int) -> float:
    """Bytes each rank sends in the ring: all_gather (M = full gathered tensor) and
    reduce_scatter (M = each rank's full-size partial) send (t-1)/t*M; all_reduce 2(t-1)/t*M."""
    if op in ("all_gather", "reduce_scatter"):
        return (t - 1) / t * M
    if op == "all_reduce":
        return 2 * (t - 1) / t * M
    raise ValueError(op)


def unidirectional_link_traffic(op: str, V: float, N: int) -> float:
    """Per-link traffic on a unidirectional ring: AllGather V(N-1)/N, AllToAll V(N-1)/(2N)."""
    if op == "all_gather":
        return V * (N - 1) / N
    if op == "all_to_all":
        return (V / N ** 2) * sum(range(1, N))
    raise ValueError(op)


def case3_compute_bound_D(N: int, flops: float, W: float) -> float:
    """Case 3 is compute-bound when 2BDF/(N C) > 4BF/W, i.e. D > 2 N C / W."""
    return 2 * N * flops / W


def tp_upper_bound(F: int, C_over_W: float) -> float:
    """A two-matrix MLP stays compute-bound under TP degree Y while Y < F * W / C."""
    return F / C_over_W


def allgather_overlap_ratio(t: int, h: int, C: float, W: float, itemsize: int = 2) -> float:
    """Time of the next layer's AllGather ((t-1)/t * b s h elements at W/itemsize elements/s)
    over the compute of one [h, h] linear (2 b s h^2 / t FLOPs at C)."""
    return ((t - 1) / (2 * h)) * C / (W / itemsize)


def llama_layer_shapes(h: int, n_h: int, n_kv: int, d_h: int, F: int, t: int):
    """Per-shard weight shapes of a Llama-style layer under TP degree t (t | n_kv case):
    fused QKV [h, (n_h/t + 2 n_kv/t) d_h], W_O [n_h d_h / t, h], gate|up [h, 2F/t], down [F/t, h]."""
    return {
        "qkv": (h, (n_h // t + 2 * (n_kv // t)) * d_h),
        "o": (n_h * d_h // t, h),
        "gate_up": (h, 2 * F // t),
        "down": (F // t, h),
    }


def params_per_layer(h: int, n_h: int, n_kv: int, d_h: int, F: int) -> int:
    """Linear-layer parameters of one Llama-style layer (norm weights left out)."""
    return h * n_h * d_h + 2 * h * n_kv * d_h + n_h * d_h * h + 2 * h * F + F * h


def params_per_shard(h: int, n_h: int, n_kv: int, d_h: int, F: int, t: int) -> int:
    return sum(prod(s) for s in llama_layer_shapes(h, n_h, n_kv, d_h, F, t).values())


def tp_layer_comm(b: int, s: int, h: int, t: int, layers: int, itemsize: int = 2):
    """Per-card ring bytes of pure TP: one AllReduce of M = itemsize*b*s*h sends 2(t-1)/t*M;
    a layer has 2 in the forward and 2 in the backward pass."""
    M = itemsize * b * s * h
    ar = ring_bytes_per_rank("all_reduce", M, t)
    return {"M": M, "per_allreduce": ar, "per_layer": 4 * ar, "model": 4 * ar * layers}


def layer_forward_flops(b: int, s: int, params: int, h: int) -> dict:
    """Forward FLOPs of one layer: 2 * tokens * params for the matmuls plus 2 b s^2 h for causal attention."""
    mm = 2 * b * s * params
    attn = 2 * b * s * s * h
    return {"matmul": mm, "attention": attn, "total": mm + attn}
