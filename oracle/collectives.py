"""Ring collectives over t shard buffers, by literal step simulation (test infrastructure).

Sources:
  * "Scaling Book 入门第 5 章：Sharded Matrices 上篇 — 集合通信原语", §5.2 环形算法: devices form a ring and
    each passes to its right-hand neighbour (device i -> i+1, the last wraps to the first); the
    unidirectional AllGather takes N-1 steps and the bidirectional one floor(N/2), with N=4 step tables.
  * same page, §5.3 四种核心通信原语: ReduceScatter leaves reduced chunk r on device r
    (device 0 = a0+b0+c0+d0, device 1 = a1+b1+c1+d1, ...); ring ReduceScatter takes N-1 steps, each
    sending 1/N of the data and adding it into the local chunk; AllReduce = ReduceScatter + AllGather.
  * "Scaling Book 入门第 6 章：分片矩阵乘法", §6.4 通信原语详解: ReduceScatter is the ring pass "with an
    accumulation at every step"; it may introduce the new sharding along either logical dimension;
    AllGather and ReduceScatter are each other's transpose.

Reading of what the pages leave open (the pages never state a summation order):
  * The order is the one the stated ring produces. At step s = 1..t-1 device i passes its running
    partial of chunk (i - s) mod t to device i+1, which adds its own copy of that chunk. Chunk c is
    therefore summed as (((U[c+1] + U[c+2]) + U[c+3]) + ... ) + U[c] (indices mod t), left to right.
  * fp32 payloads are accumulated in binary32 (one IEEE rounding per add). bf16 payloads are widened
    to binary32, accumulated in the same order and rounded once to bf16 at the end.
  * Optional per-hop rounding for bf16 (rounding="hop"): read literally, each device of the ring holds
    and passes on its running partial in the payload's own type, so when the links carry bf16 the
    partial is rounded to bf16 after every add (binary32 add, then round to nearest-even bf16), as
    a ring whose buffers are bf16 does. The default ("end") keeps the partial in binary32.
  * Chunk r of a [rows, cols] buffer is the row block [r*rows/t, (r+1)*rows/t) for axis 0 and the
    column block [r*cols/t, (r+1)*cols/t) for axis 1; AllGather concatenates in shard order.
  * In the bidirectional AllGather with even N, the antipodal shard arrives at the last step through
    the rightward direction only (the tables record contents, not links).
"""
from __future__ import annotations

import numpy as np

from .bf16 import bf16_bits_to_f32, f32_to_bf16_bits


# --------------------------------------------------------------------------------------------
# Generic ring ReduceScatter over an abstract "add": the numeric and the provenance versions
# both run these very steps.
# --------------------------------------------------------------------------------------------

def ring_reduce_scatter_steps(own, add):
    """own[i][c]: device i's own (unreduced) copy of chunk c. Returns held[j]: the reduced chunk j
    that device j ends with, built by the unidirectional ring's t-1 send-and-add steps."""
    t = len(own)
    if t == 1:
        return [own[0][0]]
    # step 1 payload: device i sends its own copy of chunk (i - 1) mod t
    sending = [own[i][(i - 1) % t] for i in range(t)]
    for s in range(1, t):
        arrived = [None] * t
        for j in range(t):
            c = (j - 1 - s) % t                       # chunk that reaches device j at step s
            incoming = sending[(j - 1) % t]           # from the left-hand neighbour
            arrived[j] = add(incoming, own[j][c])     # accumulate the local copy
        sending = arrived                             # what each device passes on next step
    return sending                                    # after step t-1 device j holds chunk j


def ring_sum_provenance(t: int):
    """For each chunk c, the order in which the shards' copies are added (a list of shard ids)."""
    own = [[(i,) for _ in range(t)] for i in range(t)]
    held = ring_reduce_scatter_steps(own, lambda a, b: a + b)
    return [list(h) for h in held]


# --------------------------------------------------------------------------------------------
# Numeric collectives
# --------------------------------------------------------------------------------------------

def _split(buf: np.ndarray, t: int, axis: int):
    if buf.shape[axis] % t != 0:
        raise ValueError(f"dimension {buf.shape[axis]} not divisible by t={t}")
    return np.split(buf, t, axis=axis)


def _as_f32(buf, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return bf16_bits_to_f32(buf)
    if dtype == "f32":
        return np.asarray(buf, dtype=np.float32)
    raise ValueError(dtype)


def _from_f32(x: np.ndarray, dtype: str) -> np.ndarray:
    return f32_to_bf16_bits(x) if dtype == "bf16" else np.asarray(x, dtype=np.float32)


def _bf16_hop_add(a, b):
    """One hop of a ring whose links carry bf16: binary32 add, then the partial rounded to bf16."""
    return bf16_bits_to_f32(f32_to_bf16_bits(np.add(a, b, dtype=np.float32)))


def reduce_scatter(bufs, axis: int = 0, dtype: str = "f32", out_dtype: str | None = None, rounding: str = "end"):
    """Ring ReduceScatter of t full-size buffers (2-D numpy arrays: float32, or uint16 bf16 bits).

    Returns t arrays, the reduced chunk r for shard r, in ``out_dtype`` (default = ``dtype``).
    Accumulation is binary32 in the ring order described in the module docstring; with
    ``rounding="hop"`` (bf16 only) the running partial is rounded to bf16 after every add."""
    out_dtype = out_dtype or dtype
    if rounding not in ("end", "hop") or (rounding == "hop" and (dtype, out_dtype) != ("bf16", "bf16")):
        raise ValueError("per-hop rounding is a bf16 -> bf16 mode")
    t = len(bufs)
    own = [_split(_as_f32(b, dtype), t, axis) for b in bufs]
    add = _bf16_hop_add if rounding == "hop" else (lambda a, b: np.add(a, b, dtype=np.float32))
    held = ring_reduce_scatter_steps(own, add)
    return [_from_f32(h.copy(), out_dtype) for h in held]


def reduce_scatter_f64(bufs, axis: int = 0):
    """The same ring steps accumulated in float64 (used for the transposition identity)."""
    t = len(bufs)
    own = [_split(np.asarray(b, dtype=np.float64), t, axis) for b in bufs]
    return [h.copy() for h in ring_reduce_scatter_steps(own, lambda a, b: a + b)]


def all_gather_steps(labels, bidirectional: bool = False):
    """Provenance simulation of the ring AllGather. labels[i]: what device i starts with.

    Returns (steps, final): steps[s][i] is device i's holdings after step s+1 in arrival order;
    final[i] is device i's gathered buffer in shard order."""
    t = len(labels)
    hold = [[labels[i]] for i in range(t)]
    steps = []
    if not bidirectional:
        fwd = list(labels)                                 # what each device passes rightwards
        for _ in range(t - 1):
            recv = [fwd[(i - 1) % t] for i in range(t)]
            for i in range(t):
                hold[i].append(recv[i])
            fwd = recv
            steps.append([list(h) for h in hold])
    else:
        right = list(labels)                               # travelling i -> i+1
        left = list(labels)                                # travelling i -> i-1
        n_right = t // 2                                   # distances the rightward direction covers
        n_left = (t - 1) // 2                              # ... and the leftward one
        for s in range(1, max(n_right, n_left) + 1):
            recv_r = [right[(i - 1) % t] for i in range(t)] if s <= n_right else None
            recv_l = [left[(i + 1) % t] for i in range(t)] if s <= n_left else None
            for i in range(t):
                if recv_r is not None:
                    hold[i].append(recv_r[i])
                if recv_l is not None:
                    hold[i].append(recv_l[i])
            if recv_r is not None:
                right = recv_r
            if recv_l is not None:
                left = recv_l
            steps.append([list(h) for h in hold])
    final = []
    for i in range(t):
        have = set(hold[i])
        if len(have) != t or len(hold[i]) != t:
            raise AssertionError("ring AllGather did not deliver every shard exactly once")
        final.append([labels[k] for k in range(t)])
    return steps, final


def all_gather(bufs, axis: int = 0):
    """Ring AllGather of t shard buffers: every shard ends with the concatenation, in shard order,
    of all shards' buffers (a bit copy; works on float32 or uint16 bf16 bits alike). The pieces are
    moved along the unidirectional ring's t-1 steps, then placed by their origin."""
    t = len(bufs)
    hold = [{i: np.asarray(bufs[i])} for i in range(t)]
    fwd = list(range(t))
    for _ in range(t - 1):
        recv = [fwd[(i - 1) % t] for i in range(t)]        # origin id of the piece each receives
        for i in range(t):
            src = (i - 1) % t
            hold[i][recv[i]] = hold[src][recv[i]]
        fwd = recv
    return [np.concatenate([hold[i][k] for k in range(t)], axis=axis) for i in range(t)]


def all_reduce(bufs, dtype: str = "f32", out_dtype: str | None = None, rounding: str = "end", axis: int = 0):
    """AllReduce = ReduceScatter followed by AllGather along the same axis: every shard ends with the
    full ring-ordered sum. The ReduceScatter may scatter along either dimension ("Scaling Book 入门第 6
    章", §6.4), which decides each element's summation order: rows (axis 0, the default) or columns
    (axis 1). With bf16 the one rounding happens at the end of the ReduceScatter (or after every hop,
    with rounding="hop")."""
    rs = reduce_scatter(bufs, axis=axis, dtype=dtype, out_dtype=out_dtype, rounding=rounding)
    return all_gather(rs, axis=axis)


def all_to_all(bufs, split_axis: int, concat_axis: int):
    """AllToAll (moves the sharded dimension): shard j receives piece j of every shard's buffer,
    concatenated in source-shard order ("Scaling Book 入门第 5 章", §5.3 AllToAll: device 0 = [A0,B0,C0,D0])."""
    t = len(bufs)
    pieces = [np.split(np.asarray(b), t, axis=split_axis) for b in bufs]
    return [np.concatenate([pieces[i][j] for i in range(t)], axis=concat_axis) for j in range(t)]
