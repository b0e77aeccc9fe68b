"""The four sharded-matmul cases of C[B,F] = X[B,D] . W[D,F] over t shards (test infrastructure).

Source: "Scaling Book 入门第 6 章：分片矩阵乘法 — 分布式计算的核心", §6.2 分片矩阵乘法的四种情况 (Cases 1-4,
the block-matrix identity), §6.4 (AllGather / ReduceScatter / AllReduce semantics), §6.9 Problems 4 and 9
(the two case-2 strategies and their costs). Products are fp64 over exactly-widened bf16 operands;
the collectives are the ring steps of ``oracle.collectives`` accumulated in fp64.

Operands per case (each list has one entry per shard; "replicated" entries are the same matrix):
  case 1: X[B_X, D] . W[D, F]            x: t x [B/t, D]  w: t x [D, F]    -> C[B_X, F], no communication
  case 2: X[B, D_X] . W[D, F]            x: t x [B, D/t]  w: t x [D, F]
          strategy "allgather": X <- AllGather(X); every shard computes the full C (replicated compute)
          strategy "allreduce": shard i multiplies by its own row block of W, then AllReduce  -> C[B, F]
  case 3: X[B, D_X] . W[D_X, F]          x: t x [B, D/t]  w: t x [D/t, F]  -> C[B,F]{U_X}, then
          "allreduce" -> C[B, F]; "rs_b" -> ReduceScatter onto B -> C[B_X, F]; "rs_f" -> C[B, F_X]
  case 4: X[B_X, D] . W[D, F_X] (illegal as is: only the diagonal blocks), fixed by
          "gather_x" -> C[B, F_X] or "gather_w" -> C[B_X, F]
"""
from __future__ import annotations

import numpy as np

from .collectives import all_gather, reduce_scatter_f64
from .mlp import matmul

STRATEGIES = {1: ("local",), 2: ("allgather", "allreduce"), 3: ("allreduce", "rs_b", "rs_f"), 4: ("gather_x", "gather_w")}


def all_reduce_f64(bufs):
    """AllReduce = ReduceScatter (rows) + AllGather, accumulated in fp64."""
    return all_gather(reduce_scatter_f64(bufs, axis=0), axis=0)


def case1(x, w):
    """Contracting dim unsharded: each shard multiplies its own rows, no communication."""
    return [matmul(xi, wi) for xi, wi in zip(x, w)]


def case2(x, w, strategy: str):
    """One operand sharded on the contracting dim."""
    t = len(x)
    if strategy == "allgather":
        xs = all_gather([np.asarray(xi, dtype=np.float64) for xi in x], axis=1)   # every shard: X[B, D]
        return [matmul(xs[i], w[i]) for i in range(t)]
    if strategy == "allreduce":
        D = np.asarray(w[0]).shape[0]
        d = D // t
        partial = [matmul(x[i], np.asarray(w[i])[i * d:(i + 1) * d, :]) for i in range(t)]   # C{U_X}
        return all_reduce_f64(partial)
    raise ValueError(strategy)


def case3(x, w, strategy: str):
    """Both operands sharded on the contracting dim: local partial C{U_X}, then AllReduce or a
    ReduceScatter that introduces the new sharding on B (rows) or F (columns)."""
    partial = [matmul(xi, wi) for xi, wi in zip(x, w)]
    if strategy == "allreduce":
        return all_reduce_f64(partial)
    if strategy == "rs_b":
        return reduce_scatter_f64(partial, axis=0)
    if strategy == "rs_f":
        return reduce_scatter_f64(partial, axis=1)
    raise ValueError(strategy)


def case4(x, w, strategy: str):
    """Both non-contracting dims on the same axis: gather one operand first."""
    t = len(x)
    if strategy == "gather_x":
        xs = all_gather([np.asarray(xi, dtype=np.float64) for xi in x], axis=0)    # X[B, D] everywhere
        return [matmul(xs[i], w[i]) for i in range(t)]
    if strategy == "gather_w":
        ws = all_gather([np.asarray(wi, dtype=np.float64) for wi in w], axis=1)    # W[D, F] everywhere
        return [matmul(x[i], ws[i]) for i in range(t)]
    raise ValueError(strategy)


def case4_naive(x, w):
    """The illegal local product: shard i only gets the diagonal block C[B-range i, F-range i]."""
    return [matmul(xi, wi) for xi, wi in zip(x, w)]


def run(case_id: int, strategy: str, x, w):
    if case_id == 1:
        return case1(x, w)
    if case_id == 2:
        return case2(x, w, strategy)
    if case_id == 3:
        return case3(x, w, strategy)
    if case_id == 4:
        return case4(x, w, strategy)
    raise ValueError(case_id)


def output_layout(case_id: int, strategy: str) -> str:
    """How the t outputs tile the logical C: "rows" (C[B_X, F]), "cols" (C[B, F_X]) or
    "replicated" (every shard holds C[B, F])."""
    table = {
        (1, "local"): "rows", (2, "allgather"): "replicated", (2, "allreduce"): "replicated",
        (3, "allreduce"): "replicated", (3, "rs_b"): "rows", (3, "rs_f"): "cols",
        (4, "gather_x"): "cols", (4, "gather_w"): "rows",
    }
    return table[(case_id, strategy)]


def to_logical(outs, layout: str):
    """Assemble the logical C from the shards' outputs (replicas must agree)."""
    if layout == "rows":
        return np.concatenate(outs, axis=0)
    if layout == "cols":
        return np.concatenate(outs, axis=1)
    if layout == "replicated":
        return outs[0]
    raise ValueError(layout)


def case4_choice(B: int, D: int, F: int) -> str:
    """Case 4 fixes the doubly-sharded contraction by gathering one operand; the page leaves which one
    open ("Scaling Book 入门第 6 章", §6.2 Case 4: it depends). Reading: gather the smaller one, as the
    byte count of an AllGather is the operand's size. X[B_X, D] has B*D elements, W[D, F_X] D*F."""
    return "gather_x" if B * D <= D * F else "gather_w"


def case2_choice(gathered_elems: int, output_elems: int) -> str:
    """Pick the case-2 strategy by bytes moved (ring, bandwidth-bound, same dtype): AllGather of the
    operand sharded on the contracting dim moves about its full size; AllReduce of the output about
    twice the output's size. ("Scaling Book 入门第 6 章", §6.2 Case 2 and §6.9 Problem 4: with the
    weight Y[D_X, F] as the gathered operand and output Z[B, F], AllReduce wins when D > 2B.)
    For the config X[B, D_X] . W[D, F] the gathered operand is X: gathered = B*D, output = B*F."""
    return "allgather" if gathered_elems <= 2 * output_elems else "allreduce"
