"""Weight shard layouts, written as plain block copies from their definitions (test infrastructure).

All weights are [in, out] row-major, as the pages write a linear layer Y = X W with W of shape [k, n]
("张量并行与序列并行", §矩阵乘法的两种切法). Arrays may be any dtype (bf16 bits as uint16 compare byte
for byte with the GPU's layout kernels).
"""
from __future__ import annotations

import numpy as np


def shard_cols(W: np.ndarray, t: int) -> np.ndarray:
    """Column-parallel split: shard r holds W[:, r*n/t:(r+1)*n/t] (shape [k, n/t]).
    ("张量并行与序列并行", §矩阵乘法的两种切法, the first identity; "Scaling Book 入门第 6 章", §6.7
    Column Parallel Linear: W1[D, F] -> W1[D, F/TP] on each device.)"""
    k, n = W.shape
    if n % t:
        raise ValueError("t must divide the column count")
    w = n // t
    out = np.empty((t, k, w), dtype=W.dtype)
    for r in range(t):
        out[r] = W[:, r * w:(r + 1) * w]
    return out


def shard_rows(W: np.ndarray, t: int) -> np.ndarray:
    """Row-parallel split: shard r holds W[r*k/t:(r+1)*k/t, :] (shape [k/t, n]).
    ("张量并行与序列并行", §矩阵乘法的两种切法, the second identity; "Scaling Book 入门第 6 章", §6.7
    Row Parallel Linear: W2[F, D] -> W2[F/TP, D].)"""
    k, n = W.shape
    if k % t:
        raise ValueError("t must divide the row count")
    h = k // t
    out = np.empty((t, h, n), dtype=W.dtype)
    for r in range(t):
        out[r] = W[r * h:(r + 1) * h, :]
    return out


def shard_gate_up(W_gate: np.ndarray, W_up: np.ndarray, t: int) -> np.ndarray:
    """Fused SwiGLU gate|up layout: shard r holds [W_gate[:, F-range r] | W_up[:, F-range r]],
    shape [h, 2F/t], so its gate and up columns cover the same F indices
    ("张量并行与序列并行", §MLP：先列后行，只通信一次, the SwiGLU paragraph).
    Reading: inside a rank's block the gate columns come first, then the up columns (naming order)."""
    h, F = W_gate.shape
    if W_up.shape != (h, F) or F % t:
        raise ValueError("gate/up shapes differ or t does not divide F")
    f = F // t
    out = np.empty((t, h, 2 * f), dtype=W_gate.dtype)
    for r in range(t):
        out[r, :, :f] = W_gate[:, r * f:(r + 1) * f]
        out[r, :, f:] = W_up[:, r * f:(r + 1) * f]
    return out


def kv_heads_of_rank(r: int, t: int, n_kv: int) -> list[int]:
    """KV heads placed on rank r ("张量并行与序列并行", §GQA：KV 头比 query 头少).
    t <= n_kv and t | n_kv: n_kv/t consecutive heads per rank. n_kv < t <= n_h: each KV head is
    replicated; reading: rank r takes head floor(r * n_kv / t), i.e. each head on t/n_kv consecutive
    ranks (the page says "replicate", not which rank gets which copy)."""
    if t <= n_kv:
        per = n_kv // t
        return list(range(r * per, (r + 1) * per))
    return [(r * n_kv) // t]


def qkv_validate(n_h: int, n_kv: int, t: int) -> None:
    """TP degree constraints: t divides n_h (Megatron's check, pufanyi.com "ml-revisit-infra",
    §Tensor Parallel; "张量并行与序列并行", §注意力 last bullet); for KV, t | n_kv or n_kv | t."""
    if n_h % t:
        raise ValueError("t must divide n_h")
    if n_h % n_kv:
        raise ValueError("n_kv must divide n_h")
    if t <= n_kv:
        if n_kv % t:
            raise ValueError("t must divide n_kv when t <= n_kv")
    elif t % n_kv:
        raise ValueError("n_kv must divide t when KV heads are replicated")


def shard_qkv(Wq: np.ndarray, Wk: np.ndarray, Wv: np.ndarray, n_h: int, n_kv: int, d_h: int, t: int) -> np.ndarray:
    """Rank-grouped fused QKV layout: shard r holds [its Q heads | its K heads | its V heads], each
    head d_h contiguous columns, heads ascending ("张量并行与序列并行", §注意力：按头切, fused-QKV bullet:
    group by TP rank first, then concatenate; an equal split of [Q|K|V] is wrong)."""
    qkv_validate(n_h, n_kv, t)
    h = Wq.shape[0]
    if Wq.shape != (h, n_h * d_h) or Wk.shape != (h, n_kv * d_h) or Wv.shape != (h, n_kv * d_h):
        raise ValueError("QKV weight shapes do not match the head counts")
    q_per = n_h // t
    kv_per = len(kv_heads_of_rank(0, t, n_kv))
    width = (q_per + 2 * kv_per) * d_h
    out = np.empty((t, h, width), dtype=Wq.dtype)
    for r in range(t):
        col = 0
        for head in range(r * q_per, (r + 1) * q_per):
            out[r, :, col:col + d_h] = Wq[:, head * d_h:(head + 1) * d_h]
            col += d_h
        for head in kv_heads_of_rank(r, t, n_kv):
            out[r, :, col:col + d_h] = Wk[:, head * d_h:(head + 1) * d_h]
            col += d_h
        for head in kv_heads_of_rank(r, t, n_kv):
            out[r, :, col:col + d_h] = Wv[:, head * d_h:(head + 1) * d_h]
            col += d_h
        assert col == width
    return out
