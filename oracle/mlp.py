"""The tensor-parallel MLP in fp64 (test infrastructure).

Sources:
  * "张量并行与序列并行", §MLP：先列后行，只通信一次: Z = GeLU(X A), Y = Z B with A [h, F] split by
    columns and B [F, h] by rows; shard i computes Z_i = GeLU(X A_i) locally (GeLU is element-wise)
    and the partial Z_i B_i of full shape [N, h]; Y = sum_i Z_i B_i after one AllReduce. SwiGLU:
    Y = (SiLU(X W_gate) * X W_up) W_down with gate and up split over the same F range.
  * pufanyi.com "ml-revisit-infra", §Tensor Parallel: MLP(x) = sigma(X W1) W2, W1 column-wise, W2 row-wise.
  * "Scaling Book 入门第 6 章", §6.2 block-matrix identity; §6.7 Column/Row Parallel Linear.

Readings: GeLU is the exact erf form (the pages do not say which); a tanh variant is provided.
SiLU(x) = x / (1 + e^-x). GEMMs sum exactly-widened bf16 inputs in float64 (numpy matmul); the
"device model" variant additionally rounds the activation Z to bf16 before the second GEMM, as a
device holding bf16 activations does (the pages keep activations in bf16, §预备).
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf

from .bf16 import round_to_bf16_f64

ACTS = ("none", "gelu", "gelu_tanh", "swiglu")


def gelu(x):
    """GeLU(x) = x * Phi(x) = x/2 * (1 + erf(x / sqrt 2))."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def gelu_tanh(x):
    """The tanh approximation of GeLU: x/2 * (1 + tanh(sqrt(2/pi) * (x + 0.044715 x^3)))."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))


def silu(x):
    """SiLU(x) = x * sigmoid(x) = x / (1 + e^-x)."""
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def activate(H, act: str):
    """Element-wise activation of the column GEMM's output H. For "swiglu" H = [gate | up] along the
    last axis (equal halves) and the result is SiLU(gate) * up."""
    if act == "none":
        return np.asarray(H, dtype=np.float64)
    if act == "gelu":
        return gelu(H)
    if act == "gelu_tanh":
        return gelu_tanh(H)
    if act == "swiglu":
        f = H.shape[-1] // 2
        return silu(H[..., :f]) * H[..., f:]
    raise ValueError(act)


def matmul(A, B):
    """fp64 product of exactly-widened operands (a library matmul used as one step)."""
    return np.asarray(A, dtype=np.float64) @ np.asarray(B, dtype=np.float64)


def mlp_unsharded(X, W_in, W_out, act: str):
    """Y = act(X W_in) W_out on the whole (unsharded) matrices. For "swiglu", W_in = [W_gate | W_up]
    ([h, 2F]) and act pairs column j of the gate half with column j of the up half."""
    return matmul(activate(matmul(X, W_in), act), W_out)


def column_linear(X, W_in_shards, act: str, device_model: bool = False):
    """Column-parallel layer: shard i computes Z_i = act(X W_in_i) from the full X, with no
    communication. W_in_shards[i] is [h, F/t] (or [h, 2F/t] = [gate_i | up_i] for "swiglu")."""
    Z = [activate(matmul(X, W), act) for W in W_in_shards]
    if device_model:
        Z = [round_to_bf16_f64(z) for z in Z]
    return Z


def row_linear(Z_shards, W_out_shards):
    """Row-parallel layer: shard i computes the full-shape partial sum U_i = Z_i W_out_i; the true
    output is sum_i U_i and needs one AllReduce (or a ReduceScatter)."""
    return [matmul(Z, W) for Z, W in zip(Z_shards, W_out_shards)]


def mlp_partials(X, W_in_shards, W_out_shards, act: str, device_model: bool = False):
    """The t unreduced partials {U} of the tensor-parallel MLP."""
    return row_linear(column_linear(X, W_in_shards, act, device_model), W_out_shards)


def row_first_mlp(X, A_row_shards, act: str):
    """What the row-first split would compute without its extra AllReduce: sum_i act(X_i A_i)
    (the page's counter-example, act(XA1 + XA2) != act(XA1) + act(XA2)). X is split by columns to
    match A's row split."""
    t = len(A_row_shards)
    Xs = np.split(np.asarray(X, dtype=np.float64), t, axis=1)
    return sum(activate(matmul(x, a), act) for x, a in zip(Xs, A_row_shards))


def sp_mlp(x_shards, W_in_shards, W_out_shards, act: str, device_model: bool = False):
    """The MLP under tensor + sequence parallelism ("张量并行与序列并行", §序列并行：把剩下的激活也切开): each
    shard holds its own block of tokens; the entry g gathers them along s (AllGather), the column and
    row layers run as in pure TP, and the exit g-bar sums and re-splits along s (ReduceScatter).
    Returns each shard's block of the output rows (fp64)."""
    from .collectives import all_gather, reduce_scatter_f64
    X = all_gather([np.asarray(x, dtype=np.float64) for x in x_shards], axis=0)[0]
    U = mlp_partials(X, W_in_shards, W_out_shards, act, device_model)
    return reduce_scatter_f64(U, axis=0)


def act_derivative(H, act: str):
    """d act / dH for the element-wise activations (SwiGLU is handled in mlp_backward):
    GeLU' = Phi(x) + x phi(x); the tanh form differentiated as written; SiLU' = s (1 + x (1 - s))."""
    x = np.asarray(H, dtype=np.float64)
    if act == "none":
        return np.ones_like(x)
    if act == "gelu":
        return 0.5 * (1.0 + erf(x / math.sqrt(2.0))) + x * np.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)
    if act == "gelu_tanh":
        c, a = math.sqrt(2.0 / math.pi), 0.044715
        th = np.tanh(c * (x + a * x ** 3))
        return 0.5 * (1.0 + th) + 0.5 * x * (1.0 - th * th) * c * (1.0 + 3.0 * a * x * x)
    raise ValueError(act)


def mlp_backward(X, W_in_shards, W_out_shards, dY, act: str):
    """Gradients of L = sum(Y * dY) for the tensor-parallel MLP, shard by shard
    ("张量并行与序列并行", §矩阵乘法的两种切法: column-parallel backward needs an AllReduce of dX, and
    row-parallel backward is local; pufanyi.com "ml-revisit-infra", §Tensor Parallel: dW_i = X^T dY_i,
    dX = sum_i dY_i W_i^T, and for the row split dW_i = X_i^T dY, dX_i = dY W_i^T).
    Returns dX (the sum over shards), its per-shard partials, dW_in / dW_out and the
    pre-activation gradient dH per shard."""
    X = np.asarray(X, dtype=np.float64)
    dY = np.asarray(dY, dtype=np.float64)
    out = {"dX_partials": [], "dW_in": [], "dW_out": [], "dH": []}
    for W_in, W_out in zip(W_in_shards, W_out_shards):
        W_in = np.asarray(W_in, dtype=np.float64)
        W_out = np.asarray(W_out, dtype=np.float64)
        H = X @ W_in
        Z = activate(H, act)
        dZ = dY @ W_out.T                       # row layer: input gradient, local
        out["dW_out"].append(Z.T @ dY)          # row layer: weight gradient, local
        if act == "swiglu":
            f = H.shape[1] // 2
            g, u = H[:, :f], H[:, f:]
            s = 1.0 / (1.0 + np.exp(-g))
            dH = np.concatenate([dZ * u * s * (1.0 + g * (1.0 - s)), dZ * g * s], axis=1)
        else:
            dH = dZ * act_derivative(H, act)
        out["dH"].append(dH)
        out["dW_in"].append(X.T @ dH)           # column layer: weight gradient, local
        out["dX_partials"].append(dH @ W_in.T)  # column layer: input gradient, a partial sum
    out["dX"] = sum(out["dX_partials"])
    return out
