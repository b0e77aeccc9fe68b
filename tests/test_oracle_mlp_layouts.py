"""Pins of the oracle's layouts, activations, MLP, sharded-matmul cases and layer (CPU only).

What fixes the expected values: textbook values of the normal CDF (GeLU = x * Phi(x)) and of the
logistic function, pure-Python brute force on tiny shapes, numpy's own split/concatenate, the
block-matrix identity, and the page statements each test names.
"""
import math

import numpy as np
import pytest

from oracle import cases, layer, layouts, mlp
from synthetic import tiny_mlp, to_f64


# ------------------------------------------------------------------------------------ activations
def test_gelu_textbook_values():
    # Phi(1) = 0.841344746068543, Phi(2) = 0.977249868051821 (standard normal CDF tables)
    assert mlp.gelu(1.0) == pytest.approx(0.841344746068543, abs=1e-14)
    assert mlp.gelu(2.0) == pytest.approx(2 * 0.977249868051821, abs=1e-14)
    assert mlp.gelu(0.0) == 0.0
    # the page's counter-example: GeLU(XA1 + XA2) != GeLU(XA1) + GeLU(XA2) ("张量并行与序列并行", §MLP)
    assert round(float(mlp.gelu(2.0)), 4) == 1.9545
    assert round(float(2 * mlp.gelu(1.0)), 4) == 1.6827


def test_gelu_symmetry_and_tanh_variant():
    x = np.linspace(-6, 6, 1001)
    assert np.allclose(mlp.gelu(x) - mlp.gelu(-x), x, atol=1e-14)
    assert np.max(np.abs(mlp.gelu_tanh(x) - mlp.gelu(x))) < 1e-3


def test_silu_values():
    assert mlp.silu(0.0) == 0.0
    assert mlp.silu(1.0) == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), abs=1e-15)
    assert mlp.silu(1.0) == pytest.approx(0.7310585786300049, abs=1e-15)
    x = np.linspace(-8, 8, 101)
    assert np.allclose(mlp.silu(x) - mlp.silu(-x), x, atol=1e-13)


# ------------------------------------------------------------------------------------ brute force MLP
def _bf_mlp(X, A, B, act):
    N, h = X.shape
    F = A.shape[1]
    H = [[sum(X[n][k] * A[k][f] for k in range(h)) for f in range(F)] for n in range(N)]
    if act == "gelu":
        Z = [[0.5 * v * (1 + math.erf(v / math.sqrt(2))) for v in row] for row in H]
    elif act == "swiglu":
        f2 = F // 2
        Z = [[(row[j] / (1 + math.exp(-row[j]))) * row[f2 + j] for j in range(f2)] for row in H]
    else:
        Z = H
    Fz = len(Z[0])
    return np.array([[sum(Z[n][f] * B[f][m] for f in range(Fz)) for m in range(B.shape[1])] for n in range(N)])


@pytest.mark.parametrize("act", ["gelu", "swiglu", "none"])
def test_mlp_unsharded_brute_force(act):
    g = np.random.default_rng(1)
    X = g.standard_normal((3, 5))
    A = g.standard_normal((5, 8))
    B = g.standard_normal((8 if act != "swiglu" else 4, 2))
    ref = _bf_mlp(X, A, B, act)
    assert np.allclose(mlp.mlp_unsharded(X, A, B, act), ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("act,t", [("gelu", 1), ("gelu", 2), ("gelu", 4), ("swiglu", 2), ("swiglu", 4), ("gelu_tanh", 4)])
def test_block_identity_sum_of_partials_is_unsharded(act, t):
    g = np.random.default_rng(t)
    N, h, F = 6, 8, 16
    X = g.standard_normal((N, h))
    if act == "swiglu":
        Wg, Wu = g.standard_normal((h, F)), g.standard_normal((h, F))
        W_in = np.concatenate([Wg, Wu], axis=1)
        shards_in = layouts.shard_gate_up(Wg, Wu, t)
    else:
        W_in = g.standard_normal((h, F))
        shards_in = layouts.shard_cols(W_in, t)
    W_out = g.standard_normal((F, h))
    Y = mlp.mlp_unsharded(X, W_in, W_out, act)
    U = mlp.mlp_partials(X, list(shards_in), list(layouts.shard_rows(W_out, t)), act)
    assert len(U) == t and all(u.shape == Y.shape for u in U)
    assert np.max(np.abs(sum(U) - Y)) <= 1e-12 * np.max(np.abs(Y))


def test_row_first_split_needs_its_allreduce():
    # "张量并行与序列并行", §MLP: splitting A by rows makes XA a partial sum, so GeLU of the pieces
    # is wrong; for a linear map (no activation) the pieces do sum to the right answer.
    X, A, _ = tiny_mlp(seed=0)
    X, A = to_f64(X), to_f64(A)
    t = 2
    rows = list(layouts.shard_rows(A, t))
    good = mlp.activate(mlp.matmul(X, A), "gelu")
    bad = mlp.row_first_mlp(X, rows, "gelu")
    assert np.max(np.abs(bad - good)) > 1e-2 * np.max(np.abs(good))
    assert np.allclose(mlp.row_first_mlp(X, rows, "none"), mlp.matmul(X, A), rtol=1e-12, atol=1e-12)


def test_tiny_config_gelu_of_sum_differs_from_sum_of_gelu():
    X, A, _ = tiny_mlp(seed=0)
    X, A = to_f64(X), to_f64(A)
    A1, A2 = A[:128], A[128:]
    X1, X2 = X[:, :128], X[:, 128:]
    lhs = mlp.gelu(X1 @ A1 + X2 @ A2)
    rhs = mlp.gelu(X1 @ A1) + mlp.gelu(X2 @ A2)
    assert not np.allclose(lhs, rhs, rtol=1e-2, atol=1e-3)


def test_swiglu_mispaired_layout_fails():
    # Splitting the fused [W_gate | W_up] into equal column blocks (no regrouping) pairs the wrong
    # columns ("张量并行与序列并行", §MLP, SwiGLU paragraph).
    g = np.random.default_rng(3)
    N, h, F, t = 4, 8, 16, 4
    X = g.standard_normal((N, h))
    Wg, Wu, Wd = g.standard_normal((h, F)), g.standard_normal((h, F)), g.standard_normal((F, h))
    Y = mlp.mlp_unsharded(X, np.concatenate([Wg, Wu], 1), Wd, "swiglu")
    right = sum(mlp.mlp_partials(X, list(layouts.shard_gate_up(Wg, Wu, t)), list(layouts.shard_rows(Wd, t)), "swiglu"))
    wrong = sum(mlp.mlp_partials(X, list(layouts.shard_cols(np.concatenate([Wg, Wu], 1), t)), list(layouts.shard_rows(Wd, t)), "swiglu"))
    assert np.allclose(right, Y, rtol=1e-12, atol=1e-12)
    assert np.max(np.abs(wrong - Y)) > 0.05 * np.max(np.abs(Y))


# ------------------------------------------------------------------------------------ layouts
@pytest.mark.parametrize("t", [1, 2, 4, 8])
def test_shard_cols_rows_match_numpy_split(t):
    W = np.arange(16 * 24, dtype=np.uint16).reshape(16, 24)
    assert np.array_equal(layouts.shard_cols(W, t), np.stack(np.split(W, t, axis=1)))
    assert np.array_equal(layouts.shard_rows(W, t), np.stack(np.split(W, t, axis=0)))


def test_gate_up_blocks_cover_same_F_range():
    h, F, t = 3, 8, 4
    Wg = np.arange(h * F).reshape(h, F) * 2          # even numbers: gate
    Wu = np.arange(h * F).reshape(h, F) * 2 + 1      # odd numbers: up
    out = layouts.shard_gate_up(Wg, Wu, t)
    f = F // t
    for r in range(t):
        assert np.array_equal(out[r][:, :f], Wg[:, r * f:(r + 1) * f])
        assert np.array_equal(out[r][:, f:], Wu[:, r * f:(r + 1) * f])
        assert np.array_equal(out[r][:, :f] + 1, out[r][:, f:])    # same F indices, paired


def _qkv_weights(h, n_h, n_kv, d_h):
    # Q heads tagged 1000+head, K heads 2000+head, V heads 3000+head (d_h columns each)
    Wq = np.repeat(1000 + np.arange(n_h), d_h)[None, :].repeat(h, 0)
    Wk = np.repeat(2000 + np.arange(n_kv), d_h)[None, :].repeat(h, 0)
    Wv = np.repeat(3000 + np.arange(n_kv), d_h)[None, :].repeat(h, 0)
    return Wq, Wk, Wv


def test_qkv_t1_is_plain_concatenation():
    Wq, Wk, Wv = _qkv_weights(2, 8, 2, 4)
    out = layouts.shard_qkv(Wq, Wk, Wv, 8, 2, 4, 1)
    assert np.array_equal(out[0], np.concatenate([Wq, Wk, Wv], axis=1))


def test_qkv_naive_equal_split_is_wrong():
    # "张量并行与序列并行", §注意力: an equal column split of the fused [Q|K|V] gives the first rank
    # only Q heads and the last rank all of V.
    n_h, n_kv, d_h, t = 8, 2, 4, 2
    Wq, Wk, Wv = _qkv_weights(1, n_h, n_kv, d_h)
    fused = np.concatenate([Wq, Wk, Wv], axis=1)
    naive = np.split(fused, t, axis=1)
    assert set(np.unique(naive[0] // 1000)) == {1}
    assert set(np.unique(naive[-1][:, -n_kv * d_h:] // 1000)) == {3}
    grouped = layouts.shard_qkv(Wq, Wk, Wv, n_h, n_kv, d_h, t)
    for r in range(t):
        kinds = grouped[r][0] // 1000
        assert list(np.unique(kinds)) == [1, 2, 3]
    assert not np.array_equal(np.stack(naive), grouped)


@pytest.mark.parametrize("n_h,n_kv,t", [(8, 8, 8), (64, 8, 8), (32, 8, 4), (32, 8, 16), (32, 8, 32), (8, 2, 4), (8, 4, 2)])
def test_gqa_query_heads_meet_their_kv_head(n_h, n_kv, t):
    # "张量并行与序列并行", §GQA: a group of query heads and the KV head it shares must be on the same
    # rank; t <= n_kv splits KV heads, n_kv < t <= n_h replicates them.
    d_h = 2
    Wq, Wk, Wv = _qkv_weights(1, n_h, n_kv, d_h)
    out = layouts.shard_qkv(Wq, Wk, Wv, n_h, n_kv, d_h, t)
    group = n_h // n_kv
    for r in range(t):
        row = out[r][0][::d_h]
        q = [v - 1000 for v in row if v // 1000 == 1]
        k = [v - 2000 for v in row if v // 1000 == 2]
        v_ = [v - 3000 for v in row if v // 1000 == 3]
        assert q == list(range(r * n_h // t, (r + 1) * n_h // t))
        assert k == v_ and {qh // group for qh in q} <= set(k)
        assert len(k) == max(1, n_kv // t)


@pytest.mark.parametrize("n_h,n_kv,t", [(8, 2, 3), (6, 2, 4), (8, 4, 16)])
def test_qkv_rejects_bad_tp_degree(n_h, n_kv, t):
    Wq, Wk, Wv = _qkv_weights(1, n_h, n_kv, 2)
    with pytest.raises(ValueError):
        layouts.shard_qkv(Wq, Wk, Wv, n_h, n_kv, 2, t)


# ------------------------------------------------------------------------------------ cases
def _case_inputs(case_id, t, B=8, D=12, F=16, seed=0):
    g = np.random.default_rng(seed + case_id)
    X, W = g.standard_normal((B, D)), g.standard_normal((D, F))
    if case_id == 1:
        x, w = np.split(X, t, 0), [W] * t
    elif case_id == 2:
        x, w = np.split(X, t, 1), [W] * t
    elif case_id == 3:
        x, w = np.split(X, t, 1), np.split(W, t, 0)
    else:
        x, w = np.split(X, t, 0), np.split(W, t, 1)
    return X, W, x, w


@pytest.mark.parametrize("case_id", [1, 2, 3, 4])
@pytest.mark.parametrize("t", [1, 2, 4])
def test_every_case_strategy_gives_the_logical_product(case_id, t):
    X, W, x, w = _case_inputs(case_id, t)
    for strategy in cases.STRATEGIES[case_id]:
        outs = cases.run(case_id, strategy, x, w)
        layout = cases.output_layout(case_id, strategy)
        if layout == "replicated":
            assert all(np.array_equal(o, outs[0]) for o in outs)
        assert np.allclose(cases.to_logical(outs, layout), X @ W, rtol=1e-12, atol=1e-12)


def test_case4_local_product_gives_only_diagonal_blocks():
    t = 2
    X, W, x, w = _case_inputs(4, t)
    C = X @ W
    naive = cases.case4_naive(x, w)
    b, f = X.shape[0] // t, W.shape[1] // t
    for i in range(t):
        assert np.allclose(naive[i], C[i * b:(i + 1) * b, i * f:(i + 1) * f])
    assert naive[0].shape != C.shape


def test_case2_choice_follows_problem4_rule():
    # Problem 4 orientation: gather Y[D, F] vs AllReduce Z[B, F] -> AllReduce when D > 2B.
    B, F = 128, 1024
    assert cases.case2_choice(gathered_elems=(2 * B + 8) * F, output_elems=B * F) == "allreduce"
    assert cases.case2_choice(gathered_elems=(2 * B - 8) * F, output_elems=B * F) == "allgather"
    # the config's orientation: X[8192, 8192/4] gathered vs C[8192, 28672] reduced -> gather X
    assert cases.case2_choice(8192 * 8192, 8192 * 28672) == "allgather"


# ------------------------------------------------------------------------------------ layer
def _tiny_layer(seed=0, N=4, h=16, n_h=4, n_kv=2, d_h=4, F=8, t=2):
    g = np.random.default_rng(seed)
    X = g.standard_normal((N, h))
    O = g.standard_normal((N, n_h * d_h))
    Wq, Wk, Wv = g.standard_normal((h, n_h * d_h)), g.standard_normal((h, n_kv * d_h)), g.standard_normal((h, n_kv * d_h))
    Wo = g.standard_normal((n_h * d_h, h))
    Wg, Wu, Wd = g.standard_normal((h, F)), g.standard_normal((h, F)), g.standard_normal((F, h))
    sh = dict(
        O=np.split(O, t, 1), qkv=list(layouts.shard_qkv(Wq, Wk, Wv, n_h, n_kv, d_h, t)),
        o=list(layouts.shard_rows(Wo, t)), gu=list(layouts.shard_gate_up(Wg, Wu, t)), d=list(layouts.shard_rows(Wd, t)))
    return X, O, Wq, Wk, Wv, Wo, Wg, Wu, Wd, sh


def test_layer_matches_unsharded_definition():
    X, O, Wq, Wk, Wv, Wo, Wg, Wu, Wd, sh = _tiny_layer()
    out = layer.layer_forward(X, sh["O"], sh["qkv"], sh["o"], sh["gu"], sh["d"])
    attn = O @ Wo
    h1 = X + attn
    from oracle.bf16 import round_to_bf16_f64
    y = h1 + mlp.mlp_unsharded(round_to_bf16_f64(h1), np.concatenate([Wg, Wu], 1), Wd, "swiglu")
    assert np.allclose(out["attn"], attn, rtol=1e-12, atol=1e-12)
    assert np.allclose(out["y"], y, rtol=1e-12, atol=1e-12)
    # each shard's QKV output is its own heads' columns of the full Q, K and V projections
    Q, K, V = X @ Wq, X @ Wk, X @ Wv
    d = 4
    for r in range(2):
        want = np.concatenate([Q[:, 2 * r * d:(2 * r + 2) * d], K[:, r * d:(r + 1) * d], V[:, r * d:(r + 1) * d]], 1)
        assert np.allclose(out["qkv"][r], want, rtol=1e-12, atol=1e-12)


def test_layer_with_zero_projections_is_identity():
    X, O, *_, sh = _tiny_layer(seed=2)
    zo = [np.zeros_like(w) for w in sh["o"]]
    zd = [np.zeros_like(w) for w in sh["d"]]
    out = layer.layer_forward(X, sh["O"], sh["qkv"], zo, sh["gu"], zd)
    assert np.array_equal(out["y"], X)


def test_layer_rows_are_independent():
    X, O, *_, sh = _tiny_layer(seed=4)
    full = layer.layer_forward(X, sh["O"], sh["qkv"], sh["o"], sh["gu"], sh["d"])
    rows = np.array([3, 1])
    part = layer.layer_forward(X, sh["O"], sh["qkv"], sh["o"], sh["gu"], sh["d"], rows=rows)
    assert np.allclose(part["y"], full["y"][rows], rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("act,t", [("gelu", 2), ("swiglu", 4)])
def test_sp_mlp_equals_pure_tp_rows(act, t):
    # "张量并行与序列并行", §序列并行: TP+SP replaces the entry f by an AllGather and the exit g by a
    # ReduceScatter along s; the result is the same tensor, each shard keeping its own block of tokens.
    g = np.random.default_rng(11)
    N, h, F = 8, 6, 8
    X = g.standard_normal((N, h))
    if act == "swiglu":
        Wg, Wu = g.standard_normal((h, F)), g.standard_normal((h, F))
        W_in, shards_in = np.concatenate([Wg, Wu], 1), list(layouts.shard_gate_up(Wg, Wu, t))
    else:
        W_in = g.standard_normal((h, F))
        shards_in = list(layouts.shard_cols(W_in, t))
    W_out = g.standard_normal((F, h))
    Y = mlp.mlp_unsharded(X, W_in, W_out, act)
    out = mlp.sp_mlp(np.split(X, t, axis=0), shards_in, list(layouts.shard_rows(W_out, t)), act)
    assert len(out) == t and all(o.shape == (N // t, h) for o in out)
    assert np.allclose(np.concatenate(out, 0), Y, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------------------------ backward
@pytest.mark.parametrize("act,t", [("gelu", 2), ("gelu_tanh", 2), ("swiglu", 2), ("none", 4)])
def test_mlp_backward_against_finite_differences(act, t):
    # Central differences of L(X, W) = sum(MLP(X) * dY) pin every gradient formula independently.
    g = np.random.default_rng(21)
    N, h, F = 3, 4, 8
    X, dY = g.standard_normal((N, h)), g.standard_normal((N, h))
    if act == "swiglu":
        Wg, Wu = g.standard_normal((h, F)) * 0.5, g.standard_normal((h, F)) * 0.5
        W_in, shards_in = np.concatenate([Wg, Wu], 1), list(layouts.shard_gate_up(Wg, Wu, t))
    else:
        W_in = g.standard_normal((h, F)) * 0.5
        shards_in = list(layouts.shard_cols(W_in, t))
    W_out = g.standard_normal((F, h)) * 0.5
    shards_out = list(layouts.shard_rows(W_out, t))
    grads = mlp.mlp_backward(X, shards_in, shards_out, dY, act)
    loss = lambda X_, Win_, Wout_: float(np.sum(mlp.mlp_unsharded(X_, Win_, Wout_, act) * dY))  # noqa: E731
    eps = 1e-6

    def num(f, A):
        G = np.zeros_like(A)
        for idx in np.ndindex(A.shape):
            Ap, Am = A.copy(), A.copy()
            Ap[idx] += eps
            Am[idx] -= eps
            G[idx] = (f(Ap) - f(Am)) / (2 * eps)
        return G

    assert np.allclose(grads["dX"], num(lambda A: loss(A, W_in, W_out), X), rtol=1e-5, atol=1e-6)
    assert np.allclose(np.concatenate(grads["dW_out"], 0), num(lambda A: loss(X, W_in, A), W_out), rtol=1e-5, atol=1e-6)
    dWin = num(lambda A: loss(X, A, W_out), W_in)
    f = F // t
    for r in range(t):
        if act == "swiglu":     # shard r's block is [gate cols r | up cols r]
            want = np.concatenate([dWin[:, r * f:(r + 1) * f], dWin[:, F + r * f:F + (r + 1) * f]], 1)
        else:
            want = dWin[:, r * f:(r + 1) * f]
        assert np.allclose(grads["dW_in"][r], want, rtol=1e-5, atol=1e-6)


def test_column_backward_needs_the_sum_over_shards():
    # "张量并行与序列并行", §矩阵乘法的两种切法: each shard's dX is only a partial sum; one shard's alone is wrong.
    g = np.random.default_rng(5)
    X, dY = g.standard_normal((4, 6)), g.standard_normal((4, 6))
    W_in, W_out = g.standard_normal((6, 8)), g.standard_normal((8, 6))
    grads = mlp.mlp_backward(X, list(layouts.shard_cols(W_in, 2)), list(layouts.shard_rows(W_out, 2)), dY, "gelu")
    full = mlp.mlp_backward(X, [W_in], [W_out], dY, "gelu")
    assert np.allclose(grads["dX"], full["dX"], rtol=1e-12, atol=1e-12)
    assert not np.allclose(grads["dX_partials"][0], full["dX"], rtol=1e-2, atol=1e-2)
