"""GPU parity of the tensor-parallel MLP, the sharded-matmul cases and the tensor-parallel layer
against the oracle, through the C ABI: the tiny GeLU MLP in full, the Llama-3-8B SwiGLU MLP, the
four cases at B=D=8192, F=28672 and the Llama-3-70B-shaped layer at full size on sampled token rows
(the oracle computes those rows one by one), plus GPU-side properties that hold at any size
(AllReduce replicas identical, RS+AG == AR bit for bit, bf16 outputs = one rounding of fp32 outputs)."""
import numpy as np
import pytest
import torch

import synthetic as S
import tensor_sharded_matmul_b200 as tp
from gpu_util import GEMM_TOL, assert_close, cuda, f64, host_bits, same_bits
from oracle import cases as OCASE
from oracle import layer as OLAYER
from oracle import layouts as OL
from oracle import mlp as OM
from oracle.bf16 import f32_to_bf16_bits

pytestmark = pytest.mark.gpu


def _status_ok():
    st, site = tp.tp_device_status(1)
    assert st == tp.TP_OK, f"device wait site {site}"


def _mlp_device(X, w_in, w_down, N, h, F, t, act, mode):
    f = F // t
    z = torch.empty((t, N, f), dtype=torch.bfloat16, device="cuda")
    partials = [torch.empty((N, h), device="cuda") for _ in range(t)]
    if mode == tp.TP_OUT_RS:
        out = [torch.empty((N // t, h), device="cuda") for _ in range(t)]
    elif mode == tp.TP_OUT_PARTIALS:
        out = None
    else:
        out = [torch.empty((N, h), device="cuda") for _ in range(t)]
    tp.tp_mlp_fwd(X, N, h, F, t, act, w_in, w_down, z, partials, mode, out)
    torch.cuda.synchronize()
    _status_ok()
    return z, partials, out


# ---------------------------------------------------------------------------------- tiny GeLU MLP
def test_tiny_gelu_mlp_all_modes():
    N, h, F, t = 64, 256, 1024, 4
    X, A, B = S.tiny_mlp(seed=0)
    dX, dA, dB = cuda(X), cuda(A), cuda(B)
    w_in = torch.empty((t, h, F // t), dtype=torch.bfloat16, device="cuda")
    w_down = torch.empty((t, F // t, h), dtype=torch.bfloat16, device="cuda")
    tp.tp_shard_cols(dA, F, h, F, t, w_in)
    tp.tp_shard_rows(dB, h, F, h, t, w_down)
    torch.cuda.synchronize()
    Xf, Af, Bf = f64(X), f64(A), f64(B)
    U = OM.mlp_partials(Xf, list(OL.shard_cols(Af, t)), list(OL.shard_rows(Bf, t)), "gelu")
    Y = OM.mlp_unsharded(Xf, Af, Bf, "gelu")
    results = {}
    for mode in (tp.TP_OUT_PARTIALS, tp.TP_OUT_RS, tp.TP_OUT_AR, tp.TP_OUT_RS_AG):
        z, partials, out = _mlp_device(dX, w_in, w_down, N, h, F, t, tp.TP_ACT_GELU, mode)
        for r in range(t):
            assert_close(f64(partials[r]), U[r], GEMM_TOL, f"partial {r}")
        if mode == tp.TP_OUT_RS:
            for r in range(t):
                assert_close(f64(out[r]), Y[r * N // t:(r + 1) * N // t], GEMM_TOL, f"RS block {r}")
        elif mode != tp.TP_OUT_PARTIALS:
            for r in range(t):
                assert_close(f64(out[r]), Y, GEMM_TOL, f"replica {r}")
        results[mode] = (partials, out)
    # GPU-side: AR replicas identical; RS+AG == AR; RS blocks == AR rows (same ring order, same partials)
    ar = [host_bits(o) for o in results[tp.TP_OUT_AR][1]]
    rsag = [host_bits(o) for o in results[tp.TP_OUT_RS_AG][1]]
    rs = [host_bits(o) for o in results[tp.TP_OUT_RS][1]]
    for r in range(t):
        assert same_bits(ar[r], ar[0]) and same_bits(rsag[r], ar[0])
        assert same_bits(rs[r], ar[0][r * N // t:(r + 1) * N // t])


# ---------------------------------------------------------------------------------- shard-count extremes
@pytest.mark.parametrize("N,h,F,t,act", [
    (512, 256, 1024, 1, "gelu"),        # t = 1: no sharding, the ring is a single chunk
    (2048, 512, 4096, 16, "swiglu"),    # t = 16 (the maximum): 128-row chunks, single-CTA fused kernel
    (4096, 512, 4096, 16, "gelu"),      # t = 16: 256-row chunks, CTA pairs, deferred replica copies
])
def test_mlp_shard_count_extremes(N, h, F, t, act):
    d = S.Draw(N + F + t)
    f = F // t
    wn = 2 * f if act == "swiglu" else f
    X = d.normal((N, h), 1.0)
    w_in = d.normal((t, h, wn), 0.05)
    w_down = d.normal((t, f, h), 0.05)
    dX, dw_in, dw_down = cuda(X), cuda(w_in), cuda(w_down)
    a = tp.TP_ACT_SWIGLU if act == "swiglu" else tp.TP_ACT_GELU
    res = {mode: _mlp_device(dX, dw_in, dw_down, N, h, F, t, a, mode)
           for mode in (tp.TP_OUT_PARTIALS, tp.TP_OUT_RS, tp.TP_OUT_AR, tp.TP_OUT_RS_AG)}
    rows = np.arange(N) if N <= 512 else np.sort(np.random.default_rng(t).choice(N, 32, replace=False))
    U = OM.mlp_partials(f64(X)[rows], [f64(w) for w in w_in], [f64(w) for w in w_down], act)
    partials = res[tp.TP_OUT_PARTIALS][1]
    for r in range(t):
        assert_close(f64(partials[r])[rows], U[r], GEMM_TOL, f"partial {r}")
    Y = sum(U)
    ar = [host_bits(o) for o in res[tp.TP_OUT_AR][2]]
    rsag = [host_bits(o) for o in res[tp.TP_OUT_RS_AG][2]]
    rs = [host_bits(o) for o in res[tp.TP_OUT_RS][2]]
    assert_close(f64(res[tp.TP_OUT_AR][2][0])[rows], Y, GEMM_TOL, "AllReduce")
    for r in range(t):
        assert same_bits(ar[r], ar[0]) and same_bits(rsag[r], ar[0]), f"replica {r}"
        assert same_bits(rs[r], ar[0][r * N // t:(r + 1) * N // t]), f"RS block {r}"


def tile_rows(n_rows: int, tile: int = 128) -> np.ndarray:
    """One row from every `tile`-row block of the output, at an offset that moves across the block
    from tile to tile (so different TMEM lanes, epilogue warps and both CTAs of a pair are checked),
    plus the first and the last row."""
    rows = {0, n_rows - 1}
    for mt in range(n_rows // tile):
        rows.add(mt * tile + (mt * 53 + 17) % tile)
    return np.array(sorted(rows))


# ---------------------------------------------------------------------------------- Llama-3-8B SwiGLU MLP
@pytest.fixture(scope="module")
def llama8b():
    N, h, F, t = 4096, 4096, 14336, 8
    X, Wgu, Wd = S.llama8b_mlp(seed=0)
    dX, dWgu, dWd = cuda(X), cuda(Wgu), cuda(Wd)
    w_in = torch.empty((t, h, 2 * F // t), dtype=torch.bfloat16, device="cuda")
    w_down = torch.empty((t, F // t, h), dtype=torch.bfloat16, device="cuda")
    tp.tp_shard_gate_up(dWgu, 2 * F, dWgu.data_ptr() + 2 * F, 2 * F, h, F, t, w_in)
    tp.tp_shard_rows(dWd, h, F, h, t, w_down)
    torch.cuda.synchronize()
    del dWgu, dWd
    return dict(N=N, h=h, F=F, t=t, X=X, Wgu=Wgu, Wd=Wd, dX=dX, w_in=w_in, w_down=w_down)


def test_llama8b_swiglu_mlp_sampled_rows(llama8b):
    m = llama8b
    N, h, F, t = m["N"], m["h"], m["F"], m["t"]
    # the reducing modes fuse the row GEMM with its collective: the partials come from PARTIALS mode
    _, partials, _ = _mlp_device(m["dX"], m["w_in"], m["w_down"], N, h, F, t, tp.TP_ACT_SWIGLU, tp.TP_OUT_PARTIALS)
    z, _, out = _mlp_device(m["dX"], m["w_in"], m["w_down"], N, h, F, t, tp.TP_ACT_SWIGLU, tp.TP_OUT_RS_AG)
    # every 128-row m-tile of the output (both GEMMs, every pair tile and the fused kernel's half-width
    # last-round tiles: whole rows cover every n-tile)
    rows = tile_rows(N)
    Xr = f64(m["X"])[rows]
    Wg = m["Wgu"][:, :F].float().numpy()
    Wu = m["Wgu"][:, F:].float().numpy()
    Wd = m["Wd"].float().numpy()
    shards_in = list(OL.shard_gate_up(Wg, Wu, t))
    shards_down = list(OL.shard_rows(Wd, t))
    U = OM.mlp_partials(Xr, shards_in, shards_down, "swiglu")
    Y = sum(U)
    for r in (0, 3, 7):
        assert_close(f64(partials[r])[rows], U[r], GEMM_TOL, f"partial {r}")
    for s in range(t):
        assert_close(f64(out[s])[rows], Y, GEMM_TOL, f"replica {s}")
    # the activation workspace itself (Z_r = SiLU(X G_r) * X U_r) on the sampled rows
    Z0 = OM.column_linear(Xr, shards_in[:1], "swiglu")[0]
    assert_close(f64(z[0])[rows], Z0, GEMM_TOL, "Z_0")
    # block identity on the device: the ring sum of the GPU's own partials (unfused GEMM) is the fused
    # kernel's output bit for bit
    from oracle import collectives as OC
    ring = OC.reduce_scatter([host_bits(p) for p in partials], axis=0)
    for r in (0, 5):
        assert same_bits(host_bits(out[r])[r * N // t:(r + 1) * N // t], ring[r])


def test_llama8b_modes_agree_bitwise(llama8b):
    m = llama8b
    N, h, F, t = m["N"], m["h"], m["F"], m["t"]
    _, p1, ar = _mlp_device(m["dX"], m["w_in"], m["w_down"], N, h, F, t, tp.TP_ACT_SWIGLU, tp.TP_OUT_AR)
    _, p2, rsag = _mlp_device(m["dX"], m["w_in"], m["w_down"], N, h, F, t, tp.TP_ACT_SWIGLU, tp.TP_OUT_RS_AG)
    _, p3, rs = _mlp_device(m["dX"], m["w_in"], m["w_down"], N, h, F, t, tp.TP_ACT_SWIGLU, tp.TP_OUT_RS)
    a0 = host_bits(ar[0])
    for s in range(t):
        assert same_bits(host_bits(ar[s]), a0)
        assert same_bits(host_bits(rsag[s]), a0)
        assert same_bits(host_bits(rs[s]), a0[s * N // t:(s + 1) * N // t])


# ---------------------------------------------------------------------------------- sharded-matmul cases
def _case_shards(X, W, case_id, t):
    if case_id == 1:
        return list(X.chunk(t, 0)), [W] * t
    if case_id == 2:
        return list(X.chunk(t, 1)), [W] * t
    if case_id == 3:
        return list(X.chunk(t, 1)), list(W.chunk(t, 0))
    return list(X.chunk(t, 0)), list(W.chunk(t, 1))


def _out_shape(case_id, strategy, B, F, t):
    layout = OCASE.output_layout(case_id, OCASE.STRATEGIES[case_id][strategy])
    return {"rows": (B // t, F), "cols": (B, F // t), "replicated": (B, F)}[layout], layout


def _run_case(case_id, strategy, xs, ws, B, D, F, t, c_dtype):
    shape, layout = _out_shape(case_id, strategy, B, F, t)
    cdt = torch.float32 if c_dtype == tp.TP_F32 else torch.bfloat16
    c = [torch.empty(shape, dtype=cdt, device="cuda") for _ in range(t)]
    nbytes = tp.tp_sharded_matmul_ws_bytes(case_id, strategy, B, D, F, t)
    ws_buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device="cuda")
    tp.tp_sharded_matmul(case_id, strategy, xs, ws, B, D, F, t, c, c_dtype, ws_buf, nbytes)
    torch.cuda.synchronize()
    _status_ok()
    return c, layout


# Two shapes: with (512, 384, 768) case 2 AllGather materialises its gather (D/t = 96 is not whole
# 64-wide k-blocks) while case 4 reads X's row pieces and W's column pieces in place; with
# (384, 512, 640) it is the other way round (D/t = 128; B/t = 96, F/t = 160).
@pytest.mark.parametrize("shape", [(512, 384, 768), (384, 512, 640)])
@pytest.mark.parametrize("case_id,strategy", [(1, 0), (2, 0), (2, 1), (3, 0), (3, 1), (3, 2), (4, 0), (4, 1)])
def test_cases_small_against_oracle(case_id, strategy, shape):
    (B, D, F), t = shape, 4
    X, W = S.case_operands(seed=case_id, B=B, D=D, F=F)
    xs, ws = _case_shards(X, W, case_id, t)
    dxs = [cuda(x) for x in xs]
    dws = [cuda(w) for w in ws]
    ref = OCASE.run(case_id, OCASE.STRATEGIES[case_id][strategy], [f64(x) for x in xs], [f64(w) for w in ws])
    c32, layout = _run_case(case_id, strategy, dxs, dws, B, D, F, t, tp.TP_F32)
    c16, _ = _run_case(case_id, strategy, dxs, dws, B, D, F, t, tp.TP_BF16)
    for i in range(t):
        assert_close(f64(c32[i]), ref[i], GEMM_TOL, f"shard {i}")
        assert_close(f64(c16[i]), ref[i], GEMM_TOL, f"shard {i} bf16")
    logical = OCASE.to_logical([f64(c) for c in c32], layout)
    assert_close(logical, f64(X) @ f64(W), GEMM_TOL, "logical C")
    if layout == "replicated":
        for i in range(t):
            assert same_bits(host_bits(c32[i]), host_bits(c32[0]))
    if case_id in (2, 3) and not (case_id == 2 and strategy == 0):
        # reduced outputs: the bf16 result is the fp32 ring sum rounded once
        for i in range(t):
            assert np.array_equal(host_bits(c16[i]), f32_to_bf16_bits(host_bits(c32[i])))


@pytest.mark.parametrize("case_id,strategy", [(2, 0), (4, 0), (4, 1)])
def test_gather_in_place_equals_gather_then_gemm(case_id, strategy):
    """Reading the gathered operand's pieces where they lie gives the same bits as the AllGather into
    a buffer followed by the plain grouped GEMM: the same MMA sequence runs on the same values."""
    B, D, F, t = 1024, 512, 1536, 4
    assert tp.tp_sharded_matmul_ws_bytes(case_id, strategy, B, D, F, t) == 0
    X, W = S.case_operands(seed=40 + case_id + strategy, B=B, D=D, F=F)
    xs, ws = _case_shards(X, W, case_id, t)
    dxs = [cuda(x) for x in xs]
    dws = [cuda(w) for w in ws]
    c, _ = _run_case(case_id, strategy, dxs, dws, B, D, F, t, tp.TP_F32)
    if case_id == 2:       # X gathered along D, every shard computes the full C
        g = [torch.empty((B, D), dtype=torch.bfloat16, device="cuda") for _ in range(t)]
        tp.tp_all_gather(dxs, g, B, D, 1, tp.TP_BF16, t)
        ref = [torch.empty((B, F), device="cuda") for _ in range(t)]
        tp.tp_grouped_gemm(t, g, dws, ref, B, F, D, tp.TP_ACT_NONE, tp.TP_F32)
    elif strategy == 0:    # X gathered along B, shard i's columns of W
        g = [torch.empty((B, D), dtype=torch.bfloat16, device="cuda") for _ in range(t)]
        tp.tp_all_gather(dxs, g, B, D, 0, tp.TP_BF16, t)
        ref = [torch.empty((B, F // t), device="cuda") for _ in range(t)]
        tp.tp_grouped_gemm(t, g, dws, ref, B, F // t, D, tp.TP_ACT_NONE, tp.TP_F32)
    else:                  # W gathered along F, shard i's rows of X
        g = [torch.empty((D, F), dtype=torch.bfloat16, device="cuda") for _ in range(t)]
        tp.tp_all_gather(dws, g, D, F, 1, tp.TP_BF16, t)
        ref = [torch.empty((B // t, F), device="cuda") for _ in range(t)]
        tp.tp_grouped_gemm(t, dxs, g, ref, B // t, F, D, tp.TP_ACT_NONE, tp.TP_F32)
    torch.cuda.synchronize()
    _status_ok()
    for i in range(t):
        assert torch.equal(c[i], ref[i]), f"shard {i}"


@pytest.fixture(scope="module")
def case_operands_full():
    """The full-size case operands and the oracle's fp64 rows of the logical C = X W for one row of
    every 128-row block (whole rows: all F columns), computed once for every strategy."""
    X, W = S.case_operands(seed=0)
    rows = tile_rows(X.shape[0])
    ref = OM.matmul(f64(X[torch.from_numpy(rows)]), f64(W))
    return X, W, rows, ref


@pytest.mark.parametrize("case_id,strategy", [(1, 0), (2, 0), (2, 1), (3, 0), (3, 1), (3, 2), (4, 0), (4, 1)])
def test_cases_full_size_sampled(case_operands_full, case_id, strategy):
    B, D, F, t = 8192, 8192, 28672, 4
    X, W, rows, ref = case_operands_full
    xs, ws = _case_shards(X, W, case_id, t)
    dxs = [cuda(x) for x in xs]
    dws = [cuda(w) for w in ws] if case_id != 1 and case_id != 2 else [cuda(W)] * t
    c, layout = _run_case(case_id, strategy, dxs, dws, B, D, F, t, tp.TP_F32)
    # whole logical rows, one from every 128-row m-tile of the output: every m-tile and n-tile of every
    # shard's output is compared (replicated outputs: the row's replica rotates over the shards)
    got = np.empty_like(ref)
    for a, r in enumerate(rows):
        r = int(r)
        if layout == "rows":
            got[a] = f64(c[r // (B // t)][r % (B // t)])
        elif layout == "cols":
            got[a] = np.concatenate([f64(c[i][r]) for i in range(t)])
        else:
            got[a] = f64(c[a % t][r])
    assert_close(got, ref, GEMM_TOL, f"case {case_id} strategy {strategy}")
    if layout == "replicated":   # AllReduce: every replica bit-identical at full size
        for i in range(1, t):
            assert torch.equal(c[i], c[0]), f"replica {i}"


# ---------------------------------------------------------------------------------- 70B-shaped layer
def _layer_device(L, N, h, n_h, n_kv, d_h, F, t, with_partials):
    d = {k: cuda(v) for k, v in L.items()}
    kv = n_kv // t if t <= n_kv else 1
    qkv_w = (n_h // t + 2 * kv) * d_h
    w_qkv = torch.empty((t, h, qkv_w), dtype=torch.bfloat16, device="cuda")
    w_o = torch.empty((t, n_h * d_h // t, h), dtype=torch.bfloat16, device="cuda")
    w_gu = torch.empty((t, h, 2 * F // t), dtype=torch.bfloat16, device="cuda")
    w_down = torch.empty((t, F // t, h), dtype=torch.bfloat16, device="cuda")
    tp.tp_shard_qkv(d["Wq"], n_h * d_h, d["Wk"], n_kv * d_h, d["Wv"], n_kv * d_h, h, n_h, n_kv, d_h, t, w_qkv)
    tp.tp_shard_rows(d["Wo"], h, n_h * d_h, h, t, w_o)
    tp.tp_shard_gate_up(d["Wg"], F, d["Wu"], F, h, F, t, w_gu)
    tp.tp_shard_rows(d["Wd"], h, F, h, t, w_down)
    o_shards = [d["O"][:, r * n_h * d_h // t:(r + 1) * n_h * d_h // t].contiguous() for r in range(t)]
    out = dict(qkv=torch.empty((t, N, qkv_w), dtype=torch.bfloat16, device="cuda"),
               h1=[torch.empty((N, h), device="cuda") for _ in range(t)],
               h1_bf16=torch.empty((N, h), dtype=torch.bfloat16, device="cuda"),
               y=[torch.empty((N, h), device="cuda") for _ in range(t)])
    z_ws = torch.empty((t, N, F // t), dtype=torch.bfloat16, device="cuda")
    partials = [torch.empty((N, h), device="cuda") for _ in range(t)] if with_partials else None
    tp.tp_layer_fwd(d["X"], o_shards, N, h, n_h, n_kv, d_h, F, t, w_qkv, w_o, w_gu, w_down, out["qkv"], out["h1"],
                    out["h1_bf16"], z_ws, partials, out["y"])
    torch.cuda.synchronize()
    _status_ok()
    return out


def _layer_oracle(L, n_h, n_kv, d_h, t, rows=None):
    f32 = lambda x: x.float().numpy()  # noqa: E731  (exact widening of bf16)
    sh_qkv = OL.shard_qkv(f32(L["Wq"]), f32(L["Wk"]), f32(L["Wv"]), n_h, n_kv, d_h, t)
    sh_o = OL.shard_rows(f32(L["Wo"]), t)
    sh_gu = OL.shard_gate_up(f32(L["Wg"]), f32(L["Wu"]), t)
    sh_d = OL.shard_rows(f32(L["Wd"]), t)
    O = f32(L["O"])
    O_sh = [O[:, r * n_h * d_h // t:(r + 1) * n_h * d_h // t] for r in range(t)]
    return OLAYER.layer_forward(f32(L["X"]), O_sh, list(sh_qkv), list(sh_o), list(sh_gu), list(sh_d), rows=rows)


# The layer's two AllReduces run fused with their row GEMMs, scattering along h when h/t is whole
# 256-column tiles (first shape), else along tokens when N/t is whole 128-row tiles (second), else
# unfused through the partials (third). Every path is compared in full with the fp64 oracle.
@pytest.mark.parametrize("N,h,n_h,n_kv,d_h,F,t,with_partials", [
    (256, 1024, 16, 4, 64, 2048, 4, False),
    (512, 512, 8, 4, 64, 1024, 4, False),
    (96, 512, 8, 2, 64, 1024, 4, True),
])
def test_layer_small_every_reduction_path(N, h, n_h, n_kv, d_h, F, t, with_partials):
    L = S.llama70b_layer(seed=3, N=N, h=h, n_h=n_h, n_kv=n_kv, d_h=d_h, F=F)
    got = _layer_device(L, N, h, n_h, n_kv, d_h, F, t, with_partials)
    ref = _layer_oracle(L, n_h, n_kv, d_h, t)
    for r in range(t):
        assert_close(f64(got["qkv"][r]), ref["qkv"][r], GEMM_TOL, f"qkv {r}")
    for s in range(t):
        assert_close(f64(got["h1"][s]), ref["h1"], GEMM_TOL, f"h1 replica {s}")
        assert_close(f64(got["y"][s]), ref["y"], GEMM_TOL, f"y replica {s}")
        assert same_bits(host_bits(got["h1"][s]), host_bits(got["h1"][0]))
        assert same_bits(host_bits(got["y"][s]), host_bits(got["y"][0]))
    # the MLP's input is h1 rounded once to bf16
    assert np.array_equal(host_bits(got["h1_bf16"]), f32_to_bf16_bits(host_bits(got["h1"][0])))
    assert_close(f64(got["y"][0]) - f64(got["h1"][0]), ref["mlp"], GEMM_TOL, "mlp part")


def test_llama70b_layer_sampled_rows():
    N, h, n_h, n_kv, d_h, F, t = 2048, 8192, 64, 8, 128, 28672, 8
    L = S.llama70b_layer(seed=0)
    d = {k: cuda(v) for k, v in L.items()}
    kv = n_kv // t
    qkv_w = (n_h // t + 2 * kv) * d_h
    w_qkv = torch.empty((t, h, qkv_w), dtype=torch.bfloat16, device="cuda")
    w_o = torch.empty((t, n_h * d_h // t, h), dtype=torch.bfloat16, device="cuda")
    w_gu = torch.empty((t, h, 2 * F // t), dtype=torch.bfloat16, device="cuda")
    w_down = torch.empty((t, F // t, h), dtype=torch.bfloat16, device="cuda")
    tp.tp_shard_qkv(d["Wq"], n_h * d_h, d["Wk"], n_kv * d_h, d["Wv"], n_kv * d_h, h, n_h, n_kv, d_h, t, w_qkv)
    tp.tp_shard_rows(d["Wo"], h, n_h * d_h, h, t, w_o)
    tp.tp_shard_gate_up(d["Wg"], F, d["Wu"], F, h, F, t, w_gu)
    tp.tp_shard_rows(d["Wd"], h, F, h, t, w_down)
    o_shards = [d["O"][:, r * n_h * d_h // t:(r + 1) * n_h * d_h // t].contiguous() for r in range(t)]
    qkv_out = torch.empty((t, N, qkv_w), dtype=torch.bfloat16, device="cuda")
    h1 = [torch.empty((N, h), device="cuda") for _ in range(t)]
    h1_bf16 = torch.empty((N, h), dtype=torch.bfloat16, device="cuda")
    z_ws = torch.empty((t, N, F // t), dtype=torch.bfloat16, device="cuda")
    partials = [torch.empty((N, h), device="cuda") for _ in range(t)]
    y = [torch.empty((N, h), device="cuda") for _ in range(t)]
    tp.tp_layer_fwd(d["X"], o_shards, N, h, n_h, n_kv, d_h, F, t, w_qkv, w_o, w_gu, w_down, qkv_out, h1, h1_bf16,
                    z_ws, partials, y)
    torch.cuda.synchronize()
    _status_ok()
    rows = tile_rows(N)   # every 128-row m-tile, whole rows (every n-tile)
    f32 = lambda x: x.float().numpy()  # noqa: E731  (exact widening of bf16)
    sh_qkv = OL.shard_qkv(f32(L["Wq"]), f32(L["Wk"]), f32(L["Wv"]), n_h, n_kv, d_h, t)
    sh_o = OL.shard_rows(f32(L["Wo"]), t)
    sh_gu = OL.shard_gate_up(f32(L["Wg"]), f32(L["Wu"]), t)
    sh_d = OL.shard_rows(f32(L["Wd"]), t)
    O = f32(L["O"])
    O_sh = [O[:, r * n_h * d_h // t:(r + 1) * n_h * d_h // t] for r in range(t)]
    ref = OLAYER.layer_forward(f32(L["X"]), O_sh, list(sh_qkv), list(sh_o), list(sh_gu), list(sh_d), rows=rows)
    for r in (0, 5):
        assert_close(f64(qkv_out[r])[rows], ref["qkv"][r], GEMM_TOL, f"qkv {r}")
    assert_close(f64(h1[3])[rows], ref["h1"], GEMM_TOL, "h1")
    for s in (0, 7):
        assert_close(f64(y[s])[rows], ref["y"], GEMM_TOL, f"y replica {s}")
        assert same_bits(host_bits(y[s]), host_bits(y[0]))
    # the MLP contribution alone, y - h1, against the oracle's
    assert_close(f64(y[0])[rows] - f64(h1[0])[rows], ref["mlp"], GEMM_TOL, "mlp part")


# ---------------------------------------------------------------------------------- TP + SP MLP
@pytest.mark.parametrize("N,h,F,t,act", [(512, 256, 1024, 4, tp.TP_ACT_GELU), (1024, 512, 2048, 4, tp.TP_ACT_SWIGLU),
                                         (2048, 1024, 4096, 8, tp.TP_ACT_SWIGLU)])
def test_sp_mlp_matches_oracle_and_tp_rows_bitwise(N, h, F, t, act):
    d = S.Draw(N + t)
    X = d.normal((N, h), 1.0)
    wn = 2 * F // t if act == tp.TP_ACT_SWIGLU else F // t
    w_in = d.normal((t, h, wn), 0.05)
    w_down = d.normal((t, F // t, h), 0.05)
    dX, dw_in, dw_down = cuda(X), cuda(w_in), cuda(w_down)
    x_shards = [cuda(xs) for xs in X.chunk(t, 0)]
    z = torch.empty((t, N, F // t), dtype=torch.bfloat16, device="cuda")
    out = [torch.empty((N // t, h), device="cuda") for _ in range(t)]
    tp.tp_mlp_fwd_sp(x_shards, N, h, F, t, act, dw_in, dw_down, z, out)
    # the column GEMM reading the shards in place gives the same activations as reading the gathered X
    z_full = torch.empty_like(z)
    tp.tp_column_linear(dX, N, h, F, t, act, dw_in, z_full)
    ref_tp = [torch.empty((N // t, h), device="cuda") for _ in range(t)]
    tp.tp_mlp_fwd(dX, N, h, F, t, act, dw_in, dw_down, torch.empty_like(z), None, tp.TP_OUT_RS, ref_tp)
    torch.cuda.synchronize()
    _status_ok()
    assert torch.equal(z, z_full)
    for r in range(t):
        assert torch.equal(out[r], ref_tp[r]), f"shard {r}"
    a = "swiglu" if act == tp.TP_ACT_SWIGLU else "gelu"
    ref = OM.sp_mlp([f64(x) for x in X.chunk(t, 0)], [f64(w) for w in w_in], [f64(w) for w in w_down], a)
    for r in range(t):
        assert_close(f64(out[r]), ref[r], GEMM_TOL, f"SP shard {r}")


# ---------------------------------------------------------------------------------- empty inputs
def test_empty_token_count_is_a_noop_then_a_normal_call_matches():
    """N = 0 launches nothing and leaves the output untouched; the next non-empty call on the same
    stream is unaffected (no error state, no device status)."""
    N, h, F, t = 64, 256, 1024, 4
    X, A, B = S.tiny_mlp(seed=3)
    dX = cuda(X)
    w_in = torch.empty((t, h, F // t), dtype=torch.bfloat16, device="cuda")
    w_down = torch.empty((t, F // t, h), dtype=torch.bfloat16, device="cuda")
    tp.tp_shard_cols(cuda(A), F, h, F, t, w_in)
    tp.tp_shard_rows(cuda(B), h, F, h, t, w_down)
    empty_x = torch.empty((0, h), dtype=torch.bfloat16, device="cuda")
    z0 = torch.empty((t, 0, F // t), dtype=torch.bfloat16, device="cuda")
    sentinel = [torch.full((4, h), 7.0, device="cuda") for _ in range(t)]
    tp.tp_mlp_fwd(empty_x, 0, h, F, t, tp.TP_ACT_GELU, w_in, w_down, z0, None, tp.TP_OUT_AR, sentinel)
    tp.tp_all_reduce(sentinel, sentinel, 0, h, tp.TP_F32, t)
    tp.tp_column_linear(empty_x, 0, h, F, t, tp.TP_ACT_GELU, w_in, z0)
    torch.cuda.synchronize()
    _status_ok()
    for s in sentinel:
        assert bool((s == 7.0).all())
    _, _, out = _mlp_device(dX, w_in, w_down, N, h, F, t, tp.TP_ACT_GELU, tp.TP_OUT_AR)
    Y = OM.mlp_unsharded(f64(X), f64(A), f64(B), "gelu")
    for r in range(t):
        assert_close(f64(out[r]), Y, GEMM_TOL, f"replica {r}")


# ---------------------------------------------------------------------------------- streams and graphs
def test_mlp_step_on_a_side_stream_and_in_a_cuda_graph():
    """The library only enqueues work on the caller's stream: the same MLP step on a side stream, and
    captured once into a CUDA graph and replayed, gives bit-identical results to the eager call on
    the default stream (no host synchronisation or allocation on the path)."""
    N, h, F, t = 1024, 512, 2048, 8
    d = S.Draw(11)
    X = cuda(d.normal((N, h), 1.0))
    w_in = cuda(d.normal((t, h, 2 * F // t), 0.05))
    w_down = cuda(d.normal((t, F // t, h), 0.05))
    z = torch.empty((t, N, F // t), dtype=torch.bfloat16, device="cuda")

    def outputs():
        return [torch.empty((N, h), device="cuda") for _ in range(t)]

    ref = outputs()
    tp.tp_mlp_fwd(X, N, h, F, t, tp.TP_ACT_SWIGLU, w_in, w_down, z, None, tp.TP_OUT_RS_AG, ref)
    torch.cuda.synchronize()
    _status_ok()

    side = torch.cuda.Stream()
    got_side = outputs()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        tp.tp_mlp_fwd(X, N, h, F, t, tp.TP_ACT_SWIGLU, w_in, w_down, z, None, tp.TP_OUT_RS_AG, got_side, side)
    side.synchronize()

    got_graph = outputs()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        tp.tp_mlp_fwd(X, N, h, F, t, tp.TP_ACT_SWIGLU, w_in, w_down, z, None, tp.TP_OUT_RS_AG, got_graph)
    for o in got_graph:
        o.zero_()
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    _status_ok()
    for r in range(t):
        assert torch.equal(got_side[r], ref[r]), f"side stream, replica {r}"
        assert torch.equal(got_graph[r], ref[r]), f"graph replay, replica {r}"
