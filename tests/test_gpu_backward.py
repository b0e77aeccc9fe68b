"""GPU parity of the backward pass of the tensor-parallel MLP and of the transposed-operand GEMM modes
it uses, against the fp64 oracle (whose gradient formulas are pinned by finite differences).

The GPU computes its own forward intermediates (H = X W_in, Z = act(H)) in bf16, as a training step
would. The oracle computes everything from the same seeded X, W and dY in fp64. Tolerance: the GEMM
tolerance, max|err| <= 2e-2 * max|ref|."""
import numpy as np
import pytest
import torch

import synthetic as S
import tensor_sharded_matmul_b200 as tp
from gpu_util import FP32_GEMM_TOL, GEMM_TOL, assert_close, cuda, f64, host_bits, same_bits
from oracle import mlp as OM

pytestmark = pytest.mark.gpu

ACT = {"gelu": tp.TP_ACT_GELU, "gelu_tanh": tp.TP_ACT_GELU_TANH, "swiglu": tp.TP_ACT_SWIGLU, "none": tp.TP_ACT_NONE}


@pytest.mark.parametrize("trans_a,trans_b", [(0, 1), (1, 0), (1, 1), (0, 0)])
@pytest.mark.parametrize("groups,M,N,K", [(2, 128, 256, 256), (3, 200, 264, 136), (2, 512, 512, 1024), (4, 1024, 768, 512)])
def test_transposed_operand_gemm(trans_a, trans_b, groups, M, N, K):
    d = S.Draw(M + N + K + 10 * trans_a + trans_b)
    A = [d.normal((M, K), 1.0) for _ in range(groups)]
    B = [d.normal((K, N), 0.05) for _ in range(groups)]
    a_st = [cuda(a.t().contiguous() if trans_a else a) for a in A]
    b_st = [cuda(b.t().contiguous() if trans_b else b) for b in B]
    C = [torch.empty((M, N), device="cuda") for _ in range(groups)]
    tp.tp_grouped_gemm_t(groups, a_st, trans_a, b_st, trans_b, C, M, N, K, tp.TP_F32)
    torch.cuda.synchronize()
    st, site = tp.tp_device_status(1)
    assert st == tp.TP_OK, f"device wait site {site}"
    for g in range(groups):
        assert_close(f64(C[g]), OM.matmul(f64(A[g]), f64(B[g])), FP32_GEMM_TOL, f"group {g}")


def _forward_intermediates(dX, dw_in, N, h, F, t, act):
    """H (pre-activations) and Z (activations) as the GPU forward produces them."""
    f = F // t
    wn = 2 * f if act == "swiglu" else f
    H = torch.empty((t, N, wn), dtype=torch.bfloat16, device="cuda")
    tp.tp_column_linear(dX, N, h, wn * t, t, tp.TP_ACT_NONE, dw_in, H)
    Z = torch.empty((t, N, f), dtype=torch.bfloat16, device="cuda")
    tp.tp_column_linear(dX, N, h, F, t, ACT[act], dw_in, Z)
    return H, Z


@pytest.mark.parametrize("N,h,F,t,act", [
    (64, 256, 1024, 4, "gelu"),        # the tiny configuration: dX through the unfused path
    (512, 256, 1024, 4, "gelu_tanh"),
    (1024, 512, 2048, 4, "swiglu"),    # dX through the fused ring GEMM (CTA pairs)
    (1024, 1024, 4096, 8, "swiglu"),
    (256, 128, 512, 2, "none"),
    (384, 256, 1088, 8, "swiglu"),     # F/t = 136: a partial 32-column chunk; a partial pair tile
    (200, 128, 544, 4, "gelu"),        # one-CTA kernel, ragged rows and columns
])
def test_mlp_backward_against_oracle(N, h, F, t, act):
    d = S.Draw(N + h + t)
    f = F // t
    wn = 2 * f if act == "swiglu" else f
    X = d.normal((N, h), 1.0)
    dY = d.normal((N, h), 1.0)
    w_in = d.normal((t, h, wn), 0.05)
    w_down = d.normal((t, f, h), 0.05)
    dX_, ddY, dw_in, dw_down = cuda(X), cuda(dY), cuda(w_in), cuda(w_down)
    H, Z = _forward_intermediates(dX_, dw_in, N, h, F, t, act)
    dz = torch.empty((t, N, f), dtype=torch.bfloat16, device="cuda")
    dh = torch.empty((t, N, wn), dtype=torch.bfloat16, device="cuda")
    g_in = torch.empty((t, h, wn), device="cuda")
    g_down = torch.empty((t, f, h), device="cuda")
    gx = [torch.empty((N, h), device="cuda") for _ in range(t)]
    tp.tp_mlp_bwd(dX_, ddY, N, h, F, t, ACT[act], dw_in, dw_down, H, Z, dz, dh, g_in, g_down, gx)
    torch.cuda.synchronize()
    st, site = tp.tp_device_status(1)
    assert st == tp.TP_OK, f"device wait site {site}"
    ref = OM.mlp_backward(f64(X), [f64(w) for w in w_in], [f64(w) for w in w_down], f64(dY), act)
    for r in range(t):
        # dH_r from the activation's backward kernel (bf16); the GPU's H is its own bf16 forward
        assert_close(f64(dh[r]), ref["dH"][r], GEMM_TOL, f"dH[{r}]")
        assert_close(f64(g_down[r]), ref["dW_out"][r], GEMM_TOL, f"dW_down[{r}]")
        assert_close(f64(g_in[r]), ref["dW_in"][r], GEMM_TOL, f"dW_in[{r}]")
        assert_close(f64(gx[r]), ref["dX"], GEMM_TOL, f"dX replica {r}")
        assert same_bits(host_bits(gx[r]), host_bits(gx[0]))   # f's backward AllReduce: identical replicas


def _sample(n: int, tile: int = 128) -> np.ndarray:
    """One index from every `tile`-wide block (at an offset that moves from block to block, so that
    different TMEM lanes, epilogue warps and both CTAs of a pair are checked), plus the first and
    the last index."""
    idx = {0, n - 1}
    for b in range(n // tile):
        idx.add(b * tile + (b * 53 + 17) % tile)
    return np.array(sorted(idx))


def test_llama8b_backward_full_size_sampled():
    """The backward at the benchmark's Llama-3-8B shape (4096 tokens, h = 4096, F = 14336, t = 8,
    SwiGLU) against the oracle, on samples the oracle computes exactly:
      * dX and dH on one row per 128-row tile: a row of either needs only the same row of X and dY,
        so the oracle runs on those rows alone;
      * dW_down rows and dW_in columns on one index per 128-wide block of F/t, for three shards: those
        slices need only the matching gate/up columns of W_in and rows of W_down, so the oracle runs
        on the sliced shards with the full X and dY."""
    from oracle import layouts as OL
    N, h, F, t = 4096, 4096, 14336, 8
    f = F // t
    X, Wgu, Wd = S.llama8b_mlp(seed=0)
    dY = S.Draw(7).normal((N, h), 1.0)
    dX_, ddY = cuda(X), cuda(dY)
    dWgu, dWd = cuda(Wgu), cuda(Wd)
    w_in = torch.empty((t, h, 2 * f), dtype=torch.bfloat16, device="cuda")
    w_down = torch.empty((t, f, h), dtype=torch.bfloat16, device="cuda")
    tp.tp_shard_gate_up(dWgu, 2 * F, dWgu.data_ptr() + 2 * F, 2 * F, h, F, t, w_in)
    tp.tp_shard_rows(dWd, h, F, h, t, w_down)
    del dWgu, dWd
    H, Z = _forward_intermediates(dX_, w_in, N, h, F, t, "swiglu")
    dz = torch.empty((t, N, f), dtype=torch.bfloat16, device="cuda")
    dh = torch.empty((t, N, 2 * f), dtype=torch.bfloat16, device="cuda")
    g_in = torch.empty((t, h, 2 * f), device="cuda")
    g_down = torch.empty((t, f, h), device="cuda")
    gx = [torch.empty((N, h), device="cuda") for _ in range(t)]
    tp.tp_mlp_bwd(dX_, ddY, N, h, F, t, tp.TP_ACT_SWIGLU, w_in, w_down, H, Z, dz, dh, g_in, g_down, gx)
    torch.cuda.synchronize()
    st, site = tp.tp_device_status(1)
    assert st == tp.TP_OK, f"device wait site {site}"
    shards_in = list(OL.shard_gate_up(Wgu[:, :F].float().numpy(), Wgu[:, F:].float().numpy(), t))
    shards_down = list(OL.shard_rows(Wd.float().numpy(), t))
    Xf, dYf = f64(X), f64(dY)

    rows = _sample(N)
    ref = OM.mlp_backward(Xf[rows], shards_in, shards_down, dYf[rows], "swiglu")
    for r in (0, 3, 7):
        assert_close(f64(gx[r])[rows], ref["dX"], GEMM_TOL, f"dX replica {r}")
        assert_close(f64(dh[r])[rows], ref["dH"][r], GEMM_TOL, f"dH[{r}]")
    for r in range(t):
        assert same_bits(host_bits(gx[r]), host_bits(gx[0]))   # the AllReduce's replicas are identical

    cols = _sample(f)
    gate_up = np.concatenate([cols, f + cols])
    for s in (0, 3, 7):
        sub = OM.mlp_backward(Xf, [shards_in[s][:, gate_up]], [shards_down[s][cols, :]], dYf, "swiglu")
        assert_close(f64(g_down[s])[cols, :], sub["dW_out"][0], GEMM_TOL, f"dW_down[{s}] rows")
        assert_close(f64(g_in[s])[:, gate_up], sub["dW_in"][0], GEMM_TOL, f"dW_in[{s}] columns")
