"""GPU parity of the tcgen05 grouped GEMM and its fused epilogues against the fp64 oracle, through the
C ABI. Shapes cover one and several tiles per dimension, ragged M/N/K tails (TMA zero fill and masked
stores), shared and per-group A operands, and every epilogue (fp32, bf16, GeLU erf/tanh, SwiGLU)."""
import numpy as np
import pytest
import torch

import synthetic as S
import tensor_sharded_matmul_b200 as tp
from gpu_util import FP32_GEMM_TOL, GEMM_TOL, assert_close, cuda, f64
from oracle import mlp as OM

pytestmark = pytest.mark.gpu

ACT = {"none": tp.TP_ACT_NONE, "gelu": tp.TP_ACT_GELU, "gelu_tanh": tp.TP_ACT_GELU_TANH, "swiglu": tp.TP_ACT_SWIGLU}


def _run(groups, M, N, K, act, c_dtype, shared_a, seed=0):
    d = S.Draw(seed)
    nb = 2 * N if act == "swiglu" else N
    A = [d.normal((M, K), 1.0) for _ in range(1 if shared_a else groups)]
    B = [d.normal((K, nb), 0.05) for _ in range(groups)]
    dA = [cuda(a) for a in A]
    dB = [cuda(b) for b in B]
    cdt = torch.float32 if c_dtype == tp.TP_F32 else torch.bfloat16
    dC = [torch.empty((M, N), dtype=cdt, device="cuda") for _ in range(groups)]
    a_ptrs = [dA[0 if shared_a else g] for g in range(groups)]
    tp.tp_grouped_gemm(groups, a_ptrs, dB, dC, M, N, K, ACT[act], c_dtype)
    torch.cuda.synchronize()
    st, site = tp.tp_device_status(1)
    assert st == tp.TP_OK, f"device wait site {site}"
    refs = [OM.activate(OM.matmul(f64(A[0 if shared_a else g]), f64(B[g])), act) for g in range(groups)]
    return [f64(c) for c in dC], refs


@pytest.mark.parametrize("groups,M,N,K,shared", [
    (1, 128, 256, 64, False),     # one tile, one k-block
    (1, 128, 256, 256, False),    # several k-blocks
    (1, 64, 256, 256, False),     # M < tile (zero-filled rows, masked stores)
    (1, 200, 264, 200, False),    # ragged M, N, K
    (3, 384, 512, 1024, False),   # several tiles per dimension, 3 groups
    (4, 256, 768, 512, True),     # shared A (column-parallel form)
    (8, 130, 520, 136, False),    # many groups, ragged
    (2, 1024, 1024, 4096, True),  # long K
    # 80 CTA-pair tiles: more than one round on the 74 pairs of a 148-SM GPU
    (2, 1024, 2560, 512, False),
    (2, 1024, 2520, 264, True),   # ... with a ragged N tail and a ragged K
    # CTA pairs take two k-blocks per pipeline stage: odd k-block counts leave the last stage half used
    (2, 256, 256, 64, False),     # one k-block
    (1, 512, 512, 136, True),     # three k-blocks, the last ragged
    # long contractions shrink the raster band (row-tiles kept in L2 together): 8 row-tiles at
    # K = 8192 (12 here: one full band and a partial one), 4 at K = 16384
    (3, 1024, 512, 8192, False),
    (2, 1280, 264, 16384, True),
])
def test_gemm_fp32_out(groups, M, N, K, shared):
    got, ref = _run(groups, M, N, K, "none", tp.TP_F32, shared, seed=M + N + K)
    for g in range(groups):
        assert_close(got[g], ref[g], FP32_GEMM_TOL, f"group {g}")


@pytest.mark.parametrize("act", ["none", "gelu", "gelu_tanh"])
@pytest.mark.parametrize("groups,M,N,K", [(2, 256, 512, 512), (4, 64, 256, 256), (3, 200, 136, 96),
                                          (2, 1024, 2560, 256),    # more tiles than CTA pairs
                                          (2, 384, 264, 128)])     # CTA pairs: a half-empty row tile, 8-column tail
def test_gemm_bf16_epilogues(act, groups, M, N, K):
    got, ref = _run(groups, M, N, K, act, tp.TP_BF16, shared_a=True, seed=N)
    for g in range(groups):
        assert_close(got[g], ref[g], GEMM_TOL, f"{act} group {g}")
        # bf16 rounding bounds the error well below the stated tolerance
        assert_close(got[g], ref[g], 1e-2, f"{act} group {g} (rounding bound)")


@pytest.mark.parametrize("groups,M,N,K", [(1, 128, 128, 64), (2, 256, 384, 512), (8, 192, 136, 264), (8, 512, 1792, 1024),
                                          (2, 1024, 1280, 512), (2, 1024, 1224, 264)])   # more tiles than CTA pairs
def test_gemm_swiglu_pairs_gate_and_up(groups, M, N, K):
    got, ref = _run(groups, M, N, K, "swiglu", tp.TP_BF16, shared_a=True, seed=K)
    for g in range(groups):
        assert_close(got[g], ref[g], GEMM_TOL, f"swiglu group {g}")


def test_gemm_output_is_deterministic():
    a, _ = _run(2, 256, 512, 512, "none", tp.TP_F32, False, seed=3)
    b, _ = _run(2, 256, 512, 512, "none", tp.TP_F32, False, seed=3)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
