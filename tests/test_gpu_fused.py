"""GPU parity of the fused row-parallel GEMM + ring reduction (tp_row_linear_reduce).

Each output tile's t shard products are computed in ring order and summed in binary32 inside the
GEMM epilogue. Two checks apply:
  * bit-identical to the unfused path, tp_row_linear (fp32 partials) followed by tp_reduce_scatter /
    tp_all_reduce: same MMA tile schedule, same ring order, one add per shard;
  * within the GEMM tolerance of the fp64 oracle (partials summed in ring order).
Shapes cover t in {2,3,4,8}, both chunk axes, ragged K and N tails, and the Llama-3-8B down-GEMM
shape at full size."""
import numpy as np
import pytest
import torch

import synthetic as S
import tensor_sharded_matmul_b200 as tp
from gpu_util import GEMM_TOL, assert_close, f64, host_bits, same_bits
from oracle import collectives as OC
from oracle import mlp as OM

pytestmark = pytest.mark.gpu


def _operands(t, N, k, n, seed):
    d = S.Draw(seed, "cuda")
    x = d.normal((t, N, k // t), 1.0)
    w = d.normal((t, k // t, n), 0.05)
    return x, w


def _out_shape(mode, axis, N, n, t):
    if mode != tp.TP_OUT_RS:
        return (N, n)
    return (N // t, n) if axis == 0 else (N, n // t)


CASES = [
    # t, N, k, n, mode, axis
    (2, 256, 512, 512, tp.TP_OUT_RS, 0),
    (4, 512, 1024, 768, tp.TP_OUT_RS, 0),
    (8, 1024, 1024, 512, tp.TP_OUT_AR, 0),
    (4, 512, 2048, 1024, tp.TP_OUT_RS, 1),
    (2, 256, 400, 264, tp.TP_OUT_AR, 0),      # ragged K (k/t = 200) and an N tail (264)
    (3, 384, 768, 512, tp.TP_OUT_RS_AG, 0),   # t without a specialised ring kernel
    (8, 2048, 8192, 8192, tp.TP_OUT_AR, 0),   # the 70B W_O shape: 1024 of k per shard
    # chunks of 256 rows: the CTA-pair variant of the fused kernel
    (2, 512, 512, 512, tp.TP_OUT_RS, 0),
    (4, 1024, 1024, 520, tp.TP_OUT_AR, 0),    # with an N tail
    (3, 768, 768, 512, tp.TP_OUT_RS_AG, 0),
    (2, 384, 512, 512, tp.TP_OUT_RS, 1),      # axis 1 on pairs with a 128-row M tail
    # more pair tiles than the 74 pairs of a 148-SM GPU, the remainder at most half of them: the last
    # round runs as 256 x 128 half tiles; AllReduce copies replica 0 into the others one slice at a time
    (4, 2048, 1024, 2560, tp.TP_OUT_AR, 0),   # 80 tiles
    (8, 2048, 1024, 2600, tp.TP_OUT_RS_AG, 0),  # 88 tiles, N tail: one half tile wholly past N
    (2, 2048, 512, 2560, tp.TP_OUT_RS, 0),
    (4, 1280, 512, 4096, tp.TP_OUT_RS, 1),    # axis 1, 80 tiles
    # shard-count extremes: t = 1 (a single chunk) and t = 16 (the maximum)
    (1, 512, 512, 512, tp.TP_OUT_AR, 0),
    (1, 384, 256, 512, tp.TP_OUT_RS, 1),
    (16, 4096, 2048, 1024, tp.TP_OUT_RS_AG, 0),   # 256-row chunks: CTA pairs, deferred replica copies
    (16, 2048, 4096, 512, tp.TP_OUT_RS, 0),       # 128-row chunks: single-CTA kernel
    # odd k-block counts per shard on CTA pairs (two k-blocks per pipeline stage)
    (4, 1024, 768, 512, tp.TP_OUT_AR, 0),         # 192 per shard: three k-blocks
    (2, 512, 80, 512, tp.TP_OUT_RS, 0),           # 40 per shard: one ragged k-block
    # axis 1 places no constraint on the row count: a partial last row-tile on the single-CTA kernel
    (2, 200, 512, 512, tp.TP_OUT_RS, 1),
    (4, 72, 256, 1024, tp.TP_OUT_RS, 1),
    # AllReduce whose ReduceScatter runs along columns (each element summed in its column chunk's
    # ring order): pairs, a 128-row M tail, the single-CTA kernel, the 70B W_O shape
    (4, 512, 1024, 1024, tp.TP_OUT_AR, 1),
    (2, 384, 512, 512, tp.TP_OUT_AR, 1),
    (4, 200, 256, 1024, tp.TP_OUT_AR, 1),
    (8, 2048, 1024, 4096, tp.TP_OUT_AR, 1),      # 8 x 16 tiles: more tiles than pairs, half-width round
    (8, 2048, 8192, 8192, tp.TP_OUT_AR, 1),
    (1, 256, 256, 512, tp.TP_OUT_AR, 1),         # a single chunk
    (16, 512, 2048, 4096, tp.TP_OUT_AR, 1),      # the maximum shard count, 256-column chunks
]


@pytest.mark.parametrize("t,N,k,n,mode,axis", CASES)
def test_fused_equals_unfused_bitwise_and_oracle(t, N, k, n, mode, axis):
    x, w = _operands(t, N, k, n, seed=t * 1000 + N + n)
    shape = _out_shape(mode, axis, N, n, t)
    fused = [torch.empty(shape, device="cuda") for _ in range(t)]
    tp.tp_row_linear_reduce(x, N, k, n, t, w, mode, axis, fused)
    partials = [torch.empty((N, n), device="cuda") for _ in range(t)]
    tp.tp_row_linear(x, N, k, n, t, w, partials)
    plain = [torch.empty(shape, device="cuda") for _ in range(t)]
    if mode == tp.TP_OUT_RS:
        tp.tp_reduce_scatter(partials, plain, N, n, axis, tp.TP_F32, t)
    elif axis == 0:
        tp.tp_all_reduce(partials, plain, N, n, tp.TP_F32, t)
    else:                   # AllReduce along columns = ReduceScatter(axis 1) then AllGather(axis 1)
        pieces = [torch.empty((N, n // t), device="cuda") for _ in range(t)]
        tp.tp_reduce_scatter(partials, pieces, N, n, 1, tp.TP_F32, t)
        tp.tp_all_gather(pieces, plain, N, n, 1, tp.TP_F32, t)
    torch.cuda.synchronize()
    st, site = tp.tp_device_status(1)
    assert st == tp.TP_OK, f"device wait site {site}"
    for r in range(t):
        assert same_bits(host_bits(fused[r]), host_bits(plain[r])), f"shard {r} differs from the unfused path"
    # oracle: fp64 partials, reduced by the oracle's ring (accumulated in fp64 here)
    rows = np.arange(N) if N <= 1024 else np.sort(np.random.default_rng(t).choice(N, 64, replace=False))
    U = [OM.matmul(f64(x[r])[rows], f64(w[r])) for r in range(t)]
    Y = sum(U)
    if mode == tp.TP_OUT_RS and axis == 0:
        for r in range(t):
            lo, hi = r * N // t, (r + 1) * N // t
            inside = (rows >= lo) & (rows < hi)          # sampled rows that land in shard r's block
            assert_close(f64(fused[r])[rows[inside] - lo], Y[inside], GEMM_TOL, f"RS block {r}")
    elif mode == tp.TP_OUT_RS:
        for r in range(t):
            assert_close(f64(fused[r])[rows], Y[:, r * n // t:(r + 1) * n // t], GEMM_TOL, f"RS column block {r}")
    else:
        for r in range(t):
            assert_close(f64(fused[r])[rows], Y, GEMM_TOL, f"replica {r}")


@pytest.mark.parametrize("t,N", [(4, 512), (4, 1024)])      # 128-row chunks (single CTA), 256 (pairs)
def test_fused_ring_order_matches_the_oracle_bitwise(t, N):
    # Feed the oracle the GPU's own fp32 partials (from the unfused GEMM): the ring sum must match bit for
    # bit, which shows that the fused epilogue adds the shards in the ring order the pages imply.
    k, n = 1024, 512
    x, w = _operands(t, N, k, n, seed=77)
    fused = [torch.empty((N // t, n), device="cuda") for _ in range(t)]
    tp.tp_row_linear_reduce(x, N, k, n, t, w, tp.TP_OUT_RS, 0, fused)
    partials = [torch.empty((N, n), device="cuda") for _ in range(t)]
    tp.tp_row_linear(x, N, k, n, t, w, partials)
    torch.cuda.synchronize()
    ref = OC.reduce_scatter([host_bits(p) for p in partials], axis=0)
    for r in range(t):
        assert same_bits(host_bits(fused[r]), ref[r])


def test_llama8b_down_gemm_fused_full_size():
    t, N, k, n = 8, 4096, 14336, 4096
    x, w = _operands(t, N, k, n, seed=8)
    fused = [torch.empty((N, n), device="cuda") for _ in range(t)]
    tp.tp_row_linear_reduce(x, N, k, n, t, w, tp.TP_OUT_RS_AG, 0, fused)
    partials = [torch.empty((N, n), device="cuda") for _ in range(t)]
    tp.tp_row_linear(x, N, k, n, t, w, partials)
    plain = [torch.empty((N, n), device="cuda") for _ in range(t)]
    tp.tp_all_reduce(partials, plain, N, n, tp.TP_F32, t)
    torch.cuda.synchronize()
    for r in range(t):
        assert torch.equal(fused[r], plain[r]), f"replica {r}"


def test_unaligned_chunks_need_partials():
    t, N, k, n = 4, 64, 256, 256          # N/t = 16 rows: no tile fits inside one chunk
    x, w = _operands(t, N, k, n, seed=5)
    out = [torch.empty((N // t, n), device="cuda") for _ in range(t)]
    with pytest.raises(tp.TPError) as e:
        tp.tp_row_linear_reduce(x, N, k, n, t, w, tp.TP_OUT_RS, 0, out)
    assert e.value.status == tp.TP_EUNSUPPORTED
    partials = [torch.empty((N, n), device="cuda") for _ in range(t)]
    tp.tp_row_linear_reduce(x, N, k, n, t, w, tp.TP_OUT_RS, 0, out, partials)
    torch.cuda.synchronize()
    Y = sum(OM.matmul(f64(x[r]), f64(w[r])) for r in range(t))
    for r in range(t):
        assert_close(f64(out[r]), Y[r * N // t:(r + 1) * N // t], GEMM_TOL, f"block {r}")


@pytest.mark.parametrize("t,N,k,n", [(4, 256, 512, 520), (3, 96, 384, 264)])
def test_unfused_all_reduce_along_columns(t, N, k, n):
    # n/t is not a whole number of 256-column tiles: the partials path with the ring kernel's
    # AllReduce along columns, bit-identical to ReduceScatter(axis 1) then AllGather(axis 1) and to
    # the oracle's ring order fed the same partials
    x, w = _operands(t, N, k, n, seed=31 + t)
    out = [torch.empty((N, n), device="cuda") for _ in range(t)]
    partials = [torch.empty((N, n), device="cuda") for _ in range(t)]
    tp.tp_row_linear_reduce(x, N, k, n, t, w, tp.TP_OUT_AR, 1, out, partials)
    torch.cuda.synchronize()
    ref = OC.all_reduce([host_bits(p) for p in partials], axis=1)
    for r in range(t):
        assert same_bits(host_bits(out[r]), ref[r]), f"replica {r}"
