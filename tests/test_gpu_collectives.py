"""GPU parity of the ring collectives and the layout kernels against the oracle (bit-exact), through
the C ABI. Shapes span several vectors per thread, ragged tails (scalar path), t in {1..16}, both
chunk axes, fp32 and bf16; the largest cases are the MLP's own full-size reduction."""
import numpy as np
import pytest
import torch

import synthetic as S
import tensor_sharded_matmul_b200 as tp
from gpu_util import cuda, host_bits, same_bits
from oracle import collectives as OC
from oracle import layouts as OL

pytestmark = pytest.mark.gpu

TPD = {"f32": tp.TP_F32, "bf16": tp.TP_BF16}
TD = {"f32": torch.float32, "bf16": torch.bfloat16}


def _payload(t, rows, cols, dtype, seed):
    return S.collective_payload(t, rows, cols, dtype, seed)


CASES = [
    # t, rows, cols, dtype, axis
    (1, 16, 64, "f32", 0), (2, 64, 256, "f32", 0), (4, 64, 256, "f32", 1), (8, 128, 512, "f32", 0),
    (8, 64, 1024, "f32", 1), (3, 96, 72, "f32", 0), (5, 40, 80, "bf16", 1), (16, 64, 128, "bf16", 0),
    (2, 6, 5, "f32", 0), (3, 9, 7, "bf16", 0), (4, 12, 20, "f32", 1), (2, 10, 3, "bf16", 0),
    (4, 256, 2048, "bf16", 0), (8, 512, 4096, "bf16", 1),
    # more than one grid-stride step per thread, with the last step of some threads partial
    (2, 2050, 4104, "f32", 0), (4, 1028, 4104, "bf16", 0), (2, 2050, 4104, "bf16", 1),
]


@pytest.mark.parametrize("t,rows,cols,dtype,axis", CASES)
def test_reduce_scatter_bit_exact(t, rows, cols, dtype, axis):
    ins = _payload(t, rows, cols, dtype, seed=S.collective_sweep_seed(t, dtype, rows * cols))
    d_in = [cuda(x) for x in ins]
    oshape = (rows // t, cols) if axis == 0 else (rows, cols // t)
    d_out = [torch.empty(oshape, dtype=TD[dtype], device="cuda") for _ in range(t)]
    tp.tp_reduce_scatter(d_in, d_out, rows, cols, axis, TPD[dtype], t)
    torch.cuda.synchronize()
    ref = OC.reduce_scatter([host_bits(x) for x in ins], axis=axis, dtype=dtype)
    for r in range(t):
        assert same_bits(host_bits(d_out[r]), ref[r]), f"shard {r}"


@pytest.mark.parametrize("t,rows,cols,dtype,axis", CASES)
def test_all_gather_bit_exact(t, rows, cols, dtype, axis):
    pieces = _payload(t, rows // t if axis == 0 else rows, cols if axis == 0 else cols // t, dtype, seed=7 + t)
    d_in = [cuda(x) for x in pieces]
    d_out = [torch.empty((rows, cols), dtype=TD[dtype], device="cuda") for _ in range(t)]
    tp.tp_all_gather(d_in, d_out, rows, cols, axis, TPD[dtype], t)
    torch.cuda.synchronize()
    ref = OC.all_gather([host_bits(x) for x in pieces], axis=axis)
    for s in range(t):
        assert same_bits(host_bits(d_out[s]), ref[s]), f"shard {s}"


@pytest.mark.parametrize("t,rows,cols,dtype", [(c[0], c[1], c[2], c[3]) for c in CASES if c[4] == 0])
def test_all_reduce_bit_exact_and_equal_to_rs_then_ag(t, rows, cols, dtype):
    ins = _payload(t, rows, cols, dtype, seed=11 * t + rows)
    d_in = [cuda(x) for x in ins]
    d_out = [torch.empty((rows, cols), dtype=TD[dtype], device="cuda") for _ in range(t)]
    tp.tp_all_reduce(d_in, d_out, rows, cols, TPD[dtype], t)
    # the same through ReduceScatter into each shard's own block, then an in-place AllGather
    d_two = [torch.empty((rows, cols), dtype=TD[dtype], device="cuda") for _ in range(t)]
    blocks = [d_two[r].view(t, rows // t, cols)[r] for r in range(t)]
    tp.tp_reduce_scatter(d_in, blocks, rows, cols, 0, TPD[dtype], t)
    tp.tp_all_gather(blocks, d_two, rows, cols, 0, TPD[dtype], t)
    torch.cuda.synchronize()
    ref = OC.all_reduce([host_bits(x) for x in ins], dtype=dtype)
    for s in range(t):
        got = host_bits(d_out[s])
        assert same_bits(got, ref[s]), f"replica {s}"
        assert same_bits(got, host_bits(d_out[0]))
        assert same_bits(host_bits(d_two[s]), got)


def test_all_reduce_in_place():
    t, rows, cols = 4, 64, 96
    ins = _payload(t, rows, cols, "f32", seed=99)
    bufs = [cuda(x) for x in ins]
    tp.tp_all_reduce(bufs, bufs, rows, cols, tp.TP_F32, t)
    torch.cuda.synchronize()
    ref = OC.all_reduce([host_bits(x) for x in ins])
    for s in range(t):
        assert same_bits(host_bits(bufs[s]), ref[s])


def test_tiny_config_collectives():
    # 4 fp32 shards ~U(-1,1): AllGather of 4 x 256 and ReduceScatter of 4 x 1024 (chunks of 256)
    ag_in, rs_in = S.tiny_collectives(seed=0)
    t = 4
    d_ag = [cuda(x.view(1, 256)) for x in ag_in]
    d_ag_out = [torch.empty((4, 256), device="cuda") for _ in range(t)]
    tp.tp_all_gather(d_ag, d_ag_out, 4, 256, 0, tp.TP_F32, t)
    d_rs = [cuda(x.view(4, 256)) for x in rs_in]
    d_rs_out = [torch.empty((1, 256), device="cuda") for _ in range(t)]
    tp.tp_reduce_scatter(d_rs, d_rs_out, 4, 256, 0, tp.TP_F32, t)
    torch.cuda.synchronize()
    ag_ref = OC.all_gather([x.view(1, 256).numpy() for x in ag_in], axis=0)
    rs_ref = OC.reduce_scatter([x.view(4, 256).numpy() for x in rs_in], axis=0)
    for s in range(t):
        assert same_bits(host_bits(d_ag_out[s]), ag_ref[s])
        assert same_bits(host_bits(d_rs_out[s]), rs_ref[s])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_full_size_mlp_reduction(dtype):
    # the 8B MLP's reduction: 8 partials [4096, 4096] (64 MiB each in fp32), ReduceScatter along tokens
    t, rows, cols = 8, 4096, 4096
    ins = _payload(t, rows, cols, dtype, seed=S.collective_sweep_seed(t, dtype, 64))
    d_in = [cuda(x) for x in ins]
    d_out = [torch.empty((rows // t, cols), dtype=TD[dtype], device="cuda") for _ in range(t)]
    tp.tp_reduce_scatter(d_in, d_out, rows, cols, 0, TPD[dtype], t)
    torch.cuda.synchronize()
    ref = OC.reduce_scatter([host_bits(x) for x in ins], axis=0, dtype=dtype)
    for r in range(t):
        assert same_bits(host_bits(d_out[r]), ref[r])


def test_selftest_wait_runs_out_and_context_survives():
    tp.tp_device_status(1)                         # clear
    tp.tp_selftest_wait_timeout(200_000)           # ~0.1 ms budget on a flag nothing sets
    st, site = tp.tp_device_status(1)
    assert st == tp.TP_ETIMEOUT and site == 1
    st, _ = tp.tp_device_status(1)
    assert st == tp.TP_OK
    # the context is still usable
    ins = _payload(2, 8, 16, "f32", seed=1)
    d_in = [cuda(x) for x in ins]
    d_out = [torch.empty((4, 16), device="cuda") for _ in range(2)]
    tp.tp_reduce_scatter(d_in, d_out, 8, 16, 0, tp.TP_F32, 2)
    torch.cuda.synchronize()
    ref = OC.reduce_scatter([host_bits(x) for x in ins], axis=0)
    assert same_bits(host_bits(d_out[0]), ref[0])


# ---------------------------------------------------------------------------------- layouts
def _w(shape, seed):
    return S.Draw(seed).normal(shape, 0.02)


@pytest.mark.parametrize("K,N,t", [(64, 256, 4), (40, 24, 3), (16, 12, 2), (256, 1024, 8)])
def test_shard_cols_rows_bit_exact(K, N, t):
    W = _w((K, N), seed=K + N)
    d = cuda(W)
    if N % t == 0:
        out = torch.empty((t, K, N // t), dtype=torch.bfloat16, device="cuda")
        tp.tp_shard_cols(d, N, K, N, t, out)
        torch.cuda.synchronize()
        assert np.array_equal(host_bits(out), OL.shard_cols(S.bf16_bits(W), t))
    if K % t == 0:
        out = torch.empty((t, K // t, N), dtype=torch.bfloat16, device="cuda")
        tp.tp_shard_rows(d, N, K, N, t, out)
        torch.cuda.synchronize()
        assert np.array_equal(host_bits(out), OL.shard_rows(S.bf16_bits(W), t))


@pytest.mark.parametrize("h,F,t", [(64, 1024, 4), (32, 48, 3), (4096, 14336, 8)])
def test_shard_gate_up_bit_exact(h, F, t):
    # gate and up given as the two halves of one fused [h, 2F] matrix (row stride 2F)
    Wgu = _w((h, 2 * F), seed=h)
    d = cuda(Wgu)
    out = torch.empty((t, h, 2 * F // t), dtype=torch.bfloat16, device="cuda")
    tp.tp_shard_gate_up(d, 2 * F, d.data_ptr() + 2 * F, 2 * F, h, F, t, out)
    torch.cuda.synchronize()
    bits = S.bf16_bits(Wgu)
    assert np.array_equal(host_bits(out), OL.shard_gate_up(bits[:, :F], bits[:, F:], t))


@pytest.mark.parametrize("h,n_h,n_kv,d_h,t", [
    (64, 8, 2, 16, 2), (64, 8, 2, 16, 4), (64, 8, 8, 16, 8), (32, 4, 2, 4, 4), (8192, 64, 8, 128, 8),
    (256, 32, 8, 8, 16), (96, 6, 3, 8, 3),
])
def test_shard_qkv_bit_exact(h, n_h, n_kv, d_h, t):
    Wq, Wk, Wv = _w((h, n_h * d_h), 1), _w((h, n_kv * d_h), 2), _w((h, n_kv * d_h), 3)
    kv = n_kv // t if t <= n_kv else 1
    width = (n_h // t + 2 * kv) * d_h
    out = torch.empty((t, h, width), dtype=torch.bfloat16, device="cuda")
    dq, dk, dv = cuda(Wq), cuda(Wk), cuda(Wv)
    tp.tp_shard_qkv(dq, n_h * d_h, dk, n_kv * d_h, dv, n_kv * d_h, h, n_h, n_kv, d_h, t, out)
    torch.cuda.synchronize()
    ref = OL.shard_qkv(S.bf16_bits(Wq), S.bf16_bits(Wk), S.bf16_bits(Wv), n_h, n_kv, d_h, t)
    assert np.array_equal(host_bits(out), ref)


# ---------------------------------------------------------------------------------- AllToAll
@pytest.mark.parametrize("t,rows,cols,split,concat,dtype", [
    (4, 64, 256, 1, 0, "f32"), (4, 64, 256, 0, 1, "bf16"), (2, 32, 64, 0, 0, "f32"), (8, 64, 512, 1, 1, "bf16"),
    (3, 9, 12, 1, 0, "f32"), (4, 8, 20, 0, 1, "bf16"), (8, 1024, 4096, 1, 0, "f32"),
])
def test_all_to_all_bit_exact(t, rows, cols, split, concat, dtype):
    ins = _payload(t, rows, cols, dtype, seed=rows + cols + t)
    ref = OC.all_to_all([host_bits(x) for x in ins], split_axis=split, concat_axis=concat)
    d_in = [cuda(x) for x in ins]
    d_out = [torch.empty(ref[0].shape, dtype=TD[dtype], device="cuda") for _ in range(t)]
    tp.tp_all_to_all(d_in, d_out, rows, cols, split, concat, TPD[dtype], t)
    torch.cuda.synchronize()
    for j in range(t):
        assert same_bits(host_bits(d_out[j]), ref[j]), f"shard {j}"


def test_all_to_all_moves_the_sharded_dim():
    # "Scaling Book 入门第 6 章", §6.4: AllToAll_{X,J}(A[I_X, J]) -> A[I, J_X]
    t, I, J = 4, 64, 128
    A = S.Draw(3).normal((I, J), 1.0, dtype=torch.float32)
    ins = [cuda(b) for b in A.chunk(t, 0)]
    outs = [torch.empty((I, J // t), device="cuda") for _ in range(t)]
    tp.tp_all_to_all(ins, outs, I // t, J, 1, 0, tp.TP_F32, t)
    torch.cuda.synchronize()
    for j in range(t):
        assert torch.equal(outs[j].cpu(), A[:, j * J // t:(j + 1) * J // t])


# ---------------------------------------------------------------------------------- per-hop bf16 mode
@pytest.mark.parametrize("t,rows,cols,axis", [(2, 64, 256, 0), (3, 96, 72, 0), (4, 64, 256, 1), (8, 512, 4096, 0),
                                              (5, 40, 80, 1), (3, 9, 7, 0), (4, 1028, 4104, 0), (16, 256, 512, 0),
                                              (16, 64, 1024, 1), (1, 8, 16, 0)])
def test_per_hop_bf16_reduce_scatter_and_all_reduce_bit_exact(t, rows, cols, axis):
    ins = _payload(t, rows, cols, "bf16", seed=900 + t * rows + cols)
    d_in = [cuda(x) for x in ins]
    oshape = (rows // t, cols) if axis == 0 else (rows, cols // t)
    rs = [torch.empty(oshape, dtype=torch.bfloat16, device="cuda") for _ in range(t)]
    tp.tp_reduce_scatter(d_in, rs, rows, cols, axis, tp.TP_BF16_RING, t)
    ar = [torch.empty((rows, cols), dtype=torch.bfloat16, device="cuda") for _ in range(t)]
    if axis == 0:
        tp.tp_all_reduce(d_in, ar, rows, cols, tp.TP_BF16_RING, t)
    torch.cuda.synchronize()
    bits = [host_bits(x) for x in ins]
    ref = OC.reduce_scatter(bits, axis=axis, dtype="bf16", rounding="hop")
    for r in range(t):
        assert same_bits(host_bits(rs[r]), ref[r]), f"RS shard {r}"
    if axis == 0:
        full = OC.all_reduce(bits, dtype="bf16", rounding="hop")
        for r in range(t):
            assert same_bits(host_bits(ar[r]), full[r]), f"AR replica {r}"


def test_per_hop_and_end_rounding_differ_where_the_oracle_says():
    # t = 3; chunk 0 sums U[1] = 1, U[2] = 2^-8, U[0] = 2^-8 in that order: one rounding at the end
    # gives 1 + 2^-7 (0x3F81), rounding after every hop gives 1 (0x3F80), as the oracle's pins state.
    t, rows, cols = 3, 3, 8
    vals = {0: 0x3B80, 1: 0x3F80, 2: 0x3B80}
    ins = []
    for d in range(t):
        b = np.zeros((rows, cols), dtype=np.uint16)
        b[0, :] = vals[d]
        ins.append(cuda(S.bits_to_bf16(b)))
    outs = {}
    for mode in (tp.TP_BF16, tp.TP_BF16_RING):
        o = [torch.empty((rows // t, cols), dtype=torch.bfloat16, device="cuda") for _ in range(t)]
        tp.tp_reduce_scatter(ins, o, rows, cols, 0, mode, t)
        torch.cuda.synchronize()
        outs[mode] = host_bits(o[0])
    assert np.all(outs[tp.TP_BF16] == 0x3F81)
    assert np.all(outs[tp.TP_BF16_RING] == 0x3F80)
