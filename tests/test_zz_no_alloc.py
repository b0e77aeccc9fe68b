"""tp_mlp_fwd_noalloc, the MLP forward for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc. One case is code inside a host framework whose caching pool
owns the GPU's memory: an allocation behind the pool's back can fail or escape its accounting.
Another is a serving loop that forbids allocation after start-up, because cudaMalloc/cudaFree can
synchronise the device. For them the library keeps the MLP's scratch (activations and fp32 partial
sums) in a fixed array of its own.

This test calls that entry point through the C ABI twice in a row, on different shapes, inputs and
modes. Both entry points launch the same kernels on the same inputs, so each result must equal
tp_mlp_fwd's bit for bit; a tolerance could hide stale scratch or a wrong offset inside the array.
Shapes with (N/t) % 128 == 0 take the fused row GEMM + reduction, which needs no room for the fp32
partials, so the Llama-3-8B-shaped MLP on 1024 tokens (29.4 MB of activations) fits the array. It
also checks that a request too large for the array is refused. It does not depend on other tests
having run first.
"""
import pytest
import torch

import synthetic as S
import tensor_sharded_matmul_b200 as tp

pytestmark = pytest.mark.gpu


def _weights(N, h, F, t, act, seed):
    d = S.Draw(seed, "cuda")
    X = d.normal((N, h), 1.0)
    wn = 2 * F // t if act == tp.TP_ACT_SWIGLU else F // t
    w_in = d.normal((t, h, wn), 0.02)
    w_down = d.normal((t, F // t, h), 0.02)
    return X, w_in, w_down


def _outs(N, h, t, mode):
    rows = N // t if mode == tp.TP_OUT_RS else N
    return [torch.empty((rows, h), device="cuda") for _ in range(t)]


def _with_workspaces(X, w_in, w_down, N, h, F, t, act, mode):
    z = torch.empty((t, N, F // t), dtype=torch.bfloat16, device="cuda")
    partials = [torch.empty((N, h), device="cuda") for _ in range(t)]
    out = _outs(N, h, t, mode)
    tp.tp_mlp_fwd(X, N, h, F, t, act, w_in, w_down, z, partials, mode, out)
    return partials if mode == tp.TP_OUT_PARTIALS else out


def _check(N, h, F, t, act, mode, seed):
    X, w_in, w_down = _weights(N, h, F, t, act, seed)
    got = _outs(N, h, t, mode)
    tp.tp_mlp_fwd_noalloc(X, N, h, F, t, act, w_in, w_down, mode, got)
    torch.cuda.synchronize()
    ref = _with_workspaces(X, w_in, w_down, N, h, F, t, act, mode)
    torch.cuda.synchronize()
    st, site = tp.tp_device_status(1)
    assert st == tp.TP_OK, f"device wait site {site}"
    for r in range(t):
        assert torch.equal(got[r], ref[r]), f"shard {r} differs from tp_mlp_fwd"


def test_two_calls_in_a_row_match_tp_mlp_fwd():
    # First call: a small SwiGLU MLP reduced by ReduceScatter + AllGather.
    _check(N=256, h=1024, F=4096, t=4, act=tp.TP_ACT_SWIGLU, mode=tp.TP_OUT_RS_AG, seed=1)
    # Second call, right after: a different shape, activation and mode. It reuses the array the
    # first call left filled.
    _check(N=64, h=256, F=1024, t=4, act=tp.TP_ACT_GELU, mode=tp.TP_OUT_AR, seed=2)


def test_partials_and_reduce_scatter_modes():
    _check(N=128, h=512, F=2048, t=8, act=tp.TP_ACT_SWIGLU, mode=tp.TP_OUT_PARTIALS, seed=3)
    _check(N=128, h=512, F=2048, t=8, act=tp.TP_ACT_SWIGLU, mode=tp.TP_OUT_RS, seed=4)


def test_fused_path_fits_where_partials_would_not():
    # N/t = 128: the row GEMM is fused with its AllReduce, so only Z (1024 x 14336 bf16, 29.4 MB) needs
    # the array; the unfused path's 8 fp32 [1024, 4096] partials (134 MB) would not fit.
    _check(N=1024, h=4096, F=14336, t=8, act=tp.TP_ACT_SWIGLU, mode=tp.TP_OUT_RS_AG, seed=5)
    # and a small fused ReduceScatter right after it, on the array the first call left filled
    _check(N=1024, h=512, F=2048, t=8, act=tp.TP_ACT_GELU, mode=tp.TP_OUT_RS, seed=6)


def test_request_beyond_the_array_is_refused():
    N, h, F, t = 4096, 4096, 14336, 8     # needs about 0.6 GiB of scratch
    X, w_in, w_down = (torch.empty(8, dtype=torch.bfloat16, device="cuda") for _ in range(3))
    out = [torch.empty(8, device="cuda") for _ in range(t)]
    with pytest.raises(tp.TPError) as e:
        tp.tp_mlp_fwd_noalloc(X, N, h, F, t, tp.TP_ACT_SWIGLU, w_in, w_down, tp.TP_OUT_AR, out)
    assert e.value.status == tp.TP_ENOSPACE
    assert "scratch" in str(e.value)
