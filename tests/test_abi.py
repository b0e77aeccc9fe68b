"""The C ABI library loads, exports every entry point include/tp.h declares, and rejects bad
arguments on the host before launching anything (CPU only: no call here reaches the GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

import tensor_sharded_matmul_b200 as tp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tp.h")


def declared_functions():
    src = open(HEADER, encoding="utf-8").read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tp_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("tp_shard_qkv", "tp_shard_gate_up", "tp_mlp_fwd", "tp_sharded_matmul", "tp_reduce_scatter",
                 "tp_all_gather", "tp_all_reduce"):
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(tp.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    out = subprocess.run(["nm", "-D", "--defined-only", tp.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (tp_\w+)", out))
    assert set(declared_functions()) <= exported


def test_binding_has_the_same_names():
    assert set(declared_functions()) == set(tp.EXPORTED)
    for n in declared_functions():
        assert callable(getattr(tp, n))


def test_status_strings():
    assert tp.tp_status_str(tp.TP_OK) == "ok"
    assert "divide" in tp.tp_status_str(tp.TP_EDIVIS)
    assert tp.tp_status_str(99) == "unknown status"


def _expect(status, fn, *args):
    with pytest.raises(tp.TPError) as e:
        fn(*args)
    assert e.value.status == status, str(e.value)


FAKE = 1 << 20   # a 16-byte aligned non-null address; never dereferenced (calls fail validation first)


def test_collectives_validate_before_launch():
    _expect(tp.TP_EINVAL, tp.tp_reduce_scatter, [FAKE] * 17, [FAKE] * 17, 16, 16, 0, tp.TP_F32, 17, 0)
    _expect(tp.TP_EINVAL, tp.tp_reduce_scatter, [FAKE], [FAKE], 16, 16, 0, tp.TP_F32, 0, 0)
    _expect(tp.TP_EDIVIS, tp.tp_reduce_scatter, [FAKE] * 3, [FAKE] * 3, 16, 16, 0, tp.TP_F32, 3, 0)
    _expect(tp.TP_EDIVIS, tp.tp_all_gather, [FAKE] * 3, [FAKE] * 3, 16, 16, 1, tp.TP_BF16, 3, 0)
    _expect(tp.TP_EINVAL, tp.tp_all_reduce, [FAKE, 0], [FAKE, FAKE], 16, 16, tp.TP_F32, 2, 0)
    _expect(tp.TP_EINVAL, tp.tp_reduce_scatter, [FAKE] * 2, [FAKE] * 2, 16, 16, 2, tp.TP_F32, 2, 0)
    _expect(tp.TP_EINVAL, tp.tp_reduce_scatter, [FAKE] * 2, [FAKE] * 2, -2, 16, 0, tp.TP_F32, 2, 0)


def test_layouts_validate_before_launch():
    _expect(tp.TP_EDIVIS, tp.tp_shard_cols, FAKE, 30, 8, 30, 4, FAKE, 0)
    _expect(tp.TP_EDIVIS, tp.tp_shard_rows, FAKE, 8, 30, 8, 4, FAKE, 0)
    _expect(tp.TP_EINVAL, tp.tp_shard_cols, FAKE, 8, 8, 16, 2, FAKE, 0)            # ld < N
    # t must divide n_h; KV heads split (t | n_kv) or replicated (n_kv | t)
    _expect(tp.TP_EDIVIS, tp.tp_shard_qkv, FAKE, 64, FAKE, 16, FAKE, 16, 64, 8, 2, 8, 3, FAKE, 0)
    _expect(tp.TP_EDIVIS, tp.tp_shard_qkv, FAKE, 48, FAKE, 16, FAKE, 16, 64, 6, 2, 8, 4, FAKE, 0)  # 2 | 4 ok, 4 | 6 no
    _expect(tp.TP_EDIVIS, tp.tp_shard_qkv, FAKE, 64, FAKE, 32, FAKE, 32, 64, 8, 4, 8, 16, FAKE, 0)  # t > n_h


def test_gemm_and_mlp_validate_before_launch():
    _expect(tp.TP_EALIGN, tp.tp_grouped_gemm, 1, [FAKE], [FAKE], [FAKE], 64, 64, 60, tp.TP_ACT_NONE, tp.TP_F32, 0)
    _expect(tp.TP_EALIGN, tp.tp_grouped_gemm, 1, [FAKE + 8], [FAKE], [FAKE], 64, 64, 64, tp.TP_ACT_NONE, tp.TP_F32, 0)
    _expect(tp.TP_EINVAL, tp.tp_grouped_gemm, 1, [FAKE], [FAKE], [FAKE], 64, 64, 64, tp.TP_ACT_GELU, tp.TP_F32, 0)
    _expect(tp.TP_EINVAL, tp.tp_grouped_gemm, 0, [], [], [], 64, 64, 64, tp.TP_ACT_NONE, tp.TP_F32, 0)
    _expect(tp.TP_EDIVIS, tp.tp_mlp_fwd, FAKE, 64, 256, 1000, 3, tp.TP_ACT_GELU, FAKE, FAKE, FAKE, [FAKE] * 3,
            tp.TP_OUT_PARTIALS, None, 0)
    _expect(tp.TP_EDIVIS, tp.tp_mlp_fwd, FAKE, 66, 256, 1024, 4, tp.TP_ACT_GELU, FAKE, FAKE, FAKE, [FAKE] * 4,
            tp.TP_OUT_RS, [FAKE] * 4, 0)
    _expect(tp.TP_EINVAL, tp.tp_mlp_fwd, FAKE, 64, 256, 1024, 4, 9, FAKE, FAKE, FAKE, [FAKE] * 4,
            tp.TP_OUT_PARTIALS, None, 0)


def test_sharded_matmul_workspace_sizes_and_validation():
    B, D, F, t = 8192, 8192, 28672, 4
    assert tp.tp_sharded_matmul_ws_bytes(1, 0, B, D, F, t) == 0
    # the gathering strategies read the gathered operand's pieces in place when they are whole
    # 64-wide k-blocks (case 2), 128-row tiles (case 4, X) or 64-column boxes (case 4, W) ...
    assert tp.tp_sharded_matmul_ws_bytes(2, tp.TP_CASE2_ALLGATHER, B, D, F, t) == 0
    assert tp.tp_sharded_matmul_ws_bytes(4, tp.TP_CASE4_GATHER_X, B, D, F, t) == 0
    assert tp.tp_sharded_matmul_ws_bytes(4, tp.TP_CASE4_GATHER_W, B, D, F, t) == 0
    # ... and materialise the gather otherwise (one gathered copy per shard)
    assert tp.tp_sharded_matmul_ws_bytes(2, tp.TP_CASE2_ALLGATHER, B, 96 * 4, F, t) == t * B * 384 * 2
    assert tp.tp_sharded_matmul_ws_bytes(4, tp.TP_CASE4_GATHER_X, 64 * 4, D, F, t) == t * 256 * D * 2
    assert tp.tp_sharded_matmul_ws_bytes(4, tp.TP_CASE4_GATHER_W, B, D, 96 * 4, t) == t * D * 384 * 2
    # the fused row GEMM + ring reduction needs no workspace when the chunks are whole tiles ...
    assert tp.tp_sharded_matmul_ws_bytes(2, tp.TP_CASE2_ALLREDUCE, B, D, F, t) == 0
    assert tp.tp_sharded_matmul_ws_bytes(3, tp.TP_CASE3_RS_F, B, D, F, t) == 0
    assert tp.tp_sharded_matmul_ws_bytes(3, tp.TP_CASE3_RS_B, B, D, F, t) == 0
    # ... and the unfused path's fp32 partials otherwise (B/t = 24 rows: no whole 128-row tile)
    assert tp.tp_sharded_matmul_ws_bytes(2, tp.TP_CASE2_ALLREDUCE, 96, D, F, t) == t * 96 * F * 4
    assert tp.tp_sharded_matmul_ws_bytes(3, tp.TP_CASE3_RS_B, 96, D, F, t) == t * 96 * F * 4
    assert tp.tp_sharded_matmul_ws_bytes(3, tp.TP_CASE3_RS_F, B, D, 1000, t) == t * B * 1000 * 4
    _expect(tp.TP_ENOSPACE, tp.tp_sharded_matmul, 3, 0, [FAKE] * 4, [FAKE] * 4, 64, 64, 64, 4, [FAKE] * 4, tp.TP_F32,
            FAKE, 10, 0)
    _expect(tp.TP_EINVAL, tp.tp_sharded_matmul, 5, 0, [FAKE] * 4, [FAKE] * 4, 64, 64, 64, 4, [FAKE] * 4, tp.TP_F32,
            FAKE, 1 << 30, 0)
    _expect(tp.TP_EDIVIS, tp.tp_sharded_matmul, 3, 0, [FAKE] * 3, [FAKE] * 3, 64, 64, 64, 3, [FAKE] * 3, tp.TP_F32,
            FAKE, 1 << 30, 0)


def test_layer_validates_head_split():
    args = [FAKE, [FAKE] * 3, 96, 256, 8, 2, 32, 768, 3, FAKE, FAKE, FAKE, FAKE, FAKE, [FAKE] * 3, FAKE, FAKE,
            [FAKE] * 3, [FAKE] * 3, 0]
    _expect(tp.TP_EDIVIS, tp.tp_layer_fwd, *args)


def test_empty_inputs_are_noops_without_a_gpu():
    """A zero token/row count returns TP_OK having read no data pointer and launched nothing, which
    is why these calls succeed on a host with no GPU (null data pointers included: an empty tensor
    may have none). t and the sizes are still validated."""
    E = [0, 0]
    tp.tp_reduce_scatter(E, E, 0, 16, 0, tp.TP_F32, 2, 0)
    tp.tp_all_gather(E, E, 16, 0, 1, tp.TP_BF16, 2, 0)
    tp.tp_all_reduce(E, E, 0, 0, tp.TP_F32, 2, 0)
    tp.tp_all_to_all(E, E, 0, 16, 0, 1, tp.TP_BF16, 2, 0)
    tp.tp_shard_cols(0, 16, 0, 16, 2, FAKE, 0)
    tp.tp_shard_gate_up(0, 16, 0, 16, 0, 16, 2, FAKE, 0)
    tp.tp_grouped_gemm(2, E, E, E, 0, 64, 64, tp.TP_ACT_NONE, tp.TP_F32, 0)
    tp.tp_grouped_gemm_t(2, E, 1, E, 1, E, 64, 0, 64, tp.TP_BF16, 0)
    tp.tp_column_linear(0, 0, 256, 1024, 4, tp.TP_ACT_GELU, 0, 0, 0)
    tp.tp_row_linear(0, 0, 1024, 256, 4, 0, [0] * 4, 0)
    tp.tp_row_linear_reduce(0, 0, 1024, 256, 4, 0, tp.TP_OUT_AR, 0, [0] * 4, None, 0)
    tp.tp_mlp_fwd(0, 0, 256, 1024, 4, tp.TP_ACT_SWIGLU, 0, 0, 0, None, tp.TP_OUT_RS, [0] * 4, 0)
    tp.tp_mlp_fwd_noalloc(0, 0, 256, 1024, 4, tp.TP_ACT_GELU, 0, 0, tp.TP_OUT_AR, [0] * 4, 0)
    tp.tp_mlp_fwd_sp([0] * 4, 0, 256, 1024, 4, tp.TP_ACT_GELU, 0, 0, 0, [0] * 4, 0)
    tp.tp_mlp_bwd(0, 0, 0, 256, 1024, 4, tp.TP_ACT_GELU, 0, 0, 0, 0, 0, 0, 0, 0, [0] * 4, 0)
    tp.tp_sharded_matmul(3, 0, [0] * 4, [0] * 4, 0, 64, 64, 4, [0] * 4, tp.TP_F32, 0, 0, 0)
    tp.tp_layer_fwd(0, [0] * 2, 0, 256, 8, 2, 32, 768, 2, 0, 0, 0, 0, 0, [0] * 2, 0, 0, None, [0] * 2, 0)
    # still validated: t, negative sizes, empty contractions
    _expect(tp.TP_EINVAL, tp.tp_column_linear, 0, 0, 256, 1024, 0, tp.TP_ACT_GELU, 0, 0, 0)
    _expect(tp.TP_EINVAL, tp.tp_column_linear, 0, -1, 256, 1024, 4, tp.TP_ACT_GELU, 0, 0, 0)
    _expect(tp.TP_EINVAL, tp.tp_grouped_gemm, 1, [FAKE], [FAKE], [FAKE], 64, 64, 0, tp.TP_ACT_NONE, tp.TP_F32, 0)
    _expect(tp.TP_EINVAL, tp.tp_mlp_fwd, 0, 0, 0, 1024, 4, tp.TP_ACT_GELU, 0, 0, 0, None, tp.TP_OUT_RS, [0] * 4, 0)


def test_oversized_problems_are_rejected_before_launch():
    """Sizes past the kernels' 32-bit tile coordinates give TP_ESHAPE on the host (no GPU needed)."""
    big = 1 << 31
    _expect(tp.TP_ESHAPE, tp.tp_grouped_gemm, 1, [FAKE], [FAKE], [FAKE], big, 64, 64, tp.TP_ACT_NONE, tp.TP_F32, 0)
    _expect(tp.TP_ESHAPE, tp.tp_grouped_gemm, 1, [FAKE], [FAKE], [FAKE], 256, 64, big, tp.TP_ACT_NONE, tp.TP_F32, 0)
    _expect(tp.TP_ESHAPE, tp.tp_grouped_gemm_t, 1, [FAKE], 1, [FAKE], 1, [FAKE], 256, big, 64, tp.TP_F32, 0)
    _expect(tp.TP_ESHAPE, tp.tp_row_linear_reduce, FAKE, big, 1024, 512, 4, FAKE, tp.TP_OUT_AR, 0, [FAKE] * 4)
    # the maximum shard count is accepted up to validation, one more is not
    _expect(tp.TP_EDIVIS, tp.tp_reduce_scatter, [FAKE] * 16, [FAKE] * 16, 24, 16, 0, tp.TP_F32, 16, 0)
    _expect(tp.TP_EINVAL, tp.tp_mlp_fwd, FAKE, 64, 256, 1024, 17, tp.TP_ACT_GELU, FAKE, FAKE, FAKE, [FAKE] * 17,
            tp.TP_OUT_PARTIALS, None, 0)


def test_noalloc_scratch_bound_cannot_wrap():
    """tp_mlp_fwd_noalloc bounds every size before multiplying it: sizes whose byte counts would wrap
    a 64-bit product (and so slip past a check done after the multiplication) give TP_ENOSPACE on
    the host, before the scratch array is looked up or anything is launched."""
    huge = 1 << 62
    A = tp.TP_ACT_GELU
    # the activations' N*F*2 alone would wrap
    _expect(tp.TP_ENOSPACE, tp.tp_mlp_fwd_noalloc, FAKE, huge, 256, 8, 4, A, FAKE, FAKE, tp.TP_OUT_PARTIALS, [FAKE] * 4, 0)
    _expect(tp.TP_ENOSPACE, tp.tp_mlp_fwd_noalloc, FAKE, 8, 256, huge, 4, A, FAKE, FAKE, tp.TP_OUT_AR, [FAKE] * 4, 0)
    # small Z, but the unfused path's t*N*h*4 partials would wrap (N/t = 1 row: not fusable)
    _expect(tp.TP_ENOSPACE, tp.tp_mlp_fwd_noalloc, FAKE, 4, huge, 8, 4, A, FAKE, FAKE, tp.TP_OUT_AR, [FAKE] * 4, 0)
    # in range but larger than the array
    _expect(tp.TP_ENOSPACE, tp.tp_mlp_fwd_noalloc, FAKE, 4096, 4096, 14336, 8, tp.TP_ACT_SWIGLU, FAKE, FAKE,
            tp.TP_OUT_PARTIALS, [FAKE] * 8, 0)


def test_per_hop_bf16_is_a_ring_collective_mode_only():
    """TP_BF16_RING is accepted by the ring collectives and refused elsewhere, on the host."""
    _expect(tp.TP_EINVAL, tp.tp_grouped_gemm, 1, [FAKE], [FAKE], [FAKE], 64, 64, 64, tp.TP_ACT_NONE, tp.TP_BF16_RING, 0)
    _expect(tp.TP_EINVAL, tp.tp_all_to_all, [FAKE] * 2, [FAKE] * 2, 16, 16, 0, 1, tp.TP_BF16_RING, 2, 0)
    _expect(tp.TP_EINVAL, tp.tp_reduce_scatter, [FAKE] * 2, [FAKE] * 2, 16, 16, 0, 3, 2, 0)   # unknown dtype
    # empty inputs pass validation in the per-hop mode like in the others
    tp.tp_reduce_scatter([0, 0], [0, 0], 0, 16, 0, tp.TP_BF16_RING, 2, 0)
    tp.tp_all_reduce([0, 0], [0, 0], 0, 16, tp.TP_BF16_RING, 2, 0)


def test_strategy_choice_matches_the_oracle_rule():
    """tp_sharded_matmul_choose applies the pages' byte rule (case 2: AllGather of X unless it moves
    more than the AllReduce of C; case 4: gather the smaller operand) like oracle.cases does."""
    from oracle import cases as OC
    code2 = {"allgather": tp.TP_CASE2_ALLGATHER, "allreduce": tp.TP_CASE2_ALLREDUCE}
    code4 = {"gather_x": tp.TP_CASE4_GATHER_X, "gather_w": tp.TP_CASE4_GATHER_W}
    shapes = [(8192, 8192, 28672), (4096, 4096, 14336), (64, 256, 1024)]
    for B in (8, 256, 4096):
        for F in (B // 2, B, 2 * B):
            for D in (2 * F - 8, 2 * F, 2 * F + 8):   # around the case-2 boundary B*D = 2*B*F
                if D > 0:
                    shapes.append((B, D, F))
    shapes += [(B, 512, B + d) for B in (16, 1024) for d in (-8, 0, 8)]   # around the case-4 boundary
    for B, D, F in shapes:
        assert tp.tp_sharded_matmul_choose(1, B, D, F, 4) == tp.TP_CASE1_LOCAL
        assert tp.tp_sharded_matmul_choose(2, B, D, F, 4) == code2[OC.case2_choice(B * D, B * F)], (B, D, F)
        assert tp.tp_sharded_matmul_choose(4, B, D, F, 4) == code4[OC.case4_choice(B, D, F)], (B, D, F)
    # the benchmark's configuration: gather X for both cases
    assert tp.tp_sharded_matmul_choose(2, 8192, 8192, 28672, 4) == tp.TP_CASE2_ALLGATHER
    assert tp.tp_sharded_matmul_choose(4, 8192, 8192, 28672, 4) == tp.TP_CASE4_GATHER_X
    # huge sizes do not overflow the comparison
    assert tp.tp_sharded_matmul_choose(2, 1 << 40, 1 << 41, 1 << 40, 4) == tp.TP_CASE2_ALLGATHER
    assert tp.tp_sharded_matmul_choose(2, 1 << 40, (1 << 41) + 8, 1 << 40, 4) == tp.TP_CASE2_ALLREDUCE
    _expect(tp.TP_EUNSUPPORTED, tp.tp_sharded_matmul_choose, 3, 8192, 8192, 28672, 4)
    _expect(tp.TP_EINVAL, tp.tp_sharded_matmul_choose, 5, 8192, 8192, 28672, 4)
    _expect(tp.TP_EINVAL, tp.tp_sharded_matmul_choose, 2, 0, 8192, 28672, 4)
    _expect(tp.TP_EINVAL, tp.tp_sharded_matmul_choose, 2, 8192, 8192, 28672, 17)

