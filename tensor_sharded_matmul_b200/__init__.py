"""Python binding of libtp (the C ABI declared in include/tp.h).

Argument marshalling only: every function has the C entry point's name and argument order, accepts
torch tensors (or raw integer addresses) where the C side takes device pointers, lists of them where
it takes a host array of shard pointers, and an optional ``stream`` (default: torch's current
stream). A non-OK status raises ``TPError``. All work runs in the library's CUDA kernels; there is no
fallback path: importing this package fails if libtp.so has not been built.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtp.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python tensor_sharded_matmul_b200/build.py` "
                      "(or __graft_entry__.build()); there is no fallback implementation")

_lib = C.CDLL(LIB_PATH)

# ---- enums (values of include/tp.h) ----------------------------------------------------------
TP_OK, TP_EINVAL, TP_ESHAPE, TP_EDIVIS, TP_EALIGN, TP_ECUDA, TP_ETIMEOUT, TP_EUNSUPPORTED, TP_ENOSPACE = range(9)
TP_F32, TP_BF16, TP_BF16_RING = 0, 1, 2
TP_ACT_NONE, TP_ACT_GELU, TP_ACT_GELU_TANH, TP_ACT_SWIGLU = 0, 1, 2, 3
TP_OUT_PARTIALS, TP_OUT_RS, TP_OUT_AR, TP_OUT_RS_AG = 0, 1, 2, 3
TP_CASE1_LOCAL = 0
TP_CASE2_ALLGATHER, TP_CASE2_ALLREDUCE = 0, 1
TP_CASE3_ALLREDUCE, TP_CASE3_RS_B, TP_CASE3_RS_F = 0, 1, 2
TP_CASE4_GATHER_X, TP_CASE4_GATHER_W = 0, 1
TP_MAX_SHARDS = 16

EXPORTED = (
    "tp_status_str", "tp_last_error", "tp_device_status", "tp_set_wait_budget", "tp_selftest_wait_timeout",
    "tp_num_sms", "tp_shard_cols", "tp_shard_rows", "tp_shard_gate_up", "tp_shard_qkv", "tp_reduce_scatter",
    "tp_all_gather", "tp_all_reduce", "tp_grouped_gemm", "tp_column_linear", "tp_row_linear", "tp_row_linear_reduce", "tp_mlp_fwd",
    "tp_sharded_matmul_ws_bytes", "tp_sharded_matmul_choose", "tp_sharded_matmul", "tp_layer_fwd", "tp_mlp_fwd_noalloc",
    "tp_column_linear_sp", "tp_mlp_fwd_sp", "tp_all_to_all", "tp_grouped_gemm_t", "tp_mlp_bwd",
)

_vp, _i64, _i32, _u64, _sz = C.c_void_p, C.c_int64, C.c_int, C.c_uint64, C.c_size_t
_pp = C.POINTER(C.c_void_p)

_SIGS = {
    "tp_status_str": (C.c_char_p, [_i32]),
    "tp_last_error": (C.c_char_p, []),
    "tp_device_status": (_i32, [_i32, C.POINTER(C.c_uint32)]),
    "tp_set_wait_budget": (None, [_u64]),
    "tp_selftest_wait_timeout": (_i32, [_u64, _vp]),
    "tp_num_sms": (_i32, []),
    "tp_shard_cols": (_i32, [_vp, _i64, _i64, _i64, _i32, _vp, _vp]),
    "tp_shard_rows": (_i32, [_vp, _i64, _i64, _i64, _i32, _vp, _vp]),
    "tp_shard_gate_up": (_i32, [_vp, _i64, _vp, _i64, _i64, _i64, _i32, _vp, _vp]),
    "tp_shard_qkv": (_i32, [_vp, _i64, _vp, _i64, _vp, _i64, _i64, _i32, _i32, _i32, _i32, _vp, _vp]),
    "tp_reduce_scatter": (_i32, [_pp, _pp, _i64, _i64, _i32, _i32, _i32, _vp]),
    "tp_all_gather": (_i32, [_pp, _pp, _i64, _i64, _i32, _i32, _i32, _vp]),
    "tp_all_reduce": (_i32, [_pp, _pp, _i64, _i64, _i32, _i32, _vp]),
    "tp_all_to_all": (_i32, [_pp, _pp, _i64, _i64, _i32, _i32, _i32, _i32, _vp]),
    "tp_grouped_gemm": (_i32, [_i32, _pp, _pp, _pp, _i64, _i64, _i64, _i32, _i32, _vp]),
    "tp_grouped_gemm_t": (_i32, [_i32, _pp, _i32, _pp, _i32, _pp, _i64, _i64, _i64, _i32, _vp]),
    "tp_mlp_bwd": (_i32, [_vp, _vp, _i64, _i64, _i64, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _pp, _vp]),
    "tp_column_linear": (_i32, [_vp, _i64, _i64, _i64, _i32, _i32, _vp, _vp, _vp]),
    "tp_row_linear": (_i32, [_vp, _i64, _i64, _i64, _i32, _vp, _pp, _vp]),
    "tp_row_linear_reduce": (_i32, [_vp, _i64, _i64, _i64, _i32, _vp, _i32, _i32, _pp, _pp, _vp]),
    "tp_mlp_fwd": (_i32, [_vp, _i64, _i64, _i64, _i32, _i32, _vp, _vp, _vp, _pp, _i32, _pp, _vp]),
    "tp_mlp_fwd_noalloc": (_i32, [_vp, _i64, _i64, _i64, _i32, _i32, _vp, _vp, _i32, _pp, _vp]),
    "tp_column_linear_sp": (_i32, [_pp, _i64, _i64, _i64, _i32, _i32, _vp, _vp, _vp]),
    "tp_mlp_fwd_sp": (_i32, [_pp, _i64, _i64, _i64, _i32, _i32, _vp, _vp, _vp, _pp, _vp]),
    "tp_sharded_matmul_ws_bytes": (_sz, [_i32, _i32, _i64, _i64, _i64, _i32]),
    "tp_sharded_matmul_choose": (_i32, [_i32, _i64, _i64, _i64, _i32, C.POINTER(C.c_int)]),
    "tp_sharded_matmul": (_i32, [_i32, _i32, _pp, _pp, _i64, _i64, _i64, _i32, _pp, _i32, _vp, _sz, _vp]),
    "tp_layer_fwd": (_i32, [_vp, _pp, _i64, _i64, _i32, _i32, _i32, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _pp,
                            _vp, _vp, _pp, _pp, _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class TPError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.tp_status_str(status).decode()
        detail = _lib.tp_last_error().decode()
        super().__init__(f"{where}: {msg} ({detail})" if detail else f"{where}: {msg}")


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _ptrs(xs):
    if xs is None:
        return None
    arr = (C.c_void_p * len(xs))(*[_ptr(x) for x in xs])
    return C.cast(arr, _pp)


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _call(name, *args):
    st = getattr(_lib, name)(*args)
    if st != TP_OK:
        raise TPError(st, name)


# ---- status -----------------------------------------------------------------------------------
def tp_status_str(status: int) -> str:
    return _lib.tp_status_str(status).decode()


def tp_last_error() -> str:
    return _lib.tp_last_error().decode()


def tp_device_status(clear: int = 1):
    """Returns (status, site) after synchronising; does not raise."""
    where = C.c_uint32(0)
    st = _lib.tp_device_status(clear, C.byref(where))
    return st, where.value


def tp_set_wait_budget(cycles: int) -> None:
    _lib.tp_set_wait_budget(cycles)


def tp_selftest_wait_timeout(budget_cycles: int, stream=None) -> None:
    _call("tp_selftest_wait_timeout", budget_cycles, _stream(stream))


def tp_num_sms() -> int:
    return _lib.tp_num_sms()


# ---- layouts ----------------------------------------------------------------------------------
def tp_shard_cols(w, ld, K, N, t, out, stream=None):
    _call("tp_shard_cols", _ptr(w), ld, K, N, t, _ptr(out), _stream(stream))


def tp_shard_rows(w, ld, K, N, t, out, stream=None):
    _call("tp_shard_rows", _ptr(w), ld, K, N, t, _ptr(out), _stream(stream))


def tp_shard_gate_up(w_gate, ld_g, w_up, ld_u, h, F, t, out, stream=None):
    _call("tp_shard_gate_up", _ptr(w_gate), ld_g, _ptr(w_up), ld_u, h, F, t, _ptr(out), _stream(stream))


def tp_shard_qkv(w_q, ld_q, w_k, ld_k, w_v, ld_v, h, n_h, n_kv, d_h, t, out, stream=None):
    _call("tp_shard_qkv", _ptr(w_q), ld_q, _ptr(w_k), ld_k, _ptr(w_v), ld_v, h, n_h, n_kv, d_h, t, _ptr(out),
          _stream(stream))


# ---- collectives ------------------------------------------------------------------------------
def tp_reduce_scatter(ins, outs, rows, cols, axis, dtype, t, stream=None):
    _call("tp_reduce_scatter", _ptrs(ins), _ptrs(outs), rows, cols, axis, dtype, t, _stream(stream))


def tp_all_gather(ins, outs, rows, cols, axis, dtype, t, stream=None):
    _call("tp_all_gather", _ptrs(ins), _ptrs(outs), rows, cols, axis, dtype, t, _stream(stream))


def tp_all_reduce(ins, outs, rows, cols, dtype, t, stream=None):
    _call("tp_all_reduce", _ptrs(ins), _ptrs(outs), rows, cols, dtype, t, _stream(stream))


def tp_all_to_all(ins, outs, rows, cols, split_axis, concat_axis, dtype, t, stream=None):
    _call("tp_all_to_all", _ptrs(ins), _ptrs(outs), rows, cols, split_axis, concat_axis, dtype, t, _stream(stream))


# ---- GEMMs, MLP, cases, layer -----------------------------------------------------------------
def tp_grouped_gemm(groups, a, b, c, M, N, K, act, c_dtype, stream=None):
    _call("tp_grouped_gemm", groups, _ptrs(a), _ptrs(b), _ptrs(c), M, N, K, act, c_dtype, _stream(stream))


def tp_grouped_gemm_t(groups, a, trans_a, b, trans_b, c, M, N, K, c_dtype, stream=None):
    _call("tp_grouped_gemm_t", groups, _ptrs(a), trans_a, _ptrs(b), trans_b, _ptrs(c), M, N, K, c_dtype,
          _stream(stream))


def tp_mlp_bwd(x, dy, N, h, F, t, act, w_in, w_down, h_pre, z, dz_ws, dh_ws, dw_in, dw_down, dx, stream=None):
    _call("tp_mlp_bwd", _ptr(x), _ptr(dy), N, h, F, t, act, _ptr(w_in), _ptr(w_down), _ptr(h_pre), _ptr(z),
          _ptr(dz_ws), _ptr(dh_ws), _ptr(dw_in), _ptr(dw_down), _ptrs(dx), _stream(stream))


def tp_column_linear(x, N, k, n, t, act, w, y, stream=None):
    _call("tp_column_linear", _ptr(x), N, k, n, t, act, _ptr(w), _ptr(y), _stream(stream))


def tp_row_linear(x, N, k, n, t, w, partials, stream=None):
    _call("tp_row_linear", _ptr(x), N, k, n, t, _ptr(w), _ptrs(partials), _stream(stream))


def tp_row_linear_reduce(x, N, k, n, t, w, mode, axis, out, partials=None, stream=None):
    _call("tp_row_linear_reduce", _ptr(x), N, k, n, t, _ptr(w), mode, axis, _ptrs(out), _ptrs(partials),
          _stream(stream))


def tp_mlp_fwd(x, N, h, F, t, act, w_in, w_down, z_ws, partials, mode, out, stream=None):
    _call("tp_mlp_fwd", _ptr(x), N, h, F, t, act, _ptr(w_in), _ptr(w_down), _ptr(z_ws), _ptrs(partials), mode,
          _ptrs(out), _stream(stream))


def tp_mlp_fwd_noalloc(x, N, h, F, t, act, w_in, w_down, mode, out, stream=None):
    """tp_mlp_fwd for callers that cannot allocate device memory: the scratch is a fixed array inside
    the library (TP_MLP_NOALLOC_SCRATCH_BYTES); see include/tp.h for its limits and sharing rules."""
    _call("tp_mlp_fwd_noalloc", _ptr(x), N, h, F, t, act, _ptr(w_in), _ptr(w_down), mode, _ptrs(out),
          _stream(stream))


TP_MLP_NOALLOC_SCRATCH_BYTES = 32 << 20


def tp_column_linear_sp(x, N, k, n, t, act, w, y, stream=None):
    _call("tp_column_linear_sp", _ptrs(x), N, k, n, t, act, _ptr(w), _ptr(y), _stream(stream))


def tp_mlp_fwd_sp(x, N, h, F, t, act, w_in, w_down, z_ws, out, stream=None):
    _call("tp_mlp_fwd_sp", _ptrs(x), N, h, F, t, act, _ptr(w_in), _ptr(w_down), _ptr(z_ws), _ptrs(out),
          _stream(stream))


def tp_sharded_matmul_ws_bytes(case_id, strategy, B, D, F, t) -> int:
    return int(_lib.tp_sharded_matmul_ws_bytes(case_id, strategy, B, D, F, t))


def tp_sharded_matmul_choose(case_id, B, D, F, t) -> int:
    """The strategy the pages' cost rule picks for case 1, 2 or 4 (see include/tp.h)."""
    out = C.c_int(-1)
    _call("tp_sharded_matmul_choose", case_id, B, D, F, t, C.byref(out))
    return out.value


def tp_sharded_matmul(case_id, strategy, x, w, B, D, F, t, c, c_dtype, ws, ws_bytes, stream=None):
    _call("tp_sharded_matmul", case_id, strategy, _ptrs(x), _ptrs(w), B, D, F, t, _ptrs(c), c_dtype, _ptr(ws),
          ws_bytes, _stream(stream))


def tp_layer_fwd(x, o, N, h, n_h, n_kv, d_h, F, t, w_qkv, w_o, w_gu, w_down, qkv_out, h1, h1_bf16, z_ws, partials,
                 y, stream=None):
    _call("tp_layer_fwd", _ptr(x), _ptrs(o), N, h, n_h, n_kv, d_h, F, t, _ptr(w_qkv), _ptr(w_o), _ptr(w_gu),
          _ptr(w_down), _ptr(qkv_out), _ptrs(h1), _ptr(h1_bf16), _ptr(z_ws), _ptrs(partials), _ptrs(y),
          _stream(stream))
