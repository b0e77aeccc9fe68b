// C entry points that compose the GEMM and ring kernels: the column/row parallel linear layers,
// the tensor-parallel MLP, the four sharded-matmul cases and one tensor-parallel layer.
// Argument validation happens here, before anything is launched.
#include <cstring>

#include "common.cuh"

namespace tpx {
namespace {

bool valid_act(tp_act a) { return a == TP_ACT_NONE || a == TP_ACT_GELU || a == TP_ACT_GELU_TANH || a == TP_ACT_SWIGLU; }
bool valid_dtype(tp_dtype d) { return d == TP_F32 || d == TP_BF16; }

EpiKind epi_for(tp_act act, tp_dtype c_dtype) {
  switch (act) {
    case TP_ACT_GELU: return EPI_GELU;
    case TP_ACT_GELU_TANH: return EPI_GELU_TANH;
    case TP_ACT_SWIGLU: return EPI_SWIGLU;
    default: return c_dtype == TP_F32 ? EPI_F32 : EPI_BF16;
  }
}

GemmArgs gemm_args(int groups, int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb, EpiKind epi) {
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  g.groups = groups; g.M = M; g.N = N; g.K = K; g.lda = lda; g.ldb = ldb; g.epi = epi;
  return g;
}

RingArgs ring_args(RingOp op, int t, int64_t rows, int64_t cols, int axis, tp_dtype din, tp_dtype dout) {
  RingArgs a;
  std::memset(&a, 0, sizeof(a));
  a.op = op; a.t = t; a.rows = rows; a.cols = cols; a.axis = axis; a.in_dtype = din; a.out_dtype = dout;
  a.resid_dtype = TP_F32;
  return a;
}

size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

// When the GEMM can read an AllGather's pieces where they lie instead of a gathered copy:
//   case 2 AllGather (X gathered along D, the contraction): every piece a whole number of 64-wide k-blocks;
//   case 4 gather X (X gathered along B, rows):             every piece a whole number of 128-row tiles;
//   case 4 gather W (W gathered along F, columns):          every piece a whole number of 64-wide column boxes.
bool gather_in_place(int case_id, int strategy, int64_t B, int64_t D, int64_t F, int t) {
  if (case_id == 2 && strategy == TP_CASE2_ALLGATHER) return D % t == 0 && (D / t) % 64 == 0;
  if (case_id == 4 && strategy == TP_CASE4_GATHER_X) return B % t == 0 && (B / t) % 128 == 0;
  if (case_id == 4 && strategy == TP_CASE4_GATHER_W) return F % t == 0 && (F / t) % 64 == 0;
  return false;
}

tp_status column_gemm(const uint16_t* x, int64_t N, int64_t k, int64_t n_shard, int t, tp_act act, const uint16_t* w,
                      uint16_t* y, cudaStream_t s) {
  const int64_t wn = act == TP_ACT_SWIGLU ? 2 * n_shard : n_shard;
  GemmArgs g = gemm_args(t, N, n_shard, k, k, wn, epi_for(act, TP_BF16));
  for (int r = 0; r < t; ++r) {
    g.a[r] = x;
    g.b[r] = w + r * k * wn;
    g.c[r] = y + r * N * n_shard;
  }
  return grouped_gemm(g, s);
}

tp_status row_gemm(const uint16_t* x, int64_t N, int64_t k_shard, int64_t n, int t, const uint16_t* w,
                   float* const* partials, cudaStream_t s) {
  GemmArgs g = gemm_args(t, N, n, k_shard, k_shard, n, EPI_F32);
  for (int r = 0; r < t; ++r) {
    if (partials[r] == nullptr) return fail(TP_EINVAL, "null partial buffer %d", r);
    g.a[r] = x + r * N * k_shard;
    g.b[r] = w + r * k_shard * n;
    g.c[r] = partials[r];
  }
  return grouped_gemm(g, s);
}

// Reduce the t fp32 partials [N, h] according to `mode` into out.
tp_status reduce_partials(float* const* partials, int64_t N, int64_t h, int t, tp_reduce mode, float* const* out,
                          const void* resid, tp_dtype resid_dtype, uint16_t* copy_bf16, cudaStream_t s) {
  if (mode == TP_OUT_PARTIALS) return TP_OK;
  if (out == nullptr) return fail(TP_EINVAL, "null output array");
  for (int r = 0; r < t; ++r)
    if (out[r] == nullptr) return fail(TP_EINVAL, "null output buffer %d", r);
  if (mode == TP_OUT_RS) {
    RingArgs a = ring_args(RING_RS, t, N, h, 0, TP_F32, TP_F32);
    for (int r = 0; r < t; ++r) { a.in[r] = partials[r]; a.out[r] = out[r]; }
    return ring_collective(a, s);
  }
  if (mode == TP_OUT_AR) {
    RingArgs a = ring_args(RING_AR, t, N, h, 0, TP_F32, TP_F32);
    for (int r = 0; r < t; ++r) { a.in[r] = partials[r]; a.out[r] = out[r]; }
    a.resid = resid; a.resid_dtype = resid_dtype; a.copy_bf16 = copy_bf16;
    return ring_collective(a, s);
  }
  if (mode == TP_OUT_RS_AG) {
    // ReduceScatter along tokens straight into each shard's own row block of its output, then an
    // in-place AllGather fills in the other shards' blocks.
    const int64_t chunk = (N / t) * h;
    RingArgs rs = ring_args(RING_RS, t, N, h, 0, TP_F32, TP_F32);
    for (int r = 0; r < t; ++r) { rs.in[r] = partials[r]; rs.out[r] = out[r] + r * chunk; }
    if (tp_status st = ring_collective(rs, s)) return st;
    RingArgs ag = ring_args(RING_AG, t, N, h, 0, TP_F32, TP_F32);
    for (int r = 0; r < t; ++r) { ag.in[r] = out[r] + r * chunk; ag.out[r] = out[r]; }
    return ring_collective(ag, s);
  }
  return fail(TP_EINVAL, "bad reduce mode %d", static_cast<int>(mode));
}

// Row-parallel GEMM fused with its collective (see gemm.cu): RS leaves chunk r on out[r]; AR and
// RS_AG (ReduceScatter with its AllGather folded into the same epilogue) write every replica.
tp_status fused_row_reduce(const uint16_t* x, int64_t N, int64_t k_shard, int64_t n, int t, const uint16_t* w,
                           tp_reduce mode, int axis, float* const* out, const void* resid, tp_dtype resid_dtype,
                           uint16_t* copy_bf16, cudaStream_t s) {
  RingGemmArgs g;
  std::memset(&g, 0, sizeof(g));
  g.t = t; g.M = N; g.N = n; g.K = k_shard; g.lda = k_shard; g.ldb = n;
  g.op = mode == TP_OUT_RS ? RING_RS : RING_AR;
  g.axis = axis;
  g.out_dtype = TP_F32;
  g.resid = resid; g.resid_dtype = resid_dtype; g.copy_bf16 = copy_bf16;
  for (int r = 0; r < t; ++r) {
    if (out[r] == nullptr) return fail(TP_EINVAL, "null output buffer %d", r);
    g.a[r] = x + r * N * k_shard;
    g.b[r] = w + r * k_shard * n;
    g.out[r] = out[r];
  }
  return ring_gemm(g, s);
}

}  // namespace
}  // namespace tpx

using namespace tpx;

extern "C" {

tp_status tp_grouped_gemm(int groups, const uint16_t* const* a, const uint16_t* const* b, void* const* c, int64_t M,
                          int64_t N, int64_t K, tp_act act, tp_dtype c_dtype, void* stream) {
  if (a == nullptr || b == nullptr || c == nullptr) return fail(TP_EINVAL, "null pointer array");
  if (groups < 1 || groups > TP_MAX_SHARDS) return fail(TP_EINVAL, "groups=%d outside 1..%d", groups, TP_MAX_SHARDS);
  if (!valid_act(act) || !valid_dtype(c_dtype)) return fail(TP_EINVAL, "bad activation or dtype");
  if (act != TP_ACT_NONE && c_dtype != TP_BF16) return fail(TP_EINVAL, "activations write bf16");
  GemmArgs g = gemm_args(groups, M, N, K, K, act == TP_ACT_SWIGLU ? 2 * N : N, epi_for(act, c_dtype));
  for (int i = 0; i < groups; ++i) { g.a[i] = a[i]; g.b[i] = b[i]; g.c[i] = c[i]; }
  return grouped_gemm(g, static_cast<cudaStream_t>(stream));
}

tp_status tp_column_linear(const uint16_t* x, int64_t N, int64_t k, int64_t n, int t, tp_act act, const uint16_t* w,
                           uint16_t* y, void* stream) {
  if (!valid_t(t)) return fail(TP_EINVAL, "t=%d outside 1..%d", t, TP_MAX_SHARDS);
  if (N < 0 || k <= 0 || n <= 0) return fail(TP_EINVAL, "negative size or empty contraction");
  if (N == 0) return TP_OK;                              // no tokens: nothing to compute
  if (x == nullptr || w == nullptr || y == nullptr) return fail(TP_EINVAL, "null pointer");
  if (!valid_act(act)) return fail(TP_EINVAL, "bad activation");
  if (n % t) return fail(TP_EDIVIS, "t=%d does not divide n=%lld", t, (long long)n);
  return column_gemm(x, N, k, n / t, t, act, w, y, static_cast<cudaStream_t>(stream));
}

tp_status tp_row_linear(const uint16_t* x, int64_t N, int64_t k, int64_t n, int t, const uint16_t* w,
                        float* const* partials, void* stream) {
  if (!valid_t(t)) return fail(TP_EINVAL, "t=%d outside 1..%d", t, TP_MAX_SHARDS);
  if (N < 0 || k <= 0 || n <= 0) return fail(TP_EINVAL, "negative size or empty contraction");
  if (N == 0) return TP_OK;                              // no tokens: nothing to compute
  if (x == nullptr || w == nullptr || partials == nullptr) return fail(TP_EINVAL, "null pointer");
  if (k % t) return fail(TP_EDIVIS, "t=%d does not divide k=%lld", t, (long long)k);
  return row_gemm(x, N, k / t, n, t, w, partials, static_cast<cudaStream_t>(stream));
}

tp_status tp_row_linear_reduce(const uint16_t* x, int64_t N, int64_t k, int64_t n, int t, const uint16_t* w,
                               tp_reduce mode, int axis, float* const* out, float* const* partials, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!valid_t(t)) return fail(TP_EINVAL, "t=%d outside 1..%d", t, TP_MAX_SHARDS);
  if (N < 0 || k <= 0 || n <= 0) return fail(TP_EINVAL, "negative size or empty contraction");
  if (N == 0) return TP_OK;                              // no tokens: nothing to compute
  if (x == nullptr || w == nullptr || out == nullptr) return fail(TP_EINVAL, "null pointer");
  if (mode != TP_OUT_RS && mode != TP_OUT_AR && mode != TP_OUT_RS_AG) return fail(TP_EINVAL, "mode must reduce");
  if (axis != 0 && axis != 1) return fail(TP_EINVAL, "axis must be 0 or 1");
  if (mode == TP_OUT_RS_AG) axis = 0;   // ReduceScatter along tokens, by definition
  if (k % t) return fail(TP_EDIVIS, "t=%d does not divide k=%lld", t, (long long)k);
  if (axis == 0 ? N % t != 0 : n % t != 0) return fail(TP_EDIVIS, "t=%d does not divide the scattered dim", t);
  if (ring_gemm_fits(N, n, t, axis))
    return fused_row_reduce(x, N, k / t, n, t, w, mode, axis, out, nullptr, TP_F32, nullptr, s);
  if (partials == nullptr)
    return fail(TP_EUNSUPPORTED, "chunks do not align with the fused kernel's 128 x 256 tiles and no partials were given");
  if (tp_status st = row_gemm(x, N, k / t, n, t, w, partials, s)) return st;
  RingArgs a = ring_args(mode == TP_OUT_RS ? RING_RS : RING_AR, t, N, n, axis, TP_F32, TP_F32);
  for (int r = 0; r < t; ++r) { a.in[r] = partials[r]; a.out[r] = out[r]; }
  return ring_collective(a, s);
}

tp_status tp_mlp_fwd(const uint16_t* x, int64_t N, int64_t h, int64_t F, int t, tp_act act, const uint16_t* w_in,
                     const uint16_t* w_down, uint16_t* z_ws, float* const* partials, tp_reduce mode, float* const* out,
                     void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!valid_t(t)) return fail(TP_EINVAL, "t=%d outside 1..%d", t, TP_MAX_SHARDS);
  if (N < 0 || h <= 0 || F <= 0) return fail(TP_EINVAL, "negative size or empty hidden/F dimension");
  if (N == 0) return TP_OK;                              // no tokens: nothing to compute
  if (x == nullptr || w_in == nullptr || w_down == nullptr || z_ws == nullptr) return fail(TP_EINVAL, "null pointer");
  if (partials == nullptr && (mode == TP_OUT_PARTIALS || N % t != 0 || !ring_gemm_fits(N, h, t, 0)))
    return fail(TP_EINVAL, "null partials: needed unless the fused row GEMM + reduction applies (N/t a multiple of 128)");
  if (!valid_act(act)) return fail(TP_EINVAL, "bad activation");
  if (mode < TP_OUT_PARTIALS || mode > TP_OUT_RS_AG) return fail(TP_EINVAL, "bad reduce mode");
  if (F % t) return fail(TP_EDIVIS, "t=%d does not divide F=%lld", t, (long long)F);
  if (mode != TP_OUT_PARTIALS && N % t) return fail(TP_EDIVIS, "t=%d does not divide the token count %lld", t, (long long)N);
  const int64_t f = F / t;
  if (tp_status st = column_gemm(x, N, h, f, t, act, w_in, z_ws, s)) return st;          // Z_r = act(X W_in[r])
  if (mode != TP_OUT_PARTIALS && ring_gemm_fits(N, h, t, 0)) {
    // U_r = Z_r W_down[r] and g (the collective) in one kernel; the partials never reach HBM
    if (out == nullptr) return fail(TP_EINVAL, "null output array");
    return fused_row_reduce(z_ws, N, f, h, t, w_down, mode, 0, out, nullptr, TP_F32, nullptr, s);
  }
  if (tp_status st = row_gemm(z_ws, N, f, h, t, w_down, partials, s)) return st;         // U_r = Z_r W_down[r]
  return reduce_partials(partials, N, h, t, mode, out, nullptr, TP_F32, nullptr, s);     // g: the collective
}

tp_status tp_column_linear_sp(const uint16_t* const* x, int64_t N, int64_t k, int64_t n, int t, tp_act act,
                              const uint16_t* w, uint16_t* y, void* stream) {
  if (!valid_t(t)) return fail(TP_EINVAL, "t=%d outside 1..%d", t, TP_MAX_SHARDS);
  if (N < 0 || k <= 0 || n <= 0) return fail(TP_EINVAL, "negative size or empty contraction");
  if (N == 0) return TP_OK;                              // no tokens: nothing to compute
  if (x == nullptr || w == nullptr || y == nullptr) return fail(TP_EINVAL, "null pointer");
  if (!valid_act(act)) return fail(TP_EINVAL, "bad activation");
  if (n % t || N % t) return fail(TP_EDIVIS, "t=%d does not divide n or the token count", t);
  if ((N / t) % 128) return fail(TP_EUNSUPPORTED, "token shards must be multiples of 128 rows");
  const int64_t n_shard = n / t;
  const int64_t wn = act == TP_ACT_SWIGLU ? 2 * n_shard : n_shard;
  GemmArgs g = gemm_args(t, N, n_shard, k, k, wn, epi_for(act, TP_BF16));
  g.a_slices = t;
  g.slice_rows = N / t;
  for (int r = 0; r < t; ++r) {
    g.a_slice[r] = x[r];
    g.b[r] = w + r * k * wn;
    g.c[r] = y + r * N * n_shard;
  }
  return grouped_gemm(g, static_cast<cudaStream_t>(stream));
}

tp_status tp_mlp_fwd_sp(const uint16_t* const* x, int64_t N, int64_t h, int64_t F, int t, tp_act act,
                        const uint16_t* w_in, const uint16_t* w_down, uint16_t* z_ws, float* const* out,
                        void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!valid_t(t)) return fail(TP_EINVAL, "t=%d outside 1..%d", t, TP_MAX_SHARDS);
  if (N < 0 || h <= 0 || F <= 0) return fail(TP_EINVAL, "negative size or empty hidden/F dimension");
  if (N == 0) return TP_OK;                              // no tokens: nothing to compute
  if (x == nullptr || w_in == nullptr || w_down == nullptr || z_ws == nullptr || out == nullptr)
    return fail(TP_EINVAL, "null pointer");
  if (F % t) return fail(TP_EDIVIS, "t=%d does not divide F=%lld", t, (long long)F);
  // g: AllGather along tokens, fused into the column GEMM's operand loads
  if (tp_status st = tp_column_linear_sp(x, N, h, F, t, act, w_in, z_ws, stream)) return st;
  // g-bar: the row GEMM fused with the ReduceScatter along tokens
  return fused_row_reduce(z_ws, N, F / t, h, t, w_down, TP_OUT_RS, 0, out, nullptr, TP_F32, nullptr, s);
}

size_t tp_sharded_matmul_ws_bytes(int case_id, int strategy, int64_t B, int64_t D, int64_t F, int t) {
  if (t < 1 || B <= 0 || D <= 0 || F <= 0) return 0;
  const size_t T = static_cast<size_t>(t);
  switch (case_id) {
    case 2:   // AllReduce: no workspace when the fused row GEMM + ring reduction applies
      if (strategy == TP_CASE2_ALLGATHER)
        return gather_in_place(case_id, strategy, B, D, F, t) ? 0 : T * align256(size_t(B) * D * 2);
      return (B % t == 0 && ring_gemm_fits(B, F, t, 0)) ? 0 : T * align256(size_t(B) * F * 4);
    case 3: {  // likewise for every case-3 strategy
      const int axis = strategy == TP_CASE3_RS_F ? 1 : 0;
      const bool divides = axis == 1 ? F % t == 0 : B % t == 0;
      return (divides && ring_gemm_fits(B, F, t, axis)) ? 0 : T * align256(size_t(B) * F * 4);
    }
    case 4:   // no workspace when the GEMM reads the gathered operand's pieces in place
      if (gather_in_place(case_id, strategy, B, D, F, t)) return 0;
      return strategy == TP_CASE4_GATHER_X ? T * align256(size_t(B) * D * 2) : T * align256(size_t(D) * F * 2);
    default: return 0;
  }
}

tp_status tp_sharded_matmul_choose(int case_id, int64_t B, int64_t D, int64_t F, int t, int* strategy) {
  if (strategy == nullptr) return fail(TP_EINVAL, "null strategy pointer");
  if (!valid_t(t)) return fail(TP_EINVAL, "t=%d outside 1..%d", t, TP_MAX_SHARDS);
  if (B <= 0 || D <= 0 || F <= 0) return fail(TP_EINVAL, "sizes must be positive");
  switch (case_id) {
    case 1: *strategy = TP_CASE1_LOCAL; return TP_OK;
    case 2: {   // gathered X: B*D elements; AllReduce of C: about 2*B*F (both in 128-bit arithmetic)
      const __int128 gathered = static_cast<__int128>(B) * D, reduced = static_cast<__int128>(2) * B * F;
      *strategy = gathered <= reduced ? TP_CASE2_ALLGATHER : TP_CASE2_ALLREDUCE;
      return TP_OK;
    }
    case 3: return fail(TP_EUNSUPPORTED, "case 3: the wanted sharding of C picks AllReduce, RS_B or RS_F");
    case 4: *strategy = B <= F ? TP_CASE4_GATHER_X : TP_CASE4_GATHER_W; return TP_OK;   // B*D <= D*F
    default: return fail(TP_EINVAL, "case %d outside 1..4", case_id);
  }
}

tp_status tp_sharded_matmul(int case_id, int strategy, const uint16_t* const* x, const uint16_t* const* w, int64_t B,
                            int64_t D, int64_t F, int t, void* const* c, tp_dtype c_dtype, void* ws, size_t ws_bytes,
                            void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!valid_t(t)) return fail(TP_EINVAL, "t=%d outside 1..%d", t, TP_MAX_SHARDS);
  if (B < 0 || D <= 0 || F <= 0) return fail(TP_EINVAL, "negative size or empty contraction");
  if (B == 0) return TP_OK;                              // no rows: nothing to compute
  if (x == nullptr || w == nullptr || c == nullptr) return fail(TP_EINVAL, "null pointer array");
  if (!valid_dtype(c_dtype)) return fail(TP_EINVAL, "bad dtype");
  for (int i = 0; i < t; ++i)
    if (x[i] == nullptr || w[i] == nullptr || c[i] == nullptr) return fail(TP_EINVAL, "null shard pointer %d", i);
  const size_t need = tp_sharded_matmul_ws_bytes(case_id, strategy, B, D, F, t);
  if (need > 0 && (ws == nullptr || ws_bytes < need))
    return fail(TP_ENOSPACE, "workspace of %zu bytes < %zu needed", ws_bytes, need);
  const EpiKind epi = c_dtype == TP_F32 ? EPI_F32 : EPI_BF16;
  char* wsb = static_cast<char*>(ws);

  if (case_id == 1) {                                   // X[B_X, D] . W[D, F]: local
    if (strategy != TP_CASE1_LOCAL) return fail(TP_EINVAL, "case 1 has one strategy");
    if (B % t) return fail(TP_EDIVIS, "t=%d does not divide B", t);
    GemmArgs g = gemm_args(t, B / t, F, D, D, F, epi);
    for (int i = 0; i < t; ++i) { g.a[i] = x[i]; g.b[i] = w[i]; g.c[i] = c[i]; }
    return grouped_gemm(g, s);
  }
  if (case_id == 2) {                                   // X[B, D_X] . W[D, F]
    if (D % t) return fail(TP_EDIVIS, "t=%d does not divide D", t);
    if (strategy == TP_CASE2_ALLGATHER) {
      if (gather_in_place(case_id, strategy, B, D, F, t)) {
        // every shard computes the full C from X's t column pieces, each k-block read from the shard
        // that holds it: the AllGather is the GEMM's operand addressing
        GemmArgs g = gemm_args(t, B, F, D, D / t, F, epi);
        g.a_kslices = t;
        g.kslice_cols = D / t;
        for (int i = 0; i < t; ++i) { g.a_kslice[i] = x[i]; g.b[i] = w[i]; g.c[i] = c[i]; }
        return grouped_gemm(g, s);
      }
      const size_t slot = align256(size_t(B) * D * 2);
      RingArgs ag = ring_args(RING_AG, t, B, D, 1, TP_BF16, TP_BF16);
      for (int i = 0; i < t; ++i) { ag.in[i] = x[i]; ag.out[i] = wsb + i * slot; }
      if (tp_status st = ring_collective(ag, s)) return st;
      GemmArgs g = gemm_args(t, B, F, D, D, F, epi);
      for (int i = 0; i < t; ++i) { g.a[i] = reinterpret_cast<const uint16_t*>(wsb + i * slot); g.b[i] = w[i]; g.c[i] = c[i]; }
      return grouped_gemm(g, s);
    }
    if (strategy == TP_CASE2_ALLREDUCE) {
      if (B % t) return fail(TP_EDIVIS, "t=%d does not divide B (AllReduce chunks)", t);
      const size_t slot = align256(size_t(B) * F * 4);
      const int64_t d = D / t;
      if (ring_gemm_fits(B, F, t, 0)) {                 // local products and AllReduce in one kernel
        RingGemmArgs rg;
        std::memset(&rg, 0, sizeof(rg));
        rg.t = t; rg.M = B; rg.N = F; rg.K = d; rg.lda = d; rg.ldb = F; rg.op = RING_AR; rg.out_dtype = c_dtype;
        for (int i = 0; i < t; ++i) { rg.a[i] = x[i]; rg.b[i] = w[i] + i * d * F; rg.out[i] = c[i]; }
        return ring_gemm(rg, s);
      }
      GemmArgs g = gemm_args(t, B, F, d, d, F, EPI_F32);
      for (int i = 0; i < t; ++i) { g.a[i] = x[i]; g.b[i] = w[i] + i * d * F; g.c[i] = wsb + i * slot; }
      if (tp_status st = grouped_gemm(g, s)) return st;
      RingArgs ar = ring_args(RING_AR, t, B, F, 0, TP_F32, c_dtype);
      for (int i = 0; i < t; ++i) { ar.in[i] = wsb + i * slot; ar.out[i] = c[i]; }
      return ring_collective(ar, s);
    }
    return fail(TP_EINVAL, "bad case-2 strategy %d", strategy);
  }
  if (case_id == 3) {                                   // X[B, D_X] . W[D_X, F] -> C{U_X}
    if (D % t) return fail(TP_EDIVIS, "t=%d does not divide D", t);
    if (strategy < TP_CASE3_ALLREDUCE || strategy > TP_CASE3_RS_F) return fail(TP_EINVAL, "bad case-3 strategy %d", strategy);
    const size_t slot = align256(size_t(B) * F * 4);
    const int64_t d = D / t;
    GemmArgs g = gemm_args(t, B, F, d, d, F, EPI_F32);
    for (int i = 0; i < t; ++i) { g.a[i] = x[i]; g.b[i] = w[i]; g.c[i] = wsb + i * slot; }
    if (strategy == TP_CASE3_RS_F ? (F % t != 0) : (B % t != 0)) return fail(TP_EDIVIS, "t=%d does not divide the scattered dim", t);
    const int axis = strategy == TP_CASE3_RS_F ? 1 : 0;
    if (ring_gemm_fits(B, F, t, axis)) {                 // local products and the reduction in one kernel
      RingGemmArgs rg;
      std::memset(&rg, 0, sizeof(rg));
      rg.t = t; rg.M = B; rg.N = F; rg.K = d; rg.lda = d; rg.ldb = F; rg.axis = axis; rg.out_dtype = c_dtype;
      rg.op = strategy == TP_CASE3_ALLREDUCE ? RING_AR : RING_RS;
      for (int i = 0; i < t; ++i) { rg.a[i] = x[i]; rg.b[i] = w[i]; rg.out[i] = c[i]; }
      return ring_gemm(rg, s);
    }
    if (tp_status st = grouped_gemm(g, s)) return st;
    RingArgs a = ring_args(strategy == TP_CASE3_ALLREDUCE ? RING_AR : RING_RS, t, B, F,
                           strategy == TP_CASE3_RS_F ? 1 : 0, TP_F32, c_dtype);
    for (int i = 0; i < t; ++i) { a.in[i] = wsb + i * slot; a.out[i] = c[i]; }
    return ring_collective(a, s);
  }
  if (case_id == 4) {                                   // X[B_X, D] . W[D, F_X]: gather one operand
    if (B % t || F % t) return fail(TP_EDIVIS, "t=%d does not divide B and F", t);
    if (strategy == TP_CASE4_GATHER_X) {
      if (gather_in_place(case_id, strategy, B, D, F, t)) {
        // shard i multiplies the gathered X by its own columns of W; each 128-row tile of X is read
        // from the shard that holds it
        GemmArgs g = gemm_args(t, B, F / t, D, D, F / t, epi);
        g.a_slices = t;
        g.slice_rows = B / t;
        for (int i = 0; i < t; ++i) { g.a_slice[i] = x[i]; g.b[i] = w[i]; g.c[i] = c[i]; }
        return grouped_gemm(g, s);
      }
      const size_t slot = align256(size_t(B) * D * 2);
      RingArgs ag = ring_args(RING_AG, t, B, D, 0, TP_BF16, TP_BF16);
      for (int i = 0; i < t; ++i) { ag.in[i] = x[i]; ag.out[i] = wsb + i * slot; }
      if (tp_status st = ring_collective(ag, s)) return st;
      GemmArgs g = gemm_args(t, B, F / t, D, D, F / t, epi);
      for (int i = 0; i < t; ++i) { g.a[i] = reinterpret_cast<const uint16_t*>(wsb + i * slot); g.b[i] = w[i]; g.c[i] = c[i]; }
      return grouped_gemm(g, s);
    }
    if (strategy == TP_CASE4_GATHER_W) {
      if (gather_in_place(case_id, strategy, B, D, F, t)) {
        // shard i multiplies its rows of X by the gathered W; each 64-column box of W is read from the
        // shard that holds it
        GemmArgs g = gemm_args(t, B / t, F, D, D, F / t, epi);
        g.b_slices = t;
        g.bslice_cols = F / t;
        for (int i = 0; i < t; ++i) { g.a[i] = x[i]; g.b_slice[i] = w[i]; g.c[i] = c[i]; }
        return grouped_gemm(g, s);
      }
      const size_t slot = align256(size_t(D) * F * 2);
      RingArgs ag = ring_args(RING_AG, t, D, F, 1, TP_BF16, TP_BF16);
      for (int i = 0; i < t; ++i) { ag.in[i] = w[i]; ag.out[i] = wsb + i * slot; }
      if (tp_status st = ring_collective(ag, s)) return st;
      GemmArgs g = gemm_args(t, B / t, F, D, D, F, epi);
      for (int i = 0; i < t; ++i) { g.a[i] = x[i]; g.b[i] = reinterpret_cast<const uint16_t*>(wsb + i * slot); g.c[i] = c[i]; }
      return grouped_gemm(g, s);
    }
    return fail(TP_EINVAL, "bad case-4 strategy %d", strategy);
  }
  return fail(TP_EINVAL, "case_id %d outside 1..4", case_id);
}

tp_status tp_layer_fwd(const uint16_t* x, const uint16_t* const* o, int64_t N, int64_t h, int n_h, int n_kv, int d_h,
                       int64_t F, int t, const uint16_t* w_qkv, const uint16_t* w_o, const uint16_t* w_gu,
                       const uint16_t* w_down, uint16_t* qkv_out, float* const* h1, uint16_t* h1_bf16, uint16_t* z_ws,
                       float* const* partials, float* const* y, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!valid_t(t)) return fail(TP_EINVAL, "t=%d outside 1..%d", t, TP_MAX_SHARDS);
  if (N < 0 || h <= 0 || F <= 0 || n_h <= 0 || n_kv <= 0 || d_h <= 0) return fail(TP_EINVAL, "non-positive size");
  if (N == 0) return TP_OK;                              // no tokens: nothing to compute
  if (!x || !o || !w_qkv || !w_o || !w_gu || !w_down || !qkv_out || !h1 || !h1_bf16 || !z_ws || !y)
    return fail(TP_EINVAL, "null pointer");
  if (n_h % t || n_h % n_kv || (t <= n_kv ? n_kv % t != 0 : t % n_kv != 0))
    return fail(TP_EDIVIS, "head counts n_h=%d n_kv=%d do not split over t=%d", n_h, n_kv, t);
  if (F % t || N % t) return fail(TP_EDIVIS, "t=%d does not divide F or the token count", t);
  const int64_t kv = t <= n_kv ? n_kv / t : 1;
  const int64_t qkv_w = (n_h / t + 2 * kv) * d_h;
  const int64_t o_w = int64_t(n_h) * d_h / t;
  // Both AllReduces are fused into their row GEMMs. Their ReduceScatter scatters along h (columns)
  // when h/t is a whole number of 256-column tiles: every row-tile of a chunk then reads the same
  // shard's weight panel at the same time, so the weights stream from DRAM about once instead of once
  // per row-tile. Otherwise along tokens (rows), else unfused through the partials.
  const int ar_axis = ring_gemm_fits(N, h, t, 1) ? 1 : 0;
  const bool need_partials = !ring_gemm_fits(N, h, t, ar_axis);
  if (need_partials && partials == nullptr) return fail(TP_EINVAL, "null partials (needed: N/t is not a multiple of 128)");
  for (int r = 0; r < t; ++r)
    if (o[r] == nullptr || h1[r] == nullptr || y[r] == nullptr || (need_partials && partials[r] == nullptr))
      return fail(TP_EINVAL, "null shard buffer %d", r);
  // 1. fused QKV projection, column-parallel on head boundaries (feeds the attention core)
  if (tp_status st = column_gemm(x, N, h, qkv_w, t, TP_ACT_NONE, w_qkv, qkv_out, s)) return st;
  const bool fused = !need_partials;
  // 2-3. attention output projection (row-parallel) and g: AllReduce, with the residual add
  //      h1 = X + attn and the bf16 copy for the MLP input
  if (fused) {
    RingGemmArgs rg;
    std::memset(&rg, 0, sizeof(rg));
    rg.t = t; rg.M = N; rg.N = h; rg.K = o_w; rg.lda = o_w; rg.ldb = h; rg.op = RING_AR; rg.out_dtype = TP_F32;
    rg.axis = ar_axis;
    rg.resid = x; rg.resid_dtype = TP_BF16; rg.copy_bf16 = h1_bf16;
    for (int r = 0; r < t; ++r) { rg.a[r] = o[r]; rg.b[r] = w_o + r * o_w * h; rg.out[r] = h1[r]; }
    if (tp_status st = ring_gemm(rg, s)) return st;
  } else {
    GemmArgs g = gemm_args(t, N, h, o_w, o_w, h, EPI_F32);
    for (int r = 0; r < t; ++r) { g.a[r] = o[r]; g.b[r] = w_o + r * o_w * h; g.c[r] = partials[r]; }
    if (tp_status st = grouped_gemm(g, s)) return st;
    if (tp_status st = reduce_partials(partials, N, h, t, TP_OUT_AR, h1, x, TP_BF16, h1_bf16, s)) return st;
  }
  // 4. SwiGLU MLP on bf16(h1), then AllReduce with y = h1 + mlp
  const int64_t f = F / t;
  if (tp_status st = column_gemm(h1_bf16, N, h, f, t, TP_ACT_SWIGLU, w_gu, z_ws, s)) return st;
  if (fused) return fused_row_reduce(z_ws, N, f, h, t, w_down, TP_OUT_AR, ar_axis, y, h1[0], TP_F32, nullptr, s);
  if (tp_status st = row_gemm(z_ws, N, f, h, t, w_down, partials, s)) return st;
  return reduce_partials(partials, N, h, t, TP_OUT_AR, y, h1[0], TP_F32, nullptr, s);
}

}  // extern "C"
