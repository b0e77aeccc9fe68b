// Weight shard layouts ("张量并行与序列并行": §矩阵乘法的两种切法 for the column/row splits, §MLP for the
// fused gate|up layout, §注意力 and §GQA for the rank-grouped fused QKV layout).
//
// Every layout is the same operation: output shard r, row k, is the concatenation of up to three
// column segments, segment s taken from source s at row (row0[s][r] + k), columns
// [col0[s][r], col0[s][r] + len[s]). One bandwidth-bound copy kernel does all of them: 16-byte
// vectors when every offset is a multiple of 8 bf16, 2-byte elements otherwise.
#include <cstring>

#include "common.cuh"
#include "ptx.cuh"

namespace tpx {

namespace {

constexpr int kMaxSeg = 3;

struct SegParams {
  const uint16_t* src[kMaxSeg];
  int64_t ld[kMaxSeg];                      // source row strides (elements)
  int64_t row0[kMaxSeg][TP_MAX_SHARDS];     // source row of output row 0, per shard
  int64_t col0[kMaxSeg][TP_MAX_SHARDS];     // source column of the segment, per shard
  int64_t len[kMaxSeg];                     // segment width (elements)
  int64_t dst0[kMaxSeg];                    // segment start inside an output row
  int nseg;
  int t;
  int64_t rows;                             // rows per output shard
  int64_t width;                            // output row width (sum of len)
  uint16_t* out;                            // stacked [t][rows][width]
};

// VEC = elements moved per step (8 -> one 16-byte vector, 1 -> one element).
template <int VEC>
__global__ void __launch_bounds__(256) segment_copy_kernel(const __grid_constant__ SegParams p) {
  const int64_t wv = p.width / VEC;
  const int64_t per_shard = p.rows * wv;
  const int64_t total = per_shard * p.t;
  for (int64_t u = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; u < total;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int r = static_cast<int>(u / per_shard);
    const int64_t rem = u - r * per_shard;
    const int64_t k = rem / wv;
    const int64_t j = (rem - k * wv) * VEC;              // output column
    int s = 0;
    while (s + 1 < p.nseg && j >= p.dst0[s + 1]) ++s;
    const int64_t scol = p.col0[s][r] + (j - p.dst0[s]);
    const uint16_t* src = p.src[s] + (p.row0[s][r] + k) * p.ld[s] + scol;
    uint16_t* dst = p.out + (static_cast<int64_t>(r) * p.rows + k) * p.width + j;
    if constexpr (VEC == 8) {
      st_v4(dst, ld_nc_v4(src));
    } else {
      *dst = *src;
    }
  }
}

tp_status launch_segments(SegParams& p, cudaStream_t stream) {
  int64_t acc = 0;
  for (int s = 0; s < p.nseg; ++s) {
    p.dst0[s] = acc;
    acc += p.len[s];
  }
  p.width = acc;
  bool vec = aligned16(p.out) && (p.width % 8 == 0);
  for (int s = 0; s < p.nseg && vec; ++s) {
    vec = aligned16(p.src[s]) && p.ld[s] % 8 == 0 && p.len[s] % 8 == 0;
    for (int r = 0; r < p.t && vec; ++r) vec = p.col0[s][r] % 8 == 0;
  }
  const int64_t units = p.t * p.rows * (p.width / (vec ? 8 : 1));
  if (units == 0) return TP_OK;                         // empty weight: nothing to copy
  const int sms = sm_count();
  if (sms <= 0) return fail(TP_ECUDA, "cannot query the SM count");
  const int64_t want = (units + 255) / 256;
  const int blocks = static_cast<int>(want < static_cast<int64_t>(sms) * 8 ? want : static_cast<int64_t>(sms) * 8);
  if (vec)
    segment_copy_kernel<8><<<blocks, 256, 0, stream>>>(p);
  else
    segment_copy_kernel<1><<<blocks, 256, 0, stream>>>(p);
  return check_launch("segment_copy_kernel");
}

// Sets *empty (and returns TP_OK) for a weight with no elements: nothing is read or launched then.
tp_status common_checks(const void* out, int t, int64_t rows, int64_t cols, bool* empty) {
  if (!valid_t(t)) return fail(TP_EINVAL, "t=%d outside 1..%d", t, TP_MAX_SHARDS);
  if (rows < 0 || cols < 0) return fail(TP_EINVAL, "negative size %lld x %lld", (long long)rows, (long long)cols);
  *empty = rows == 0 || cols == 0;
  if (*empty) return TP_OK;
  if (out == nullptr) return fail(TP_EINVAL, "null output");
  return TP_OK;
}

}  // namespace
}  // namespace tpx

using namespace tpx;

extern "C" {

tp_status tp_shard_cols(const uint16_t* w, int64_t ld, int64_t K, int64_t N, int t, uint16_t* out, void* stream) {
  bool empty = false;
  if (tp_status s = common_checks(out, t, K, N, &empty)) return s;
  if (empty) return TP_OK;
  if (w == nullptr || ld < N) return fail(TP_EINVAL, "null weight or row stride %lld < %lld", (long long)ld, (long long)N);
  if (N % t) return fail(TP_EDIVIS, "t=%d does not divide N=%lld", t, (long long)N);
  SegParams p;
  std::memset(&p, 0, sizeof(p));
  p.nseg = 1; p.t = t; p.rows = K; p.out = out;
  p.src[0] = w; p.ld[0] = ld; p.len[0] = N / t;
  for (int r = 0; r < t; ++r) { p.row0[0][r] = 0; p.col0[0][r] = r * (N / t); }
  return launch_segments(p, static_cast<cudaStream_t>(stream));
}

tp_status tp_shard_rows(const uint16_t* w, int64_t ld, int64_t K, int64_t N, int t, uint16_t* out, void* stream) {
  bool empty = false;
  if (tp_status s = common_checks(out, t, K, N, &empty)) return s;
  if (empty) return TP_OK;
  if (w == nullptr || ld < N) return fail(TP_EINVAL, "null weight or row stride %lld < %lld", (long long)ld, (long long)N);
  if (K % t) return fail(TP_EDIVIS, "t=%d does not divide K=%lld", t, (long long)K);
  SegParams p;
  std::memset(&p, 0, sizeof(p));
  p.nseg = 1; p.t = t; p.rows = K / t; p.out = out;
  p.src[0] = w; p.ld[0] = ld; p.len[0] = N;
  for (int r = 0; r < t; ++r) { p.row0[0][r] = r * (K / t); p.col0[0][r] = 0; }
  return launch_segments(p, static_cast<cudaStream_t>(stream));
}

tp_status tp_shard_gate_up(const uint16_t* w_gate, int64_t ld_g, const uint16_t* w_up, int64_t ld_u, int64_t h,
                           int64_t F, int t, uint16_t* out, void* stream) {
  bool empty = false;
  if (tp_status s = common_checks(out, t, h, F, &empty)) return s;
  if (empty) return TP_OK;
  if (w_gate == nullptr || w_up == nullptr || ld_g < F || ld_u < F) return fail(TP_EINVAL, "null weight or short row stride");
  if (F % t) return fail(TP_EDIVIS, "t=%d does not divide F=%lld", t, (long long)F);
  SegParams p;
  std::memset(&p, 0, sizeof(p));
  p.nseg = 2; p.t = t; p.rows = h; p.out = out;
  const int64_t f = F / t;
  p.src[0] = w_gate; p.ld[0] = ld_g; p.len[0] = f;
  p.src[1] = w_up;   p.ld[1] = ld_u; p.len[1] = f;
  for (int r = 0; r < t; ++r) {
    p.row0[0][r] = p.row0[1][r] = 0;
    p.col0[0][r] = p.col0[1][r] = r * f;
  }
  return launch_segments(p, static_cast<cudaStream_t>(stream));
}

tp_status tp_shard_qkv(const uint16_t* w_q, int64_t ld_q, const uint16_t* w_k, int64_t ld_k, const uint16_t* w_v,
                       int64_t ld_v, int64_t h, int n_h, int n_kv, int d_h, int t, uint16_t* out, void* stream) {
  bool empty = false;
  if (tp_status s = common_checks(out, t, h, 1, &empty)) return s;
  if (empty) return TP_OK;
  if (w_q == nullptr || w_k == nullptr || w_v == nullptr) return fail(TP_EINVAL, "null QKV weight");
  if (n_h <= 0 || n_kv <= 0 || d_h <= 0) return fail(TP_EINVAL, "non-positive head counts");
  if (ld_q < int64_t(n_h) * d_h || ld_k < int64_t(n_kv) * d_h || ld_v < int64_t(n_kv) * d_h)
    return fail(TP_EINVAL, "QKV row strides shorter than the head columns");
  if (n_h % t) return fail(TP_EDIVIS, "t=%d does not divide n_h=%d", t, n_h);
  if (n_h % n_kv) return fail(TP_EDIVIS, "n_kv=%d does not divide n_h=%d", n_kv, n_h);
  if (t <= n_kv ? (n_kv % t != 0) : (t % n_kv != 0))
    return fail(TP_EDIVIS, "KV heads n_kv=%d cannot be split or replicated over t=%d", n_kv, t);
  const int q_per = n_h / t;
  const int kv_per = t <= n_kv ? n_kv / t : 1;
  SegParams p;
  std::memset(&p, 0, sizeof(p));
  p.nseg = 3; p.t = t; p.rows = h; p.out = out;
  p.src[0] = w_q; p.ld[0] = ld_q; p.len[0] = int64_t(q_per) * d_h;
  p.src[1] = w_k; p.ld[1] = ld_k; p.len[1] = int64_t(kv_per) * d_h;
  p.src[2] = w_v; p.ld[2] = ld_v; p.len[2] = int64_t(kv_per) * d_h;
  for (int r = 0; r < t; ++r) {
    const int kv_first = t <= n_kv ? r * kv_per : (r * n_kv) / t;   // a rank's first KV head
    p.col0[0][r] = int64_t(r) * q_per * d_h;
    p.col0[1][r] = p.col0[2][r] = int64_t(kv_first) * d_h;
  }
  return launch_segments(p, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
