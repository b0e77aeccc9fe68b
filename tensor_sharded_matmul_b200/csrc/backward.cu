// Backward pass of the tensor-parallel MLP ("张量并行与序列并行", §矩阵乘法的两种切法, the backward
// bullets, and §f 和 g; pufanyi.com "ml-revisit-infra", §Tensor Parallel, the gradient identities).
//
//   row-parallel layer (W_down): dY is the same on every shard (g's backward is the identity)
//       dZ_r = dY W_down[r]^T                 local
//       dW_down[r] = Z_r^T dY                 local
//   activation (element-wise, local):  dH_r = act'(H_r) * dZ_r  (SwiGLU: dG = dZ*U*SiLU'(G), dU = dZ*SiLU(G))
//   column-parallel layer (W_in):
//       dW_in[r] = X^T dH_r                   local
//       dX = sum_r dH_r W_in[r]^T             the AllReduce of f's backward (ring order)
//
// The transposed products use the GEMM's transposed-operand modes (A stored [K][M], B stored
// [N][K]), so no transposed copy of any tensor is made. The final sum over shards runs in the fused
// ring GEMM when the token count allows it.
#include <cuda_bf16.h>

#include <cstring>

#include "common.cuh"
#include "ptx.cuh"

namespace tpx {
namespace {

__device__ __forceinline__ float gelu_grad(float x) {
  // d/dx [x Phi(x)] = Phi(x) + x phi(x)
  return 0.5f * (1.0f + erff(x * 0.70710678118654752f)) + x * 0.39894228040143268f * __expf(-0.5f * x * x);
}
__device__ __forceinline__ float gelu_tanh_grad(float x) {
  const float c = 0.79788456080286536f, a = 0.044715f;
  const float th = tanhf(c * (x + a * x * x * x));
  return 0.5f * (1.0f + th) + 0.5f * x * (1.0f - th * th) * c * (1.0f + 3.0f * a * x * x);
}

__device__ __forceinline__ float bf(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }
__device__ __forceinline__ uint16_t to_bf(float x) { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }

// rows = t*N stacked rows; f = columns of dZ. H and dH have wn = f (GeLU) or 2f (SwiGLU) columns.
// VEC consecutive columns per step.
template <int ACT, int VEC>
__global__ void __launch_bounds__(256) act_backward_kernel(const uint16_t* __restrict__ h, const uint16_t* __restrict__ dz,
                                                           uint16_t* __restrict__ dh, int64_t rows, int64_t f) {
  const int64_t per_row = f / VEC;
  const int64_t units = rows * per_row;
  const int64_t wn = ACT == TP_ACT_SWIGLU ? 2 * f : f;
  for (int64_t u = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; u < units;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = u / per_row;
    const int64_t j = (u - r * per_row) * VEC;
    uint16_t d[VEC], a[VEC], b[VEC], o1[VEC], o2[VEC];
    if constexpr (VEC == 8) {
      *reinterpret_cast<uint4*>(d) = ld_nc_v4(dz + r * f + j);
      *reinterpret_cast<uint4*>(a) = ld_nc_v4(h + r * wn + j);
      if constexpr (ACT == TP_ACT_SWIGLU) *reinterpret_cast<uint4*>(b) = ld_nc_v4(h + r * wn + f + j);
    } else {
      d[0] = dz[r * f + j];
      a[0] = h[r * wn + j];
      if constexpr (ACT == TP_ACT_SWIGLU) b[0] = h[r * wn + f + j];
    }
#pragma unroll
    for (int v = 0; v < VEC; ++v) {
      const float dzv = bf(d[v]);
      if constexpr (ACT == TP_ACT_SWIGLU) {
        const float g = bf(a[v]), up = bf(b[v]);
        const float s = 1.0f / (1.0f + __expf(-g));
        const float silu = g * s;
        o1[v] = to_bf(dzv * up * (s * (1.0f + g * (1.0f - s))));   // dG
        o2[v] = to_bf(dzv * silu);                                  // dU
      } else if constexpr (ACT == TP_ACT_GELU) {
        o1[v] = to_bf(dzv * gelu_grad(bf(a[v])));
      } else if constexpr (ACT == TP_ACT_GELU_TANH) {
        o1[v] = to_bf(dzv * gelu_tanh_grad(bf(a[v])));
      } else {
        o1[v] = d[v];
      }
    }
    if constexpr (VEC == 8) {
      st_v4(dh + r * wn + j, *reinterpret_cast<uint4*>(o1));
      if constexpr (ACT == TP_ACT_SWIGLU) st_v4(dh + r * wn + f + j, *reinterpret_cast<uint4*>(o2));
    } else {
      dh[r * wn + j] = o1[0];
      if constexpr (ACT == TP_ACT_SWIGLU) dh[r * wn + f + j] = o2[0];
    }
  }
}

template <int ACT>
tp_status launch_act_bwd(const uint16_t* h, const uint16_t* dz, uint16_t* dh, int64_t rows, int64_t f, cudaStream_t s) {
  const bool vec = f % 8 == 0 && aligned16(h) && aligned16(dz) && aligned16(dh);
  const int64_t units = rows * f / (vec ? 8 : 1);
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  const int64_t want = (units + 255) / 256;
  const int blocks = static_cast<int>(want < cap ? want : cap);
  if (blocks <= 0) return fail(TP_ECUDA, "cannot query the SM count");
  if (vec)
    act_backward_kernel<ACT, 8><<<blocks, 256, 0, s>>>(h, dz, dh, rows, f);
  else
    act_backward_kernel<ACT, 1><<<blocks, 256, 0, s>>>(h, dz, dh, rows, f);
  return check_launch("act_backward_kernel");
}

bool valid_act(tp_act a) { return a == TP_ACT_NONE || a == TP_ACT_GELU || a == TP_ACT_GELU_TANH || a == TP_ACT_SWIGLU; }

GemmArgs args(int groups, int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb, EpiKind epi, bool a_mn, bool b_km) {
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  g.groups = groups; g.M = M; g.N = N; g.K = K; g.lda = lda; g.ldb = ldb; g.epi = epi; g.a_mn = a_mn; g.b_km = b_km;
  return g;
}

}  // namespace
}  // namespace tpx

using namespace tpx;

extern "C" {

tp_status tp_grouped_gemm_t(int groups, const uint16_t* const* a, int trans_a, const uint16_t* const* b, int trans_b,
                            void* const* c, int64_t M, int64_t N, int64_t K, tp_dtype c_dtype, void* stream) {
  if (a == nullptr || b == nullptr || c == nullptr) return fail(TP_EINVAL, "null pointer array");
  if (groups < 1 || groups > TP_MAX_SHARDS) return fail(TP_EINVAL, "groups=%d outside 1..%d", groups, TP_MAX_SHARDS);
  if (c_dtype != TP_F32 && c_dtype != TP_BF16) return fail(TP_EINVAL, "bad dtype");
  GemmArgs g = args(groups, M, N, K, trans_a ? M : K, trans_b ? K : N, c_dtype == TP_F32 ? EPI_F32 : EPI_BF16,
                    trans_a != 0, trans_b != 0);
  for (int i = 0; i < groups; ++i) { g.a[i] = a[i]; g.b[i] = b[i]; g.c[i] = c[i]; }
  return grouped_gemm(g, static_cast<cudaStream_t>(stream));
}

tp_status tp_mlp_bwd(const uint16_t* x, const uint16_t* dy, int64_t N, int64_t h, int64_t F, int t, tp_act act,
                     const uint16_t* w_in, const uint16_t* w_down, const uint16_t* h_pre, const uint16_t* z,
                     uint16_t* dz_ws, uint16_t* dh_ws, float* dw_in, float* dw_down, float* const* dx, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!valid_t(t)) return fail(TP_EINVAL, "t=%d outside 1..%d", t, TP_MAX_SHARDS);
  if (N < 0 || h <= 0 || F <= 0) return fail(TP_EINVAL, "negative size or empty hidden/F dimension");
  if (N == 0) return TP_OK;                              // no tokens: nothing to compute
  if (!x || !dy || !w_in || !w_down || !h_pre || !z || !dz_ws || !dh_ws || !dw_in || !dw_down || !dx)
    return fail(TP_EINVAL, "null pointer");
  if (!valid_act(act)) return fail(TP_EINVAL, "bad activation");
  if (F % t || N % t) return fail(TP_EDIVIS, "t=%d does not divide F or the token count", t);
  if (N % 8 || h % 8 || (F / t) % 8) return fail(TP_EALIGN, "token count, h and F/t must be multiples of 8");
  for (int r = 0; r < t; ++r)
    if (dx[r] == nullptr) return fail(TP_EINVAL, "null dX buffer %d", r);
  const int64_t f = F / t;
  const int64_t wn = act == TP_ACT_SWIGLU ? 2 * f : f;
  // 1. row layer, input gradient: dZ_r = dY W_down[r]^T      (W_down[r] [f][h] is B^T)
  {
    GemmArgs g = args(t, N, f, h, h, h, EPI_BF16, false, true);
    for (int r = 0; r < t; ++r) { g.a[r] = dy; g.b[r] = w_down + r * f * h; g.c[r] = dz_ws + r * N * f; }
    if (tp_status st = grouped_gemm(g, s)) return st;
  }
  // 2. row layer, weight gradient: dW_down[r] = Z_r^T dY     (Z_r [N][f] is A^T)
  {
    GemmArgs g = args(t, f, h, N, f, h, EPI_F32, true, false);
    for (int r = 0; r < t; ++r) { g.a[r] = z + r * N * f; g.b[r] = dy; g.c[r] = dw_down + r * f * h; }
    if (tp_status st = grouped_gemm(g, s)) return st;
  }
  // 3. activation: dH_r = act'(H_r) * dZ_r
  {
    tp_status st;
    switch (act) {
      case TP_ACT_SWIGLU: st = launch_act_bwd<TP_ACT_SWIGLU>(h_pre, dz_ws, dh_ws, t * N, f, s); break;
      case TP_ACT_GELU: st = launch_act_bwd<TP_ACT_GELU>(h_pre, dz_ws, dh_ws, t * N, f, s); break;
      case TP_ACT_GELU_TANH: st = launch_act_bwd<TP_ACT_GELU_TANH>(h_pre, dz_ws, dh_ws, t * N, f, s); break;
      default: st = launch_act_bwd<TP_ACT_NONE>(h_pre, dz_ws, dh_ws, t * N, f, s); break;
    }
    if (st) return st;
  }
  // 4. column layer, weight gradient: dW_in[r] = X^T dH_r    (X [N][h] is A^T)
  {
    GemmArgs g = args(t, h, wn, N, h, wn, EPI_F32, true, false);
    for (int r = 0; r < t; ++r) { g.a[r] = x; g.b[r] = dh_ws + r * N * wn; g.c[r] = dw_in + r * h * wn; }
    if (tp_status st = grouped_gemm(g, s)) return st;
  }
  // 5. column layer, input gradient: dX = sum_r dH_r W_in[r]^T, summed in ring order and replicated
  //    (the AllReduce of f's backward). W_in[r] [h][wn] is B^T.
  if (ring_gemm_fits(N, h, t, 0)) {
    RingGemmArgs rg;
    std::memset(&rg, 0, sizeof(rg));
    rg.t = t; rg.M = N; rg.N = h; rg.K = wn; rg.lda = wn; rg.ldb = wn; rg.op = RING_AR; rg.out_dtype = TP_F32;
    rg.b_km = true;
    for (int r = 0; r < t; ++r) { rg.a[r] = dh_ws + r * N * wn; rg.b[r] = w_in + r * h * wn; rg.out[r] = dx[r]; }
    return ring_gemm(rg, s);
  }
  // unfused: each shard's partial into its own dX buffer, then an in-place ring AllReduce
  GemmArgs g = args(t, N, h, wn, wn, wn, EPI_F32, false, true);
  for (int r = 0; r < t; ++r) { g.a[r] = dh_ws + r * N * wn; g.b[r] = w_in + r * h * wn; g.c[r] = dx[r]; }
  if (tp_status st = grouped_gemm(g, s)) return st;
  RingArgs a;
  std::memset(&a, 0, sizeof(a));
  a.op = RING_AR; a.t = t; a.rows = N; a.cols = h; a.in_dtype = a.out_dtype = TP_F32; a.resid_dtype = TP_F32;
  for (int r = 0; r < t; ++r) { a.in[r] = dx[r]; a.out[r] = dx[r]; }
  return ring_collective(a, s);
}

}  // extern "C"
