// Grouped bf16 GEMM on the 5th-generation tensor cores (tcgen05) with fused epilogues.
//
// Used for the column-parallel GEMM Z_r = act(X W_r) and the row-parallel GEMM U_r = Z_r W_r of the
// tensor-parallel MLP ("张量并行与序列并行", §矩阵乘法的两种切法 and §MLP：先列后行，只通信一次), and for
// the local products of the sharded-matmul cases ("Scaling Book 入门第 6 章", §6.2). All t shards
// of one layer run in ONE persistent launch: the tile space is (shard, m-tile, n-tile).
//
// Design (sm_100a):
//   * persistent CTAs, one per SM, each looping over tiles (raster: bands of row-tiles swept across
//     the n-tiles so that concurrently running CTAs share operand panels in L2);
//   * warp 0, one lane: TMA producer. A [M,K] is K-major (box 64 x 128, 128-byte swizzle); B [K,N]
//     is the weight as stored, [in, out] row-major, i.e. MN-major (boxes 64 x 64, 128-byte swizzle);
//   * warp 1, one lane: tcgen05.mma issuer (M=128, N=256, K=16 per instruction, fp32 accumulator in
//     TMEM). 4-stage shared-memory ring, two TMEM accumulators (2 x 256 columns) so the epilogue of
//     one tile overlaps the main loop of the next;
//   * warps 2..5: epilogue. tcgen05.ld 32 columns at a time, apply the activation in fp32, store.
//     SwiGLU tiles carry 128 gate columns and the 128 up columns of the same F indices in one
//     N=256 accumulator, so SiLU(gate)*up is formed in registers without another pass.
//   * every mbarrier wait is bounded; on expiry the kernel records the site in the status word,
//     raises a shared abort flag, drains its in-flight copies and MMAs and frees TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "common.cuh"
#include "ptx.cuh"

namespace tpx {

namespace {

constexpr int BM = 128;
constexpr int BN = 256;                  // MMA N (output tile width; 128 for SwiGLU)
constexpr int BK = 64;                   // one 128-byte swizzle atom of bf16
constexpr int STAGES = 4;
constexpr int THREADS = 192;
constexpr uint32_t A_STAGE = BM * BK * 2;        // 16 KiB
constexpr uint32_t B_STAGE = BN * BK * 2;        // 32 KiB
constexpr uint32_t B_BOX = 64 * BK * 2;          // one 64(N) x 64(K) box, 8 KiB
constexpr uint32_t TMEM_COLS = 512;              // two 128 x 256 fp32 accumulators
constexpr int RASTER_BAND = 16;                  // row-tiles per raster band
constexpr size_t SMEM_BYTES = 1024 + STAGES * (A_STAGE + B_STAGE) + 256;
constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, /*a_mn=*/false, /*b_mn=*/true);

struct GemmParams {
  CUtensorMap ta[TP_MAX_SHARDS];    // A views
  CUtensorMap tb[TP_MAX_SHARDS];    // B views (the gate half for SwiGLU)
  CUtensorMap tb2[TP_MAX_SHARDS];   // up-half views (SwiGLU only)
  void* c[TP_MAX_SHARDS];
  int M, N, K;                      // N = output columns
  int groups, tiles_m, tiles_n, row_tiles, num_tiles, num_kb;
  uint32_t* status;
  unsigned long long budget;
};

struct Tile {
  int g, m0, n0;
};

// Tile index -> (shard, m0, n0). Row-tiles of all shards form one sequence (shard-major); it is cut
// into bands of RASTER_BAND row-tiles and each band is swept across all n-tiles, row-tile fastest.
__device__ __forceinline__ Tile decode_tile(const GemmParams& p, int tile, int tile_n_cols) {
  const int band_tiles = RASTER_BAND * p.tiles_n;
  const int band = tile / band_tiles;
  const int first = band * RASTER_BAND;
  const int in_band = min(RASTER_BAND, p.row_tiles - first);
  const int local = tile - band * band_tiles;
  const int rt = first + local % in_band;
  const int nt = local / in_band;
  Tile t;
  t.g = rt / p.tiles_m;
  t.m0 = (rt - t.g * p.tiles_m) * BM;
  t.n0 = nt * tile_n_cols;
  return t;
}

__device__ __forceinline__ float gelu_erf(float x) { return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f)); }
__device__ __forceinline__ float gelu_tanh(float x) {
  return 0.5f * x * (1.0f + tanhf(0.79788456080286536f * (x + 0.044715f * x * x * x)));
}
__device__ __forceinline__ float silu(float x) { return x / (1.0f + __expf(-x)); }

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(lo))) |
         (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(hi))) << 16);
}

// Store 32 consecutive output columns [col0, col0+32) of one row.
template <int EPI>
__device__ __forceinline__ void store_row_chunk(void* cbase, int N, int row, int col0, const uint32_t (&v)[32],
                                                const uint32_t (&u)[32]) {
  if constexpr (EPI == EPI_F32) {
    float* dst = static_cast<float*>(cbase) + static_cast<int64_t>(row) * N + col0;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (col0 + 4 * j < N) st_v4(dst + 4 * j, make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
  } else {
    float f[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float x = __uint_as_float(v[j]);
      if constexpr (EPI == EPI_BF16) f[j] = x;
      else if constexpr (EPI == EPI_GELU) f[j] = gelu_erf(x);
      else if constexpr (EPI == EPI_GELU_TANH) f[j] = gelu_tanh(x);
      else f[j] = silu(x) * __uint_as_float(u[j]);
    }
    uint16_t* dst = static_cast<uint16_t*>(cbase) + static_cast<int64_t>(row) * N + col0;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (col0 + 8 * j < N)
        st_v4(dst + 8 * j, make_uint4(pack2(f[8 * j], f[8 * j + 1]), pack2(f[8 * j + 2], f[8 * j + 3]),
                                      pack2(f[8 * j + 4], f[8 * j + 5]), pack2(f[8 * j + 6], f[8 * j + 7])));
  }
}

template <int EPI>
__global__ void __launch_bounds__(THREADS, 1) gemm_tcgen05_kernel(const __grid_constant__ GemmParams p) {
  constexpr bool SWIGLU = EPI == EPI_SWIGLU;
  constexpr int TILE_N = SWIGLU ? BN / 2 : BN;   // output columns per tile

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + STAGES * B_STAGE);
  // bars: full[STAGES], empty[STAGES], acc_full[2], acc_empty[2], drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * STAGES;
  const uint32_t accf0 = empty0 + 8 * STAGES;
  const uint32_t acce0 = accf0 + 16;
  const uint32_t drain = acce0 + 16;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(accf0 + 8 * a, 1);
      mbar_init(acce0 + 8 * a, 4);   // one arrive per epilogue warp
    }
    mbar_init(drain, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int g = 0; g < p.groups; ++g) {
      prefetch_tmap(&p.ta[g]);
      prefetch_tmap(&p.tb[g]);
      if (SWIGLU) prefetch_tmap(&p.tb2[g]);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // producer bookkeeping, used again at teardown
  int last_phase[STAGES];
  bool issued[STAGES];
#pragma unroll
  for (int s = 0; s < STAGES; ++s) { last_phase[s] = 0; issued[s] = false; }
  bool mma_issued = false;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
        const Tile tl = decode_tile(p, tile, TILE_N);
        bool ok = true;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait_bounded(empty0 + 8 * stage, phase ^ 1u, p.budget, abort_flag)) {
            if (!*abort_flag) record_timeout(p.status, WAIT_PRODUCER_EMPTY);
            *abort_flag = 1u;
            ok = false;
            break;
          }
          const uint32_t fb = full0 + 8 * stage;
          mbar_arrive_expect_tx(fb, A_STAGE + B_STAGE);
          const uint32_t a_dst = smem_u32(sA + stage * A_STAGE);
          const uint32_t b_dst = smem_u32(sB + stage * B_STAGE);
          const int k0 = kb * BK;
          tma_load_2d(a_dst, &p.ta[tl.g], k0, tl.m0, fb);
          if constexpr (SWIGLU) {
            tma_load_2d(b_dst + 0 * B_BOX, &p.tb[tl.g], tl.n0, k0, fb);
            tma_load_2d(b_dst + 1 * B_BOX, &p.tb[tl.g], tl.n0 + 64, k0, fb);
            tma_load_2d(b_dst + 2 * B_BOX, &p.tb2[tl.g], tl.n0, k0, fb);
            tma_load_2d(b_dst + 3 * B_BOX, &p.tb2[tl.g], tl.n0 + 64, k0, fb);
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) tma_load_2d(b_dst + j * B_BOX, &p.tb[tl.g], tl.n0 + 64 * j, k0, fb);
          }
          issued[stage] = true;
          last_phase[stage] = static_cast<int>(phase);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
        bool ok = mbar_wait_bounded(acce0 + 8 * acc, acc_phase ^ 1u, p.budget, abort_flag);
        if (!ok) {
          if (!*abort_flag) record_timeout(p.status, WAIT_MMA_ACC_EMPTY);
          *abort_flag = 1u;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait_bounded(full0 + 8 * stage, phase, p.budget, abort_flag)) {
            if (!*abort_flag) record_timeout(p.status, WAIT_MMA_FULL);
            *abort_flag = 1u;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * A_STAGE);
          const uint32_t b_base = smem_u32(sB + stage * B_STAGE);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            // K-major A: advance 16 elements = 32 bytes inside the swizzle atom.
            const uint64_t ad = smem_desc_sw128(a_base + 32u * k, 16u, 1024u);
            // MN-major B: advance 16 K rows = two 8-row groups of 1 KiB; 64-wide N blocks 8 KiB apart.
            const uint64_t bd = smem_desc_sw128(b_base + 2048u * k, B_BOX, 1024u);
            umma_bf16(d_tmem, ad, bd, IDESC, (kb | k) != 0 ? 1u : 0u);
          }
          mma_issued = true;
          umma_commit(empty0 + 8 * stage);   // frees the stage once these MMAs have read it
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(accf0 + 8 * acc);        // accumulator complete
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
    }
  } else {
    // epilogue warps 2..5; TMEM lane quadrant = warp % 4
    const int quad = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
      const Tile tl = decode_tile(p, tile, TILE_N);
      if (!mbar_wait_bounded(accf0 + 8 * acc, acc_phase, p.budget, abort_flag)) {
        if (!*abort_flag) record_timeout(p.status, WAIT_EPI_ACC_FULL);
        *abort_flag = 1u;
        break;
      }
      tc_fence_after();
      const int row = tl.m0 + quad * 32 + lane;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(acc * BN);
      void* cbase = p.c[tl.g];
#pragma unroll 1
      for (int ch = 0; ch < TILE_N / 32; ++ch) {
        uint32_t v[32], u[32];
        tmem_ld32(t_row + ch * 32, v);
        if constexpr (SWIGLU) tmem_ld32(t_row + 128 + ch * 32, u);
        tmem_ld_wait();
        const int col0 = tl.n0 + ch * 32;
        if (row < p.M && col0 < p.N) store_row_chunk<EPI>(cbase, p.N, row, col0, v, u);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce0 + 8 * acc);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  // ---- teardown: drain in-flight TMA and MMA work before TMEM is released -------------------
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (*abort_flag != 0u) {
    const unsigned long long drain_budget = 4000000000ull;
    if (warp == 0 && lane == 0) {
      for (int s = 0; s < STAGES; ++s)
        if (issued[s] && !mbar_wait_bounded(full0 + 8 * s, static_cast<uint32_t>(last_phase[s]), drain_budget, nullptr))
          record_timeout(p.status, WAIT_TEARDOWN);
    }
    if (warp == 1 && lane == 0 && mma_issued) {
      umma_commit(drain);
      if (!mbar_wait_bounded(drain, 0, drain_budget, nullptr)) record_timeout(p.status, WAIT_TEARDOWN);
    }
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D bf16 view [outer, inner] with row stride `ld` elements, 128-byte swizzled boxes.
bool encode_bf16_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t ld,
                    uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int EPI>
tp_status launch(GemmParams& p, cudaStream_t s) {
  static int configured_for[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(TP_ECUDA, "cudaGetDevice failed");
  if (dev >= 0 && dev < 64 && !configured_for[dev]) {
    if (cudaFuncSetAttribute(gemm_tcgen05_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(SMEM_BYTES)) != cudaSuccess)
      return fail(TP_ECUDA, "cannot reserve %zu bytes of shared memory", SMEM_BYTES);
    configured_for[dev] = 1;
  }
  const int sms = sm_count();
  const int grid = p.num_tiles < sms ? p.num_tiles : sms;
  gemm_tcgen05_kernel<EPI><<<grid, THREADS, SMEM_BYTES, s>>>(p);
  return check_launch("gemm_tcgen05_kernel");
}

}  // namespace

tp_status grouped_gemm(const GemmArgs& g, cudaStream_t s) {
  if (g.groups < 1 || g.groups > TP_MAX_SHARDS) return fail(TP_EINVAL, "groups=%d outside 1..%d", g.groups, TP_MAX_SHARDS);
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return fail(TP_EINVAL, "non-positive GEMM size");
  if (g.M > INT32_MAX / 2 || g.N > INT32_MAX / 2 || g.K > INT32_MAX / 2) return fail(TP_ESHAPE, "GEMM size too large");
  const bool swiglu = g.epi == EPI_SWIGLU;
  if (g.K % 8 || g.N % 8 || g.lda % 8 || g.ldb % 8) return fail(TP_EALIGN, "K, N and row strides must be multiples of 8");
  if (g.lda < g.K || g.ldb < (swiglu ? 2 * g.N : g.N)) return fail(TP_ESHAPE, "row stride shorter than the row");
  for (int i = 0; i < g.groups; ++i) {
    if (g.a[i] == nullptr || g.b[i] == nullptr || g.c[i] == nullptr) return fail(TP_EINVAL, "null GEMM operand %d", i);
    if (!aligned16(g.a[i]) || !aligned16(g.b[i]) || !aligned16(g.c[i])) return fail(TP_EALIGN, "GEMM operand %d not 16-byte aligned", i);
  }
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  const int tile_n = swiglu ? BN / 2 : BN;
  for (int i = 0; i < g.groups; ++i) {
    if (!encode_bf16_2d(&p.ta[i], g.a[i], g.K, g.M, g.lda, BK, BM))
      return fail(TP_ECUDA, "cannot encode the TMA descriptor of A[%d]", i);
    if (!encode_bf16_2d(&p.tb[i], g.b[i], g.N, g.K, g.ldb, 64, BK))
      return fail(TP_ECUDA, "cannot encode the TMA descriptor of B[%d]", i);
    if (swiglu && !encode_bf16_2d(&p.tb2[i], g.b[i] + g.N, g.N, g.K, g.ldb, 64, BK))
      return fail(TP_ECUDA, "cannot encode the TMA descriptor of the up half of B[%d]", i);
    p.c[i] = g.c[i];
  }
  p.M = static_cast<int>(g.M);
  p.N = static_cast<int>(g.N);
  p.K = static_cast<int>(g.K);
  p.tiles_m = static_cast<int>((g.M + BM - 1) / BM);
  p.tiles_n = static_cast<int>((g.N + tile_n - 1) / tile_n);
  p.groups = g.groups;
  p.row_tiles = g.groups * p.tiles_m;
  const int64_t tiles = static_cast<int64_t>(g.groups) * p.tiles_m * p.tiles_n;
  if (tiles > INT32_MAX) return fail(TP_ESHAPE, "too many tiles");
  p.num_tiles = static_cast<int>(tiles);
  p.num_kb = static_cast<int>((g.K + BK - 1) / BK);
  p.status = status_word();
  p.budget = wait_budget();
  if (p.status == nullptr) return fail(TP_ECUDA, "cannot resolve the device status word");
  switch (g.epi) {
    case EPI_F32: return launch<EPI_F32>(p, s);
    case EPI_BF16: return launch<EPI_BF16>(p, s);
    case EPI_GELU: return launch<EPI_GELU>(p, s);
    case EPI_GELU_TANH: return launch<EPI_GELU_TANH>(p, s);
    case EPI_SWIGLU: return launch<EPI_SWIGLU>(p, s);
  }
  return fail(TP_EINVAL, "bad epilogue");
}

}  // namespace tpx
