// bf16 GEMMs on the 5th-generation tensor cores (tcgen05) with fused epilogues.
//
// Four persistent, warp-specialised kernels share one TMA -> shared memory -> tcgen05.mma -> TMEM
// pipeline, in a single-CTA form and a CTA-pair form (cluster 2x1, tcgen05 cta_group::2):
//
//  gemm_tcgen05_kernel / gemm_pair_kernel: grouped GEMM C_g = epi(A_g B_g). They serve the
//    column-parallel GEMM Z_r = act(X W_r), the row-parallel GEMM U_r = Z_r W_r when the partials
//    themselves are wanted ("张量并行与序列并行", §矩阵乘法的两种切法 and §MLP：先列后行，只通信一次),
//    and the local products of the sharded-matmul cases ("Scaling Book 入门第 6 章", §6.2). All t
//    shards of one layer run in ONE launch over the tile space (shard, m-tile, n-tile). An operand
//    may be given as the t pieces of an AllGather, each box read from the piece that holds it: A's
//    row pieces (TP+SP input, case 4 gather X), A's K pieces (case 2 AllGather) or B's column pieces
//    (case 4 gather W). The gather then never reaches memory ("Scaling Book 入门第 6 章", §6.6).
//
//  gemm_ring_kernel / gemm_ring_pair_kernel: the row-parallel GEMM fused with its collective, the
//    one-GPU form of the pages' collective matmul ("Scaling Book 入门第 6 章", §6.6;
//    "张量并行与序列并行", §把通信藏到计算后面). For each output tile they compute the t shards' partial
//    tiles U_s = A_s B_s one after another IN RING ORDER (s = c+1, c+2, ..., c for the tile's chunk
//    c) into alternating TMEM accumulators. The epilogue adds them into an fp32 running sum in
//    registers, one binary32 add per shard, which is exactly the ReduceScatter's summation order. It
//    then writes the tile once: to shard c's output (ReduceScatter) or to all t outputs (AllReduce =
//    ReduceScatter followed by AllGather, its chunks rows or columns), optionally adding a residual
//    and writing a bf16 copy. The fp32 partials never reach HBM. Each U_s tile comes from the same
//    MMA instruction sequence as the plain GEMM's, so the results are bit-identical to the unfused
//    GEMM followed by the ring kernel.
//
// Pipeline (sm_100a):
//   * warp 0, one lane: TMA producer. A [M,K] is K-major (64 x 128 boxes, 128-byte swizzle); B [K,N]
//     is the weight as stored, [in, out] row-major, i.e. MN-major (64 x 64 boxes, 128-byte swizzle);
//     the transposed forms (A stored [K][M], B stored [N][K]) swap the box shapes;
//   * warp 1, one lane: tcgen05.mma issuer, K=16 per instruction, fp32 in TMEM. Single CTA: M=128,
//     N=256, a 4-stage ring of 48 KB stages. CTA pair: M=256 over the pair (each CTA holds 128 rows
//     of A and half of B's 256 columns), a 3-stage ring of 64 KB stages per CTA, each stage two
//     64-deep k-blocks (eight MMAs per barrier round trip), issued by the pair's leader, whose
//     barriers count both CTAs' TMA bytes;
//   * two TMEM accumulators of 256 columns, so the epilogue of one unit overlaps the main loop of the
//     next;
//   * tiles in raster bands of row-tiles swept across the n-tiles, each band holding about 32 MiB
//     of A rows so that they stay in L2 while the band's B panels stream past;
//   * the remaining warps: epilogue (tcgen05.ld 32 columns at a time; the plain GEMMs stage each
//     warp's 32 x 32 output block through shared memory so that every store instruction writes
//     whole row segments of 64 or 128 bytes);
//   * every mbarrier wait is bounded: on expiry the kernel records the site in the status word,
//     raises a shared abort flag, drains its in-flight copies and MMAs and frees TMEM.
// No TMA load uses cluster multicast; the pair's commits reach both CTAs through tcgen05.commit's
// multicast form.
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
constexpr uint32_t A_STAGE = BM * BK * 2;        // 16 KiB
constexpr uint32_t B_STAGE = BN * BK * 2;        // 32 KiB
constexpr uint32_t B_BOX = 64 * BK * 2;          // one 64(N) x 64(K) box, 8 KiB
constexpr uint32_t TMEM_COLS = 512;              // two 128 x 256 fp32 accumulators
constexpr int RASTER_BAND_MAX = 16;              // row-tiles per raster band, at most
constexpr int64_t RASTER_A_BYTES = 32ll << 20;   // A rows one band keeps in L2 while its B panels stream

constexpr int GEMM_THREADS = 192;                // producer, MMA, 4 epilogue warps
constexpr int RING_THREADS = 320;                // producer, MMA, 8 epilogue warps
constexpr uint32_t STAGING_PER_WARP = 32 * 128;  // 32 rows x 128 bytes
constexpr size_t GEMM_SMEM = 1024 + STAGES * (A_STAGE + B_STAGE) + 256;
// CTA-pair (cta_group::2) variant: a 256 x 256 tile per pair, each CTA holding 128 rows of A and
// 128 of B's columns per k-block. A stage holds TWO 64-deep k-blocks (K = 128), so each barrier
// round trip and each commit covers eight MMAs instead of four; 3 such stages fit. Measured against
// 6 stages of one k-block: 9-19% faster (and 2 stages of three k-blocks: 20% slower).
constexpr int PAIR_KB = 2;                           // k-blocks per stage
constexpr int PAIR_STAGES = 3;
constexpr uint32_t PAIR_A_HALF = 128 * BK * 2;       // one k-block of this CTA's 128 A rows: 16 KiB
constexpr uint32_t PAIR_B_HALF = 128 * BK * 2;       // one k-block of its 128 B columns: 16 KiB
constexpr uint32_t PAIR_A_STAGE = PAIR_KB * PAIR_A_HALF;   // 32 KiB
constexpr uint32_t PAIR_B_STAGE = PAIR_KB * PAIR_B_HALF;   // 32 KiB
constexpr size_t PAIR_SMEM = 1024 + PAIR_STAGES * (PAIR_A_STAGE + PAIR_B_STAGE) + 256;
constexpr size_t RING_SMEM = 1024 + STAGES * (A_STAGE + B_STAGE) + 8 * STAGING_PER_WARP + 256;
constexpr size_t RING_PAIR_SMEM = 1024 + PAIR_STAGES * (PAIR_A_STAGE + PAIR_B_STAGE) + 8 * STAGING_PER_WARP + 256;

// ------------------------------------------------------------------ shared pipeline pieces
struct Ring {
  int stage = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void advance() {
    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
  }
};

struct Ctl {
  uint8_t* sA;
  uint8_t* sB;
  uint32_t full0, empty0, accf0, acce0, drain;
  volatile uint32_t* abort_flag;
  uint32_t* status;
  unsigned long long budget;
  uint64_t b_policy;                       // L2 policy of the B (weight) loads
  bool a_mn;                               // A given transposed: stored [K][M] (M contiguous)
  bool b_km;                               // B given transposed: stored [N][K] (K contiguous)
  uint32_t idesc;                          // instruction descriptor for these major-nesses
};

__device__ __forceinline__ bool wait_or_abort(const Ctl& c, uint32_t bar, uint32_t parity, uint32_t site) {
  if (mbar_wait_bounded(bar, parity, c.budget, c.abort_flag)) return true;
  if (!*c.abort_flag) record_timeout(c.status, site);
  *c.abort_flag = 1u;
  return false;
}

// Lays out barriers and the TMEM slot after the operand stages (and the staging area, if any).
__device__ __forceinline__ Ctl setup_ctl(uint8_t* smem, uint32_t extra_bytes, uint32_t*& tmem_slot, uint32_t* status,
                                         unsigned long long budget, bool keep_b, bool a_mn, bool b_km) {
  Ctl c;
  c.sA = smem;
  c.sB = smem + STAGES * A_STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(c.sB + STAGES * B_STAGE + extra_bytes);
  c.full0 = smem_u32(bars);
  c.empty0 = c.full0 + 8 * STAGES;
  c.accf0 = c.empty0 + 8 * STAGES;
  c.acce0 = c.accf0 + 16;
  c.drain = c.acce0 + 16;
  tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  c.abort_flag = tmem_slot + 1;
  c.status = status;
  c.budget = budget;
  c.b_policy = keep_b ? l2_policy_evict_last() : l2_policy_evict_normal();
  c.a_mn = a_mn;
  c.b_km = b_km;
  c.idesc = idesc_bf16_f32(BM, BN, a_mn, !b_km);
  return c;
}

__device__ __forceinline__ void init_barriers(const Ctl& c, uint32_t epilogue_warps) {
  for (int s = 0; s < STAGES; ++s) {
    mbar_init(c.full0 + 8 * s, 1);
    mbar_init(c.empty0 + 8 * s, 1);
  }
  for (int a = 0; a < 2; ++a) {
    mbar_init(c.accf0 + 8 * a, 1);
    mbar_init(c.acce0 + 8 * a, epilogue_warps);   // one arrive per epilogue warp
  }
  mbar_init(c.drain, 1);
  *c.abort_flag = 0u;
  fence_mbar_init();
}

// Operand pieces of a sliced operand: the view that holds element `x` of the sliced dimension, and
// x's place inside it. Past the last piece the last view is used with an out-of-range coordinate,
// which TMA fills with zeros (the padding k-block of an odd k-block count, a partial last tile).
__device__ __forceinline__ const CUtensorMap* slice_view(const CUtensorMap* base, int width, int count, int x, int& lx) {
  if (width == 0) {
    lx = x;
    return base;
  }
  int sl = x / width;
  if (sl > count - 1) sl = count - 1;
  lx = x - sl * width;
  return base + sl;
}

// Producer: the num_kb k-blocks of one unit. B is four 64-wide boxes of `b` at n0 (b2 == nullptr),
// or two boxes of `b` and two of `b2`, both at n0 (SwiGLU: gate and up halves). a_kslice != 0: A is
// a_kslices views of a_kslice columns each, starting at `a` (A split along K). b_nslice != 0: B is
// b_nslices views of b_nslice columns each, starting at `b` (B split along N).
__device__ __forceinline__ bool produce_unit(const Ctl& c, Ring& r, const CUtensorMap* a, const CUtensorMap* b,
                                             const CUtensorMap* b2, int m0, int n0, int num_kb, int* last_phase,
                                             bool* issued, int a_kslice = 0, int a_kslices = 1, int b_nslice = 0,
                                             int b_nslices = 1) {
  // Slice views are chosen without divisions in the loop: B's four boxes once per unit, A's piece by
  // counting k-blocks (the producer's per-stage latency paces the whole pipeline).
  const CUtensorMap* bv[4];
  int bn[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) bv[j] = slice_view(b, b_nslice, b_nslices, n0 + 64 * j, bn[j]);
  const int a_kbs = a_kslice / BK;      // k-blocks per A piece (0: A not split along K)
  int a_sl = 0, a_lk = 0;
  for (int kb = 0; kb < num_kb; ++kb) {
    if (!wait_or_abort(c, c.empty0 + 8 * r.stage, r.phase ^ 1u, WAIT_PRODUCER_EMPTY)) return false;
    const uint32_t fb = c.full0 + 8 * r.stage;
    mbar_arrive_expect_tx(fb, A_STAGE + B_STAGE);
    const uint32_t a_dst = smem_u32(c.sA + r.stage * A_STAGE);
    const uint32_t b_dst = smem_u32(c.sB + r.stage * B_STAGE);
    const int k0 = kb * BK;
    if (c.a_mn) {                       // A^T [K][M]: two 64(M) x 64(K) boxes
      tma_load_2d(a_dst, a, m0, k0, fb);
      tma_load_2d(a_dst + B_BOX, a, m0 + 64, k0, fb);
    } else {                            // A [M][K]: one 64(K) x 128(M) box
      const CUtensorMap* av = a;
      int ak0 = k0;
      if (a_kbs) {
        if (a_lk == a_kbs && a_sl < a_kslices - 1) { ++a_sl; a_lk = 0; }
        av = a + a_sl;
        ak0 = a_lk++ * BK;
      }
      tma_load_2d(a_dst, av, ak0, m0, fb);
    }
    // B (the weights) is re-read by every row-tile: the fused kernel keeps its lines in L2 longest
    if (c.b_km) {                       // B^T [N][K]: one 64(K) x 256(N) box
      tma_load_2d_hint(b_dst, b, k0, n0, fb, c.b_policy);
    } else if (b2 != nullptr) {
      tma_load_2d_hint(b_dst + 0 * B_BOX, b, n0, k0, fb, c.b_policy);
      tma_load_2d_hint(b_dst + 1 * B_BOX, b, n0 + 64, k0, fb, c.b_policy);
      tma_load_2d_hint(b_dst + 2 * B_BOX, b2, n0, k0, fb, c.b_policy);
      tma_load_2d_hint(b_dst + 3 * B_BOX, b2, n0 + 64, k0, fb, c.b_policy);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) tma_load_2d_hint(b_dst + j * B_BOX, bv[j], bn[j], k0, fb, c.b_policy);
    }
    issued[r.stage] = true;
    last_phase[r.stage] = static_cast<int>(r.phase);
    r.advance();
  }
  return true;
}

// MMA issuer: accumulate one unit's num_kb k-blocks into d_tmem (the first one overwrites).
__device__ __forceinline__ bool mma_unit(const Ctl& c, Ring& r, uint32_t d_tmem, int num_kb, bool& mma_issued) {
  for (int kb = 0; kb < num_kb; ++kb) {
    if (!wait_or_abort(c, c.full0 + 8 * r.stage, r.phase, WAIT_MMA_FULL)) return false;
    tc_fence_after();
    const uint32_t a_base = smem_u32(c.sA + r.stage * A_STAGE);
    const uint32_t b_base = smem_u32(c.sB + r.stage * B_STAGE);
#pragma unroll
    for (int k = 0; k < BK / 16; ++k) {
      // K-major: advance 16 elements = 32 bytes inside the swizzle atom (8-row atoms of 1 KiB).
      // MN-major: advance 16 K rows = two 8-row groups of 1 KiB; 64-wide MN blocks 8 KiB apart.
      const uint64_t ad = c.a_mn ? smem_desc_sw128(a_base + 2048u * k, B_BOX, 1024u)
                                 : smem_desc_sw128(a_base + 32u * k, 16u, 1024u);
      const uint64_t bd = c.b_km ? smem_desc_sw128(b_base + 32u * k, 16u, 1024u)
                                 : smem_desc_sw128(b_base + 2048u * k, B_BOX, 1024u);
      umma_bf16(d_tmem, ad, bd, c.idesc, (kb | k) != 0 ? 1u : 0u);
    }
    mma_issued = true;
    umma_commit(c.empty0 + 8 * r.stage);   // frees the stage once these MMAs have read it
    r.advance();
  }
  return true;
}

// After all roles left their loops: if the kernel aborted, wait (bounded) for the copies and MMAs
// still in flight, then free TMEM. Called by every thread.
__device__ __forceinline__ void teardown(const Ctl& c, int warp, int lane, const int* last_phase, const bool* issued,
                                         bool mma_issued, uint32_t tmem_base) {
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (*c.abort_flag != 0u) {
    const unsigned long long drain_budget = 4000000000ull;
    if (warp == 0 && lane == 0) {
      for (int s = 0; s < STAGES; ++s)
        if (issued[s] && !mbar_wait_bounded(c.full0 + 8 * s, static_cast<uint32_t>(last_phase[s]), drain_budget, nullptr))
          record_timeout(c.status, WAIT_TEARDOWN);
    }
    if (warp == 1 && lane == 0 && mma_issued) {
      umma_commit(c.drain);
      if (!mbar_wait_bounded(c.drain, 0, drain_budget, nullptr)) record_timeout(c.status, WAIT_TEARDOWN);
    }
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
}

// Tile index -> (row-tile, n-tile). Row-tiles form one sequence; it is cut into bands of `band_rows`
// row-tiles and each band is swept across all n-tiles, row-tile fastest.
__device__ __forceinline__ void raster(int tile, int row_tiles, int tiles_n, int band_rows, int& rt, int& nt) {
  const int band_tiles = band_rows * tiles_n;
  const int band = tile / band_tiles;
  const int first = band * band_rows;
  const int in_band = min(band_rows, row_tiles - first);
  const int local = tile - band * band_tiles;
  rt = first + local % in_band;
  nt = local / in_band;
}

// Fused-kernel tile order: chunk by chunk, so that every running tile streams the same shard's
// operands at about the same time (all tiles of a chunk follow the same ring order). Axis 0: the
// chunk's row-tiles fastest, then its n-tiles. Axis 1: all row-tiles fastest, then the chunk's n-tiles.
__device__ __forceinline__ void raster_by_chunk(int tile, int tiles_m, int tiles_n, int axis, int chunk_tiles, int& rt,
                                                int& nt) {
  if (axis == 0) {
    const int per_chunk = chunk_tiles * tiles_n;           // chunk_tiles row-tiles per chunk
    const int c = tile / per_chunk;
    const int local = tile - c * per_chunk;
    rt = c * chunk_tiles + local % chunk_tiles;
    nt = local / chunk_tiles;
  } else {
    const int per_chunk = tiles_m * chunk_tiles;           // chunk_tiles n-tiles per chunk
    const int c = tile / per_chunk;
    const int local = tile - c * per_chunk;
    rt = local % tiles_m;
    nt = c * chunk_tiles + local / tiles_m;
  }
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

__device__ __forceinline__ void st_shared_v4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}
__device__ __forceinline__ void st_shared_u4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}
__device__ __forceinline__ uint4 ld_shared_u4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ float4 ld_shared_v4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr) : "memory");
  return v;
}

// ------------------------------------------------------------------ grouped GEMM
struct GemmParams {
  CUtensorMap ta[TP_MAX_SHARDS];    // A views
  CUtensorMap tb[TP_MAX_SHARDS];    // B views (the gate half for SwiGLU)
  CUtensorMap tb2[TP_MAX_SHARDS];   // up-half views (SwiGLU only)
  void* c[TP_MAX_SHARDS];
  int M, N, K;                      // N = output columns
  int groups, tiles_m, tiles_n, row_tiles, num_tiles, num_kb;
  // A given as row slices shared by all groups (the sequence-parallel entry: A = AllGather of t
  // row shards): row m of A is row m % slice_rows of ta[m / slice_rows]. 0 = one A per group.
  int a_slices, slice_rows;
  // A given as a_kslices column slices of a_kslice columns shared by all groups (the AllGather along
  // the contraction): column k of A is column k % a_kslice of ta[k / a_kslice]. 0 = not sliced.
  int a_kslice, a_kslices;
  // B given as b_nslices column slices of b_nslice columns shared by all groups (the AllGather of a
  // column-split weight): column n of B is column n % b_nslice of tb[n / b_nslice]. 0 = not sliced.
  int b_nslice, b_nslices;
  int n_amaps, n_bmaps;             // tensor maps in ta[] / tb[] (prefetched at start)
  int band;                         // row-tiles per raster band
  bool a_mn, b_km;                  // A stored [K][M] / B stored [N][K] (transposed operands)
  uint32_t* status;
  unsigned long long budget;
};

// Tensor map and local row of A for a tile starting at row m0 of group g.
__device__ __forceinline__ const CUtensorMap* a_view(const GemmParams& p, int g, int m0, int& am0) {
  if (p.a_kslice) {                 // every group reads the same K slices (chosen per k-block)
    am0 = m0;
    return &p.ta[0];
  }
  if (p.a_slices) {
    const int sl = m0 / p.slice_rows;
    am0 = m0 - sl * p.slice_rows;
    return &p.ta[sl];
  }
  am0 = m0;
  return &p.ta[g];
}


// fp32 output of one warp: a 32 x 32 block held one row per lane (lane i: row row0 + i, columns col0..
// col0+31), written through the warp's 4 KiB staging buffer. Its 16-byte pieces are XOR-swizzled by
// row, so that the row-wise writes and the column-wise reads are free of bank conflicts, and each
// store instruction covers four rows x 128 contiguous bytes instead of 32 rows x 16 bytes.
__device__ __forceinline__ void store_f32_staged(void* cbase, int M, int N, uint32_t stg, int lane,
                                                 const uint32_t (&v)[32], int row0, int col0) {
#pragma unroll
  for (int j = 0; j < 8; ++j)
    st_shared_v4(stg + lane * 128 + ((j ^ (lane & 7)) << 4), __uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                 __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
  __syncwarp();
  const int sub = lane & 7;
  float* c = static_cast<float*>(cbase);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int r = 4 * k + (lane >> 3);
    const float4 x = ld_shared_v4(stg + r * 128 + ((sub ^ (r & 7)) << 4));
    const int row = row0 + r;
    const int col = col0 + 4 * sub;   // N % 8 == 0: a vector inside N lies wholly inside it
    if (row < M && col < N)
      st_v4(c + static_cast<int64_t>(row) * N + col,
            make_uint4(__float_as_uint(x.x), __float_as_uint(x.y), __float_as_uint(x.z), __float_as_uint(x.w)));
  }
  __syncwarp();
}

// bf16 output of one warp: 32 rows x 32 columns (64 bytes a row), one row per lane, formed by the
// epilogue in registers (f: 32 values of this lane's row). Staged like store_f32_staged, with the
// 64-byte swizzle (piece j of row r at piece j ^ ((r / 2) % 4)); each store instruction then covers
// eight rows x 64 contiguous bytes.
__device__ __forceinline__ void store_bf16_staged(void* cbase, int M, int N, uint32_t stg, int lane, const float (&f)[32],
                                                  int row0, int col0) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
    st_shared_u4(stg + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4),
                 make_uint4(pack2(f[8 * j], f[8 * j + 1]), pack2(f[8 * j + 2], f[8 * j + 3]),
                            pack2(f[8 * j + 4], f[8 * j + 5]), pack2(f[8 * j + 6], f[8 * j + 7])));
  __syncwarp();
  const int q = lane & 3;
  uint16_t* c = static_cast<uint16_t*>(cbase);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = 8 * k + (lane >> 2);
    const uint4 x = ld_shared_u4(stg + r * 64 + ((q ^ ((r >> 1) & 3)) << 4));
    const int row = row0 + r;
    const int col = col0 + 8 * q;   // N % 8 == 0: a vector inside N lies wholly inside it
    if (row < M && col < N) st_v4(c + static_cast<int64_t>(row) * N + col, x);
  }
  __syncwarp();
}

// Applies the epilogue's activation to 32 accumulator columns (u: SwiGLU's up half).
template <int EPI>
__device__ __forceinline__ void activate32(const uint32_t (&v)[32], const uint32_t (&u)[32], float (&f)[32]) {
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float x = __uint_as_float(v[j]);
    if constexpr (EPI == EPI_BF16) f[j] = x;
    else if constexpr (EPI == EPI_GELU) f[j] = gelu_erf(x);
    else if constexpr (EPI == EPI_GELU_TANH) f[j] = gelu_tanh(x);
    else f[j] = silu(x) * __uint_as_float(u[j]);
  }
}

template <int EPI>
__global__ void __launch_bounds__(GEMM_THREADS, 1) gemm_tcgen05_kernel(const __grid_constant__ GemmParams p) {
  constexpr bool SWIGLU = EPI == EPI_SWIGLU;
  constexpr int TILE_N = SWIGLU ? BN / 2 : BN;   // output columns per tile

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* tmem_slot;
  constexpr uint32_t STAGING = 4 * STAGING_PER_WARP;   // output staging, one buffer per epilogue warp
  const Ctl c = setup_ctl(smem, STAGING, tmem_slot, p.status, p.budget, false, p.a_mn, p.b_km);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) init_barriers(c, 4);
  if (warp == 0 && lane == 0) {
    for (int g = 0; g < p.n_bmaps; ++g) {
      prefetch_tmap(&p.tb[g]);
      if (SWIGLU) prefetch_tmap(&p.tb2[g]);
    }
    for (int g = 0; g < p.n_amaps; ++g) prefetch_tmap(&p.ta[g]);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  int last_phase[STAGES];
  bool issued[STAGES];
#pragma unroll
  for (int s = 0; s < STAGES; ++s) { last_phase[s] = 0; issued[s] = false; }
  bool mma_issued = false;

  if (warp == 0) {
    if (lane == 0) {
      Ring r;
      for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
        int rt, nt;
        raster(tile, p.row_tiles, p.tiles_n, p.band, rt, nt);
        const int g = rt / p.tiles_m;
        const int m0 = (rt - g * p.tiles_m) * BM;
        int am0;
        const CUtensorMap* ta = a_view(p, g, m0, am0);
        if (!produce_unit(c, r, ta, p.b_nslice ? &p.tb[0] : &p.tb[g], SWIGLU ? &p.tb2[g] : nullptr, am0,
                          nt * TILE_N, p.num_kb, last_phase, issued, p.a_kslice, p.a_kslices, p.b_nslice,
                          p.b_nslices))
          break;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      Ring r;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
        if (!wait_or_abort(c, c.acce0 + 8 * acc, acc_phase ^ 1u, WAIT_MMA_ACC_EMPTY)) break;
        tc_fence_after();
        if (!mma_unit(c, r, tmem_base + static_cast<uint32_t>(acc * BN), p.num_kb, mma_issued)) break;
        umma_commit(c.accf0 + 8 * acc);   // accumulator complete
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
    }
  } else {
    // epilogue warps 2..5; TMEM lane quadrant = warp % 4
    const int quad = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
      int rt, nt;
      raster(tile, p.row_tiles, p.tiles_n, p.band, rt, nt);
      const int g = rt / p.tiles_m;
      const int m0 = (rt - g * p.tiles_m) * BM;
      const int n0 = nt * TILE_N;
      if (!wait_or_abort(c, c.accf0 + 8 * acc, acc_phase, WAIT_EPI_ACC_FULL)) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(acc * BN);
      void* cbase = p.c[g];
      const uint32_t stg = smem_u32(smem + STAGES * (A_STAGE + B_STAGE)) + (warp - 2) * STAGING_PER_WARP;
#pragma unroll 1
      for (int ch = 0; ch < TILE_N / 32; ++ch) {
        uint32_t v[32], u[32];
        tmem_ld32(t_row + ch * 32, v);
        if constexpr (SWIGLU) tmem_ld32(t_row + 128 + ch * 32, u);
        tmem_ld_wait();
        const int col0 = n0 + ch * 32;
        if constexpr (EPI == EPI_F32) {
          store_f32_staged(cbase, p.M, p.N, stg, lane, v, m0 + quad * 32, col0);
        } else {
          float f[32];
          activate32<EPI>(v, u, f);
          store_bf16_staged(cbase, p.M, p.N, stg, lane, f, m0 + quad * 32, col0);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(c.acce0 + 8 * acc);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }
  teardown(c, warp, lane, last_phase, issued, mma_issued, tmem_base);
}

// ------------------------------------------------------------------ CTA-pair pipeline
// The two CTAs of a cluster share 256-row tiles. Each CTA loads its 128 rows of A and its half of
// B's 256 columns (SwiGLU: CTA 0 the gate half, CTA 1 the up half) into its own shared memory, and
// the copies of both CTAs count on the leader's (CTA 0's) full barrier. The leader's single MMA
// thread issues tcgen05.mma.cta_group::2 (M=256, N=256). Its commits arrive on the barrier at the
// same offset in both CTAs (stage free, accumulator ready). Each CTA's TMEM receives its own 128
// rows. The epilogue warps of BOTH CTAs release an accumulator on the leader's barrier.
struct PairCtl {
  uint8_t* sA;
  uint8_t* sB;
  uint32_t full0, empty0, accf0, acce0, drain;
  uint32_t full0_leader, acce0_leader;       // shared::cluster addresses in CTA 0
  volatile uint32_t* abort_flag;
  uint32_t* status;
  unsigned long long budget;
  uint32_t rank;
  uint64_t b_policy;                         // L2 policy of the B (weight) loads
  bool a_mn, b_km;                           // transposed operand storage (see Ctl)
  uint32_t idesc;                            // M=256, N=256
  uint32_t idesc_half;                       // M=256, N=128 (half-width tiles)
};

struct PairRing {
  int stage = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void advance() {
    if (++stage == PAIR_STAGES) { stage = 0; phase ^= 1u; }
  }
};

__device__ __forceinline__ PairCtl pair_setup(uint8_t* smem, uint32_t extra_bytes, uint32_t*& tmem_slot,
                                              uint32_t epilogue_warps_per_cta, uint32_t* status,
                                              unsigned long long budget, bool keep_b, bool a_mn, bool b_km) {
  PairCtl c;
  c.sA = smem;
  c.sB = smem + PAIR_STAGES * PAIR_A_STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(c.sB + PAIR_STAGES * PAIR_B_STAGE + extra_bytes);
  c.full0 = smem_u32(bars);
  c.empty0 = c.full0 + 8 * PAIR_STAGES;
  c.accf0 = c.empty0 + 8 * PAIR_STAGES;
  c.acce0 = c.accf0 + 16;
  c.drain = c.acce0 + 16;
  tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * PAIR_STAGES + 5);
  c.abort_flag = tmem_slot + 1;
  c.status = status;
  c.budget = budget;
  c.rank = cluster_ctarank();
  c.b_policy = keep_b ? l2_policy_evict_last() : l2_policy_evict_normal();
  c.a_mn = a_mn;
  c.b_km = b_km;
  c.idesc = idesc_bf16_f32(2 * BM, BN, a_mn, !b_km);
  c.idesc_half = idesc_bf16_f32(2 * BM, BN / 2, a_mn, !b_km);
  if (threadIdx.x == 0) {
    for (int s = 0; s < PAIR_STAGES; ++s) {
      mbar_init(c.full0 + 8 * s, 1);
      mbar_init(c.empty0 + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(c.accf0 + 8 * a, 1);
      mbar_init(c.acce0 + 8 * a, 2 * epilogue_warps_per_cta);   // epilogue warps of both CTAs
    }
    mbar_init(c.drain, 1);
    *c.abort_flag = 0u;
    fence_mbar_init();
  }
  if (threadIdx.x / 32 == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();   // barriers of both CTAs initialised, TMEM allocated in both
  tc_fence_after();
  c.full0_leader = mapa_shared(c.full0, 0);
  c.acce0_leader = mapa_shared(c.acce0, 0);
  return c;
}

__device__ __forceinline__ bool pair_fail(const PairCtl& c, uint32_t site) {
  if (!*c.abort_flag) record_timeout(c.status, site);
  *c.abort_flag = 1u;
  return false;
}

// Producer of one CTA: the num_kb k-blocks of one unit, PAIR_KB per stage (a k-block past K loads
// zeros and is not multiplied). m0 is this CTA's first row, nb its first B column: two 64-wide boxes
// of `tb` per k-block for a full tile, one for a half-width tile (wide == false, B stored [K][N] only).
__device__ __forceinline__ bool pair_produce_unit(const PairCtl& c, PairRing& r, const CUtensorMap* ta, int m0,
                                                  const CUtensorMap* tb, int nb, int num_kb, bool wide = true,
                                                  int a_kslice = 0, int a_kslices = 1, int b_nslice = 0,
                                                  int b_nslices = 1) {
  const uint32_t tx = 2 * (PAIR_A_STAGE + (wide ? PAIR_B_STAGE : PAIR_B_STAGE / 2));
  // slice views without divisions in the loop (see produce_unit)
  int bn0, bn1;
  const CUtensorMap* bv0 = slice_view(tb, b_nslice, b_nslices, nb, bn0);
  const CUtensorMap* bv1 = slice_view(tb, b_nslice, b_nslices, nb + 64, bn1);
  const int a_kbs = a_kslice / BK;
  int a_sl = 0, a_lk = 0;
  for (int kb = 0; kb < num_kb; kb += PAIR_KB) {
    if (!mbar_wait_bounded(c.empty0 + 8 * r.stage, r.phase ^ 1u, c.budget, c.abort_flag))
      return pair_fail(c, WAIT_PRODUCER_EMPTY);
    if (c.rank == 0) mbar_arrive_expect_tx(c.full0 + 8 * r.stage, tx);
    const uint32_t fb = c.full0_leader + 8 * r.stage;
#pragma unroll
    for (int h = 0; h < PAIR_KB; ++h) {
      const uint32_t a_dst = smem_u32(c.sA + r.stage * PAIR_A_STAGE + h * PAIR_A_HALF);
      const uint32_t b_dst = smem_u32(c.sB + r.stage * PAIR_B_STAGE + h * PAIR_B_HALF);
      const int k0 = (kb + h) * BK;
      if (c.a_mn) {                     // A^T [K][M]: two 64(M) x 64(K) boxes of this CTA's 128 rows
        tma_load_2d_pair(a_dst, ta, m0, k0, fb);
        tma_load_2d_pair(a_dst + B_BOX, ta, m0 + 64, k0, fb);
      } else {
        const CUtensorMap* av = ta;
        int ak0 = k0;
        if (a_kbs) {
          if (a_lk == a_kbs && a_sl < a_kslices - 1) { ++a_sl; a_lk = 0; }
          av = ta + a_sl;
          ak0 = a_lk++ * BK;
        }
        tma_load_2d_pair(a_dst, av, ak0, m0, fb);
      }
      if (c.b_km) {                     // B^T [N][K]: one 64(K) x 128(N) box of this CTA's columns
        tma_load_2d_pair_hint(b_dst, tb, k0, nb, fb, c.b_policy);
      } else {
        tma_load_2d_pair_hint(b_dst, bv0, bn0, k0, fb, c.b_policy);
        if (wide) tma_load_2d_pair_hint(b_dst + B_BOX, bv1, bn1, k0, fb, c.b_policy);
      }
    }
    r.advance();
  }
  return true;
}

// Leader's MMA thread: wait until both CTAs' epilogues released accumulator `acc`.
__device__ __forceinline__ bool pair_wait_acc_empty(const PairCtl& c, int acc, uint32_t parity) {
  bool got = mbar_try_wait_cluster(c.acce0 + 8 * acc, parity);
  if (!got) {
    const long long t0 = clock64();
    while (!(got = mbar_try_wait_cluster(c.acce0 + 8 * acc, parity))) {
      if (*c.abort_flag || static_cast<unsigned long long>(clock64() - t0) > c.budget) break;
    }
  }
  if (!got) return pair_fail(c, WAIT_MMA_ACC_EMPTY);
  tc_fence_after();
  return true;
}

// Leader's MMA thread: one unit's num_kb k-blocks into d_tmem (M=256 over the pair; N=256, or 128
// with c.idesc_half), four K=16 MMAs per k-block, one commit per stage. Only k-blocks below num_kb
// are multiplied, so the MMA sequence is the same as the single-CTA kernels'.
__device__ __forceinline__ bool pair_mma_unit(const PairCtl& c, PairRing& r, uint32_t d_tmem, int num_kb,
                                              bool& mma_issued, uint32_t idesc) {
  for (int kb = 0; kb < num_kb; kb += PAIR_KB) {
    if (!mbar_wait_bounded(c.full0 + 8 * r.stage, r.phase, c.budget, c.abort_flag)) return pair_fail(c, WAIT_MMA_FULL);
    tc_fence_after();
#pragma unroll
    for (int h = 0; h < PAIR_KB; ++h) {
      if (kb + h < num_kb) {
        const uint32_t a_base = smem_u32(c.sA + r.stage * PAIR_A_STAGE + h * PAIR_A_HALF);
        const uint32_t b_base = smem_u32(c.sB + r.stage * PAIR_B_STAGE + h * PAIR_B_HALF);
#pragma unroll
        for (int k = 0; k < BK / 16; ++k) {
          const uint64_t ad = c.a_mn ? smem_desc_sw128(a_base + 2048u * k, B_BOX, 1024u)
                                     : smem_desc_sw128(a_base + 32u * k, 16u, 1024u);
          const uint64_t bd = c.b_km ? smem_desc_sw128(b_base + 32u * k, 16u, 1024u)
                                     : smem_desc_sw128(b_base + 2048u * k, B_BOX, 1024u);
          umma_bf16_pair(d_tmem, ad, bd, idesc, (kb + h) != 0 || k != 0 ? 1u : 0u);
        }
      }
    }
    mma_issued = true;
    umma_commit_pair_mc(c.empty0 + 8 * r.stage, 0x3);   // frees the stage in both CTAs
    r.advance();
  }
  return true;
}

// Epilogue warp: wait for accumulator `acc` in this CTA.
__device__ __forceinline__ bool pair_wait_acc_full(const PairCtl& c, int acc, uint32_t parity) {
  if (!mbar_wait_bounded(c.accf0 + 8 * acc, parity, c.budget, c.abort_flag)) return pair_fail(c, WAIT_EPI_ACC_FULL);
  tc_fence_after();
  return true;
}

// Epilogue warp: hand accumulator `acc` back to the leader's MMA thread.
__device__ __forceinline__ void pair_release_acc(const PairCtl& c, int acc, int lane) {
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive_cluster(c.acce0_leader + 8 * acc);
}

// All pair MMAs complete (they read both CTAs' shared memory and write both TMEMs), then both
// CTAs meet before either releases TMEM or exits.
__device__ __forceinline__ void pair_teardown(const PairCtl& c, int warp, int lane, bool mma_issued,
                                              uint32_t tmem_base) {
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1 && lane == 0 && c.rank == 0 && mma_issued) {
    umma_commit_pair(c.drain);
    if (!mbar_wait_bounded(c.drain, 0, 4000000000ull, nullptr)) record_timeout(c.status, WAIT_TEARDOWN);
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, TMEM_COLS);
}

// ------------------------------------------------------------------ CTA-pair grouped GEMM
// Same computation as gemm_tcgen05_kernel on 256-row tiles shared by the two CTAs of a cluster.
template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GEMM_THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ GemmParams p) {
  constexpr bool SWIGLU = EPI == EPI_SWIGLU;
  constexpr int TILE_N = SWIGLU ? BN / 2 : BN;
  constexpr int TILE_M = 2 * BM;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (warp == 0 && lane == 0) {
    for (int g = 0; g < p.n_bmaps; ++g) {
      prefetch_tmap(&p.tb[g]);
      if (SWIGLU) prefetch_tmap(&p.tb2[g]);
    }
    for (int g = 0; g < p.n_amaps; ++g) prefetch_tmap(&p.ta[g]);
  }
  uint32_t* tmem_slot;
  constexpr uint32_t STAGING = 4 * STAGING_PER_WARP;   // output staging, one buffer per epilogue warp
  const PairCtl c = pair_setup(smem, STAGING, tmem_slot, 4, p.status, p.budget, false, p.a_mn, p.b_km);
  const uint32_t tmem_base = *tmem_slot;
  const int pair = blockIdx.x >> 1;
  const int pairs = gridDim.x >> 1;
  const int tiles_m = (p.M + TILE_M - 1) / TILE_M;
  const int row_tiles = p.groups * tiles_m;
  const int num_tiles = row_tiles * p.tiles_n;
  bool mma_issued = false;

  if (warp == 0) {
    if (lane == 0) {
      PairRing r;
      for (int tile = pair; tile < num_tiles; tile += pairs) {
        int rt, nt;
        raster(tile, row_tiles, p.tiles_n, p.band, rt, nt);
        const int g = rt / tiles_m;
        const int m0 = (rt - g * tiles_m) * TILE_M + static_cast<int>(c.rank) * BM;
        const int n0 = nt * TILE_N;
        const CUtensorMap* tb = SWIGLU ? (c.rank == 0 ? &p.tb[g] : &p.tb2[g]) : p.b_nslice ? &p.tb[0] : &p.tb[g];
        const int nb = SWIGLU ? n0 : n0 + static_cast<int>(c.rank) * 128;
        int am0;
        const CUtensorMap* ta = a_view(p, g, m0, am0);
        if (!pair_produce_unit(c, r, ta, am0, tb, nb, p.num_kb, true, p.a_kslice, p.a_kslices, p.b_nslice,
                               p.b_nslices))
          break;
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && c.rank == 0) {
      PairRing r;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int tile = pair; tile < num_tiles; tile += pairs) {
        if (!pair_wait_acc_empty(c, acc, acc_phase ^ 1u)) break;
        if (!pair_mma_unit(c, r, tmem_base + static_cast<uint32_t>(acc * BN), p.num_kb, mma_issued, c.idesc)) break;
        umma_commit_pair_mc(c.accf0 + 8 * acc, 0x3);   // both halves of the accumulator ready
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
    }
  } else {
    const int quad = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < num_tiles; tile += pairs) {
      int rt, nt;
      raster(tile, row_tiles, p.tiles_n, p.band, rt, nt);
      const int g = rt / tiles_m;
      const int m0 = (rt - g * tiles_m) * TILE_M + static_cast<int>(c.rank) * BM;
      const int n0 = nt * TILE_N;
      if (!pair_wait_acc_full(c, acc, acc_phase)) break;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(acc * BN);
      void* cbase = p.c[g];
      const uint32_t stg = smem_u32(smem + PAIR_STAGES * (PAIR_A_STAGE + PAIR_B_STAGE)) + (warp - 2) * STAGING_PER_WARP;
#pragma unroll 1
      for (int ch = 0; ch < TILE_N / 32; ++ch) {
        uint32_t v[32], u[32];
        tmem_ld32(t_row + ch * 32, v);
        if constexpr (SWIGLU) tmem_ld32(t_row + 128 + ch * 32, u);
        tmem_ld_wait();
        const int col0 = n0 + ch * 32;
        if constexpr (EPI == EPI_F32) {
          store_f32_staged(cbase, p.M, p.N, stg, lane, v, m0 + quad * 32, col0);
        } else {
          float f[32];
          activate32<EPI>(v, u, f);
          store_bf16_staged(cbase, p.M, p.N, stg, lane, f, m0 + quad * 32, col0);
        }
      }
      pair_release_acc(c, acc, lane);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }
  pair_teardown(c, warp, lane, mma_issued, tmem_base);
}

// ------------------------------------------------------------------ fused row GEMM + ring reduction
struct RingGemmParams {
  CUtensorMap ta[TP_MAX_SHARDS];    // A_s [M, K] (K-major)
  CUtensorMap tb[TP_MAX_SHARDS];    // B_s [K, N] (MN-major)
  void* out[TP_MAX_SHARDS];
  const void* resid;                // AllReduce only: added after the ring sum (f32 or bf16 [M, N])
  uint16_t* copy_bf16;              // AllReduce only: bf16 copy of the result [M, N]
  int M, N, t;
  int tiles_m, tiles_n, num_tiles, num_kb;
  int axis;                         // chunk axis of the reduction
  int chunk;                        // rows (axis 0) or columns (axis 1) per chunk
  int chunk_tiles;                  // row-tiles (axis 0) or n-tiles (axis 1) per chunk
  int resid_bf16;
  bool b_km;                        // B stored [N][K] (transposed)
  // CTA-pair kernel schedule: units [0, full_units) are 256 x 256 tiles in raster order; the
  // remaining tiles are cut into two 256 x 128 halves each, units [full_units, num_units).
  int full_units, num_units;
  // AllReduce on CTA pairs with t >= 8: write replica 0 at the tile's end and copy it into the other
  // t - 1 replicas a slice at a time while the next tile's shards run.
  bool defer_replicas;
  uint32_t* status;
  unsigned long long budget;
};


// Writes a 32 x 32 fp32 block held one row per lane (lane i: row row0+i, columns col0..col0+31)
// with coalesced global stores. The block passes through the warp's 4 KiB staging buffer, with its
// 16-byte chunks XOR-swizzled by row so both the row-wise writes and the column-wise reads are free
// of bank conflicts. Each store instruction then covers four rows x 128 contiguous bytes (64 for bf16).
template <bool OUT_BF16, bool AR>
__device__ __forceinline__ void store_block32(const RingGemmParams& p, uint32_t stg, int lane, const float (&v)[32],
                                              int row0, int col0, int c, bool defer = false) {
#pragma unroll
  for (int j = 0; j < 8; ++j)
    st_shared_v4(stg + lane * 128 + ((j ^ (lane & 7)) << 4), v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
  __syncwarp();
  const int sub = lane & 7;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int r = 4 * k + (lane >> 3);
    float4 x = ld_shared_v4(stg + r * 128 + ((sub ^ (r & 7)) << 4));
    const int row = row0 + r;
    const int col = col0 + 4 * sub;
    if (row < p.M && col < p.N) {
      const int64_t e = static_cast<int64_t>(row) * p.N + col;
      if constexpr (AR) {
        if (p.resid != nullptr) {
          float4 q;
          if (p.resid_bf16) {
            const uint2 w = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(p.resid) + e);
            q = make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u), __uint_as_float(w.y << 16),
                            __uint_as_float(w.y & 0xFFFF0000u));
          } else {
            q = *reinterpret_cast<const float4*>(static_cast<const float*>(p.resid) + e);
          }
          x.x = __fadd_rn(x.x, q.x); x.y = __fadd_rn(x.y, q.y); x.z = __fadd_rn(x.z, q.z); x.w = __fadd_rn(x.w, q.w);
        }
        if (defer) {   // replica 0 only, kept in L2 for the copies that follow
          if constexpr (OUT_BF16)
            st_v2(static_cast<uint16_t*>(p.out[0]) + e, make_uint2(pack2(x.x, x.y), pack2(x.z, x.w)));
          else
            st_v4(static_cast<float*>(p.out[0]) + e, make_uint4(__float_as_uint(x.x), __float_as_uint(x.y),
                                                               __float_as_uint(x.z), __float_as_uint(x.w)));
        } else {
          for (int s = 0; s < p.t; ++s) {
            if constexpr (OUT_BF16)
              st_cs_v2(static_cast<uint16_t*>(p.out[s]) + e, make_uint2(pack2(x.x, x.y), pack2(x.z, x.w)));
            else
              st_cs_v4(static_cast<float*>(p.out[s]) + e, make_uint4(__float_as_uint(x.x), __float_as_uint(x.y),
                                                                    __float_as_uint(x.z), __float_as_uint(x.w)));
          }
        }
        if (p.copy_bf16 != nullptr) st_cs_v2(p.copy_bf16 + e, make_uint2(pack2(x.x, x.y), pack2(x.z, x.w)));
      } else {
        // ReduceScatter: chunk c lands in shard c's output, at its place inside the chunk
        const int64_t o = p.axis == 0 ? static_cast<int64_t>(row - c * p.chunk) * p.N + col
                                      : static_cast<int64_t>(row) * p.chunk + (col - c * p.chunk);
        if constexpr (OUT_BF16)
          st_cs_v2(static_cast<uint16_t*>(p.out[c]) + o, make_uint2(pack2(x.x, x.y), pack2(x.z, x.w)));
        else
          st_cs_v4(static_cast<float*>(p.out[c]) + o, make_uint4(__float_as_uint(x.x), __float_as_uint(x.y),
                                                                __float_as_uint(x.z), __float_as_uint(x.w)));
      }
    }
  }
  __syncwarp();
}

// Deferred AllGather leg of the CTA-pair AllReduce: rows [r_begin, r_end) of one warp's region
// (first row row0, first column col0, ncols columns) are copied from replica 0, which this warp
// wrote, into replicas 1..t-1. Copying moves bits, so the replicas stay identical. Loads go out in
// batches of four per lane before their stores, so that a read-back that missed L2 does not
// serialise the loop.
template <bool OUT_BF16>
__device__ __forceinline__ void copy_replica_rows(const RingGemmParams& p, int lane, int row0, int col0, int ncols,
                                                  int r_begin, int r_end) {
  constexpr int PER16 = OUT_BF16 ? 8 : 4;          // elements per 16-byte vector
  constexpr int ESIZE = OUT_BF16 ? 2 : 4;
  constexpr int BATCH = 4;
  const int vec_per_row = ncols / PER16;
  const int total = (r_end - r_begin) * vec_per_row;
  const uint8_t* src = static_cast<const uint8_t*>(p.out[0]);
  for (int base = 0; base < total; base += 32 * BATCH) {
    uint4 v[BATCH];
    int64_t off[BATCH];
#pragma unroll
    for (int b = 0; b < BATCH; ++b) {
      const int idx = base + 32 * b + lane;
      const int row = row0 + r_begin + idx / vec_per_row;
      const int col = col0 + (idx % vec_per_row) * PER16;
      off[b] = (idx < total && row < p.M && col < p.N) ? (static_cast<int64_t>(row) * p.N + col) * ESIZE : -1;
      if (off[b] >= 0) v[b] = ld_cg_v4(src + off[b]);
    }
#pragma unroll
    for (int b = 0; b < BATCH; ++b)
      if (off[b] >= 0)
        for (int s = 1; s < p.t; ++s) st_cs_v4(static_cast<uint8_t*>(p.out[s]) + off[b], v[b]);
  }
}

template <bool OUT_BF16, bool AR>
__global__ void __launch_bounds__(RING_THREADS, 1) gemm_ring_kernel(const __grid_constant__ RingGemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* tmem_slot;
  // the fused kernel re-reads every shard's weight panels from each chunk: keep them in L2
  const Ctl c = setup_ctl(smem, 8 * STAGING_PER_WARP, tmem_slot, p.status, p.budget, true, false, p.b_km);
  const uint32_t staging0 = smem_u32(smem + STAGES * (A_STAGE + B_STAGE));
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int t = p.t;

  if (threadIdx.x == 0) init_barriers(c, 8);
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < t; ++s) {
      prefetch_tmap(&p.ta[s]);
      prefetch_tmap(&p.tb[s]);
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

  int last_phase[STAGES];
  bool issued[STAGES];
#pragma unroll
  for (int s = 0; s < STAGES; ++s) { last_phase[s] = 0; issued[s] = false; }
  bool mma_issued = false;

  if (warp == 0) {
    if (lane == 0) {
      Ring r;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        int mt, nt;
        raster_by_chunk(tile, p.tiles_m, p.tiles_n, p.axis, p.chunk_tiles, mt, nt);
        const int m0 = mt * BM, n0 = nt * BN;
        const int ch = (p.axis == 0 ? m0 : n0) / p.chunk;
        for (int j = 0; ok && j < t; ++j) {
          const int s = (ch + 1 + j) % t;              // ring order of this chunk
          ok = produce_unit(c, r, &p.ta[s], &p.tb[s], nullptr, m0, n0, p.num_kb, last_phase, issued);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      Ring r;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        for (int j = 0; ok && j < t; ++j) {
          ok = wait_or_abort(c, c.acce0 + 8 * acc, acc_phase ^ 1u, WAIT_MMA_ACC_EMPTY);
          if (!ok) break;
          tc_fence_after();
          ok = mma_unit(c, r, tmem_base + static_cast<uint32_t>(acc * BN), p.num_kb, mma_issued);
          if (!ok) break;
          umma_commit(c.accf0 + 8 * acc);
          if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
      }
    }
  } else {
    // epilogue warps 2..9: TMEM lane quadrant = warp % 4; warps 2..5 take columns 0..127 of the
    // tile and warps 6..9 columns 128..255. Each thread keeps its row's 128 running sums.
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const uint32_t stg = staging0 + static_cast<uint32_t>(warp - 2) * STAGING_PER_WARP;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    float sum[4][32];
    for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
      int mt, nt;
      raster_by_chunk(tile, p.tiles_m, p.tiles_n, p.axis, p.chunk_tiles, mt, nt);
      const int m0 = mt * BM, n0 = nt * BN;
      const int ch = (p.axis == 0 ? m0 : n0) / p.chunk;
      for (int j = 0; j < t; ++j) {
        ok = wait_or_abort(c, c.accf0 + 8 * acc, acc_phase, WAIT_EPI_ACC_FULL);
        if (!ok) break;
        tc_fence_after();
        const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                               static_cast<uint32_t>(acc * BN + half * 128);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t v[32];
          tmem_ld32(t_row + q * 32, v);
          tmem_ld_wait();
          if (j == 0) {
#pragma unroll
            for (int i = 0; i < 32; ++i) sum[q][i] = __uint_as_float(v[i]);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) sum[q][i] = __fadd_rn(sum[q][i], __uint_as_float(v[i]));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(c.acce0 + 8 * acc);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok) break;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        store_block32<OUT_BF16, AR>(p, stg, lane, sum[q], m0 + quad * 32, n0 + half * 128 + q * 32, ch);
    }
  }
  teardown(c, warp, lane, last_phase, issued, mma_issued, tmem_base);
}

// Unit u of the CTA-pair fused kernel -> its tile's first row-tile, first column and width.
__device__ __forceinline__ void ring_pair_unit(const RingGemmParams& p, int u, int tiles_m, int& mt, int& n0,
                                               bool& wide) {
  int tile = u, hsel = 0;
  wide = u < p.full_units;
  if (!wide) {
    const int h = u - p.full_units;
    tile = p.full_units + (h >> 1);
    hsel = h & 1;
  }
  int nt;
  raster_by_chunk(tile, tiles_m, p.tiles_n, p.axis, p.chunk_tiles, mt, nt);
  n0 = nt * BN + hsel * (BN / 2);
}

// Fused row GEMM + ring reduction on CTA pairs: the same ring-ordered epilogue as
// gemm_ring_kernel, each CTA summing and storing its own 128 rows of a 256-row pair tile.
//  * Tiles are 256 x 256. For AllReduce, when the last round of tiles would leave at least half of
//    the pairs idle, those tiles are cut into 256 x 128 halves (MMA N = 128) over twice the pairs.
//  * AllReduce with t >= 8: at a tile's end only replica 0 is written; the copies into replicas
//    1..t-1 are spread over the next tile's t shard steps (1/t of the rows after each step), so the
//    t-fold write traffic overlaps the tensor-core work instead of arriving as one burst per tile.
template <bool OUT_BF16, bool AR>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(RING_THREADS, 1)
    gemm_ring_pair_kernel(const __grid_constant__ RingGemmParams p) {
  constexpr int TILE_M = 2 * BM;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int t = p.t;
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < t; ++s) {
      prefetch_tmap(&p.ta[s]);
      prefetch_tmap(&p.tb[s]);
    }
  }
  uint32_t* tmem_slot;
  // the fused kernel re-reads every shard's weight panels from each chunk: keep them in L2
  const PairCtl c = pair_setup(smem, 8 * STAGING_PER_WARP, tmem_slot, 8, p.status, p.budget, true, false, p.b_km);
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t staging0 = smem_u32(smem + PAIR_STAGES * (PAIR_A_STAGE + PAIR_B_STAGE));
  const int pair = blockIdx.x >> 1;
  const int pairs = gridDim.x >> 1;
  const int tiles_m = (p.M + TILE_M - 1) / TILE_M;
  bool mma_issued = false;

  if (warp == 0) {
    if (lane == 0) {
      PairRing r;
      bool ok = true;
      for (int u = pair; ok && u < p.num_units; u += pairs) {
        int mt, n0;
        bool wide;
        ring_pair_unit(p, u, tiles_m, mt, n0, wide);
        const int ch = (p.axis == 0 ? mt * TILE_M : n0) / p.chunk;
        const int m0 = mt * TILE_M + static_cast<int>(c.rank) * BM;
        const int nb = n0 + static_cast<int>(c.rank) * (wide ? 128 : 64);
        for (int j = 0; ok && j < t; ++j) {
          const int s = (ch + 1 + j) % t;              // ring order of this chunk
          ok = pair_produce_unit(c, r, &p.ta[s], m0, &p.tb[s], nb, p.num_kb, wide);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && c.rank == 0) {
      PairRing r;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int u = pair; ok && u < p.num_units; u += pairs) {
        const uint32_t idesc = u < p.full_units ? c.idesc : c.idesc_half;
        for (int j = 0; ok && j < t; ++j) {
          ok = pair_wait_acc_empty(c, acc, acc_phase ^ 1u);
          if (!ok) break;
          ok = pair_mma_unit(c, r, tmem_base + static_cast<uint32_t>(acc * BN), p.num_kb, mma_issued, idesc);
          if (!ok) break;
          umma_commit_pair_mc(c.accf0 + 8 * acc, 0x3);
          if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
      }
    }
  } else {
    // warps 2..9: TMEM lane quadrant = warp % 4; warps 2..5 take the tile's left half of the
    // columns and warps 6..9 the right half. Each thread keeps its row's running sums.
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const uint32_t stg = staging0 + static_cast<uint32_t>(warp - 2) * STAGING_PER_WARP;
    const bool defer = AR && p.defer_replicas;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    bool pending = false;                 // a region of replica 0 still to copy into the others
    int pend_row0 = 0, pend_col0 = 0, pend_cols = 0;
    float sum[4][32];
    for (int u = pair; ok && u < p.num_units; u += pairs) {
      int mt, n0;
      bool wide;
      ring_pair_unit(p, u, tiles_m, mt, n0, wide);
      const int ch = (p.axis == 0 ? mt * TILE_M : n0) / p.chunk;
      const int m0 = mt * TILE_M + static_cast<int>(c.rank) * BM;
      const int cols = wide ? BN / 2 : BN / 4;       // this warp's columns: 128 or 64
      const int nq = cols / 32;
      for (int j = 0; j < t; ++j) {
        ok = pair_wait_acc_full(c, acc, acc_phase);
        if (!ok) break;
        const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                               static_cast<uint32_t>(acc * BN + half * cols);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (q < nq) {
            uint32_t v[32];
            tmem_ld32(t_row + q * 32, v);
            tmem_ld_wait();
            if (j == 0) {
#pragma unroll
              for (int i = 0; i < 32; ++i) sum[q][i] = __uint_as_float(v[i]);
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) sum[q][i] = __fadd_rn(sum[q][i], __uint_as_float(v[i]));
            }
          }
        }
        pair_release_acc(c, acc, lane);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        if (pending) copy_replica_rows<OUT_BF16>(p, lane, pend_row0, pend_col0, pend_cols, (32 * j) / t, (32 * (j + 1)) / t);
      }
      if (!ok) break;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (q < nq) store_block32<OUT_BF16, AR>(p, stg, lane, sum[q], m0 + quad * 32, n0 + half * cols + q * 32, ch, defer);
      pending = defer;
      pend_row0 = m0 + quad * 32;
      pend_col0 = n0 + half * cols;
      pend_cols = cols;
    }
    if (ok && pending) copy_replica_rows<OUT_BF16>(p, lane, pend_row0, pend_col0, pend_cols, 0, 32);
  }
  pair_teardown(c, warp, lane, mma_issued, tmem_base);
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

// Reserve the dynamic shared memory of a kernel once per device.
template <typename K>
tp_status reserve_smem(K kernel, size_t bytes, int* done_for) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(TP_ECUDA, "cudaGetDevice failed");
  if (dev >= 0 && dev < 64 && !done_for[dev]) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)) != cudaSuccess)
      return fail(TP_ECUDA, "cannot reserve %zu bytes of shared memory", bytes);
    done_for[dev] = 1;
  }
  return TP_OK;
}

template <int EPI>
tp_status launch(GemmParams& p, cudaStream_t s) {
  static int configured_for[64] = {};
  constexpr size_t smem = GEMM_SMEM + 4 * STAGING_PER_WARP;
  if (tp_status st = reserve_smem(gemm_tcgen05_kernel<EPI>, smem, configured_for)) return st;
  const int sms = sm_count();
  const int grid = p.num_tiles < sms ? p.num_tiles : sms;
  gemm_tcgen05_kernel<EPI><<<grid, GEMM_THREADS, smem, s>>>(p);
  return check_launch("gemm_tcgen05_kernel");
}

template <int EPI>
tp_status launch_pair(GemmParams& p, cudaStream_t s) {
  static int configured_for[64] = {};
  constexpr size_t smem = PAIR_SMEM + 4 * STAGING_PER_WARP;
  if (tp_status st = reserve_smem(gemm_pair_kernel<EPI>, smem, configured_for)) return st;
  const int sms = sm_count();
  const int tiles = p.groups * ((p.M + 2 * BM - 1) / (2 * BM)) * p.tiles_n;
  int grid = 2 * tiles < sms ? 2 * tiles : (sms & ~1);
  if (grid < 2) grid = 2;
  gemm_pair_kernel<EPI><<<grid, GEMM_THREADS, smem, s>>>(p);
  return check_launch("gemm_pair_kernel");
}

template <bool OUT_BF16, bool AR>
tp_status launch_ring(RingGemmParams& p, bool pair, cudaStream_t s) {
  const int sms = sm_count();
  if (pair) {
    static int configured_for[64] = {};
    if (tp_status st = reserve_smem(gemm_ring_pair_kernel<OUT_BF16, AR>, RING_PAIR_SMEM, configured_for)) return st;
    const int tiles = ((p.M + 2 * BM - 1) / (2 * BM)) * p.tiles_n;
    int grid = 2 * tiles < sms ? 2 * tiles : (sms & ~1);
    if (grid < 2) grid = 2;
    // AllReduce: half-width tiles for a last round that would leave at least half of the pairs idle
    // (B stored [K][N]: a half tile loads one 64-column box per CTA). The last tiles then carry the
    // replica writes over twice as many pairs; measured 4-5% faster on the 8B and case-3 AllReduce,
    // while a ReduceScatter's short last round runs faster as whole tiles.
    const int pairs = grid / 2;
    const int rem = tiles % pairs;
    const bool halves = AR && !p.b_km && tiles > pairs && rem > 0 && 2 * rem <= pairs;
    p.full_units = halves ? tiles - rem : tiles;
    p.num_units = halves ? tiles + rem : tiles;
    // Deferring costs one read-back of the tile and saves a burst of t - 1 copies: measured a gain at
    // t = 8 (Llama-3-8B down GEMM, 70B layer) and a loss at t = 4 with 0.9 GB replicas (case 3).
    p.defer_replicas = AR && p.t >= 8;
    gemm_ring_pair_kernel<OUT_BF16, AR><<<grid, RING_THREADS, RING_PAIR_SMEM, s>>>(p);
    return check_launch("gemm_ring_pair_kernel");
  }
  static int configured_for[64] = {};
  if (tp_status st = reserve_smem(gemm_ring_kernel<OUT_BF16, AR>, RING_SMEM, configured_for)) return st;
  const int grid = p.num_tiles < sms ? p.num_tiles : sms;
  gemm_ring_kernel<OUT_BF16, AR><<<grid, RING_THREADS, RING_SMEM, s>>>(p);
  return check_launch("gemm_ring_kernel");
}

tp_status check_operands(int n, const uint16_t* const* a, const uint16_t* const* b, void* const* c) {
  for (int i = 0; i < n; ++i) {
    if (a[i] == nullptr || b[i] == nullptr || c[i] == nullptr) return fail(TP_EINVAL, "null GEMM operand %d", i);
    if (!aligned16(a[i]) || !aligned16(b[i]) || !aligned16(c[i])) return fail(TP_EALIGN, "GEMM operand %d not 16-byte aligned", i);
  }
  return TP_OK;
}

}  // namespace

tp_status grouped_gemm(const GemmArgs& g, cudaStream_t s) {
  if (g.groups < 1 || g.groups > TP_MAX_SHARDS) return fail(TP_EINVAL, "groups=%d outside 1..%d", g.groups, TP_MAX_SHARDS);
  if (g.M < 0 || g.N < 0 || g.K <= 0) return fail(TP_EINVAL, "negative GEMM size or empty contraction (K = 0)");
  if (g.M == 0 || g.N == 0) return TP_OK;               // empty output: nothing to compute
  if (g.M > INT32_MAX / 2 || g.N > INT32_MAX / 2 || g.K > INT32_MAX / 2) return fail(TP_ESHAPE, "GEMM size too large");
  const bool swiglu = g.epi == EPI_SWIGLU;
  const bool a_sliced = g.a_slices || g.a_kslices;
  if (g.K % 8 || g.N % 8 || g.lda % 8 || g.ldb % 8) return fail(TP_EALIGN, "K, N and row strides must be multiples of 8");
  if (g.M % 8 && g.a_mn) return fail(TP_EALIGN, "M must be a multiple of 8 for a transposed A");
  const int64_t a_row = g.a_kslices ? g.kslice_cols : (g.a_mn ? g.M : g.K);
  const int64_t b_row = g.b_slices ? g.bslice_cols : (g.b_km ? g.K : (swiglu ? 2 * g.N : g.N));
  if (g.lda < a_row || g.ldb < b_row) return fail(TP_ESHAPE, "row stride shorter than the row");
  for (int i = 0; i < g.groups; ++i) {
    if ((!a_sliced && g.a[i] == nullptr) || (!g.b_slices && g.b[i] == nullptr) || g.c[i] == nullptr)
      return fail(TP_EINVAL, "null GEMM operand %d", i);
    if ((!a_sliced && !aligned16(g.a[i])) || (!g.b_slices && !aligned16(g.b[i])) || !aligned16(g.c[i]))
      return fail(TP_EALIGN, "GEMM operand %d not 16-byte aligned", i);
  }
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  const int tile_n = swiglu ? BN / 2 : BN;
  const bool pair = g.M >= 2 * BM && (g.a_slices == 0 || g.slice_rows % (2 * BM) == 0);
  if (g.a_slices && g.a_mn) return fail(TP_EUNSUPPORTED, "row slices of a transposed A are not supported");
  if (g.a_kslices && (g.a_mn || g.a_slices)) return fail(TP_EUNSUPPORTED, "K slices need A as [M][K] and no row slices");
  if (g.b_slices && (g.b_km || swiglu)) return fail(TP_EUNSUPPORTED, "column slices need B as [K][N], no SwiGLU");
  if (swiglu && g.b_km) return fail(TP_EUNSUPPORTED, "SwiGLU needs B as [K][2N]");
  if (g.a_slices) {
    if (g.a_slices > TP_MAX_SHARDS || g.slice_rows <= 0 || g.slice_rows % BM != 0 || g.slice_rows * g.a_slices != g.M)
      return fail(TP_ESHAPE, "A row slices must tile M in multiples of %d rows", BM);
    for (int i = 0; i < g.a_slices; ++i) {
      if (g.a_slice[i] == nullptr) return fail(TP_EINVAL, "null A slice %d", i);
      if (!aligned16(g.a_slice[i])) return fail(TP_EALIGN, "A slice %d not 16-byte aligned", i);
      if (!encode_bf16_2d(&p.ta[i], g.a_slice[i], g.K, g.slice_rows, g.lda, BK, BM))
        return fail(TP_ECUDA, "cannot encode the TMA descriptor of A slice %d", i);
    }
    p.a_slices = g.a_slices;
    p.slice_rows = static_cast<int>(g.slice_rows);
  }
  if (g.a_kslices) {   // A split along K: each k-block is read from the piece that holds it
    if (g.a_kslices > TP_MAX_SHARDS || g.kslice_cols <= 0 || g.kslice_cols % BK != 0 || g.kslice_cols * g.a_kslices != g.K)
      return fail(TP_ESHAPE, "A's K slices must tile K in multiples of %d columns", BK);
    for (int i = 0; i < g.a_kslices; ++i) {
      if (g.a_kslice[i] == nullptr) return fail(TP_EINVAL, "null A K slice %d", i);
      if (!aligned16(g.a_kslice[i])) return fail(TP_EALIGN, "A K slice %d not 16-byte aligned", i);
      if (!encode_bf16_2d(&p.ta[i], g.a_kslice[i], g.kslice_cols, g.M, g.lda, BK, BM))
        return fail(TP_ECUDA, "cannot encode the TMA descriptor of A K slice %d", i);
    }
    p.a_kslice = static_cast<int>(g.kslice_cols);
    p.a_kslices = g.a_kslices;
  }
  if (g.b_slices) {    // B split along N: each 64-column box is read from the piece that holds it
    if (g.b_slices > TP_MAX_SHARDS || g.bslice_cols <= 0 || g.bslice_cols % 64 != 0 || g.bslice_cols * g.b_slices != g.N)
      return fail(TP_ESHAPE, "B's column slices must tile N in multiples of 64 columns");
    for (int i = 0; i < g.b_slices; ++i) {
      if (g.b_slice[i] == nullptr) return fail(TP_EINVAL, "null B column slice %d", i);
      if (!aligned16(g.b_slice[i])) return fail(TP_EALIGN, "B column slice %d not 16-byte aligned", i);
      if (!encode_bf16_2d(&p.tb[i], g.b_slice[i], g.bslice_cols, g.K, g.ldb, 64, BK))
        return fail(TP_ECUDA, "cannot encode the TMA descriptor of B column slice %d", i);
    }
    p.b_nslice = static_cast<int>(g.bslice_cols);
    p.b_nslices = g.b_slices;
  }
  p.n_amaps = g.a_slices ? g.a_slices : g.a_kslices ? g.a_kslices : g.groups;
  p.n_bmaps = g.b_slices ? g.b_slices : g.groups;
  for (int i = 0; i < g.groups; ++i) {
    const bool a_ok = a_sliced ? true
                      : g.a_mn ? encode_bf16_2d(&p.ta[i], g.a[i], g.M, g.K, g.lda, 64, BK)
                               : encode_bf16_2d(&p.ta[i], g.a[i], g.K, g.M, g.lda, BK, BM);
    if (!a_ok) return fail(TP_ECUDA, "cannot encode the TMA descriptor of A[%d]", i);
    const bool b_ok = g.b_slices ? true
                      : g.b_km ? encode_bf16_2d(&p.tb[i], g.b[i], g.K, g.N, g.ldb, BK, pair ? 128 : BN)
                               : encode_bf16_2d(&p.tb[i], g.b[i], g.N, g.K, g.ldb, 64, BK);
    if (!b_ok) return fail(TP_ECUDA, "cannot encode the TMA descriptor of B[%d]", i);
    if (swiglu && !encode_bf16_2d(&p.tb2[i], g.b[i] + g.N, g.N, g.K, g.ldb, 64, BK))
      return fail(TP_ECUDA, "cannot encode the TMA descriptor of the up half of B[%d]", i);
    p.c[i] = g.c[i];
  }
  p.M = static_cast<int>(g.M);
  p.N = static_cast<int>(g.N);
  p.K = static_cast<int>(g.K);
  p.a_mn = g.a_mn;
  p.b_km = g.b_km;
  p.tiles_m = static_cast<int>((g.M + BM - 1) / BM);
  p.tiles_n = static_cast<int>((g.N + tile_n - 1) / tile_n);
  p.groups = g.groups;
  p.row_tiles = g.groups * p.tiles_m;
  const int64_t tiles = static_cast<int64_t>(g.groups) * p.tiles_m * p.tiles_n;
  if (tiles > INT32_MAX) return fail(TP_ESHAPE, "too many tiles");
  p.num_tiles = static_cast<int>(tiles);
  p.num_kb = static_cast<int>((g.K + BK - 1) / BK);
  // Raster band: as many row-tiles as keep about RASTER_A_BYTES of A rows, so that the band's A stays in
  // L2 while its B panels stream past. Measured on the sharded-matmul cases (K = 8192, 256-row tiles):
  // 8 row-tiles instead of 16 read 0.4-0.9 GB less from DRAM per launch and ran 1-4% faster.
  {
    const int64_t a_tile = static_cast<int64_t>(pair ? 2 * BM : BM) * g.K * 2;
    const int64_t fit = RASTER_A_BYTES / a_tile;
    p.band = static_cast<int>(fit < 1 ? 1 : fit > RASTER_BAND_MAX ? RASTER_BAND_MAX : fit);
  }
  p.status = status_word();
  p.budget = wait_budget();
  if (p.status == nullptr) return fail(TP_ECUDA, "cannot resolve the device status word");
  // CTA pairs for problems with at least one full 256-row tile per group (and slices of whole pair tiles).
  if (pair) {
    switch (g.epi) {
      case EPI_F32: return launch_pair<EPI_F32>(p, s);
      case EPI_BF16: return launch_pair<EPI_BF16>(p, s);
      case EPI_GELU: return launch_pair<EPI_GELU>(p, s);
      case EPI_GELU_TANH: return launch_pair<EPI_GELU_TANH>(p, s);
      case EPI_SWIGLU: return launch_pair<EPI_SWIGLU>(p, s);
    }
  }
  switch (g.epi) {
    case EPI_F32: return launch<EPI_F32>(p, s);
    case EPI_BF16: return launch<EPI_BF16>(p, s);
    case EPI_GELU: return launch<EPI_GELU>(p, s);
    case EPI_GELU_TANH: return launch<EPI_GELU_TANH>(p, s);
    case EPI_SWIGLU: return launch<EPI_SWIGLU>(p, s);
  }
  return fail(TP_EINVAL, "bad epilogue");
}

bool ring_gemm_fits(int64_t M, int64_t N, int t, int axis) {
  if (axis == 0) return M % t == 0 && (M / t) % BM == 0;
  return N % t == 0 && (N / t) % BN == 0;
}

tp_status ring_gemm(const RingGemmArgs& g, cudaStream_t s) {
  if (!valid_t(g.t)) return fail(TP_EINVAL, "t=%d outside 1..%d", g.t, TP_MAX_SHARDS);
  if (g.M < 0 || g.N < 0 || g.K <= 0) return fail(TP_EINVAL, "negative GEMM size or empty contraction (K = 0)");
  if (g.M == 0 || g.N == 0) return TP_OK;               // empty output: nothing to compute
  if (g.M > INT32_MAX / 2 || g.N > INT32_MAX / 2 || g.K > INT32_MAX / 2) return fail(TP_ESHAPE, "GEMM size too large");
  if (g.op != RING_RS && g.op != RING_AR) return fail(TP_EINVAL, "fused GEMM reduces by RS or AR only");
  if (g.axis != 0 && g.axis != 1) return fail(TP_EINVAL, "axis must be 0 or 1");
  const int axis = g.axis;              // AllReduce: the axis of its ReduceScatter (the summation order)
  if (!ring_gemm_fits(g.M, g.N, g.t, axis)) return fail(TP_EUNSUPPORTED, "chunks do not align with 128 x 256 tiles");
  if (g.K % 8 || g.N % 8 || g.lda % 8 || g.ldb % 8) return fail(TP_EALIGN, "K, N and row strides must be multiples of 8");
  if (g.lda < g.K || g.ldb < (g.b_km ? g.K : g.N)) return fail(TP_ESHAPE, "row stride shorter than the row");
  if (tp_status st = check_operands(g.t, g.a, g.b, g.out)) return st;
  if ((g.resid && !aligned16(g.resid)) || (g.copy_bf16 && !aligned16(g.copy_bf16)))
    return fail(TP_EALIGN, "residual or bf16 copy not 16-byte aligned");
  RingGemmParams p;
  std::memset(&p, 0, sizeof(p));
  const int64_t chunk0 = axis == 0 ? g.M / g.t : g.N / g.t;
  const bool pair = axis == 0 ? chunk0 % (2 * BM) == 0 : g.M >= 2 * BM;
  for (int i = 0; i < g.t; ++i) {
    if (!encode_bf16_2d(&p.ta[i], g.a[i], g.K, g.M, g.lda, BK, BM))
      return fail(TP_ECUDA, "cannot encode the TMA descriptor of A[%d]", i);
    const bool b_ok = g.b_km ? encode_bf16_2d(&p.tb[i], g.b[i], g.K, g.N, g.ldb, BK, pair ? 128 : BN)
                             : encode_bf16_2d(&p.tb[i], g.b[i], g.N, g.K, g.ldb, 64, BK);
    if (!b_ok) return fail(TP_ECUDA, "cannot encode the TMA descriptor of B[%d]", i);
    p.out[i] = g.out[i];
  }
  p.b_km = g.b_km;
  p.resid = g.op == RING_AR ? g.resid : nullptr;
  p.resid_bf16 = g.resid_dtype == TP_BF16;
  p.copy_bf16 = g.op == RING_AR ? g.copy_bf16 : nullptr;
  p.M = static_cast<int>(g.M);
  p.N = static_cast<int>(g.N);
  p.t = g.t;
  p.axis = axis;
  p.chunk = static_cast<int>(axis == 0 ? g.M / g.t : g.N / g.t);
  // CTA pairs when every chunk is a whole number of 256-row (axis 0) or 256-column (axis 1) tiles
  p.chunk_tiles = axis == 0 ? p.chunk / (pair ? 2 * BM : BM) : p.chunk / BN;
  // axis 0 has M a multiple of 128 (whole-tile chunks); axis 1 may end in a partial row-tile
  p.tiles_m = static_cast<int>((g.M + BM - 1) / BM);
  p.tiles_n = static_cast<int>((g.N + BN - 1) / BN);
  p.num_tiles = p.tiles_m * p.tiles_n;
  p.num_kb = static_cast<int>((g.K + BK - 1) / BK);
  p.status = status_word();
  p.budget = wait_budget();
  if (p.status == nullptr) return fail(TP_ECUDA, "cannot resolve the device status word");
  const bool bf16 = g.out_dtype == TP_BF16;
  if (g.op == RING_AR) return bf16 ? launch_ring<true, true>(p, pair, s) : launch_ring<false, true>(p, pair, s);
  return bf16 ? launch_ring<true, false>(p, pair, s) : launch_ring<false, false>(p, pair, s);
}

}  // namespace tpx
