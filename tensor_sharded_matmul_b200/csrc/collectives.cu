// Ring-order ReduceScatter, AllGather and AllReduce over t shard buffers resident in this GPU's HBM
// ("Scaling Book 入门第 5 章：Sharded Matrices 上篇 — 集合通信原语", §5.2 环形算法 and §5.3;
//  "Scaling Book 入门第 6 章", §6.4 通信原语详解).
//
// The ring is kept as a SUMMATION ORDER, not as data movement. The ring passes from device i to
// i+1, each device adds its own copy at every step, and device r ends with chunk r. That fixes
// chunk c's sum as (((U[c+1] + U[c+2]) + U[c+3]) + ... ) + U[c] (indices mod t). On one GPU
// every shard's buffer is directly addressable, so each output element is produced by ONE thread.
// That thread reads the t inputs, adds them in that order in binary32 and writes once.
//   ReduceScatter: reads t*M bytes, writes M.
//   AllReduce: reads t*M, writes t*M.
//   AllGather: reads M, writes t*M.
//   AllToAll (a bit copy, "Scaling Book 入门第 5 章", §5.3): reads t*M, writes t*M.
// No atomics, no reassociation, and the result does not depend on grid size.
// A thread's unit is one 16-byte vector of the input type, so every warp-wide load is 32 consecutive
// vectors; a thread takes a few units a grid stride apart and issues all their loads before any add,
// and grids give every thread the same number of steps. bf16 inputs are widened (exact), summed in
// binary32 and rounded once to bf16
// (nearest-even) at the end; the optional per-hop mode (TP_BF16_RING) instead rounds the running
// partial to bf16 after every add, as a ring whose links carry bf16 does.
#include <cuda_bf16.h>

#include <cstring>

#include "common.cuh"
#include "ptx.cuh"

namespace tpx {

namespace {

struct RingParams {
  const void* in[TP_MAX_SHARDS];
  void* out[TP_MAX_SHARDS];
  const void* resid;
  uint16_t* copy_bf16;
  int64_t rows, cols;
  int64_t chunk_elems;   // axis 0: (rows/t)*cols
  int64_t chunk_cols;    // axis 1: cols/t
  int t, axis;
  int resid_bf16;
  int skip_self;         // AllGather in place: do not rewrite a shard's own piece
};

// ------------------------------------------------------------------ element groups of VEC values
template <typename T, int VEC>
struct IO;

template <>
struct IO<float, 8> {
  static __device__ __forceinline__ void load(const void* base, int64_t i, float (&f)[8]) {
    const float* p = static_cast<const float*>(base) + i;
    const uint4 a = ld_nc_v4(p), b = ld_nc_v4(p + 4);
    f[0] = __uint_as_float(a.x); f[1] = __uint_as_float(a.y); f[2] = __uint_as_float(a.z); f[3] = __uint_as_float(a.w);
    f[4] = __uint_as_float(b.x); f[5] = __uint_as_float(b.y); f[6] = __uint_as_float(b.z); f[7] = __uint_as_float(b.w);
  }
  static __device__ __forceinline__ void store(void* base, int64_t i, const float (&f)[8]) {
    float* p = static_cast<float*>(base) + i;
    st_v4(p, make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3])));
    st_v4(p + 4, make_uint4(__float_as_uint(f[4]), __float_as_uint(f[5]), __float_as_uint(f[6]), __float_as_uint(f[7])));
  }
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const uint32_t a = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
  const uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
  return a | (b << 16);
}

template <>
struct IO<uint16_t, 8> {
  static __device__ __forceinline__ void load(const void* base, int64_t i, float (&f)[8]) {
    const uint4 a = ld_nc_v4(static_cast<const uint16_t*>(base) + i);
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      f[2 * k] = __uint_as_float(w[k] << 16);
      f[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
  }
  static __device__ __forceinline__ void store(void* base, int64_t i, const float (&f)[8]) {
    st_v4(static_cast<uint16_t*>(base) + i,
          make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7])));
  }
};

template <>
struct IO<float, 4> {
  static __device__ __forceinline__ void load(const void* base, int64_t i, float (&f)[4]) {
    const uint4 a = ld_nc_v4(static_cast<const float*>(base) + i);
    f[0] = __uint_as_float(a.x); f[1] = __uint_as_float(a.y); f[2] = __uint_as_float(a.z); f[3] = __uint_as_float(a.w);
  }
  static __device__ __forceinline__ void store(void* base, int64_t i, const float (&f)[4]) {
    st_v4(static_cast<float*>(base) + i, make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                                                    __float_as_uint(f[3])));
  }
};

template <>
struct IO<uint16_t, 4> {
  static __device__ __forceinline__ void load(const void* base, int64_t i, float (&f)[4]) {
    const uint2 a = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(base) + i);
    f[0] = __uint_as_float(a.x << 16); f[1] = __uint_as_float(a.x & 0xFFFF0000u);
    f[2] = __uint_as_float(a.y << 16); f[3] = __uint_as_float(a.y & 0xFFFF0000u);
  }
  static __device__ __forceinline__ void store(void* base, int64_t i, const float (&f)[4]) {
    st_v2(static_cast<uint16_t*>(base) + i, make_uint2(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3])));
  }
};

template <>
struct IO<float, 1> {
  static __device__ __forceinline__ void load(const void* base, int64_t i, float (&f)[1]) {
    f[0] = __ldg(static_cast<const float*>(base) + i);
  }
  static __device__ __forceinline__ void store(void* base, int64_t i, const float (&f)[1]) {
    static_cast<float*>(base)[i] = f[0];
  }
};

template <>
struct IO<uint16_t, 1> {
  static __device__ __forceinline__ void load(const void* base, int64_t i, float (&f)[1]) {
    f[0] = __uint_as_float(static_cast<uint32_t>(__ldg(static_cast<const unsigned short*>(base) + i)) << 16);
  }
  static __device__ __forceinline__ void store(void* base, int64_t i, const float (&f)[1]) {
    static_cast<uint16_t*>(base)[i] = __bfloat16_as_ushort(__float2bfloat16_rn(f[0]));
  }
};

// Widening of one raw 16-byte vector of the input type (4 fp32 or 8 bf16 values) to binary32.
template <typename T, int VEC>
__device__ __forceinline__ void unpack16(const uint4& r, float (&f)[VEC]) {
  if constexpr (sizeof(T) == 4) {
    f[0] = __uint_as_float(r.x); f[1] = __uint_as_float(r.y); f[2] = __uint_as_float(r.z); f[3] = __uint_as_float(r.w);
  } else {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      f[2 * k] = __uint_as_float(w[k] << 16);
      f[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
  }
}

// Chunk of full-tensor element e, and e's offset inside that chunk's shard buffer.
__device__ __forceinline__ void locate(const RingParams& p, int64_t e, int& c, int64_t& local) {
  if (p.axis == 0) {
    c = static_cast<int>(e / p.chunk_elems);
    local = e - c * p.chunk_elems;
  } else {
    const int64_t row = e / p.cols;
    const int64_t col = e - row * p.cols;
    c = static_cast<int>(col / p.chunk_cols);
    local = row * p.chunk_cols + (col - c * p.chunk_cols);
  }
}

// The ring sum of the unit starting at full-tensor element e (chunk c) goes out: AllReduce adds the
// residual (if any) and writes every replica (and the bf16 copy); ReduceScatter writes shard c's
// piece.
template <typename Tout, int VEC, bool AR>
__device__ __forceinline__ void finish_unit(const RingParams& p, int64_t e, int c, int64_t local, float (&acc)[VEC],
                                            int t) {
  if constexpr (AR) {
    if (p.resid != nullptr) {
      float r[VEC];
      if (p.resid_bf16)
        IO<uint16_t, VEC>::load(p.resid, e, r);
      else
        IO<float, VEC>::load(p.resid, e, r);
#pragma unroll
      for (int i = 0; i < VEC; ++i) acc[i] = __fadd_rn(acc[i], r[i]);
    }
    for (int s = 0; s < t; ++s) IO<Tout, VEC>::store(p.out[s], e, acc);
    if (p.copy_bf16 != nullptr) IO<uint16_t, VEC>::store(p.copy_bf16, e, acc);
  } else {
    IO<Tout, VEC>::store(p.out[c], local, acc);
  }
}

// Round a binary32 value to bfloat16 (nearest-even) and widen it back: one hop of a bf16 ring.
__device__ __forceinline__ float hop_round(float x) {
  return __uint_as_float(static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(x))) << 16);
}

// ReduceScatter (AR == false) or AllReduce (AR == true). TT = compile-time t (0: runtime t).
// HOP: round the running partial to bf16 after every add (bf16 in and out only).
// A unit is VEC consecutive elements: one 16-byte vector of the input type (VEC = 1 on the unaligned
// path), so every warp-wide load is 32 consecutive vectors. A thread takes UNR units per step, a
// grid stride apart, and issues all their loads before the adds (UNR * t vectors in flight).
template <typename Tin, typename Tout, int VEC, int TT, bool AR, int UNR, bool HOP>
__global__ void __launch_bounds__(256) ring_reduce_kernel(const __grid_constant__ RingParams p) {
  const int t = TT > 0 ? TT : p.t;
  const int64_t units = p.rows * p.cols / VEC;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t u0 = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; u0 < units; u0 += UNR * stride) {
    if constexpr (TT > 0 && VEC * sizeof(Tin) == 16) {
      // raw 16-byte vectors: every load of the step is issued before any value is widened or added
      uint4 raw[UNR][TT];
      int cs[UNR];
      int64_t locs[UNR];
#pragma unroll
      for (int k = 0; k < UNR; ++k) {
        const int64_t u = u0 + k * stride;
        if (u < units) {
          locate(p, u * VEC, cs[k], locs[k]);
#pragma unroll
          for (int j = 0; j < TT; ++j)
            raw[k][j] = ld_nc_v4(static_cast<const Tin*>(p.in[(cs[k] + 1 + j) % TT]) + u * VEC);
        }
      }
#pragma unroll
      for (int k = 0; k < UNR; ++k) {
        const int64_t u = u0 + k * stride;
        if (u >= units) break;
        float acc[VEC];
        unpack16<Tin, VEC>(raw[k][0], acc);
#pragma unroll
        for (int j = 1; j < TT; ++j) {
          float v[VEC];
          unpack16<Tin, VEC>(raw[k][j], v);
#pragma unroll
          for (int i = 0; i < VEC; ++i) {
            acc[i] = __fadd_rn(acc[i], v[i]);
            if constexpr (HOP) acc[i] = hop_round(acc[i]);
          }
        }
        finish_unit<Tout, VEC, AR>(p, u * VEC, cs[k], locs[k], acc, t);
      }
    } else {
#pragma unroll 1
      for (int k = 0; k < UNR; ++k) {
        const int64_t u = u0 + k * stride;
        if (u >= units) break;
        const int64_t e = u * VEC;
        int c;
        int64_t local;
        locate(p, e, c, local);
        float acc[VEC];
        IO<Tin, VEC>::load(p.in[(c + 1) % t], e, acc);
        for (int j = 2; j <= t; ++j) {
          float v[VEC];
          IO<Tin, VEC>::load(p.in[(c + j) % t], e, v);
#pragma unroll
          for (int i = 0; i < VEC; ++i) {
            acc[i] = __fadd_rn(acc[i], v[i]);
            if constexpr (HOP) acc[i] = hop_round(acc[i]);
          }
        }
        finish_unit<Tout, VEC, AR>(p, e, c, local, acc, t);
      }
    }
  }
}

// AllGather as a bit copy: every shard receives every piece. UNIT = bytes moved per step
// (16 = one vector, or the element size for the unaligned path); ES = element size. A thread takes
// UNR units a grid stride apart and loads them all before its stores.
template <int ES, int UNIT, int UNR>
__global__ void __launch_bounds__(256) ring_gather_kernel(const __grid_constant__ RingParams p) {
  constexpr int EPU = UNIT / ES;   // elements per unit
  const int64_t units = p.rows * p.cols / EPU;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t u0 = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; u0 < units; u0 += UNR * stride) {
    if constexpr (UNIT == 16) {
      uint4 v[UNR];
      int cs[UNR];
#pragma unroll
      for (int k = 0; k < UNR; ++k) {
        const int64_t u = u0 + k * stride;
        if (u < units) {
          int64_t local;
          locate(p, u * EPU, cs[k], local);
          v[k] = ld_nc_v4(static_cast<const char*>(p.in[cs[k]]) + local * ES);
        }
      }
#pragma unroll
      for (int k = 0; k < UNR; ++k) {
        const int64_t u = u0 + k * stride;
        if (u >= units) break;
        for (int s = 0; s < p.t; ++s) {
          if (p.skip_self && s == cs[k]) continue;
          st_v4(static_cast<char*>(p.out[s]) + u * EPU * ES, v[k]);
        }
      }
    } else {
#pragma unroll 1
      for (int k = 0; k < UNR; ++k) {
        const int64_t u = u0 + k * stride;
        if (u >= units) break;
        const int64_t e = u * EPU;
        int c;
        int64_t local;
        locate(p, e, c, local);
        const char* src = static_cast<const char*>(p.in[c]) + local * ES;
        if constexpr (ES == 4) {
          const uint32_t v = *reinterpret_cast<const uint32_t*>(src);
          for (int s = 0; s < p.t; ++s)
            if (!(p.skip_self && s == c)) reinterpret_cast<uint32_t*>(p.out[s])[e] = v;
        } else {
          const uint16_t v = *reinterpret_cast<const uint16_t*>(src);
          for (int s = 0; s < p.t; ++s)
            if (!(p.skip_self && s == c)) reinterpret_cast<uint16_t*>(p.out[s])[e] = v;
        }
      }
    }
  }
}

// AllToAll: out[j] = concatenation along concat_axis of piece j (split along split_axis) of every
// shard's buffer. Each output element has exactly one source, and each row of a piece lands as one
// contiguous run of an output row.
struct A2AParams {
  const void* in[TP_MAX_SHARDS];
  void* out[TP_MAX_SHARDS];
  int64_t rows, cols;        // each shard's input shape
  int64_t pr, pc;            // piece shape
  int64_t orow, ocol;        // each shard's output shape
  int t, split, concat;
};

// One task = one contiguous run of a piece: destination shard j, source shard i, row lr of the
// piece. The run is pc elements long on both sides, so a block copies it with plain coalesced
// vectors and all index arithmetic happens once per run. Loads go out four per thread before their
// stores.
template <int ES, bool VEC>
__global__ void __launch_bounds__(256, 4) all_to_all_kernel(const __grid_constant__ A2AParams p) {
  const int64_t P = p.pr;                                  // rows per piece
  const int64_t L = p.pc;                                  // elements per run
  const int64_t per_j = static_cast<int64_t>(p.t) * P;
  const int64_t tasks = static_cast<int64_t>(p.t) * per_j;
  for (int64_t task = blockIdx.x; task < tasks; task += gridDim.x) {
    const int j = static_cast<int>(task / per_j);
    const int64_t rem = task - j * per_j;
    const int i = static_cast<int>(rem / P);
    const int64_t lr = rem - i * P;
    const int64_t sr = p.split == 0 ? j * P + lr : lr;     // source row and first column
    const int64_t sc = p.split == 0 ? 0 : j * L;
    const int64_t dr = p.concat == 0 ? i * P + lr : lr;    // destination row and first column
    const int64_t dc = p.concat == 0 ? 0 : i * L;
    const char* src = static_cast<const char*>(p.in[i]) + (sr * p.cols + sc) * ES;
    char* dst = static_cast<char*>(p.out[j]) + (dr * p.ocol + dc) * ES;
    if constexpr (VEC) {
      const int64_t nv = L * ES / 16;
      for (int64_t v = threadIdx.x; v < nv; v += 4 * static_cast<int64_t>(blockDim.x)) {
        uint4 x[4];
#pragma unroll
        for (int b = 0; b < 4; ++b)
          if (v + b * blockDim.x < nv) x[b] = ld_nc_v4(src + (v + b * blockDim.x) * 16);
#pragma unroll
        for (int b = 0; b < 4; ++b)
          if (v + b * blockDim.x < nv) st_v4(dst + (v + b * blockDim.x) * 16, x[b]);
      }
    } else {
      for (int64_t e = threadIdx.x; e < L; e += blockDim.x) {
        if constexpr (ES == 4) reinterpret_cast<uint32_t*>(dst)[e] = reinterpret_cast<const uint32_t*>(src)[e];
        else reinterpret_cast<uint16_t*>(dst)[e] = reinterpret_cast<const uint16_t*>(src)[e];
      }
    }
  }
}

// Grid for `units` of work at `unr` units per thread step: at most 8 blocks of 256 threads per SM
// (a full SM), and no more threads than needed to give every thread the same number of steps, so
// the last step is not a partial wave.
int grid_for(int64_t units, int unr) {
  const int sms = sm_count();
  const int64_t cap_threads = static_cast<int64_t>(sms) * 8 * 256;
  const int64_t steps = (units + unr * cap_threads - 1) / (unr * cap_threads);        // per thread
  const int64_t threads = (units + unr * steps - 1) / (unr * steps);
  return static_cast<int>((threads + 255) / 256);
}

// Units per thread step: 4-8 input vectors in flight per thread. Measured on one B200 against
// 4 units for t = 2: 2 units were 3-8% faster at 64-256 MiB (fp32 and bf16), equal elsewhere.
template <int TT>
constexpr int unroll_for() {
  return TT == 2 || TT == 4 ? 2 : 1;
}

template <typename Tin, typename Tout, int VEC, bool AR, bool HOP = false>
tp_status launch_reduce(const RingParams& p, int64_t units, cudaStream_t s) {
  switch (p.t) {
    case 2: ring_reduce_kernel<Tin, Tout, VEC, 2, AR, unroll_for<2>(), HOP><<<grid_for(units, unroll_for<2>()), 256, 0, s>>>(p); break;
    case 4: ring_reduce_kernel<Tin, Tout, VEC, 4, AR, unroll_for<4>(), HOP><<<grid_for(units, unroll_for<4>()), 256, 0, s>>>(p); break;
    case 8: ring_reduce_kernel<Tin, Tout, VEC, 8, AR, 1, HOP><<<grid_for(units, 1), 256, 0, s>>>(p); break;
    default: ring_reduce_kernel<Tin, Tout, VEC, 0, AR, 1, HOP><<<grid_for(units, 1), 256, 0, s>>>(p); break;
  }
  return TP_OK;
}

// Vector width: one 16-byte vector of the input type (fp32: 4, bf16: 8), or 1 on the unaligned path.
template <bool AR>
tp_status dispatch_reduce(const RingParams& p, tp_dtype din, tp_dtype dout, bool vec, cudaStream_t s) {
  const int64_t n = p.rows * p.cols;
  if (din == TP_BF16_RING)   // bf16 in and out, the partial rounded after every hop
    return vec ? launch_reduce<uint16_t, uint16_t, 8, AR, true>(p, n / 8, s)
               : launch_reduce<uint16_t, uint16_t, 1, AR, true>(p, n, s);
  if (!vec) {
    if (din == TP_F32 && dout == TP_F32) return launch_reduce<float, float, 1, AR>(p, n, s);
    if (din == TP_BF16 && dout == TP_BF16) return launch_reduce<uint16_t, uint16_t, 1, AR>(p, n, s);
    if (din == TP_F32 && dout == TP_BF16) return launch_reduce<float, uint16_t, 1, AR>(p, n, s);
    return launch_reduce<uint16_t, float, 1, AR>(p, n, s);
  }
  if (din == TP_F32 && dout == TP_F32) return launch_reduce<float, float, 4, AR>(p, n / 4, s);
  if (din == TP_BF16 && dout == TP_BF16) return launch_reduce<uint16_t, uint16_t, 8, AR>(p, n / 8, s);
  if (din == TP_F32 && dout == TP_BF16) return launch_reduce<float, uint16_t, 4, AR>(p, n / 4, s);
  return launch_reduce<uint16_t, float, 8, AR>(p, n / 8, s);
}

bool ring_dtype_ok(tp_dtype d) { return d == TP_F32 || d == TP_BF16 || d == TP_BF16_RING; }

}  // namespace

tp_status ring_collective(const RingArgs& a, cudaStream_t stream) {
  if (!valid_t(a.t)) return fail(TP_EINVAL, "t=%d outside 1..%d", a.t, TP_MAX_SHARDS);
  if (a.rows < 0 || a.cols < 0) return fail(TP_EINVAL, "negative size");
  if (a.rows == 0 || a.cols == 0) return TP_OK;         // empty buffers: nothing to move
  if (a.axis != 0 && a.axis != 1) return fail(TP_EINVAL, "axis must be 0 or 1");
  const bool hop = a.in_dtype == TP_BF16_RING || a.out_dtype == TP_BF16_RING;
  if (hop && a.in_dtype != a.out_dtype) return fail(TP_EINVAL, "per-hop bf16 rounding needs bf16 in and out");
  if (!ring_dtype_ok(a.in_dtype) || !ring_dtype_ok(a.out_dtype)) return fail(TP_EINVAL, "bad dtype");
  if (a.op == RING_AG && a.in_dtype != a.out_dtype) return fail(TP_EINVAL, "AllGather copies bits: dtypes must match");
  const int axis = a.axis;   // AllReduce: the axis of its ReduceScatter (each element's summation order)
  if (axis == 0 && a.rows % a.t) return fail(TP_EDIVIS, "t=%d does not divide rows=%lld", a.t, (long long)a.rows);
  if (axis == 1 && a.cols % a.t) return fail(TP_EDIVIS, "t=%d does not divide cols=%lld", a.t, (long long)a.cols);
  for (int i = 0; i < a.t; ++i)
    if (a.in[i] == nullptr || a.out[i] == nullptr) return fail(TP_EINVAL, "null shard pointer %d", i);

  RingParams p;
  std::memset(&p, 0, sizeof(p));
  for (int i = 0; i < a.t; ++i) { p.in[i] = a.in[i]; p.out[i] = a.out[i]; }
  p.rows = a.rows; p.cols = a.cols; p.t = a.t; p.axis = axis;
  p.chunk_elems = (a.rows / a.t) * a.cols;
  p.chunk_cols = a.cols / a.t;
  p.resid = a.op == RING_AR ? a.resid : nullptr;
  p.resid_bf16 = a.resid_dtype == TP_BF16;
  p.copy_bf16 = a.op == RING_AR ? a.copy_bf16 : nullptr;

  // Pointer checks for every buffer a kernel touches (alignment decides the vector path).
  bool all16 = true;
  for (int i = 0; i < a.t; ++i) all16 = all16 && aligned16(a.in[i]) && aligned16(a.out[i]);
  if (p.resid) all16 = all16 && aligned16(p.resid);
  if (p.copy_bf16) all16 = all16 && aligned16(p.copy_bf16);

  const int sms = sm_count();
  if (sms <= 0) return fail(TP_ECUDA, "cannot query the SM count");

  if (a.op == RING_AG) {   // a bit copy: TP_BF16_RING moves bf16 like TP_BF16
    const int es = a.in_dtype == TP_F32 ? 4 : 2;
    const int epu = 16 / es;
    bool vec = all16 && (axis == 0 ? p.chunk_elems % epu == 0 : (p.chunk_cols % epu == 0 && a.cols % epu == 0));
    // In place: shard r's piece already sits at its place in out[r].
    bool in_place = axis == 0;
    for (int i = 0; i < a.t && in_place; ++i)
      in_place = static_cast<const char*>(a.in[i]) == static_cast<const char*>(a.out[i]) + i * p.chunk_elems * es;
    p.skip_self = in_place ? 1 : 0;
    const int64_t units = a.rows * a.cols / (vec ? epu : 1);
    // vectors per thread step: 4 for t = 2 (one store per vector and replica, few stores), 2
    // otherwise (measured: 4 was 5% faster at t = 2 and 256 MiB, 1-2% slower at t = 8)
    if (a.t <= 2) {
      const int blocks = grid_for(units, 4);
      if (es == 4) {
        if (vec) ring_gather_kernel<4, 16, 4><<<blocks, 256, 0, stream>>>(p);
        else ring_gather_kernel<4, 4, 4><<<blocks, 256, 0, stream>>>(p);
      } else {
        if (vec) ring_gather_kernel<2, 16, 4><<<blocks, 256, 0, stream>>>(p);
        else ring_gather_kernel<2, 2, 4><<<blocks, 256, 0, stream>>>(p);
      }
      return check_launch("ring_gather_kernel");
    }
    const int blocks = grid_for(units, 2);
    if (es == 4) {
      if (vec) ring_gather_kernel<4, 16, 2><<<blocks, 256, 0, stream>>>(p);
      else ring_gather_kernel<4, 4, 2><<<blocks, 256, 0, stream>>>(p);
    } else {
      if (vec) ring_gather_kernel<2, 16, 2><<<blocks, 256, 0, stream>>>(p);
      else ring_gather_kernel<2, 2, 2><<<blocks, 256, 0, stream>>>(p);
    }
    return check_launch("ring_gather_kernel");
  }

  // A unit (one 16-byte vector of the input type) must not straddle a chunk (or, for axis 1, a row).
  // Checking multiples of 8 elements covers both vector widths (4 fp32, 8 bf16).
  const bool vec = all16 && (axis == 0 ? p.chunk_elems % 8 == 0 : (p.chunk_cols % 8 == 0 && a.cols % 8 == 0));
  if (a.op == RING_RS) dispatch_reduce<false>(p, a.in_dtype, a.out_dtype, vec, stream);
  else dispatch_reduce<true>(p, a.in_dtype, a.out_dtype, vec, stream);
  return check_launch("ring_reduce_kernel");
}

tp_status all_to_all(const void* const* in, void* const* out, int64_t rows, int64_t cols, int split, int concat,
                     tp_dtype dtype, int t, cudaStream_t stream) {
  if (in == nullptr || out == nullptr) return fail(TP_EINVAL, "null pointer array");
  if (!valid_t(t)) return fail(TP_EINVAL, "t=%d outside 1..%d", t, TP_MAX_SHARDS);
  if (rows < 0 || cols < 0) return fail(TP_EINVAL, "negative size");
  if (rows == 0 || cols == 0) return TP_OK;             // empty buffers: nothing to move
  if ((split != 0 && split != 1) || (concat != 0 && concat != 1)) return fail(TP_EINVAL, "axes must be 0 or 1");
  if (dtype != TP_F32 && dtype != TP_BF16) return fail(TP_EINVAL, "bad dtype");
  if (split == 0 ? rows % t : cols % t) return fail(TP_EDIVIS, "t=%d does not divide the split dimension", t);
  A2AParams p;
  std::memset(&p, 0, sizeof(p));
  bool all16 = true;
  for (int i = 0; i < t; ++i) {
    if (in[i] == nullptr || out[i] == nullptr) return fail(TP_EINVAL, "null shard pointer %d", i);
    for (int k = 0; k < t; ++k)
      if (i != k && in[i] == out[k]) return fail(TP_EINVAL, "AllToAll cannot run in place");
    p.in[i] = in[i];
    p.out[i] = out[i];
    all16 = all16 && aligned16(in[i]) && aligned16(out[i]);
  }
  p.rows = rows; p.cols = cols; p.t = t; p.split = split; p.concat = concat;
  p.pr = split == 0 ? rows / t : rows;
  p.pc = split == 1 ? cols / t : cols;
  p.orow = concat == 0 ? t * p.pr : p.pr;
  p.ocol = concat == 1 ? t * p.pc : p.pc;
  const int es = dtype == TP_F32 ? 4 : 2;
  const int epu = 16 / es;
  // a vector never straddles a piece: the piece width, both row lengths and every column offset
  // are multiples of the vector length
  const bool vec = all16 && p.pc % epu == 0 && cols % epu == 0 && p.ocol % epu == 0;
  const int64_t tasks = static_cast<int64_t>(t) * t * p.pr;     // one block-sized copy per run
  const int cap = sm_count() * 4;                               // 4 resident blocks per SM
  if (cap <= 0) return fail(TP_ECUDA, "cannot query the SM count");
  const int blocks = static_cast<int>(tasks < cap ? tasks : cap);
  if (es == 4) {
    if (vec) all_to_all_kernel<4, true><<<blocks, 256, 0, stream>>>(p);
    else all_to_all_kernel<4, false><<<blocks, 256, 0, stream>>>(p);
  } else {
    if (vec) all_to_all_kernel<2, true><<<blocks, 256, 0, stream>>>(p);
    else all_to_all_kernel<2, false><<<blocks, 256, 0, stream>>>(p);
  }
  return check_launch("all_to_all_kernel");
}

}  // namespace tpx

using namespace tpx;

extern "C" {

tp_status tp_all_to_all(const void* const* in, void* const* out, int64_t rows, int64_t cols, int split_axis,
                        int concat_axis, tp_dtype dtype, int t, void* stream) {
  return all_to_all(in, out, rows, cols, split_axis, concat_axis, dtype, t, static_cast<cudaStream_t>(stream));
}

tp_status tp_reduce_scatter(const void* const* in, void* const* out, int64_t rows, int64_t cols, int axis,
                            tp_dtype dtype, int t, void* stream) {
  if (in == nullptr || out == nullptr) return fail(TP_EINVAL, "null pointer array");
  if (!valid_t(t)) return fail(TP_EINVAL, "t=%d outside 1..%d", t, TP_MAX_SHARDS);
  RingArgs a;
  std::memset(&a, 0, sizeof(a));
  a.op = RING_RS; a.in_dtype = a.out_dtype = dtype; a.rows = rows; a.cols = cols; a.axis = axis; a.t = t;
  for (int i = 0; i < t; ++i) { a.in[i] = in[i]; a.out[i] = out[i]; }
  return ring_collective(a, static_cast<cudaStream_t>(stream));
}

tp_status tp_all_gather(const void* const* in, void* const* out, int64_t rows, int64_t cols, int axis, tp_dtype dtype,
                        int t, void* stream) {
  if (in == nullptr || out == nullptr) return fail(TP_EINVAL, "null pointer array");
  if (!valid_t(t)) return fail(TP_EINVAL, "t=%d outside 1..%d", t, TP_MAX_SHARDS);
  RingArgs a;
  std::memset(&a, 0, sizeof(a));
  a.op = RING_AG; a.in_dtype = a.out_dtype = dtype; a.rows = rows; a.cols = cols; a.axis = axis; a.t = t;
  for (int i = 0; i < t; ++i) { a.in[i] = in[i]; a.out[i] = out[i]; }
  return ring_collective(a, static_cast<cudaStream_t>(stream));
}

tp_status tp_all_reduce(const void* const* in, void* const* out, int64_t rows, int64_t cols, tp_dtype dtype, int t,
                        void* stream) {
  if (in == nullptr || out == nullptr) return fail(TP_EINVAL, "null pointer array");
  if (!valid_t(t)) return fail(TP_EINVAL, "t=%d outside 1..%d", t, TP_MAX_SHARDS);
  RingArgs a;
  std::memset(&a, 0, sizeof(a));
  a.op = RING_AR; a.in_dtype = a.out_dtype = dtype; a.rows = rows; a.cols = cols; a.axis = 0; a.t = t;
  for (int i = 0; i < t; ++i) { a.in[i] = in[i]; a.out[i] = out[i]; }
  // Chunks are row blocks (AllReduce = ReduceScatter along rows + AllGather), so t must divide rows.
  return ring_collective(a, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
