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
// Memory traffic is coalesced 16-byte vectors; grids are a multiple of the SM count with
// grid-stride loops. bf16 inputs are widened (exact), summed in binary32 and rounded once to bf16
// (nearest-even) at the end.
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

// ReduceScatter (AR == false) or AllReduce (AR == true). TT = compile-time t (0: runtime t).
template <typename Tin, typename Tout, int VEC, int TT, bool AR>
__global__ void __launch_bounds__(256) ring_reduce_kernel(const __grid_constant__ RingParams p) {
  const int t = TT > 0 ? TT : p.t;
  const int64_t units = p.rows * p.cols / VEC;
  for (int64_t u = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; u < units;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t e = u * VEC;
    int c;
    int64_t local;
    locate(p, e, c, local);
    float acc[VEC];
    if constexpr (TT > 0) {
      float v[TT][VEC];
#pragma unroll
      for (int j = 0; j < TT; ++j) IO<Tin, VEC>::load(p.in[(c + 1 + j) % TT], e, v[j]);   // issue all loads first
#pragma unroll
      for (int i = 0; i < VEC; ++i) acc[i] = v[0][i];
#pragma unroll
      for (int j = 1; j < TT; ++j) {
#pragma unroll
        for (int i = 0; i < VEC; ++i) acc[i] = __fadd_rn(acc[i], v[j][i]);
      }
    } else {
      IO<Tin, VEC>::load(p.in[(c + 1) % t], e, acc);
      for (int j = 2; j <= t; ++j) {
        float v[VEC];
        IO<Tin, VEC>::load(p.in[(c + j) % t], e, v);
#pragma unroll
        for (int i = 0; i < VEC; ++i) acc[i] = __fadd_rn(acc[i], v[i]);
      }
    }
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
}

// AllGather as a bit copy: every shard receives every piece. UNIT = bytes moved per step
// (16 = one vector, or the element size for the unaligned path); ES = element size.
template <int ES, int UNIT>
__global__ void __launch_bounds__(256) ring_gather_kernel(const __grid_constant__ RingParams p) {
  constexpr int EPU = UNIT / ES;   // elements per unit
  const int64_t units = p.rows * p.cols / EPU;
  for (int64_t u = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; u < units;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t e = u * EPU;
    int c;
    int64_t local;
    locate(p, e, c, local);
    const char* src = static_cast<const char*>(p.in[c]) + local * ES;
    if constexpr (UNIT == 16) {
      const uint4 v = ld_nc_v4(src);
      for (int s = 0; s < p.t; ++s) {
        if (p.skip_self && s == c) continue;
        st_v4(static_cast<char*>(p.out[s]) + e * ES, v);
      }
    } else if constexpr (ES == 4) {
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

int grid_for(int64_t units) {
  const int sms = sm_count();
  const int64_t cap = static_cast<int64_t>(sms) * 8;   // 8 x 256 threads: a full SM
  const int64_t want = (units + 255) / 256;
  return static_cast<int>(want < cap ? want : cap);
}

template <typename Tin, typename Tout, int VEC, bool AR>
void launch_reduce(const RingParams& p, int blocks, cudaStream_t s) {
  switch (p.t) {
    case 2: ring_reduce_kernel<Tin, Tout, VEC, 2, AR><<<blocks, 256, 0, s>>>(p); break;
    case 4: ring_reduce_kernel<Tin, Tout, VEC, 4, AR><<<blocks, 256, 0, s>>>(p); break;
    case 8: ring_reduce_kernel<Tin, Tout, VEC, 8, AR><<<blocks, 256, 0, s>>>(p); break;
    default: ring_reduce_kernel<Tin, Tout, VEC, 0, AR><<<blocks, 256, 0, s>>>(p); break;
  }
}

template <int VEC, bool AR>
void dispatch_reduce(const RingParams& p, tp_dtype din, tp_dtype dout, int blocks, cudaStream_t s) {
  if (din == TP_F32 && dout == TP_F32) launch_reduce<float, float, VEC, AR>(p, blocks, s);
  else if (din == TP_BF16 && dout == TP_BF16) launch_reduce<uint16_t, uint16_t, VEC, AR>(p, blocks, s);
  else if (din == TP_F32 && dout == TP_BF16) launch_reduce<float, uint16_t, VEC, AR>(p, blocks, s);
  else launch_reduce<uint16_t, float, VEC, AR>(p, blocks, s);
}

}  // namespace

tp_status ring_collective(const RingArgs& a, cudaStream_t stream) {
  if (!valid_t(a.t)) return fail(TP_EINVAL, "t=%d outside 1..%d", a.t, TP_MAX_SHARDS);
  if (a.rows < 0 || a.cols < 0) return fail(TP_EINVAL, "negative size");
  if (a.rows == 0 || a.cols == 0) return TP_OK;         // empty buffers: nothing to move
  if (a.axis != 0 && a.axis != 1) return fail(TP_EINVAL, "axis must be 0 or 1");
  if ((a.in_dtype != TP_F32 && a.in_dtype != TP_BF16) || (a.out_dtype != TP_F32 && a.out_dtype != TP_BF16))
    return fail(TP_EINVAL, "bad dtype");
  if (a.op == RING_AG && a.in_dtype != a.out_dtype) return fail(TP_EINVAL, "AllGather copies bits: dtypes must match");
  const int axis = a.op == RING_AR ? 0 : a.axis;
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

  if (a.op == RING_AG) {
    const int es = a.in_dtype == TP_F32 ? 4 : 2;
    const int epu = 16 / es;
    bool vec = all16 && (axis == 0 ? p.chunk_elems % epu == 0 : (p.chunk_cols % epu == 0 && a.cols % epu == 0));
    // In place: shard r's piece already sits at its place in out[r].
    bool in_place = axis == 0;
    for (int i = 0; i < a.t && in_place; ++i)
      in_place = static_cast<const char*>(a.in[i]) == static_cast<const char*>(a.out[i]) + i * p.chunk_elems * es;
    p.skip_self = in_place ? 1 : 0;
    const int64_t units = a.rows * a.cols / (vec ? epu : 1);
    const int blocks = grid_for(units);
    if (es == 4) {
      if (vec) ring_gather_kernel<4, 16><<<blocks, 256, 0, stream>>>(p);
      else ring_gather_kernel<4, 4><<<blocks, 256, 0, stream>>>(p);
    } else {
      if (vec) ring_gather_kernel<2, 16><<<blocks, 256, 0, stream>>>(p);
      else ring_gather_kernel<2, 2><<<blocks, 256, 0, stream>>>(p);
    }
    return check_launch("ring_gather_kernel");
  }

  // Vectors of 8 elements must not straddle a chunk (or, for axis 1, a row).
  const bool vec = all16 && (axis == 0 ? p.chunk_elems % 8 == 0 : (p.chunk_cols % 8 == 0 && a.cols % 8 == 0));
  const int64_t units = a.rows * a.cols / (vec ? 8 : 1);
  const int blocks = grid_for(units);
  if (a.op == RING_RS) {
    if (vec) dispatch_reduce<8, false>(p, a.in_dtype, a.out_dtype, blocks, stream);
    else dispatch_reduce<1, false>(p, a.in_dtype, a.out_dtype, blocks, stream);
  } else {
    if (vec) dispatch_reduce<8, true>(p, a.in_dtype, a.out_dtype, blocks, stream);
    else dispatch_reduce<1, true>(p, a.in_dtype, a.out_dtype, blocks, stream);
  }
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
