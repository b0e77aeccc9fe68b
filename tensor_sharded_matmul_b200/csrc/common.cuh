// Host-side plumbing shared by the libtp translation units: error reporting, per-device caches,
// argument checks. Device code lives in ptx.cuh and the kernel files.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "tp.h"

namespace tpx {

// Codes recorded in the device status word (which bounded wait ran out).
enum WaitSite : uint32_t {
  WAIT_SELFTEST = 1,
  WAIT_PRODUCER_EMPTY = 2,   // TMA producer waiting for a free shared-memory stage
  WAIT_MMA_FULL = 3,         // MMA issuer waiting for a stage's TMA bytes
  WAIT_MMA_ACC_EMPTY = 4,    // MMA issuer waiting for the epilogue to drain an accumulator
  WAIT_EPI_ACC_FULL = 5,     // epilogue waiting for an accumulator
  WAIT_TEARDOWN = 6          // draining in-flight copies / MMAs before exit
};

// Records a failure message for the calling host thread and returns `s`.
tp_status fail(tp_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
// Returns TP_ECUDA (with message) if the last launch failed, TP_OK otherwise.
tp_status check_launch(const char* what);
// Per-device address of the status word (nullptr when the runtime call fails).
uint32_t* status_word();
// Current budget of bounded device waits, in SM cycles.
unsigned long long wait_budget();
// Cached SM count of the current device (0 on failure).
int sm_count();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool valid_t(int t) { return t >= 1 && t <= TP_MAX_SHARDS; }

// ---- internal entry points shared between translation units -------------------------------------
enum RingOp { RING_RS = 0, RING_AG = 1, RING_AR = 2 };

struct RingArgs {
  RingOp op;
  const void* in[TP_MAX_SHARDS];
  void* out[TP_MAX_SHARDS];
  tp_dtype in_dtype, out_dtype;
  int64_t rows, cols;        // the full logical [rows, cols] matrix
  int axis;                  // chunk axis (RS, AG)
  int t;
  const void* resid;         // AR only: optional residual added after the ring sum
  tp_dtype resid_dtype;
  uint16_t* copy_bf16;       // AR only: optional bf16 copy of the result (one buffer)
};
tp_status ring_collective(const RingArgs& a, cudaStream_t s);

enum EpiKind { EPI_F32 = 0, EPI_BF16 = 1, EPI_GELU = 2, EPI_GELU_TANH = 3, EPI_SWIGLU = 4 };

struct GemmArgs {
  int groups;
  const uint16_t* a[TP_MAX_SHARDS];  // [M, K] row-major, row stride lda elements
  const uint16_t* b[TP_MAX_SHARDS];  // [K, Nb] row-major, row stride ldb (SwiGLU: [gate | up], up at +N)
  void* c[TP_MAX_SHARDS];            // [M, N] row-major, row stride N
  int64_t M, N, K, lda, ldb;
  EpiKind epi;
  // Optional: A given as a_slices row slices [slice_rows, K] shared by every group (a[] is then
  // ignored); row m of A is row m % slice_rows of a_slice[m / slice_rows].
  int a_slices;
  int64_t slice_rows;
  const uint16_t* a_slice[TP_MAX_SHARDS];
  // Optional: A given as a_kslices column slices [M, kslice_cols] (row stride lda) shared by every
  // group (a[] is then ignored); column k of A is column k % kslice_cols of a_kslice[k / kslice_cols]
  // (an AllGather along the contraction, read where each piece lies).
  int a_kslices;
  int64_t kslice_cols;
  const uint16_t* a_kslice[TP_MAX_SHARDS];
  // Optional: B given as b_slices column slices [K, bslice_cols] (row stride ldb) shared by every
  // group (b[] is then ignored); column n of B is column n % bslice_cols of b_slice[n / bslice_cols].
  int b_slices;
  int64_t bslice_cols;
  const uint16_t* b_slice[TP_MAX_SHARDS];
  // Transposed storage: a_mn = A given as A^T [K][M] (row stride lda >= M); b_km = B given as
  // B^T [N][K] (row stride ldb >= K).
  bool a_mn, b_km;
};
tp_status grouped_gemm(const GemmArgs& g, cudaStream_t s);

// Row-parallel GEMM fused with its ring reduction: out = Reduce_s(a[s] . b[s]) over the t shards.
// RING_RS: out[c] receives chunk c (rows for axis 0, columns for axis 1); RING_AR: every out[s]
// receives the whole sum (+ resid), and copy_bf16 (optional) a bf16 copy.
struct RingGemmArgs {
  int t;
  const uint16_t* a[TP_MAX_SHARDS];  // [M, K] row-major, row stride lda
  const uint16_t* b[TP_MAX_SHARDS];  // [K, N] row-major, row stride ldb
  void* out[TP_MAX_SHARDS];
  int64_t M, N, K, lda, ldb;
  RingOp op;                         // RING_RS or RING_AR
  int axis;                          // RS chunk axis
  tp_dtype out_dtype;
  const void* resid;                 // RING_AR only, [M, N]
  tp_dtype resid_dtype;
  uint16_t* copy_bf16;               // RING_AR only, [M, N]
  bool b_km;                         // B given as B^T [N][K] (row stride ldb >= K)
};
// True when every 128 x 256 output tile lies inside one chunk (the fused kernel's requirement).
bool ring_gemm_fits(int64_t M, int64_t N, int t, int axis);
tp_status ring_gemm(const RingGemmArgs& g, cudaStream_t s);

}  // namespace tpx
