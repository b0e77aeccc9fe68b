// tp_mlp_fwd_noalloc: the tensor-parallel MLP forward for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc. One case is code inside a host framework whose caching pool
// owns the GPU's memory: an allocation behind the pool's back can fail once the pool has reserved
// the device, and it escapes the pool's accounting. Another is a serving loop that forbids
// allocation after start-up, because cudaMalloc and cudaFree can synchronise the device and stall
// other streams. This entry point therefore takes only its inputs and outputs. Its scratch (the
// activations Z and the fp32 partial sums) lives in the fixed array below, compiled into the
// library; the caller passes no workspace.
//
// Properties callers must know:
//   * Every GPU that loads the library holds TP_MLP_NOALLOC_SCRATCH_BYTES of device memory for this
//     array until the process exits.
//   * Requests whose scratch does not fit are rejected with TP_ENOSPACE before anything is launched.
//   * All calls share the one array, and it keeps the last call's contents. Nothing in it needs to
//     start at zero: every call overwrites all the scratch it reads. Calls that overlap on the GPU
//     (for example on two streams without ordering between them) race on the array and give wrong
//     results.
//   * The first call on a device resolves the array's device address (cudaGetSymbolAddress, which
//     may load the module). Make that first call before any stream capture.
//   * Nothing here calls cudaMalloc, cudaFree or any allocating library routine. The kernels are
//     the ones tp_mlp_fwd launches.
#include <atomic>

#include "common.cuh"

// The scratch: file scope, one copy per device that loads the library.
static __device__ __align__(256) unsigned char g_mlp_scratch[TP_MLP_NOALLOC_SCRATCH_BYTES];

namespace tpx {
namespace {

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_addr[kMaxDevices];

// Device address of the scratch array on the current device (nullptr on failure).
void* scratch_address(tp_status* st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *st = fail(TP_ECUDA, "cannot query the current device");
    return nullptr;
  }
  void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    cudaError_t e = cudaGetSymbolAddress(&p, g_mlp_scratch);
    if (e != cudaSuccess || p == nullptr) {
      *st = fail(TP_ECUDA, "cannot resolve the built-in scratch array: %s", cudaGetErrorString(e));
      return nullptr;
    }
    g_scratch_addr[dev].store(p, std::memory_order_release);
  }
  *st = TP_OK;
  return p;
}

size_t round256(size_t n) { return (n + 255) & ~size_t(255); }

}  // namespace
}  // namespace tpx

using namespace tpx;

extern "C" tp_status tp_mlp_fwd_noalloc(const uint16_t* x, int64_t N, int64_t h, int64_t F, int t, tp_act act,
                                        const uint16_t* w_in, const uint16_t* w_down, tp_reduce mode,
                                        float* const* out, void* stream) {
  if (!valid_t(t)) return fail(TP_EINVAL, "t=%d outside 1..%d", t, TP_MAX_SHARDS);
  if (out == nullptr) return fail(TP_EINVAL, "null output array");
  if (N < 0 || h <= 0 || F <= 0) return fail(TP_EINVAL, "negative size or empty hidden/F dimension");
  if (N == 0) return TP_OK;                              // no tokens: nothing to compute
  if (mode < TP_OUT_PARTIALS || mode > TP_OUT_RS_AG) return fail(TP_EINVAL, "bad reduce mode");
  // Scratch: Z as bf16 [t][N][F/t], plus t fp32 [N, h] partials when a reducing mode takes the
  // unfused path. When (N/t) % 128 == 0 the row GEMM is fused with its reduction and never touches
  // partials. Every size is bounded before it is multiplied, so no product can wrap around.
  const uint64_t cap = TP_MLP_NOALLOC_SCRATCH_BYTES;
  const uint64_t n = static_cast<uint64_t>(N);
  if (static_cast<uint64_t>(F) > cap / 2 || n > cap / (2 * static_cast<uint64_t>(F)))
    return fail(TP_ENOSPACE, "the activations need more scratch than the built-in %u-byte array holds",
                (unsigned)TP_MLP_NOALLOC_SCRATCH_BYTES);
  const size_t z_bytes = round256(n * static_cast<uint64_t>(F) * 2);
  const bool fused = mode != TP_OUT_PARTIALS && ring_gemm_fits(N, h, t, 0);
  const bool use_partials = mode != TP_OUT_PARTIALS && !fused;
  size_t part_bytes = 0;
  if (use_partials) {
    if (static_cast<uint64_t>(h) > cap / 4 || n > cap / (4 * static_cast<uint64_t>(h)))
      return fail(TP_ENOSPACE, "the partial sums need more scratch than the built-in %u-byte array holds",
                  (unsigned)TP_MLP_NOALLOC_SCRATCH_BYTES);
    part_bytes = round256(n * static_cast<uint64_t>(h) * 4);
  }
  const uint64_t need = z_bytes + static_cast<uint64_t>(t) * part_bytes;   // t <= 16: no wrap
  if (need > cap)
    return fail(TP_ENOSPACE, "this request needs %llu bytes of scratch; the built-in array holds %u",
                (unsigned long long)need, (unsigned)TP_MLP_NOALLOC_SCRATCH_BYTES);
  tp_status st = TP_OK;
  char* base = static_cast<char*>(scratch_address(&st));
  if (base == nullptr) return st;
  uint16_t* z = reinterpret_cast<uint16_t*>(base);
  if (mode == TP_OUT_PARTIALS)   // the partials are the result: write them straight into out
    return tp_mlp_fwd(x, N, h, F, t, act, w_in, w_down, z, out, mode, nullptr, stream);
  if (!use_partials)             // the fused row GEMM + reduction keeps the partials on chip
    return tp_mlp_fwd(x, N, h, F, t, act, w_in, w_down, z, nullptr, mode, out, stream);
  float* partials[TP_MAX_SHARDS];
  for (int r = 0; r < t; ++r) partials[r] = reinterpret_cast<float*>(base + z_bytes + size_t(r) * part_bytes);
  return tp_mlp_fwd(x, N, h, F, t, act, w_in, w_down, z, partials, mode, out, stream);
}
