// Status reporting of libtp: status strings, the per-thread error message, the device status word
// that bounded waits write to, the wait budget, and the failure-path self test.
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "common.cuh"
#include "ptx.cuh"

namespace tpx {

namespace {
thread_local char g_msg[512] = "";
constexpr int kMaxDevices = 64;
uint32_t* g_status_ptr[kMaxDevices] = {};
int g_sms[kMaxDevices] = {};
unsigned long long g_budget = 0;                                  // 0 = default
constexpr unsigned long long kDefaultBudget = 4000000000ull;      // ~2 s at the SM clock
}  // namespace

// Bit 31: a bounded wait ran out; low bits: the first site that did.
__device__ uint32_t g_tp_status_word = 0;

tp_status fail(tp_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return s;
}

tp_status check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(TP_ECUDA, "%s: %s", what, cudaGetErrorString(e));
  return TP_OK;
}

uint32_t* status_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  if (g_status_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_tp_status_word) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<uint32_t*>(p);
  }
  return g_status_ptr[dev];
}

unsigned long long wait_budget() { return g_budget ? g_budget : kDefaultBudget; }

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  if (g_sms[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    g_sms[dev] = n;
  }
  return g_sms[dev];
}

// One CTA waits, bounded, on an mbarrier phase that nothing completes.
__global__ void selftest_wait_kernel(uint32_t* status, unsigned long long budget) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!mbar_wait_bounded(b, 0, budget, nullptr)) record_timeout(status, WAIT_SELFTEST);
  }
}

}  // namespace tpx

using namespace tpx;

extern "C" {

const char* tp_status_str(tp_status s) {
  switch (s) {
    case TP_OK: return "ok";
    case TP_EINVAL: return "invalid argument";
    case TP_ESHAPE: return "inconsistent shapes";
    case TP_EDIVIS: return "t does not divide a split dimension";
    case TP_EALIGN: return "pointer or stride not 16-byte aligned";
    case TP_ECUDA: return "CUDA error";
    case TP_ETIMEOUT: return "a bounded device wait ran out";
    case TP_EUNSUPPORTED: return "unsupported";
    case TP_ENOSPACE: return "workspace too small (the caller's, or the built-in no-alloc array)";
  }
  return "unknown status";
}

const char* tp_last_error(void) { return g_msg; }

tp_status tp_device_status(int clear, uint32_t* where) {
  uint32_t* p = status_word();
  if (p == nullptr) return fail(TP_ECUDA, "cannot resolve the device status word");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return fail(TP_ECUDA, "synchronize: %s", cudaGetErrorString(e));
  uint32_t v = 0;
  e = cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(TP_ECUDA, "read status word: %s", cudaGetErrorString(e));
  if (where != nullptr) *where = v & 0x7FFFFFFFu;
  if (clear) {
    const uint32_t zero = 0;
    e = cudaMemcpy(p, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return fail(TP_ECUDA, "clear status word: %s", cudaGetErrorString(e));
  }
  if (v & 0x80000000u) return fail(TP_ETIMEOUT, "device wait site %u ran out", v & 0x7FFFFFFFu);
  return TP_OK;
}

void tp_set_wait_budget(uint64_t cycles) { g_budget = cycles; }

tp_status tp_selftest_wait_timeout(uint64_t budget_cycles, void* stream) {
  uint32_t* p = status_word();
  if (p == nullptr) return fail(TP_ECUDA, "cannot resolve the device status word");
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(p, budget_cycles);
  return check_launch("selftest_wait_kernel");
}

int tp_num_sms(void) {
  int n = sm_count();
  return n > 0 ? n : -1;
}

}  // extern "C"
