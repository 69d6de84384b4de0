// api.cu -- library-wide entry points of libnvfp4qad: status strings, ABI
// version and the device error word that bounded waits report into.
#include "common.cuh"

#include <nvtx3/nvToolsExt.h>

#include <atomic>
#include <cstdlib>

namespace nvfp4 {
__device__ int g_device_error = 0;

static std::atomic<uint64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

// Fault injection: outermost entries counted since arming; the armed index
// (0 = disarmed).  Read from NVFP4QAD_FAIL_AT when the library loads.
static std::atomic<int64_t> g_fail_at{0};
static std::atomic<int64_t> g_entries{0};
static thread_local int t_depth = 0;

static int64_t fail_at_from_env() {
  const char* v = std::getenv("NVFP4QAD_FAIL_AT");
  if (!v || !*v) return 0;
  char* end = nullptr;
  const long long n = std::strtoll(v, &end, 10);
  return (end && *end == 0 && n > 0) ? (int64_t)n : 0;
}
static const bool g_env_armed = [] {
  const int64_t n = fail_at_from_env();
  if (n > 0) g_fail_at.store(n);
  return n > 0;
}();

EntryScope::EntryScope(const char* name) : inject(false) {
  nvtxRangePushA(name);
  if (t_depth++ == 0) {
    const int64_t armed = g_fail_at.load(std::memory_order_relaxed);
    if (armed > 0) {
      const int64_t k = g_entries.fetch_add(1, std::memory_order_relaxed) + 1;
      if (k == armed) {
        inject = true;
        g_fail_at.store(0, std::memory_order_relaxed);  // one failure per arming
      }
    }
  }
}

EntryScope::~EntryScope() {
  --t_depth;
  nvtxRangePop();
}
}  // namespace nvfp4

extern "C" {

const char* nvfp4_status_string(nvfp4_status status) {
  switch (status) {
    case NVFP4_OK: return "NVFP4_OK";
    case NVFP4_ERR_ARG: return "NVFP4_ERR_ARG: invalid argument";
    case NVFP4_ERR_SHAPE: return "NVFP4_ERR_SHAPE: unsupported shape";
    case NVFP4_ERR_ALIGN: return "NVFP4_ERR_ALIGN: pointer or stride not aligned";
    case NVFP4_ERR_DTYPE: return "NVFP4_ERR_DTYPE: unsupported dtype";
    case NVFP4_ERR_CUDA: return "NVFP4_ERR_CUDA: CUDA runtime or launch error";
    case NVFP4_ERR_TIMEOUT: return "NVFP4_ERR_TIMEOUT: bounded device wait expired";
    case NVFP4_ERR_DEVICE: return "NVFP4_ERR_DEVICE: device error word set";
    case NVFP4_ERR_WORKSPACE: return "NVFP4_ERR_WORKSPACE: workspace missing or too small";
    case NVFP4_ERR_UNSUPPORTED: return "NVFP4_ERR_UNSUPPORTED: no kernel for this device or configuration";
  }
  return "NVFP4 unknown status";
}

int nvfp4_abi_version(void) { return NVFP4QAD_ABI_VERSION; }

void nvfp4_fault_inject(int64_t nth) {
  nvfp4::g_entries.store(0, std::memory_order_relaxed);
  nvfp4::g_fail_at.store(nth > 0 ? nth : 0, std::memory_order_relaxed);
}

uint64_t nvfp4_launch_count(void) { return nvfp4::g_launches.load(std::memory_order_relaxed); }

nvfp4_status nvfp4_device_error(void* stream, int32_t* code_out) {
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaStreamSynchronize(s) != cudaSuccess) return NVFP4_ERR_CUDA;
  int word = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbol(&word, nvfp4::g_device_error, sizeof(int)) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (word != 0 && cudaMemcpyToSymbol(nvfp4::g_device_error, &zero, sizeof(int)) != cudaSuccess)
    return NVFP4_ERR_CUDA;
  if (code_out) *code_out = word;
  if (word == 0) return NVFP4_OK;
  return word == nvfp4::kErrWaitTimeout ? NVFP4_ERR_TIMEOUT : NVFP4_ERR_DEVICE;
}

}  // extern "C"
