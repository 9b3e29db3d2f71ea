// capi.cu -- status strings, version and the per-thread record of the last
// CUDA error for the tree verification C ABI.
#include <atomic>

#include "tv_common.cuh"

namespace tv {
namespace {
thread_local int g_last_cuda_error = 0;
std::atomic<uint64_t> g_wait_limit_ns{0};  // 0: kWaitLimitNs
}  // namespace

uint64_t pipeline_wait_limit_ns() {
  const uint64_t v = g_wait_limit_ns.load(std::memory_order_relaxed);
  return v == 0 ? kWaitLimitNs : v;
}

tv_status record_cuda_error(cudaError_t e) {
  g_last_cuda_error = static_cast<int>(e);
  (void)cudaGetLastError();  // clear the sticky-free launch error so later calls start clean
  return TV_ERR_CUDA;
}

}  // namespace tv

extern "C" const char* tv_status_string(tv_status s) {
  switch (s) {
    case TV_OK:
      return "TV_OK";
    case TV_ERR_INVALID_ARG:
      return "TV_ERR_INVALID_ARG";
    case TV_ERR_UNSUPPORTED:
      return "TV_ERR_UNSUPPORTED";
    case TV_ERR_CUDA:
      return "TV_ERR_CUDA";
  }
  return "TV_ERR_UNKNOWN";
}

extern "C" int tv_last_cuda_error(void) { return tv::g_last_cuda_error; }

extern "C" int tv_version(void) { return 200; }

extern "C" void tv_set_wait_limit_ns(uint64_t ns) {
  tv::g_wait_limit_ns.store(ns > tv::kWaitLimitNs ? tv::kWaitLimitNs : ns, std::memory_order_relaxed);
}
