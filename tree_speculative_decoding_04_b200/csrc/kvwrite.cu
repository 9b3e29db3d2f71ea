// kvwrite.cu -- tree_kv_write: the K and V rows of the step's M+1 tree nodes go
// right behind each sequence's committed prefix, in every layer.
//
// This is the cache layout the other calls read: "EAGLE-Pangu: Accelerator-Safe
// Tree Speculative Decoding on Ascend NPUs", methodology C runs one batched
// teacher pass over all speculative tokens against the cached prefix; here the
// speculative tokens' own K/V rows sit in the same per-layer cache, at columns
// kv_start + kv_len + r, so that the tree mask alone separates the branches.
//
// Design: a pure copy, HBM-bound.  The source [L][B][Hkv][M+1][D] is read in
// order, 16 bytes per thread and access, a few accesses in flight per thread
// (all loads of a batch before its stores); each destination row is D * 2
// contiguous bytes.  The grid is a multiple of the SM count, grid-stride.
#include <algorithm>

#include "tv_common.cuh"

namespace tv {
namespace {

constexpr int kWriteThreads = 256;
constexpr int kWriteUnroll = 4;

__global__ void __launch_bounds__(kWriteThreads) kv_write_kernel(
    uint16_t* const* __restrict__ k_layers, uint16_t* const* __restrict__ v_layers,
    const uint4* __restrict__ tree_k, const uint4* __restrict__ tree_v, int B, int Hkv, int RV, int64_t S_cap,
    int M, const int32_t* __restrict__ kv_start, const int32_t* __restrict__ kv_len, int64_t per_kv) {
  pdl_wait_primary();
  pdl_launch_dependents();
  const int n = M + 1;
  const int64_t total = 2 * per_kv;  // 16-byte units: K then V
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; base < total;
       base += stride * kWriteUnroll) {
    uint4 val[kWriteUnroll];
    uint4* dst[kWriteUnroll];
#pragma unroll
    for (int t = 0; t < kWriteUnroll; ++t) {
      dst[t] = nullptr;
      const int64_t u = base + (int64_t)t * stride;
      if (u >= total) continue;
      const int kv = u >= per_kv;
      const int64_t w = kv ? u - per_kv : u;  // index inside [L][B][Hkv][n][RV]
      const int c = (int)(w % RV);
      const int64_t row = w / RV;  // ((l * B + b) * Hkv + h) * n + r
      const int r = (int)(row % n);
      const int64_t run = row / n;
      const int h = (int)(run % Hkv);
      const int64_t lb = run / Hkv;
      const int b = (int)(lb % B);
      const int l = (int)(lb / B);
      const int32_t ks = kv_start[b], kl = kv_len[b];
      if (!geometry_ok(ks, kl, M, S_cap)) continue;
      val[t] = kv ? tree_v[w] : tree_k[w];
      uint4* cache = reinterpret_cast<uint4*>((kv ? v_layers : k_layers)[l]);
      dst[t] = cache + (((int64_t)b * Hkv + h) * S_cap + ks + kl + r) * RV + c;
    }
#pragma unroll
    for (int t = 0; t < kWriteUnroll; ++t)
      if (dst[t]) *dst[t] = val[t];
  }
}

}  // namespace
}  // namespace tv

extern "C" tv_status tree_kv_write(uint16_t* const* k_layers, uint16_t* const* v_layers, const uint16_t* tree_k,
                                   const uint16_t* tree_v, int L, int B, int Hkv, int D, int64_t S_cap, int M,
                                   const int32_t* kv_start, const int32_t* kv_len, tv_stream_t stream) {
  using namespace tv;
  if (L < 0 || B < 0 || Hkv < 0 || M < 0 || S_cap < 0) return TV_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return TV_ERR_UNSUPPORTED;
  if (M + 1 > kMaxRows) return TV_ERR_UNSUPPORTED;
  if (S_cap > 0x7fffffffLL) return TV_ERR_UNSUPPORTED;
  const int64_t per_kv = (int64_t)L * B * Hkv * (M + 1) * (D / 8);
  if (per_kv == 0) return TV_OK;
  if (!k_layers || !v_layers || !tree_k || !tree_v || !kv_start || !kv_len) return TV_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(tree_k) | reinterpret_cast<uintptr_t>(tree_v)) & 15) return TV_ERR_INVALID_ARG;
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda_error(e);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t need = (2 * per_kv + (int64_t)kWriteThreads * kWriteUnroll - 1) / ((int64_t)kWriteThreads * kWriteUnroll);
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>(need, (int64_t)sms * 8));
  return launch(kv_write_kernel, dim3((unsigned)blocks), dim3(kWriteThreads), 0,
                reinterpret_cast<cudaStream_t>(stream), 1, true, k_layers, v_layers,
                reinterpret_cast<const uint4*>(tree_k), reinterpret_cast<const uint4*>(tree_v), B, Hkv, D / 8, S_cap,
                M, kv_start, kv_len, per_kv);
}
