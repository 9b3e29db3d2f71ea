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
//
// Rotary position embedding (optional): the K rows are rotated to their tree
// position kv_len + depth (position-ID contiguity, "Batch Speculative Decoding
// Done Right", section 2) on the way into the cache, so the committed cache
// holds rotated keys as the attention expects; V rows are copied as they are.
//
// Slot map (optional): batch row b writes into cache slot slot[b] of a pool of
// n_slots sequences, whose geometry is kv_start[slot[b]], kv_len[slot[b]].
#include <algorithm>

#include "tv_common.cuh"

namespace tv {
namespace {

constexpr int kWriteThreads = 256;
constexpr int kWriteUnroll = 4;

// One launch for the whole append.  Work items: without rotation, 16-byte
// units of K then V; with rotation, the K rows as pairs of 16-byte chunks (c,
// c + RV/2) rotated to position kv_len + depth[b][r], then the V units.
__global__ void __launch_bounds__(kWriteThreads) kv_write_kernel(
    uint16_t* const* __restrict__ k_layers, uint16_t* const* __restrict__ v_layers,
    const uint4* __restrict__ tree_k, const uint4* __restrict__ tree_v, int B, int Hkv, int RV, int64_t S_cap,
    int M, const int32_t* __restrict__ kv_start, const int32_t* __restrict__ kv_len,
    const int32_t* __restrict__ slot, int n_slots, int64_t per_kv, const int32_t* __restrict__ depth,
    const __grid_constant__ RopeFreqs fr) {
  pdl_wait_primary();
  pdl_launch_dependents();
  const int n = M + 1;
  const bool rope = depth != nullptr;
  const int half = RV / 2;
  const int64_t k_items = rope ? per_kv / 2 : per_kv;  // K work items
  const int64_t total = k_items + per_kv;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; base < total;
       base += stride * kWriteUnroll) {
    uint4 val[kWriteUnroll], val2[kWriteUnroll];
    uint4* dst[kWriteUnroll];
    int dst2_off[kWriteUnroll];  // second chunk of a rotated pair (0: none)
#pragma unroll
    for (int t = 0; t < kWriteUnroll; ++t) {
      dst[t] = nullptr;
      dst2_off[t] = 0;
      const int64_t u = base + (int64_t)t * stride;
      if (u >= total) continue;
      const bool is_k = u < k_items;
      const int units = (is_k && rope) ? half : RV;  // items per row
      const int64_t w = is_k ? u : u - k_items;
      const int c = (int)(w % units);
      const int64_t row = w / units;  // ((l * B + b) * Hkv + h) * n + r
      const int r = (int)(row % n);
      const int64_t run = row / n;
      const int h = (int)(run % Hkv);
      const int64_t lb = run / Hkv;
      const int b = (int)(lb % B);
      const int l = (int)(lb / B);
      const int sl = cache_slot(slot, b, n_slots);
      if (sl < 0) continue;
      const int32_t ks = kv_start[sl], kl = kv_len[sl];
      if (!geometry_ok(ks, kl, M, S_cap)) continue;
      uint4* cache = reinterpret_cast<uint4*>((is_k ? k_layers : v_layers)[l]) +
                     (((int64_t)sl * Hkv + h) * S_cap + ks + kl + r) * RV;
      if (is_k && rope) {
        val[t] = tree_k[row * RV + c];
        val2[t] = tree_k[row * RV + c + half];
        rope_rotate8(val[t], val2[t], kl + depth[(int64_t)b * n + r], fr.f, 8 * c);
        dst2_off[t] = half;
      } else {
        val[t] = is_k ? tree_k[row * RV + c] : tree_v[row * RV + c];
      }
      dst[t] = cache + c;
    }
#pragma unroll
    for (int t = 0; t < kWriteUnroll; ++t)
      if (dst[t]) {
        *dst[t] = val[t];
        if (dst2_off[t]) dst[t][dst2_off[t]] = val2[t];
      }
  }
}

}  // namespace
}  // namespace tv

extern "C" tv_status tree_kv_write(uint16_t* const* k_layers, uint16_t* const* v_layers, const uint16_t* tree_k,
                                   const uint16_t* tree_v, int L, int B, int Hkv, int D, int64_t S_cap, int M,
                                   const int32_t* kv_start, const int32_t* kv_len, const int32_t* depth,
                                   float rope_theta, const int32_t* slot, int n_slots, tv_stream_t stream) {
  using namespace tv;
  if (L < 0 || B < 0 || Hkv < 0 || M < 0 || S_cap < 0) return TV_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return TV_ERR_UNSUPPORTED;
  if (M + 1 > kMaxRows) return TV_ERR_UNSUPPORTED;
  if (S_cap > 0x7fffffffLL) return TV_ERR_UNSUPPORTED;
  if (slot && n_slots < 1) return TV_ERR_INVALID_ARG;
  const bool rope = depth != nullptr;
  if (rope && !(rope_theta > 1.0f)) return TV_ERR_INVALID_ARG;
  const int64_t per_kv = (int64_t)L * B * Hkv * (M + 1) * (D / 8);
  if (per_kv == 0) return TV_OK;
  if (!k_layers || !v_layers || !tree_k || !tree_v || !kv_start || !kv_len) return TV_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(tree_k) | reinterpret_cast<uintptr_t>(tree_v)) & 15) return TV_ERR_INVALID_ARG;
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda_error(e);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  RopeFreqs fr;
  rope_freqs(rope ? (double)rope_theta : 2.0, D, fr);
  const int64_t units = (rope ? per_kv / 2 : per_kv) + per_kv;
  const int64_t need = (units + (int64_t)kWriteThreads * kWriteUnroll - 1) / ((int64_t)kWriteThreads * kWriteUnroll);
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>(need, (int64_t)sms * 8));
  return launch(kv_write_kernel, dim3((unsigned)blocks), dim3(kWriteThreads), 0, s, 1, true, k_layers, v_layers,
                reinterpret_cast<const uint4*>(tree_k), reinterpret_cast<const uint4*>(tree_v), B, Hkv, D / 8, S_cap,
                M, kv_start, kv_len, slot, slot ? n_slots : B, per_kv, rope ? depth : (const int32_t*)nullptr, fr);
}
