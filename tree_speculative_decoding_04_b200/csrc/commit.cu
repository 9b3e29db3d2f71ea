// commit.cu -- kv_commit_realign: path-index commit of the accepted branch into
// every layer of the KV cache, and EQSPEC unpad-append-repad for left-padded
// batches.
//
// "EAGLE-Pangu: Accelerator-Safe Tree Speculative Decoding on Ascend NPUs",
// methodology A: after acceptance only the new segment is reordered by the
// accepted path ("fast reorder") while the committed prefix keeps its order.
// "Batch Speculative Decoding Done Right", methodology: every round the ragged
// batch is unpadded, the accepted tokens are appended and the batch is repadded
// so that pad + length equals the batch maximum for every sequence and position
// IDs run contiguously from 0 over the attended columns.
//
// Design: one CTA per run (layer, K|V, sequence, kv head).  A run's content is
// one contiguous block of kv_len rows, so the repad is an in-place memmove by
// s = kv_start' - kv_start rows.  The CTA (1) stages the committed tail rows in
// shared memory, (2) moves the content in 16-byte vectors, chunk by chunk, in
// the order that never overwrites an unread source (from the top when s > 0,
// from the bottom when s < 0), loading chunk c+1 while storing chunk c, and
// (3) writes the staged tail rows behind the moved content.  Extra CTAs write
// the attention mask and position IDs; a one-CTA kernel, launched as a
// programmatic dependent, publishes the new kv_start / kv_len / max_len after
// every run has read the old ones.
//
// Slot map (optional): batch row b lives in cache slot slot[b] of a pool; the
// geometry and the mask / position rows belong to the slot, so a batch can be
// any set of the pool's sequences (cross-batch scheduling, "Batch Speculative
// Decoding Done Right", section 2, EXSPEC) without moving their caches.
#include <algorithm>

#include "tv_common.cuh"

namespace tv {
namespace {

constexpr int kMoveThreads = 128;
constexpr int kMoveUnroll = 4;  // uint4 per thread per chunk
constexpr int kPlanThreads = 256;

struct Plan {
  int good;  // slot and geometry in range
  int nb;    // committed rows (0 or accept_len + 1)
  int sl;    // cache slot of the batch row
  int ks, len;
};

// Slot map: batch row b lives in cache slot slot[b] (slot == null: slot b);
// the geometry arrays and the mask / position rows are indexed by slot.
struct Slots {
  const int32_t* slot;
  int n;
};

__device__ __forceinline__ Plan seq_plan(int b, int M, int64_t S_cap, int max_depth, const int32_t* path,
                                         const int32_t* accept_len, const int32_t* status, const int32_t* kv_start,
                                         const int32_t* kv_len, Slots slots) {
  Plan p;
  p.sl = cache_slot(slots.slot, b, slots.n);
  p.ks = p.sl >= 0 ? kv_start[p.sl] : 0;
  p.len = p.sl >= 0 ? kv_len[p.sl] : 0;
  p.good = (p.sl >= 0 && geometry_ok(p.ks, p.len, M, S_cap)) ? 1 : 0;
  const int a = accept_len[b];
  int nb = 0;
  if (p.good && status[b] == 0 && a >= 0 && a <= max_depth && a <= M) {
    nb = a + 1;
    const int32_t* pb = path + (int64_t)b * (max_depth + 1);
    for (int j = 0; j < nb; ++j) {
      const int r = pb[j];
      if (r < 0 || r > M) {
        nb = 0;
        break;
      }
    }
  }
  p.nb = nb;
  return p;
}

// Lmax' over the batch (block-wide reduction; every thread gets the result).
__device__ int batch_new_max(int B, int M, int64_t S_cap, int max_depth, int realign, const int32_t* path,
                             const int32_t* accept_len, const int32_t* status, const int32_t* kv_start,
                             const int32_t* kv_len, Slots slots, int* red) {
  int mx = 0;
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const Plan p = seq_plan(b, M, S_cap, max_depth, path, accept_len, status, kv_start, kv_len, slots);
    if (p.good) mx = max(mx, realign ? p.len + p.nb : p.ks + p.len + p.nb);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  int r = 0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r = max(r, red[w]);
  __syncthreads();
  return r;
}

// grid.x = runs (+ B mask/pos CTAs when the mask or pos output is requested).
// run = ((layer * 2 + kv) * B + b) * Hkv + h.
__global__ void __launch_bounds__(kMoveThreads) kv_move_kernel(
    uint16_t* const* __restrict__ k_layers, uint16_t* const* __restrict__ v_layers, int B, int Hkv, int D,
    int64_t S_cap, int M, const int32_t* __restrict__ path, const int32_t* __restrict__ accept_len,
    const int32_t* __restrict__ status, int max_depth, const int32_t* __restrict__ kv_start,
    const int32_t* __restrict__ kv_len, int realign, int64_t runs, uint8_t* __restrict__ attn_mask,
    int32_t* __restrict__ pos_ids, Slots slots) {
  pdl_wait_primary();
  pdl_launch_dependents();
  extern __shared__ uint4 tail[];  // [max_depth + 1][D / 8]
  __shared__ int red[kMoveThreads / 32];
  const int64_t run = blockIdx.x;
  int b;
  if (run >= runs) {
    b = (int)(run - runs);
  } else {
    b = (int)((run / Hkv) % B);
  }
  const Plan me = seq_plan(b, M, S_cap, max_depth, path, accept_len, status, kv_start, kv_len, slots);
  int new_start = me.ks;
  if (realign) {
    const int lmax =
        batch_new_max(B, M, S_cap, max_depth, realign, path, accept_len, status, kv_start, kv_len, slots, red);
    new_start = lmax - (me.len + me.nb);
  }
  if (run >= runs) {  // mask / position-ID row of sequence b (row of its slot)
    if (me.sl < 0) return;
    const int lo = new_start, hi = new_start + me.len + me.nb;
    for (int64_t t = threadIdx.x; t < S_cap; t += blockDim.x) {
      const bool in = me.good && t >= lo && t < hi;
      if (attn_mask) attn_mask[(int64_t)me.sl * S_cap + t] = in ? 1 : 0;
      if (pos_ids) pos_ids[(int64_t)me.sl * S_cap + t] = in ? (int32_t)(t - lo) : 0;
    }
    return;
  }
  if (!me.good) return;
  const int shift = new_start - me.ks;
  if (shift == 0) {
    // Nothing moves when every committed row already sits at its place (a
    // chain accepted in order): the length-based commit of "EAGLE-Pangu",
    // methodology A -- only kv_len grows, which kv_finalize_kernel publishes.
    const int32_t* pb = path + (int64_t)b * (max_depth + 1);
    bool in_place = true;
    for (int j = 0; j < me.nb; ++j) in_place = in_place && pb[j] == j;
    if (in_place) return;
  }
  const int h = (int)(run % Hkv);
  const int kvsel = (int)((run / ((int64_t)Hkv * B)) & 1);
  const int layer = (int)(run / ((int64_t)Hkv * B * 2));
  uint16_t* base = (kvsel ? v_layers : k_layers)[layer];
  const int RV = D >> 3;  // uint4 per row
  uint4* cache = reinterpret_cast<uint4*>(base + ((int64_t)me.sl * Hkv + h) * S_cap * D);
  const int32_t* pb = path + (int64_t)b * (max_depth + 1);

  // (1) stage the committed tail rows (all of them are read before any store)
  const int64_t tail0 = (int64_t)me.ks + me.len;
  for (int i = threadIdx.x; i < me.nb * RV; i += blockDim.x) {
    const int j = i / RV, c = i - j * RV;
    tail[i] = cache[(tail0 + pb[j]) * RV + c];
  }
  __syncthreads();

  // (2) move the content block [ks, ks + len) to [ks + shift, ...), in place
  if (shift != 0 && me.len > 0) {
    const int64_t total = (int64_t)me.len * RV;
    const uint4* src = cache + (int64_t)me.ks * RV;
    uint4* dst = cache + ((int64_t)me.ks + shift) * RV;
    const int64_t chunk = (int64_t)kMoveThreads * kMoveUnroll;
    const int64_t nch = (total + chunk - 1) / chunk;
    const bool top_down = shift > 0;
    // chunk c covers [c0, c0 + chunk) clipped to [0, total)
    auto chunk_lo = [&](int64_t c) -> int64_t { return top_down ? total - (c + 1) * chunk : c * chunk; };
    uint4 cur[kMoveUnroll], nxt[kMoveUnroll];
    {
      const int64_t c0 = chunk_lo(0);
#pragma unroll
      for (int t = 0; t < kMoveUnroll; ++t) {
        const int64_t i = c0 + threadIdx.x + (int64_t)t * kMoveThreads;
        if (i >= 0 && i < total) cur[t] = src[i];
      }
    }
    for (int64_t c = 0; c < nch; ++c) {
      __syncthreads();  // every load of chunk c (and before) has been performed
      if (c + 1 < nch) {
        const int64_t c1 = chunk_lo(c + 1);
#pragma unroll
        for (int t = 0; t < kMoveUnroll; ++t) {
          const int64_t i = c1 + threadIdx.x + (int64_t)t * kMoveThreads;
          if (i >= 0 && i < total) nxt[t] = src[i];
        }
      }
      const int64_t c0 = chunk_lo(c);
#pragma unroll
      for (int t = 0; t < kMoveUnroll; ++t) {
        const int64_t i = c0 + threadIdx.x + (int64_t)t * kMoveThreads;
        if (i >= 0 && i < total) dst[i] = cur[t];
      }
#pragma unroll
      for (int t = 0; t < kMoveUnroll; ++t) cur[t] = nxt[t];
    }
    __syncthreads();  // all content loads done before tail rows land on old content columns
  }

  // (3) the committed rows go right behind the (moved) content
  const int64_t out0 = (int64_t)new_start + me.len;
  for (int i = threadIdx.x; i < me.nb * RV; i += blockDim.x) {
    const int j = i / RV, c = i - j * RV;
    if (shift == 0 && pb[j] == j) continue;  // already in place
    cache[(out0 + j) * RV + c] = tail[i];
  }
}

// One CTA: publish the new geometry after every run has read the old one.
__global__ void __launch_bounds__(kPlanThreads) kv_finalize_kernel(
    int B, int M, int64_t S_cap, int max_depth, int realign, const int32_t* __restrict__ path,
    const int32_t* __restrict__ accept_len, int32_t* __restrict__ status, int32_t* __restrict__ kv_start,
    int32_t* __restrict__ kv_len, int32_t* __restrict__ max_len, Slots slots) {
  __shared__ int red[kPlanThreads / 32];
  pdl_wait_primary();
  pdl_launch_dependents();
  const int lmax =
      batch_new_max(B, M, S_cap, max_depth, realign, path, accept_len, status, kv_start, kv_len, slots, red);
  // every thread finished reading the old values inside batch_new_max (it ends with a barrier)
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const Plan p = seq_plan(b, M, S_cap, max_depth, path, accept_len, status, kv_start, kv_len, slots);
    if (!p.good) {
      status[b] |= kSeqBadGeometry;
      continue;
    }
    kv_len[p.sl] = p.len + p.nb;
    kv_start[p.sl] = realign ? lmax - (p.len + p.nb) : p.ks;
  }
  if (threadIdx.x == 0) *max_len = lmax;
}

}  // namespace
}  // namespace tv

extern "C" tv_status kv_commit_realign(uint16_t* const* k_layers, uint16_t* const* v_layers, int L, int B, int Hkv,
                                       int D, int64_t S_cap, int M, const int32_t* path, const int32_t* accept_len,
                                       int32_t* status, int max_depth, int32_t* kv_start, int32_t* kv_len,
                                       int32_t* max_len, int realign, uint8_t* attn_mask, int32_t* pos_ids,
                                       const int32_t* slot, int n_slots, tv_stream_t stream) {
  using namespace tv;
  if (L < 0 || B < 0 || Hkv < 0 || M < 0 || max_depth < 0 || S_cap < 0 || (realign != 0 && realign != 1))
    return TV_ERR_INVALID_ARG;
  if (slot && n_slots < 1) return TV_ERR_INVALID_ARG;
  const Slots slots{slot, slot ? n_slots : B};
  if (D != 64 && D != 128) return TV_ERR_UNSUPPORTED;
  if (M + 1 > kMaxRows || max_depth + 1 > kMaxRows) return TV_ERR_UNSUPPORTED;
  if (S_cap > 0x7fffffffLL) return TV_ERR_UNSUPPORTED;
  if (!path || !accept_len || !status || !kv_start || !kv_len || !max_len) return TV_ERR_INVALID_ARG;
  if (L > 0 && B > 0 && Hkv > 0 && (!k_layers || !v_layers)) return TV_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t runs = (int64_t)L * 2 * B * Hkv;
  const int64_t extra = (attn_mask || pos_ids) ? B : 0;
  if (runs + extra > 0x7fffffffLL) return TV_ERR_UNSUPPORTED;
  if (runs + extra > 0) {
    const size_t smem = (size_t)(max_depth + 1) * D * 2;
    cudaError_t e = cudaFuncSetAttribute(kv_move_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return record_cuda_error(e);
    tv_status r = launch(kv_move_kernel, dim3((unsigned)(runs + extra)), dim3(kMoveThreads), smem, s, 1, true,
                         k_layers, v_layers, B, Hkv, D, S_cap, M, path, accept_len, (const int32_t*)status, max_depth,
                         (const int32_t*)kv_start, (const int32_t*)kv_len, realign, runs, attn_mask, pos_ids, slots);
    if (r != TV_OK) return r;
  }
  return launch(kv_finalize_kernel, dim3(1), dim3(kPlanThreads), 0, s, 1, true, B, M, S_cap, max_depth,
                realign, path, accept_len, status, kv_start, kv_len, max_len, slots);
}
