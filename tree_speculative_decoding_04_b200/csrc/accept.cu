// accept.cu -- tree_accept: per-node greedy argmax over the teacher logits,
// fused with the selection of the longest accepted root-to-node path.
//
// "EAGLE-Pangu: Accelerator-Safe Tree Speculative Decoding on Ascend NPUs",
// results section: the accepted length of one verification step is the number
// of speculative tokens on which the teacher's greedy choice agrees.  For a
// tree: node i is accepted iff its parent is accepted and its draft token is
// the teacher's argmax at the parent; the deepest accepted node (lowest row on
// ties) is committed and the teacher's argmax there is the bonus token.
//
// Kernel 1 streams the logits once (HBM-bound): each row is split over a
// thread-block cluster of up to 8 CTAs, every thread issues independent 16-byte
// loads, (value, index) pairs are reduced with warp shuffles and the CTAs of a
// cluster merge through distributed shared memory -- no global scratch.
// Kernel 2 (one CTA per sequence, launched as a programmatic dependent of
// kernel 1) turns the argmax rows into the accepted set with one ballot per 32
// rows and the ancestor bitmask (accepted == every ancestor matched), then picks
// the endpoint with a block max-reduction and writes the path.
#include <cooperative_groups.h>

#include <algorithm>
#include <climits>

#include "tv_common.cuh"

namespace cg = cooperative_groups;

namespace tv {
namespace {

constexpr int kArgmaxThreads = 256;
constexpr int kUnroll = 4;

struct Best {
  float v;
  int i;
};

// (value desc, index asc): true if (v2, i2) beats (v1, i1)
__device__ __forceinline__ bool better(float v2, int i2, float v1, int i1) {
  return v2 > v1 || (v2 == v1 && i2 < i1);
}

__device__ __forceinline__ void take(Best& b, float v, int i) {
  if (better(v, i, b.v, b.i)) {
    b.v = v;
    b.i = i;
  }
}

__device__ __forceinline__ Best warp_best(Best b) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float v2 = __shfl_xor_sync(0xffffffffu, b.v, off);
    const int i2 = __shfl_xor_sync(0xffffffffu, b.i, off);
    take(b, v2, i2);
  }
  return b;
}

// grid.x = rows * nsplit, cluster (nsplit, 1, 1); CTA s of a cluster scans
// columns [s * chunk, min(V, (s + 1) * chunk)) of row blockIdx.x / nsplit.
__global__ void __launch_bounds__(kArgmaxThreads) accept_argmax_kernel(const float* __restrict__ logits, int V,
                                                                       int chunk, int nsplit,
                                                                       int32_t* __restrict__ argmax_out) {
  pdl_wait_primary();
  pdl_launch_dependents();
  __shared__ Best warp_res[kArgmaxThreads / 32];
  __shared__ Best cta_res;
  const int64_t row = blockIdx.x / nsplit;
  const int s = blockIdx.x % nsplit;
  const int lo = s * chunk;
  const int hi = min(V, lo + chunk);
  const float* x = logits + row * (int64_t)V;
  Best best{-INFINITY, INT_MAX};
  if (lo < hi) {
    // scalar head up to a 16-byte boundary, then float4 body, then scalar tail
    const int mis = (int)((reinterpret_cast<uintptr_t>(x + lo) >> 2) & 3);  // floats past a 16-byte boundary
    int a0 = lo + ((4 - mis) & 3);
    if (a0 > hi) a0 = hi;
    const int nvec = (hi - a0) >> 2;
    const int a1 = a0 + 4 * nvec;
    for (int i = lo + threadIdx.x; i < a0; i += kArgmaxThreads) take(best, __ldcs(x + i), i);
    const float4* xv = reinterpret_cast<const float4*>(x + a0);
    int j = threadIdx.x;
    for (; j + (kUnroll - 1) * kArgmaxThreads < nvec; j += kUnroll * kArgmaxThreads) {
      float4 r[kUnroll];
#pragma unroll
      for (int t = 0; t < kUnroll; ++t) r[t] = __ldcs(xv + j + t * kArgmaxThreads);
#pragma unroll
      for (int t = 0; t < kUnroll; ++t) {
        const int base = a0 + 4 * (j + t * kArgmaxThreads);
        take(best, r[t].x, base);
        take(best, r[t].y, base + 1);
        take(best, r[t].z, base + 2);
        take(best, r[t].w, base + 3);
      }
    }
    for (; j < nvec; j += kArgmaxThreads) {
      const float4 r = __ldcs(xv + j);
      const int base = a0 + 4 * j;
      take(best, r.x, base);
      take(best, r.y, base + 1);
      take(best, r.z, base + 2);
      take(best, r.w, base + 3);
    }
    for (int i = a1 + threadIdx.x; i < hi; i += kArgmaxThreads) take(best, __ldcs(x + i), i);
  }
  best = warp_best(best);
  if ((threadIdx.x & 31) == 0) warp_res[threadIdx.x >> 5] = best;
  __syncthreads();
  if (threadIdx.x < 32) {
    Best b = threadIdx.x < kArgmaxThreads / 32 ? warp_res[threadIdx.x] : Best{-INFINITY, INT_MAX};
    b = warp_best(b);
    if (threadIdx.x == 0) cta_res = b;
  }
  if (nsplit == 1) {
    __syncthreads();
    if (threadIdx.x == 0) argmax_out[row] = cta_res.i == INT_MAX ? 0 : cta_res.i;
    return;
  }
  cg::cluster_group cluster = cg::this_cluster();
  cluster.sync();
  if (cluster.block_rank() == 0 && threadIdx.x < 32) {
    Best b{-INFINITY, INT_MAX};
    if ((int)threadIdx.x < nsplit) b = *cluster.map_shared_rank(&cta_res, (unsigned)threadIdx.x);
    b = warp_best(b);
    if (threadIdx.x == 0) argmax_out[row] = b.i == INT_MAX ? 0 : b.i;
  }
  cluster.sync();  // keep every CTA's shared memory alive until rank 0 has read it
}

// One CTA per sequence, blockDim = 32 * ceil((M+1)/32).
__global__ void __launch_bounds__(kMaxRows) accept_walk_kernel(
    const int32_t* __restrict__ argmax, const int32_t* __restrict__ draft, const int32_t* __restrict__ parent,
    const int32_t* __restrict__ depth, const uint32_t* __restrict__ anc, int32_t* __restrict__ status, int M,
    int max_depth, int32_t* __restrict__ accept_len, int32_t* __restrict__ path, int32_t* __restrict__ bonus) {
  __shared__ uint32_t ok_bits[kMaxRows / 32];
  __shared__ int red[kMaxRows / 32];
  __shared__ uint32_t e_row[kMaxRows / 32];
  const int b = blockIdx.x;
  const int u = threadIdx.x;
  const int n = M + 1;
  const int W = (n + 31) >> 5;
  const int64_t rbase = (int64_t)b * n;
  int32_t* pth = path + (int64_t)b * (max_depth + 1);

  // parent, depth and draft are written by no kernel of the step after
  // tree_build_mask, and the argmax kernel triggers this launch only after its
  // own wait returned, so they may be read before waiting on it.  status may
  // still gain a bit from the attention launches, so it is read after the wait.
  pdl_launch_dependents();
  const bool in = u < n;
  const int p = in ? parent[rbase + u] : 0;
  const int dp = in ? depth[rbase + u] : 0;
  const int dr = in ? draft[rbase + u] : 0;
  const bool bad_par = in && (u == 0 ? p != 0 : (p < 0 || p >= u));
  const bool bad_dep = in && (dp < 0 || dp > max_depth || dp > M || (u == 0 && dp != 0));
  const int flag = (__syncthreads_or(bad_par) ? kSeqBadParent : 0) | (__syncthreads_or(bad_dep) ? kSeqTooDeep : 0);
  pdl_wait_primary();
  const int st0 = status[b];
  if (st0 != 0 || flag != 0) {
    for (int j = u; j <= max_depth; j += blockDim.x) pth[j] = 0;
    if (u == 0) {
      accept_len[b] = -1;
      bonus[b] = 0;
      if (flag) status[b] = st0 | flag;
    }
    return;
  }
  const bool ok = in && (u == 0 || dr == argmax[rbase + p]);
  const uint32_t ballot = __ballot_sync(0xffffffffu, ok);
  if ((u & 31) == 0) ok_bits[u >> 5] = ballot;
  __syncthreads();
  // accepted iff every ancestor (itself included) matched its parent's argmax
  bool acc = in;
  if (in) {
    const uint32_t* a = anc + (rbase + u) * W;
    for (int w = 0; w < W; ++w) acc = acc && ((a[w] & ~ok_bits[w]) == 0u);
  }
  // deepest accepted row, lowest index on ties: maximise (depth, -row)
  int key = acc ? ((dp << 16) | (0xffff - u)) : -1;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) key = max(key, __shfl_xor_sync(0xffffffffu, key, off));
  if ((u & 31) == 0) red[u >> 5] = key;
  __syncthreads();
  if (u < 32) {
    int k2 = u < (int)(blockDim.x >> 5) ? red[u] : -1;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) k2 = max(k2, __shfl_xor_sync(0xffffffffu, k2, off));
    if (u == 0) red[0] = k2;
  }
  __syncthreads();
  const int best = red[0];  // the root is always accepted, so best >= 0
  const int e = 0xffff - (best & 0xffff);
  const int de = best >> 16;
  if (u < W) e_row[u] = anc[(rbase + e) * W + u];
  __syncthreads();
  if (in && ((e_row[u >> 5] >> (u & 31)) & 1u)) pth[dp] = u;
  for (int j = de + 1 + u; j <= max_depth; j += blockDim.x) pth[j] = 0;
  if (u == 0) {
    accept_len[b] = de;
    bonus[b] = argmax[rbase + e];
  }
}

}  // namespace

tv_status launch_accept_walk(const int32_t* argmax, const int32_t* draft, const int32_t* parent,
                             const int32_t* depth, const uint32_t* anc_mask, int32_t* status, int B, int M,
                             int max_depth, int32_t* accept_len, int32_t* path, int32_t* bonus, cudaStream_t s) {
  const int threads = 32 * ((M + 1 + 31) / 32);
  return launch(accept_walk_kernel, dim3(B), dim3(threads), 0, s, 1, true, argmax, draft, parent, depth, anc_mask,
                status, M, max_depth, accept_len, path, bonus);
}

}  // namespace tv

extern "C" tv_status tree_accept(const float* logits, const int32_t* draft, const int32_t* parent,
                                 const int32_t* depth, const uint32_t* anc_mask, int32_t* status, int B, int M,
                                 int V, int max_depth, int32_t* argmax, int32_t* accept_len, int32_t* path,
                                 int32_t* bonus, tv_stream_t stream) {
  using namespace tv;
  if (B < 0 || M < 0 || V < 1 || max_depth < 0) return TV_ERR_INVALID_ARG;
  if (M + 1 > kMaxRows) return TV_ERR_UNSUPPORTED;
  if (B == 0) return TV_OK;
  if (!logits || !draft || !parent || !depth || !anc_mask || !status || !argmax || !accept_len || !path || !bonus)
    return TV_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(logits) & 3u) != 0) return TV_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t rows = (int64_t)B * (M + 1);
  // Split each row over a cluster until the grid covers the GPU about four
  // times, keeping every CTA at >= 2048 columns.
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t target = 4LL * sms;
  int nsplit = (int)std::min<int64_t>(8, std::max<int64_t>(1, (target + rows - 1) / rows));
  nsplit = std::min(nsplit, std::max(1, (V + 2047) / 2048));
  int chunk = (V + nsplit - 1) / nsplit;
  chunk = (chunk + 3) & ~3;
  nsplit = (V + chunk - 1) / chunk;
  if (rows * nsplit > 0x7fffffffLL) return TV_ERR_UNSUPPORTED;
  tv_status r = launch(accept_argmax_kernel, dim3((unsigned)(rows * nsplit)), dim3(kArgmaxThreads), 0, s, nsplit,
                       true, logits, V, chunk, nsplit, argmax);
  if (r != TV_OK) return r;
  return launch_accept_walk(argmax, draft, parent, depth, anc_mask, status, B, M, max_depth, accept_len, path,
                            bonus, s);
}
