// mask.cu -- tree_build_mask: validate sentinel-free parent arrays and expand
// them into ancestor bitmasks.
//
// "EAGLE-Pangu: Accelerator-Safe Tree Speculative Decoding on Ascend NPUs",
// methodology B: a dummy root at row 0, every parent pointer inside [0, M], and
// cheap structural checks (range, acyclicity) before the fused kernels run;
// methodology C: node k may attend node j only if j is an ancestor of k.
//
// Both kernels use pointer jumping: every row u keeps (mask of the path u..nxt,
// edge count u..nxt, nxt) and repeatedly absorbs the record of nxt, so a tree of
// depth d is finished in ceil(log2(d)) + 1 rounds instead of d serial steps.
// Trees of at most 32 rows live in one warp's registers (shuffles + ballots);
// larger ones (up to 256 rows, 8 mask words) use one CTA and shared memory.
#include "tv_common.cuh"

namespace tv {
namespace {

constexpr unsigned kFull = 0xffffffffu;

// One warp per tree, M + 1 <= 32 (one mask word per row).
__global__ void __launch_bounds__(128) tb_mask_warp_kernel(const int32_t* __restrict__ parent, int B, int M,
                                                           int max_depth, uint32_t* __restrict__ anc,
                                                           int32_t* __restrict__ depth,
                                                           int32_t* __restrict__ status) {
  pdl_wait_primary();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (b >= B) return;  // warp-uniform
  const int n = M + 1;
  const bool in = lane < n;
  const int p = in ? parent[(int64_t)b * n + lane] : 0;
  const bool bad = in && (lane == 0 ? p != 0 : (p < 0 || p >= lane));
  int st = __ballot_sync(kFull, bad) ? kSeqBadParent : 0;
  uint32_t m = 0;
  int d = 0;
  if (!st) {
    int nx = p;  // lanes >= n hold 0 and point at the root
    m = in ? ((1u << lane) | (1u << p)) : 0u;
    d = (in && lane != 0) ? 1 : 0;
    // parent[i] < i guarantees termination after at most 6 rounds
    while (__any_sync(kFull, nx != 0)) {
      const uint32_t m2 = __shfl_sync(kFull, m, nx);
      const int d2 = __shfl_sync(kFull, d, nx);
      const int n2 = __shfl_sync(kFull, nx, nx);
      m |= m2;
      d += d2;
      nx = n2;
    }
    if (__ballot_sync(kFull, in && d > max_depth)) st = kSeqTooDeep;
  }
  if (st) {
    m = 0;
    d = 0;
  }
  if (in) {
    anc[(int64_t)b * n + lane] = m;
    depth[(int64_t)b * n + lane] = d;
  }
  if (lane == 0) status[b] = st;
}

// One CTA per tree, 32 < M + 1 <= 256; blockDim = 32 * ceil((M+1)/32).
__global__ void __launch_bounds__(kMaxRows) tb_mask_block_kernel(const int32_t* __restrict__ parent, int M,
                                                                 int max_depth, uint32_t* __restrict__ anc,
                                                                 int32_t* __restrict__ depth,
                                                                 int32_t* __restrict__ status) {
  __shared__ uint32_t msk[2][kMaxRows][kMaxRows / 32];
  __shared__ int nxt[2][kMaxRows];
  __shared__ int dep[2][kMaxRows];
  pdl_wait_primary();
  pdl_launch_dependents();
  const int b = blockIdx.x;
  const int u = threadIdx.x;
  const int n = M + 1;
  const int W = (n + 31) >> 5;
  const bool in = u < n;
  const int p = in ? parent[(int64_t)b * n + u] : 0;
  const bool bad = in && (u == 0 ? p != 0 : (p < 0 || p >= u));
  uint32_t* anc_row = anc + ((int64_t)b * n + u) * W;
  if (__syncthreads_or(bad)) {
    if (in) {
      for (int w = 0; w < W; ++w) anc_row[w] = 0u;
      depth[(int64_t)b * n + u] = 0;
    }
    if (u == 0) status[b] = kSeqBadParent;
    return;  // block-uniform
  }
  nxt[0][u] = p;
  dep[0][u] = (in && u != 0) ? 1 : 0;
  for (int w = 0; w < W; ++w) {
    uint32_t x = 0;
    if (in) {
      if ((u >> 5) == w) x |= 1u << (u & 31);
      if ((p >> 5) == w) x |= 1u << (p & 31);
    }
    msk[0][u][w] = x;
  }
  __syncthreads();
  int cur = 0;
  for (;;) {
    const int j = nxt[cur][u];
    for (int w = 0; w < W; ++w) msk[cur ^ 1][u][w] = msk[cur][u][w] | msk[cur][j][w];
    dep[cur ^ 1][u] = dep[cur][u] + dep[cur][j];
    const int nj = nxt[cur][j];
    nxt[cur ^ 1][u] = nj;
    cur ^= 1;
    if (!__syncthreads_or(nj != 0)) break;
  }
  const int d = dep[cur][u];
  const bool deep = __syncthreads_or(in && d > max_depth);
  if (in) {
    for (int w = 0; w < W; ++w) anc_row[w] = deep ? 0u : msk[cur][u][w];
    depth[(int64_t)b * n + u] = deep ? 0 : d;
  }
  if (u == 0) status[b] = deep ? kSeqTooDeep : 0;
}

}  // namespace
}  // namespace tv

extern "C" tv_status tree_build_mask(const int32_t* parent, int B, int M, int max_depth, uint32_t* anc_mask,
                                     int32_t* depth, int32_t* status, tv_stream_t stream) {
  using namespace tv;
  if (B < 0 || M < 0 || max_depth < 0) return TV_ERR_INVALID_ARG;
  if (M + 1 > kMaxRows) return TV_ERR_UNSUPPORTED;
  if (B == 0) return TV_OK;
  if (!parent || !anc_mask || !depth || !status) return TV_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (M + 1 <= 32) {
    const int warps = 4;
    return launch(tb_mask_warp_kernel, dim3((B + warps - 1) / warps), dim3(32 * warps), 0, s, 1, true, parent, B,
                  M, max_depth, anc_mask, depth, status);
  }
  const int threads = 32 * ((M + 1 + 31) / 32);
  return launch(tb_mask_block_kernel, dim3(B), dim3(threads), 0, s, 1, true, parent, M, max_depth, anc_mask, depth,
                status);
}
