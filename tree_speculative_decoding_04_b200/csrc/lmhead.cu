// lmhead.cu -- tree_accept_lm_head: the teacher's LM-head GEMM with the greedy
// argmax fused into its epilogue, then the acceptance walk of tree_accept.
//
// "EAGLE-Pangu: Accelerator-Safe Tree Speculative Decoding on Ascend NPUs",
// methodology C: the teacher evaluates every speculative token in one batched
// pass, and its greedy choice at node u is the argmax of u's logits.  Here the
// logits logit[u][v] = sum_h hidden[u][h] * W[v][h] are formed tile by tile in
// tensor memory and reduced to (max, first index) on the spot, so the
// [rows][V] logits never reach HBM.
//
// Design (one CTA per output tile of 128 rows x bn vocabulary columns, bn = 256
// or, for grids of a few waves, the multiple of 32 that fills the SMs best;
// rows = B * (M+1) tree nodes, H the hidden size):
//   warp 0      TMA producer: per 64-wide K slab, the hidden tile (128 x 64,
//               16 KB) and the weight tile (bn x 64, up to 32 KB), both K-major
//               with the 128-byte swizzle, into a 4-stage ring
//   warp 1      TMEM owner (256 columns) and MMA issuer: 4 x tcgen05.mma
//               (M=128, N=bn, K=16) per slab, fp32 accumulation in TMEM
//   warps 2-5   epilogue: thread t owns TMEM lane t (= tile row t); it reads its
//               bn logits 32 at a time and keeps the first maximum, then merges
//               (max, index) into the row's 64-bit key with one atomicMax: the
//               key orders by value first and by lower index second, so the
//               merge over the vocabulary tiles keeps the first maximum.
// Tiles are numbered row tile fastest, so the CTAs that share a weight tile run
// side by side and read it from HBM once (the hidden rows stay in L2).
#include <algorithm>

#include "attention_common.cuh"  // tensor-map encoder
#include "tcgen05.cuh"

namespace tv {
namespace {

constexpr int kLmThreads = 192;
constexpr int kBM = 128;  // rows per tile (TMEM lanes)
constexpr int kBN = 256;  // most vocabulary columns per tile (TMEM columns)
constexpr int kBK = 64;   // K slab: 128 bytes of bf16, one swizzle row
constexpr int kLmStages = 4;
constexpr int kABytes = kBM * kBK * 2;  // 16 KB
constexpr int kBBytes = kBN * kBK * 2;  // 32 KB
constexpr int kLmStageBytes = kABytes + kBBytes;

struct LmSmem {
  uint64_t full[kLmStages];
  uint64_t empty[kLmStages];
  uint64_t acc;    // the last MMA of the tile has completed
  uint64_t drain;  // every MMA issued has completed (before TMEM is freed)
  uint32_t tmem_base;
  int timed_out;
};

// float -> unsigned with the same order (finite values and infinities)
__device__ __forceinline__ uint32_t ordered_bits(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(kLmThreads) lm_keys_init_kernel(unsigned long long* keys, int64_t rows) {
  pdl_wait_primary();
  pdl_launch_dependents();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < rows; i += (int64_t)gridDim.x * blockDim.x)
    keys[i] = 0ull;  // below every real key
}

__global__ void __launch_bounds__(kLmThreads, 1) lm_head_argmax_kernel(
    const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b, int rows, int H, int V,
    int m_tiles, int bn, int node_rows, unsigned long long* __restrict__ keys, int32_t* __restrict__ status,
    uint64_t lim) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const bool aligned_ok = (smem_u32(smem) & 1023u) == 0;
  LmSmem* sh = reinterpret_cast<LmSmem*>(smem + kLmStages * kLmStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x;
  const int row0 = (tile % m_tiles) * kBM;
  const int col0 = (tile / m_tiles) * bn;
  const int nk = H / kBK;

  if (threadIdx.x == 0) {
    sh->timed_out = aligned_ok ? 0 : 1;
    for (int s = 0; s < kLmStages; ++s) {
      mbar_init(&sh->full[s], 1);
      mbar_init(&sh->empty[s], 1);
    }
    mbar_init(&sh->acc, 1);
    mbar_init(&sh->drain, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tma_a);
    prefetch_tensormap(&tma_b);
  }
  if (warp == 1) {
    __syncwarp();  // tcgen05.alloc is warp-collective
    tmem_alloc(&sh->tmem_base, kBN);
    tmem_relinquish();
  }
  pdl_wait_primary();  // the hidden states and the cleared keys are ready
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  const bool run = aligned_ok;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0 && run) {
      int issued = 0;
      bool to = false;
      for (int kt = 0; kt < nk; ++kt) {
        const int s = kt % kLmStages;
        if (kt >= kLmStages && !mbar_wait(&sh->empty[s], ((kt / kLmStages) - 1) & 1, lim)) {
          to = true;
          break;
        }
        uint8_t* a = smem + s * kLmStageBytes;
        mbar_arrive_expect_tx(&sh->full[s], kABytes + bn * kBK * 2);
        tma_load_2d(a, &tma_a, &sh->full[s], kt * kBK, row0);
        tma_load_2d(a + kABytes, &tma_b, &sh->full[s], kt * kBK, col0);
        ++issued;
      }
      if (to) atomicExch(&sh->timed_out, 1);
      // every copy issued lands before the CTA's shared memory is released
      for (int i = max(0, issued - kLmStages); i < issued; ++i)
        mbar_wait(&sh->full[i % kLmStages], (i / kLmStages) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0 && run) {
      const uint32_t idesc = idesc_bf16(kBM, bn, 0);
      bool to = false;
      for (int kt = 0; kt < nk; ++kt) {
        const int s = kt % kLmStages;
        if (!mbar_wait(&sh->full[s], (kt / kLmStages) & 1, lim)) {
          to = true;
          break;
        }
        tc_fence_after();
        const uint32_t a = smem_u32(smem + s * kLmStageBytes);
        const uint32_t b = a + kABytes;
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k)
          mma_ss(tmem, sw128_desc(a + k * 32, 16), sw128_desc(b + k * 32, 16), idesc, (kt > 0 || k > 0) ? 1u : 0u);
        tc_commit(&sh->empty[s]);
      }
      if (to) atomicExch(&sh->timed_out, 1);
      tc_commit(&sh->acc);
      // every MMA retires before TMEM and shared memory are released
      tc_commit(&sh->drain);
      mbar_wait(&sh->drain, 0);
    }
  } else {
    // ---------------------------------------------------------------- epilogue: row argmax
    const int r = (warp & 3) * 32 + lane;  // TMEM lane == tile row
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    // decided for the whole warp: tcgen05.ld is warp-collective
    const bool ready = run && __all_sync(0xffffffffu, mbar_wait(&sh->acc, 0, lim));
    tc_fence_after();
    const int grow = row0 + r;
    if (ready && !*(volatile int*)&sh->timed_out) {
      float best = -INFINITY;
      int bi = -1;
#pragma unroll 1
      for (int c = 0; c < bn / 32; ++c) {
        uint32_t x[32];
        tmem_ld32(tmem + lane_off + c * 32, x);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int col = col0 + c * 32 + j;
          const float v = __uint_as_float(x[j]);
          if (col < V && (bi < 0 || v > best)) {  // strict: the first maximum stays
            best = v;
            bi = col;
          }
        }
      }
      if (grow < rows && bi >= 0)
        atomicMax(keys + grow,
                  ((unsigned long long)ordered_bits(best) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)bi));
    } else if (!ready) {
      atomicExch(&sh->timed_out, 1);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();  // tcgen05.dealloc is warp-collective
    tc_fence_after();
    tmem_dealloc(tmem, kBN);
  }
  // a tile that gave up marks the sequences of its real rows
  if (sh->timed_out && threadIdx.x < kBM && row0 + (int)threadIdx.x < rows)
    atomicOr(&status[(row0 + threadIdx.x) / node_rows], kSeqTimeout);
}

// key -> argmax index (the key was built from (value, 0xFFFFFFFF - index))
__global__ void __launch_bounds__(256) lm_keys_decode_kernel(const unsigned long long* __restrict__ keys,
                                                             int32_t* __restrict__ argmax, int64_t rows) {
  pdl_wait_primary();
  pdl_launch_dependents();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < rows; i += (int64_t)gridDim.x * blockDim.x) {
    const unsigned long long k = keys[i];
    argmax[i] = k == 0ull ? 0 : (int32_t)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFull));
  }
}

// [outer][inner] bf16, K-major, boxes of 64 (128 bytes) x box_rows, 128-byte swizzle
bool encode_kmajor_map(CUtensorMap* map, const void* base, int64_t outer, int inner, int box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  cuuint64_t strides[1] = {(cuuint64_t)inner * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace
}  // namespace tv

extern "C" size_t tree_accept_lm_head_workspace_size(int B, int M) {
  if (B <= 0 || M < 0 || M + 1 > TV_MAX_TREE_ROWS) return 0;
  return (size_t)B * (M + 1) * sizeof(unsigned long long);
}

extern "C" tv_status tree_accept_lm_head(const uint16_t* hidden, const uint16_t* w_lm, const int32_t* draft,
                                         const int32_t* parent, const int32_t* depth, const uint32_t* anc_mask,
                                         int32_t* status, int B, int M, int H, int V, int max_depth,
                                         int32_t* argmax, int32_t* accept_len, int32_t* path, int32_t* bonus,
                                         void* workspace, size_t workspace_bytes, tv_stream_t stream) {
  using namespace tv;
  if (B < 0 || M < 0 || H < 1 || V < 1 || max_depth < 0) return TV_ERR_INVALID_ARG;
  if (M + 1 > kMaxRows) return TV_ERR_UNSUPPORTED;
  if (H % kBK != 0) return TV_ERR_UNSUPPORTED;  // whole 64-wide K slabs
  if (B == 0) return TV_OK;
  if (!hidden || !w_lm || !draft || !parent || !depth || !anc_mask || !status || !argmax || !accept_len || !path ||
      !bonus || !workspace)
    return TV_ERR_INVALID_ARG;
  if (!aligned16(hidden) || !aligned16(w_lm) || (reinterpret_cast<uintptr_t>(workspace) & 7u) != 0)
    return TV_ERR_INVALID_ARG;
  const int64_t rows = (int64_t)B * (M + 1);
  if (workspace_bytes < (size_t)rows * sizeof(unsigned long long)) return TV_ERR_INVALID_ARG;
  const int m_tiles = (int)((rows + kBM - 1) / kBM);
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda_error(e);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // Tile width: 256 columns, unless the grid is a few waves of one CTA per SM
  // (few rows: the weights stream at the SMs' pull rate); then the multiple of
  // 32 in [128, 256] with the fewest waves x columns, so that the last wave is
  // not left mostly empty (V = 32000: 125 tiles of 256 leave 23 of 148 SMs
  // idle, 143 tiles of 224 leave 5).
  int bn = kBN;
  if ((int64_t)m_tiles * (((int64_t)V + kBN - 1) / kBN) <= 8LL * sms) {
    int64_t best = -1;
    for (int cand = kBN; cand >= 128; cand -= 32) {
      const int64_t tiles = (int64_t)m_tiles * (((int64_t)V + cand - 1) / cand);
      const int64_t cost = (tiles + sms - 1) / sms * cand;
      if (best < 0 || cost < best) {
        best = cost;
        bn = cand;
      }
    }
  }
  const int64_t n_tiles = ((int64_t)V + bn - 1) / bn;
  if ((int64_t)m_tiles * n_tiles > 0x7fffffffLL) return TV_ERR_UNSUPPORTED;
  CUtensorMap ta, tb;
  if (!encode_kmajor_map(&ta, hidden, rows, H, kBM) || !encode_kmajor_map(&tb, w_lm, V, H, bn))
    return TV_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned long long* keys = static_cast<unsigned long long*>(workspace);
  const unsigned small_grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>((rows + 255) / 256, sms));
  tv_status r = launch(lm_keys_init_kernel, dim3(small_grid), dim3(kLmThreads), 0, s, 1, true, keys, rows);
  if (r != TV_OK) return r;
  const size_t smem = (size_t)kLmStages * kLmStageBytes + sizeof(LmSmem);
  e = cudaFuncSetAttribute(lm_head_argmax_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return record_cuda_error(e);
  r = launch(lm_head_argmax_kernel, dim3((unsigned)(m_tiles * n_tiles)), dim3(kLmThreads), smem, s, 1, true, ta, tb,
             (int)rows, H, V, m_tiles, bn, M + 1, keys, status, pipeline_wait_limit_ns());
  if (r != TV_OK) return r;
  r = launch(lm_keys_decode_kernel, dim3(small_grid), dim3(256), 0, s, 1, true, (const unsigned long long*)keys,
             argmax, rows);
  if (r != TV_OK) return r;
  return launch_accept_walk(argmax, draft, parent, depth, anc_mask, status, B, M, max_depth, accept_len, path, bonus,
                            s);
}
