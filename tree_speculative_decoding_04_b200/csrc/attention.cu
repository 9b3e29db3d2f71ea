// attention.cu -- tree_attention: tree-masked GQA attention of the M+1 tree
// queries of every sequence over its committed KV prefix and its tree rows.
//
// "EAGLE-Pangu: Accelerator-Safe Tree Speculative Decoding on Ascend NPUs",
// methodology C: all speculative tokens are verified in one batched teacher
// pass; a 4D tree mask lets node k attend node j only if j is an ancestor of k.
// Here the mask is never materialised: prefix keys are unmasked and the tree
// block (the last M+1 key columns) is masked from the ancestor bitmask.
//
// Decomposition (split-KV flash decoding).  A CTA owns one (sequence, kv head,
// query tile, key split).  The query tile stacks (node, q head of the group)
// rows, 16 per consumer warp, so the K/V tiles a CTA streams from HBM are
// shared by every q head of the GQA group and every tree node.  One producer
// warp streams 64-key K and V tiles with TMA (128-byte swizzle, no multicast)
// into a ring of shared-memory stages guarded by mbarriers; the consumer warps
// run bf16 mma.sync (fp32 accumulate) for S = Q K^T and O += P V with an online
// softmax in registers.  The key splits of one query tile form a thread-block
// cluster and merge their partial (max, sum, O) through distributed shared
// memory, so no partial result touches global memory.
#include <cooperative_groups.h>

#include <algorithm>
#include <mutex>

#include "attention_common.cuh"

namespace cg = cooperative_groups;

namespace tv {
namespace {

constexpr int KT = kKeyTile;
constexpr int kMaxCWarps = 8;   // consumer warps per CTA (16 query rows each)
constexpr int kMaxSplit = 8;    // portable cluster size



__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Byte offset of 16-byte chunk c (of D/8) in row r of a tile stored as D/64
// TMA boxes of [64 rows][128 B] with the 128-byte swizzle.
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return (uint32_t)((c >> 3) * kBoxBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__((kMaxCWarps + 1) * 32) tree_attn_mma_kernel(const __grid_constant__ CUtensorMap tmk,
                                                                         const __grid_constant__ CUtensorMap tmv,
                                                                         const __grid_constant__ AttnParams p) {
  constexpr int kTileBytes = KT * D * 2;
  constexpr int kStageBytes = 2 * kTileBytes;
  constexpr int KS = D / 16;  // k-steps of the QK^T product
  constexpr int DT = D / 8;   // n8 tiles of the output

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int stages = p.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)stages * kStageBytes);
  uint64_t* empty = full + stages;
  float* m_st = reinterpret_cast<float*>(empty + stages);  // [RT] row max (log2 domain)
  float* l_st = m_st + kMaxCWarps * 16;                     // [RT] row sum
  __shared__ int timed_out;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ncw = (blockDim.x >> 5) - 1;  // consumer warps
  const int RT = ncw * 16;
  const int split = blockIdx.x;
  const int qtile = blockIdx.y;
  const int bh = blockIdx.z;
  const int b = bh / p.Hkv;
  const int hk = bh - b * p.Hkv;

  if (threadIdx.x == 0) {
    timed_out = 0;
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], ncw);
    }
    fence_mbar_init();
  }
  if (warp == ncw && lane == 0) {
    prefetch_tensormap(&tmk);
    prefetch_tensormap(&tmv);
  }
  // everything above overlaps the previous kernel; inputs are read below
  pdl_wait_primary();
  pdl_launch_dependents();
  __syncthreads();

  const int sl = cache_slot(p.slot, b, p.n_slots);  // cache slot of this batch row
  const int32_t ks = sl >= 0 ? p.kv_start[sl] : 0;
  const int32_t kl = sl >= 0 ? p.kv_len[sl] : 0;
  const bool valid = sl >= 0 && p.status[b] == 0 && geometry_ok(ks, kl, p.M, p.S_cap);
  const int zc = sl * p.Hkv + hk;  // tensor-map row block of this (slot, kv head)
  const int N = kl + p.M + 1;  // keys of this sequence
  const int t0 = split * p.tiles_per_split;
  const int ntiles = valid ? max(0, min(p.tiles_per_split, (N + KT - 1) / KT - t0)) : 0;
  const int k_lo = t0 * KT;

  if (warp == ncw) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && ntiles > 0) {
      int issued = 0;
      bool to = false;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % stages;
        if (i >= stages && !mbar_wait(&empty[s], ((i / stages) - 1) & 1)) {
          to = true;
          break;
        }
        mbar_arrive_expect_tx(&full[s], kStageBytes);
        const int col = ks + k_lo + i * KT;
        uint8_t* kt = smem + (size_t)s * kStageBytes;
#pragma unroll
        for (int bx = 0; bx < D / 64; ++bx) {
          tma_load_3d(kt + bx * kBoxBytes, &tmk, &full[s], bx * 64, col, zc);
          tma_load_3d(kt + kTileBytes + bx * kBoxBytes, &tmv, &full[s], bx * 64, col, zc);
        }
        ++issued;
      }
      if (to) atomicExch(&timed_out, 1);
      // on a timeout, wait (bounded) for the copies still in flight before leaving
      if (to || *(volatile int*)&timed_out) {
        for (int i = max(0, issued - stages); i < issued; ++i) mbar_wait(&full[i % stages], (i / stages) & 1);
      }
    }
  }

  // ------------------------------------------------------------ consumers
  float o[DT][4];
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
#pragma unroll
  for (int dt = 0; dt < DT; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
  const int g = lane >> 2, c4 = lane & 3;
  const int rl0 = warp * 16 + g;  // local rows of this thread: rl0 and rl0 + 8
  const int gr0 = qtile * RT + rl0, gr1 = gr0 + 8;
  const int u0 = min(gr0 / p.G, p.M), u1 = min(gr1 / p.G, p.M);

  if (warp < ncw) {
    // Q fragments (A operand, row-major 16 x D) straight from global memory
    uint32_t qa[KS][4];
    {
      const int h0 = hk * p.G + gr0 % p.G, h1 = hk * p.G + gr1 % p.G;
      const uint32_t* q0 = reinterpret_cast<const uint32_t*>(p.q + (((int64_t)b * (p.M + 1) + u0) * p.Hq + h0) * D);
      const uint32_t* q1 = reinterpret_cast<const uint32_t*>(p.q + (((int64_t)b * (p.M + 1) + u1) * p.Hq + h1) * D);
      const bool r0ok = gr0 < p.rows_total, r1ok = gr1 < p.rows_total;
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        qa[k][0] = r0ok ? __ldg(q0 + k * 8 + c4) : 0u;
        qa[k][1] = r1ok ? __ldg(q1 + k * 8 + c4) : 0u;
        qa[k][2] = r0ok ? __ldg(q0 + k * 8 + 4 + c4) : 0u;
        qa[k][3] = r1ok ? __ldg(q1 + k * 8 + 4 + c4) : 0u;
      }
    }
    const uint32_t* anc0 = p.anc + ((int64_t)b * (p.M + 1) + u0) * p.W;
    const uint32_t* anc1 = p.anc + ((int64_t)b * (p.M + 1) + u1) * p.W;
    const uint32_t sbase = smem_u32(smem);
    for (int i = 0; i < ntiles; ++i) {
      const int s = i % stages;
      // decided for the whole warp: the ldmatrix / mma.sync below are warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (i / stages) & 1))) {
        atomicExch(&timed_out, 1);
        break;
      }
      const uint32_t kt = sbase + (uint32_t)(s * kStageBytes);
      const uint32_t vt = kt + kTileBytes;
      const int key0 = k_lo + i * KT;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int kb = key0 + half * 32;
        float sc[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.f;
#pragma unroll
        for (int kp = 0; kp < KS / 2; ++kp) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4(kt + swz(half * 32 + 8 * j + (lane & 7), 4 * kp + (lane >> 3)), b0, b1, b2, b3);
            mma_bf16(sc[j], qa[2 * kp], b0, b1);
            mma_bf16(sc[j], qa[2 * kp + 1], b2, b3);
          }
        }
        // scale into the log2 domain and apply the tree mask / key-range end
        const bool edge = kb + 32 > kl;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float x = sc[j][e] * p.scale_log2;
            if (edge) {
              const int key = kb + 8 * j + 2 * c4 + (e & 1);
              bool ok = key < kl;
              if (!ok && key < N) {
                const int r = key - kl;
                const uint32_t w = __ldg((e < 2 ? anc0 : anc1) + (r >> 5));
                ok = (w >> (r & 31)) & 1u;
              }
              if (!ok) x = -INFINITY;
            }
            sc[j][e] = x;
          }
        }
        float mx0 = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
        mx0 = fmaxf(mx0, fmaxf(fmaxf(sc[2][0], sc[2][1]), fmaxf(sc[3][0], sc[3][1])));
        float mx1 = fmaxf(fmaxf(sc[0][2], sc[0][3]), fmaxf(sc[1][2], sc[1][3]));
        mx1 = fmaxf(mx1, fmaxf(fmaxf(sc[2][2], sc[2][3]), fmaxf(sc[3][2], sc[3][3])));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float ms0 = mn0 == -INFINITY ? 0.f : mn0, ms1 = mn1 == -INFINITY ? 0.f : mn1;
        const float cr0 = fast_exp2(m0 - ms0), cr1 = fast_exp2(m1 - ms1);
        m0 = mn0;
        m1 = mn1;
        float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          sc[j][0] = fast_exp2(sc[j][0] - ms0);
          sc[j][1] = fast_exp2(sc[j][1] - ms0);
          sc[j][2] = fast_exp2(sc[j][2] - ms1);
          sc[j][3] = fast_exp2(sc[j][3] - ms1);
          rs0 += sc[j][0] + sc[j][1];
          rs1 += sc[j][2] + sc[j][3];
        }
        l0 = l0 * cr0 + rs0;
        l1 = l1 * cr1 + rs1;
#pragma unroll
        for (int dt = 0; dt < DT; ++dt) {
          o[dt][0] *= cr0;
          o[dt][1] *= cr0;
          o[dt][2] *= cr1;
          o[dt][3] *= cr1;
        }
        // P (16 x 32) as two A fragments of 16 keys each
        uint32_t pa[2][4];
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          pa[kk][0] = pack_bf16x2(sc[2 * kk][0], sc[2 * kk][1]);
          pa[kk][1] = pack_bf16x2(sc[2 * kk][2], sc[2 * kk][3]);
          pa[kk][2] = pack_bf16x2(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
          pa[kk][3] = pack_bf16x2(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
        }
        // keys past the end of the range may hold anything: zero their V words
        const int kend = N - kb;  // valid keys in this half: [0, kend)
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const int vrow = half * 32 + 16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8;
          // V fragment key rows held by this thread: 16kk + 2c4 (+1) and +8 (+9)
          const int kr = 16 * kk + 2 * c4;
#pragma unroll
          for (int dp = 0; dp < DT / 2; ++dp) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(vt + swz(vrow, 2 * dp + (lane >> 4)), b0, b1, b2, b3);
            if (kend < 32) {
              const uint32_t lo0 = kr < kend ? 0x0000ffffu : 0u, hi0 = kr + 1 < kend ? 0xffff0000u : 0u;
              const uint32_t lo1 = kr + 8 < kend ? 0x0000ffffu : 0u, hi1 = kr + 9 < kend ? 0xffff0000u : 0u;
              b0 &= lo0 | hi0;
              b1 &= lo1 | hi1;
              b2 &= lo0 | hi0;
              b3 &= lo1 | hi1;
            }
            mma_bf16(o[2 * dp], pa[kk], b0, b1);
            mma_bf16(o[2 * dp + 1], pa[kk], b2, b3);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  }

  const int64_t orow0 = (((int64_t)b * (p.M + 1) + gr0 / p.G) * p.Hq + hk * p.G + gr0 % p.G) * D;
  const int64_t orow1 = (((int64_t)b * (p.M + 1) + gr1 / p.G) * p.Hq + hk * p.G + gr1 % p.G) * D;
  const bool w0 = warp < ncw && gr0 < p.rows_total, w1 = warp < ncw && gr1 < p.rows_total;

  if (p.nsplit == 1) {
    if (warp < ncw) {
      const float i0 = (valid && l0 > 0.f) ? 1.f / l0 : 0.f, i1 = (valid && l1 > 0.f) ? 1.f / l1 : 0.f;
#pragma unroll
      for (int dt = 0; dt < DT; ++dt) {
        const int d = dt * 8 + 2 * c4;
        if (w0) *reinterpret_cast<uint32_t*>(p.out + orow0 + d) = pack_bf16x2(o[dt][0] * i0, o[dt][1] * i0);
        if (w1) *reinterpret_cast<uint32_t*>(p.out + orow1 + d) = pack_bf16x2(o[dt][2] * i1, o[dt][3] * i1);
      }
    }
    __syncthreads();
    if (threadIdx.x == 0 && timed_out) atomicOr(&p.status[b], kSeqTimeout);
    if (threadIdx.x == 0 && sl < 0) atomicOr(&p.status[b], kSeqBadGeometry);
    return;
  }

  // ------------------------------------------------------------ cluster combine
  __syncthreads();  // every warp is done with the stage buffers
  float* ost = reinterpret_cast<float*>(smem);  // [RT][D] unnormalised partial O
  if (warp < ncw) {
#pragma unroll
    for (int dt = 0; dt < DT; ++dt) {
      const int d = dt * 8 + 2 * c4;
      *reinterpret_cast<float2*>(ost + rl0 * D + d) = make_float2(o[dt][0], o[dt][1]);
      *reinterpret_cast<float2*>(ost + (rl0 + 8) * D + d) = make_float2(o[dt][2], o[dt][3]);
    }
    if (c4 == 0) {
      m_st[rl0] = m0;
      m_st[rl0 + 8] = m1;
      l_st[rl0] = l0;
      l_st[rl0 + 8] = l1;
    }
  }
  cg::cluster_group cluster = cg::this_cluster();
  cluster.sync();
  const int ns = p.nsplit;
  const int rank = (int)cluster.block_rank();
  const int r_lo = rank * RT / ns, r_hi = (rank + 1) * RT / ns;
  const int per_row = D / 4;
  for (int idx = threadIdx.x; idx < (r_hi - r_lo) * per_row; idx += blockDim.x) {
    const int rl = r_lo + idx / per_row;
    const int d = (idx % per_row) * 4;
    const int gr = qtile * RT + rl;
    if (gr >= p.rows_total) continue;
    float mmax = -INFINITY;
    for (int j = 0; j < ns; ++j) mmax = fmaxf(mmax, *cluster.map_shared_rank(m_st + rl, (unsigned)j));
    const float msafe = mmax == -INFINITY ? 0.f : mmax;
    float L = 0.f, a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    for (int j = 0; j < ns; ++j) {
      const float wj = fast_exp2(*cluster.map_shared_rank(m_st + rl, (unsigned)j) - msafe);
      L += wj * *cluster.map_shared_rank(l_st + rl, (unsigned)j);
      const float4 oj = *reinterpret_cast<const float4*>(cluster.map_shared_rank(ost + rl * D + d, (unsigned)j));
      a0 += wj * oj.x;
      a1 += wj * oj.y;
      a2 += wj * oj.z;
      a3 += wj * oj.w;
    }
    const float inv = (valid && L > 0.f) ? 1.f / L : 0.f;
    const int64_t orow = (((int64_t)b * (p.M + 1) + gr / p.G) * p.Hq + hk * p.G + gr % p.G) * D;
    uint2 pk;
    pk.x = pack_bf16x2(a0 * inv, a1 * inv);
    pk.y = pack_bf16x2(a2 * inv, a3 * inv);
    *reinterpret_cast<uint2*>(p.out + orow + d) = pk;
  }
  cluster.sync();  // peers may still be reading this CTA's shared memory
  if (threadIdx.x == 0 && timed_out) atomicOr(&p.status[b], kSeqTimeout);
  if (threadIdx.x == 0 && sl < 0) atomicOr(&p.status[b], kSeqBadGeometry);
}

struct LaunchPlan {
  int ncw, tiles_q, nsplit, tiles_per_split, stages;
  size_t smem;
};

template <int D>
size_t smem_bytes(int stages) {
  return 1024 + (size_t)stages * (2 * KT * D * 2) + 2 * stages * sizeof(uint64_t) + 2 * kMaxCWarps * 16 * sizeof(float);
}

template <int D>
tv_status plan_launch(const AttnParams& p, LaunchPlan& lp) {
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda_error(e);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int warps_needed = (p.rows_total + 15) / 16;
  lp.tiles_q = (warps_needed + kMaxCWarps - 1) / kMaxCWarps;
  lp.ncw = (warps_needed + lp.tiles_q - 1) / lp.tiles_q;
  const int64_t units = (int64_t)p.B * p.Hkv * lp.tiles_q;
  const int key_tiles = (int)std::max<int64_t>(1, (p.S_cap + KT - 1) / KT);
  int ns = (int)std::min<int64_t>(kMaxSplit, std::max<int64_t>(1, (2LL * sms + units - 1) / units));
  ns = std::min(ns, key_tiles);
  lp.tiles_per_split = (key_tiles + ns - 1) / ns;
  lp.nsplit = (key_tiles + lp.tiles_per_split - 1) / lp.tiles_per_split;
  // deepest ring that still keeps the whole grid resident (when it can be)
  const int64_t ctas = units * lp.nsplit;
  const int threads = (lp.ncw + 1) * 32;
  auto kern = tree_attn_mma_kernel<D>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes<D>(6));
  if (e != cudaSuccess) return record_cuda_error(e);
  int occ2 = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ2, kern, threads, smem_bytes<D>(2));
  if (e != cudaSuccess) return record_cuda_error(e);
  const int64_t want = std::min<int64_t>(std::max(1, occ2), (ctas + sms - 1) / sms);
  lp.stages = 2;
  for (int st = std::min(6, std::max(2, lp.tiles_per_split)); st > 2; --st) {
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, threads, smem_bytes<D>(st));
    if (e != cudaSuccess) return record_cuda_error(e);
    if (occ >= want) {
      lp.stages = st;
      break;
    }
  }
  lp.smem = smem_bytes<D>(lp.stages);
  return TV_OK;
}

template <int D>
tv_status run(const CUtensorMap& tmk, const CUtensorMap& tmv, AttnParams p, cudaStream_t s) {
  LaunchPlan lp;
  tv_status r = plan_launch<D>(p, lp);
  if (r != TV_OK) return r;
  p.nsplit = lp.nsplit;
  p.tiles_per_split = lp.tiles_per_split;
  p.stages = lp.stages;
  if ((int64_t)p.B * p.Hkv > 65535 || lp.tiles_q > 65535) return TV_ERR_UNSUPPORTED;
  dim3 grid(lp.nsplit, lp.tiles_q, p.B * p.Hkv);
  return launch(tree_attn_mma_kernel<D>, grid, dim3((lp.ncw + 1) * 32), lp.smem, s, lp.nsplit, true, tmk, tmv, p);
}

}  // namespace
}  // namespace tv

namespace tv {

tv_status prepare_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t S_cap,
                            const int32_t* kv_start, const int32_t* kv_len, const uint32_t* anc_mask,
                            int32_t* status, int B, int M, int Hq, int Hkv, int D, float scale, uint16_t* out,
                            unsigned flags, const int32_t* depth, float rope_theta, const int32_t* slot,
                            int n_slots, AttnCall& call) {
  call.nothing_to_do = false;
  if (B < 0 || M < 0 || Hq <= 0 || Hkv <= 0 || S_cap < 0 || !(scale > 0.f)) return TV_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return TV_ERR_INVALID_ARG;
  if ((flags & ~(unsigned)(TV_ATTN_PREFIX_READY | TV_ATTN_ROPE)) != 0) return TV_ERR_INVALID_ARG;
  const bool rope = (flags & TV_ATTN_ROPE) != 0;
  if (rope && (!depth || !(rope_theta > 1.0f))) return TV_ERR_INVALID_ARG;
  if (slot && n_slots < 1) return TV_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return TV_ERR_UNSUPPORTED;
  if (rope && D != 128) return TV_ERR_UNSUPPORTED;
  if (M + 1 > kMaxRows || S_cap > 0x7fffffffLL) return TV_ERR_UNSUPPORTED;
  if (B == 0) {
    call.nothing_to_do = true;
    return TV_OK;
  }
  if (!q || !k || !v || !kv_start || !kv_len || !anc_mask || !status || !out) return TV_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return TV_ERR_INVALID_ARG;
  AttnParams& p = call.p;
  p.q = q;
  p.kv_start = kv_start;
  p.kv_len = kv_len;
  p.anc = anc_mask;
  p.status = status;
  p.out = out;
  p.S_cap = S_cap;
  p.B = B;
  p.M = M;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.W = (M + 1 + 31) / 32;
  p.rows_total = p.G * (M + 1);
  p.nsplit = p.tiles_per_split = p.stages = p.v_stages = 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.flags = flags;
  p.wait_limit_ns = pipeline_wait_limit_ns();
  p.depth = rope ? depth : nullptr;
  p.slot = slot;
  p.n_slots = slot ? n_slots : B;
  rope_freqs(rope ? (double)rope_theta : 2.0, D, p.rope);
  p.ws = nullptr;
  if ((int64_t)p.n_slots * Hkv > 0x7fffffffLL) return TV_ERR_UNSUPPORTED;
  p.kv_4d = 0;
  if (D == 128 && encode_kv_map_4d(&call.tmk, k, p.n_slots * Hkv, S_cap) &&
      encode_kv_map_4d(&call.tmv, v, p.n_slots * Hkv, S_cap)) {
    p.kv_4d = 1;
  } else if (!encode_kv_map(&call.tmk, k, p.n_slots * Hkv, S_cap, D) ||
             !encode_kv_map(&call.tmv, v, p.n_slots * Hkv, S_cap, D)) {
    return TV_ERR_INVALID_ARG;
  }
  if (D == 128) return plan_attention_tc(B, M, Hq, Hkv, S_cap, call.plan);
  return TV_OK;
}

tv_status launch_attention(AttnCall& call, int D, cudaStream_t s) {
  if (D == 64) return run<64>(call.tmk, call.tmv, call.p, s);  // warp-MMA kernel, merge through DSMEM
  return run_attention_tc(call.tmk, call.tmv, call.p, call.plan, s);  // tcgen05 kernel
}

}  // namespace tv

extern "C" size_t tree_attention_workspace_size(int B, int M, int Hq, int Hkv, int D, int64_t S_cap) {
  using namespace tv;
  if (B <= 0 || M < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || S_cap < 0 || D != 128) return 0;
  if (M + 1 > kMaxRows || S_cap > 0x7fffffffLL) return 0;
  TcPlan plan;
  if (plan_attention_tc(B, M, Hq, Hkv, S_cap, plan) != TV_OK) return 0;
  return plan.ws_bytes;
}

extern "C" tv_status tree_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t S_cap,
                                    const int32_t* kv_start, const int32_t* kv_len, const uint32_t* anc_mask,
                                    int32_t* status, int B, int M, int Hq, int Hkv, int D, float scale,
                                    uint16_t* out, void* workspace, size_t workspace_bytes, unsigned flags,
                                    const int32_t* depth, float rope_theta, const int32_t* slot, int n_slots,
                                    tv_stream_t stream) {
  using namespace tv;
  AttnCall call;
  tv_status r = prepare_attention(q, k, v, S_cap, kv_start, kv_len, anc_mask, status, B, M, Hq, Hkv, D, scale,
                                  out, flags, depth, rope_theta, slot, n_slots, call);
  if (r != TV_OK || call.nothing_to_do) return r;
  if (D == 128 && call.plan.ws_bytes > 0) {
    if (!workspace || workspace_bytes < call.plan.ws_bytes || !aligned16(workspace)) return TV_ERR_INVALID_ARG;
    call.p.ws = static_cast<float*>(workspace);
  }
  return launch_attention(call, D, reinterpret_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// tree_attention_noalloc: the same computation for callers that cannot
// allocate device memory -- for example a serving process whose memory pool
// already owns the whole GPU, or a plugin whose host framework hands it no
// device allocator.  The split partials then live in a fixed array compiled
// into this library instead of a caller-provided workspace.
// ---------------------------------------------------------------------------
namespace tv {
namespace {

// 32 MiB of scratch; every GPU that loads this library holds it until the
// process exits.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code the
// array's name only stands in for it, so the address is looked up once per
// device, with that device current, and cached.  The cache assumes that each
// device keeps one primary context for the life of the process: after a
// cudaDeviceReset the cached address would be stale, so a process that resets
// a device must not call tree_attention_noalloc on it again.
tv_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda_error(e);
  if (dev < 0 || dev >= kMaxDevices) return TV_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return record_cuda_error(e);
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return TV_OK;
}

}  // namespace
}  // namespace tv

extern "C" size_t tree_attention_noalloc_max_scratch(void) { return tv::kNoAllocScratchBytes; }

extern "C" tv_status tree_attention_noalloc(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                            int64_t S_cap, const int32_t* kv_start, const int32_t* kv_len,
                                            const uint32_t* anc_mask, int32_t* status, int B, int M, int Hq,
                                            int Hkv, int D, float scale, uint16_t* out, tv_stream_t stream) {
  using namespace tv;
  AttnCall call;
  tv_status r = prepare_attention(q, k, v, S_cap, kv_start, kv_len, anc_mask, status, B, M, Hq, Hkv, D, scale,
                                  out, 0u, nullptr, 0.f, nullptr, 0, call);
  if (r != TV_OK || call.nothing_to_do) return r;
  if (D == 128 && call.plan.ws_bytes > 0) {  // D = 64 keeps its partials on chip
    if (call.plan.ws_bytes > kNoAllocScratchBytes) return TV_ERR_UNSUPPORTED;  // too large for the fixed scratch
    void* scratch = nullptr;
    r = noalloc_scratch(&scratch);
    if (r != TV_OK) return r;
    call.p.ws = static_cast<float*>(scratch);
  }
  return launch_attention(call, D, reinterpret_cast<cudaStream_t>(stream));
}
