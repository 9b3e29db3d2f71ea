// tv_common.cuh -- small device/host helpers shared by the kernels of the
// tree verification library: bounded mbarrier waits, TMA / bulk-copy wrappers
// (no multicast anywhere), warp reductions and host-side launch plumbing.
#pragma once

#include <cuda.h>  // CUtensorMap and driver enums (types only; the driver is reached through the runtime)
#include <math.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "treeverify.h"

namespace tv {

constexpr int kSeqBadParent = TV_SEQ_BAD_PARENT;
constexpr int kSeqTooDeep = TV_SEQ_TOO_DEEP;
constexpr int kSeqTimeout = TV_SEQ_TIMEOUT;
constexpr int kSeqBadGeometry = TV_SEQ_BAD_GEOMETRY;
constexpr int kMaxRows = TV_MAX_TREE_ROWS;

// A device wait gives up after this long (ns) and reports TV_SEQ_TIMEOUT.
constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;
// Second, independent bound on the number of polls.
constexpr uint32_t kWaitLimitPolls = 1u << 28;

__host__ __device__ inline bool geometry_ok(int32_t ks, int32_t kl, int M, int64_t S_cap) {
  return ks >= 0 && kl >= 0 && (int64_t)ks + kl + M + 1 <= S_cap;
}

// Largest head dim with a rotary table: D / 2 angle frequencies.
constexpr int kMaxRopePairs = 64;

// Inverse frequencies theta^(-2i/D), i < D/2, computed on the host in double.
struct RopeFreqs {
  double f[kMaxRopePairs];
};

inline void rope_freqs(double theta, int D, RopeFreqs& r) {
  for (int i = 0; i < kMaxRopePairs; ++i) r.f[i] = i < D / 2 ? pow(theta, -2.0 * i / D) : 0.0;
}

// Cache slot of batch row b: slot[b] when a slot map is given, else b; -1 if
// the map points outside [0, n_slots).
__host__ __device__ inline int cache_slot(const int32_t* slot, int b, int n_slots) {
  if (!slot) return b;
  const int s = slot[b];
  return (s >= 0 && s < n_slots) ? s : -1;
}

#if defined(__CUDACC__)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}
// Bounded wait on the phase with the given parity; false if it gave up (after
// Non-blocking: has the phase with this parity completed?
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// limit_ns, or kWaitLimitPolls polls, whichever comes first).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 0; i < kWaitLimitPolls; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
  return false;
}

// ---------------------------------------------------------------- TMA (tensor) loads, no multicast
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
// A 4-D box (here: 64 columns x rows x both 64-column halves of a 128-wide row
// x 1), landing as [half][row][128 B].
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2,
                                            int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
__device__ __forceinline__ void tma_prefetch_4d(const CUtensorMap* map, int c0, int c1, int c2, int c3) {
  asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// L2 prefetch of one tensor tile (no shared memory, no barrier: nothing waits on it)
__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap* map, int x, int y, int z) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(z)
               : "memory");
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// ---------------------------------------------------------------- programmatic dependent launch
__device__ __forceinline__ void pdl_wait_primary() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- misc
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// three-input maximum (one instruction on sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// packed pairs of fp32 for the sm_100 two-wide FP32 instructions
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {  // a * b + c, per lane
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 2^a for a pair of floats on the FMA pipe instead of the MUFU: a = n + f with
// n the nearest integer (the 1.5 * 2^23 rounding constant) and f in [-1/2, 1/2];
// 2^f by a cubic fitted to it (least squares at Chebyshev nodes, relative error
// below 7.5e-5 -- far below the bf16 rounding of the probabilities), scaled by
// 2^n through the exponent field.  Arguments below -125 are clamped there
// (result about 2e-38, nothing that moves an fp32 sum of terms near 1).
__device__ __forceinline__ uint64_t f2_exp2_poly(uint64_t a) {
  float a0, a1;
  f2_unpack(a, a0, a1);
  a = f2_pack(fmaxf(a0, -125.f), fmaxf(a1, -125.f));
  const uint64_t magic = f2_pack(12582912.f, 12582912.f);
  const uint64_t t = f2_add(a, magic);                                          // n in the low mantissa bits
  const uint64_t fr = f2_fma(f2_add(t, f2_pack(-12582912.f, -12582912.f)), f2_pack(-1.f, -1.f), a);  // a - n
  uint64_t p = f2_fma(f2_pack(0.055171613f, 0.055171613f), fr, f2_pack(0.24261113f, 0.24261113f));
  p = f2_fma(p, fr, f2_pack(0.69326097f, 0.69326097f));
  p = f2_fma(p, fr, f2_pack(0.99992806f, 0.99992806f));
  float t0, t1, p0, p1;
  f2_unpack(t, t0, t1);
  f2_unpack(p, p0, p1);
  const int k = 0x4B400000;  // bits of 1.5 * 2^23
  const float r0 = __int_as_float(__float_as_int(p0) + ((__float_as_int(t0) - k) << 23));
  const float r1 = __int_as_float(__float_as_int(p1) + ((__float_as_int(t1) - k) << 23));
  return f2_pack(r0, r1);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// ---------------------------------------------------------------- rotary embedding
// cos and sin of the angle pos * inv_freq.  The angle is formed and reduced to
// [-pi, pi] in double precision (two-part 2 pi, Cody-Waite style), so that the
// hardware sine and cosine (MUFU, absolute error below 4e-7 on [-pi, pi]) see
// an argument accurate to float rounding even at positions of tens of
// thousands.
__device__ __forceinline__ void rope_cos_sin(int pos, double inv_freq, float& c, float& s) {
  const double a = (double)pos * inv_freq;
  const double k = rint(a * 0.15915494309189535);   // a / (2 pi), nearest integer
  double r = fma(-k, 6.283185307179586, a);         // 2 pi, leading double
  r = fma(-k, 2.4492935982947064e-16, r);           // 2 pi, remainder
  const float rf = (float)r;
  s = __sinf(rf);
  c = __cosf(rf);
}

// Rotate 8 pairs: lo holds elements i0 .. i0+7 of a row, hi the elements
// i0 + D/2 .. i0 + D/2 + 7; pair (x, y) becomes (x cos - y sin, y cos + x sin),
// rounded to bf16.
__device__ __forceinline__ void rope_rotate8(uint4& lo, uint4& hi, int pos, const double* inv_freq, int i0) {
  uint32_t* l = reinterpret_cast<uint32_t*>(&lo);
  uint32_t* h = reinterpret_cast<uint32_t*>(&hi);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&l[w]));
    const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&h[w]));
    float c0, s0, c1, s1;
    rope_cos_sin(pos, inv_freq[i0 + 2 * w], c0, s0);
    rope_cos_sin(pos, inv_freq[i0 + 2 * w + 1], c1, s1);
    l[w] = pack_bf16x2(fmaf(x.x, c0, -y.x * s0), fmaf(x.y, c1, -y.y * s1));
    h[w] = pack_bf16x2(fmaf(y.x, c0, x.x * s0), fmaf(y.y, c1, x.y * s1));
  }
}

#endif  // __CUDACC__

// ---------------------------------------------------------------- host side
// Records the last CUDA error for tv_last_cuda_error(); returns TV_ERR_CUDA.
tv_status record_cuda_error(cudaError_t e);

// Limit (ns) of the pipeline waits of the next attention launches
// (tv_set_wait_limit_ns); kWaitLimitNs unless a test shortened it.
uint64_t pipeline_wait_limit_ns();

// The acceptance walk of tree_accept (accept.cu) on a per-node argmax that is
// already in device memory: accepted = ancestors all matched, endpoint =
// deepest accepted node (lowest row on ties), path / accept_len / bonus.
tv_status launch_accept_walk(const int32_t* argmax, const int32_t* draft, const int32_t* parent,
                             const int32_t* depth, const uint32_t* anc_mask, int32_t* status, int B, int M,
                             int max_depth, int32_t* accept_len, int32_t* path, int32_t* bonus, cudaStream_t s);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Launch with optional cluster dims and programmatic-dependent-launch attribute.
template <typename Kern, typename... Args>
tv_status launch(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, int cluster_x, bool pdl,
                 Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attrs[2];
  int na = 0;
  if (cluster_x > 1) {
    attrs[na].id = cudaLaunchAttributeClusterDimension;
    attrs[na].val.clusterDim.x = cluster_x;
    attrs[na].val.clusterDim.y = 1;
    attrs[na].val.clusterDim.z = 1;
    ++na;
  }
  if (pdl) {
    attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attrs;
  cfg.numAttrs = na;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  if (e != cudaSuccess) return record_cuda_error(e);
  return TV_OK;
}

}  // namespace tv
