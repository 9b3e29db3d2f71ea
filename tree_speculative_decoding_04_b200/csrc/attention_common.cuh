// attention_common.cuh -- pieces shared by the two tree-attention kernels:
// launch parameters and the TMA descriptor of one KV-cache layer.
#pragma once

#include <mutex>

#include "tv_common.cuh"

namespace tv {

constexpr int kKeyTile = 64;             // keys per pipeline stage
constexpr int kBoxBytes = kKeyTile * 128;  // one 64-row x 128-byte swizzled TMA box

struct AttnParams {
  const uint16_t* q;
  const int32_t* kv_start;
  const int32_t* kv_len;
  const uint32_t* anc;
  int32_t* status;
  uint16_t* out;
  int64_t S_cap;
  int B, M, Hq, Hkv, G, W;
  int rows_total;       // G * (M + 1) query rows per (sequence, kv head)
  int nsplit;           // key splits (cluster size along x)
  int tiles_per_split;  // 64-key tiles per split
  int stages;           // key-tile ring depth (K ring of the tensor-core kernel)
  int v_stages;         // V ring depth of the tensor-core kernel
  float scale_log2;     // softmax scale * log2(e)
  unsigned flags;       // TV_ATTN_* launch flags
  const int32_t* depth; // [B][M+1] node depths (rotary positions kv_len + depth), TV_ATTN_ROPE only
  const int32_t* slot;  // [B] cache slot of each batch row, or null (slot = row)
  int n_slots;          // slots of the cache pool (B without a slot map)
  int kv_4d;            // the K/V maps are 4-D (one 16 KB box per tile), else 3-D (two 8 KB boxes)
  RopeFreqs rope;       // inverse frequencies, TV_ATTN_ROPE only
  uint64_t wait_limit_ns;  // limit of the pipeline waits (the drain waits keep kWaitLimitNs)
  float* ws;            // split partials: [units][nsplit][128 rows][128] O, then [units][nsplit][128][2] (m, l)
};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// [B*Hkv][S_cap][128] bf16 as a 4-D tensor {64 columns, S_cap rows, 2 halves,
// BH} (strides: row 256 B, half 128 B, head S_cap * 256 B) with boxes of 64 x 64
// x 2 x 1: one 16 KB copy brings a whole 64-key tile, landing as [half][row][128
// B] -- the layout of two 8 KB boxes -- with one copy instead of two.  Returns
// false if the driver refuses the layout (the caller then uses the 3-D map).
inline bool encode_kv_map_4d(CUtensorMap* map, const void* base, int BH, int64_t S_cap) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {64, (cuuint64_t)S_cap, 2, (cuuint64_t)BH};
  cuuint64_t strides[3] = {256, 128, (cuuint64_t)S_cap * 256};
  cuuint32_t box[4] = {64, (cuuint32_t)kKeyTile, 2, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// [B*Hkv][S_cap][D] bf16 -> boxes of 64 columns (128 B) x 64 rows, 128-byte swizzle.
inline bool encode_kv_map(CUtensorMap* map, const void* base, int BH, int64_t S_cap, int D) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)S_cap, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)S_cap * D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)kKeyTile, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}


// Tensor-core (tcgen05) path for head dim 128; defined in attention_tc.cu.
struct TcPlan {
  int tiles_q, nq, nsplit, tiles_per_split, stages, v_stages;  // nq: query tiles per CTA
  int per_sm;  // CTAs the plan sizes to be resident on one SM
  size_t smem, ws_bytes;
};
tv_status plan_attention_tc(int B, int M, int Hq, int Hkv, int64_t S_cap, TcPlan& plan);
tv_status run_attention_tc(const CUtensorMap& tmk, const CUtensorMap& tmv, AttnParams p, const TcPlan& plan,
                           cudaStream_t s);

// Argument checks and launch parameters shared by every tree-attention entry
// point.  Returns TV_OK with *nothing_to_do set for an empty batch.
struct AttnCall {
  AttnParams p;
  CUtensorMap tmk, tmv;
  TcPlan plan;  // filled for D = 128
  bool nothing_to_do;
};
tv_status prepare_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t S_cap,
                            const int32_t* kv_start, const int32_t* kv_len, const uint32_t* anc_mask,
                            int32_t* status, int B, int M, int Hq, int Hkv, int D, float scale, uint16_t* out,
                            unsigned flags, const int32_t* depth, float rope_theta, const int32_t* slot,
                            int n_slots, AttnCall& call);
tv_status launch_attention(AttnCall& call, int D, cudaStream_t s);

}  // namespace tv
