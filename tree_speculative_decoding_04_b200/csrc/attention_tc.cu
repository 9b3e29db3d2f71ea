// attention_tc.cu -- tree_attention on the 5th-generation tensor cores
// (tcgen05 + TMEM) for head dim 128.
//
// "EAGLE-Pangu: Accelerator-Safe Tree Speculative Decoding on Ascend NPUs",
// methodology C: one batched teacher pass over all speculative tokens with a
// tree mask (node k attends node j only if j is an ancestor of k).  The mask is
// applied from the ancestor bitmask on the last M+1 key columns only.
//
// One CTA owns 128 query rows (tree node x q head of one GQA group) of one
// (sequence, kv head) and one split of that sequence's key range.  The splits
// of a query tile form a thread-block cluster: each writes its partial (max,
// sum, O) to a workspace in L2, the cluster barrier orders the writes, and each
// CTA then merges 1/nsplit of the output columns.  (Keeping the partials in
// each CTA's shared memory and merging over distributed shared memory gave the
// same bits and measured no faster on B200.)
// Warp roles (192 threads):
//   warp 0      TMA producer: lane 0 streams 64-key K tiles and lane 1 V tiles
//               into two separate smem rings (two slots each with two CTAs per
//               SM) -- a K slot is freed once S = QK^T has read it, a V slot
//               after O += PV
//   warp 1      TMEM owner and MMA issuer (one thread):
//                 S_i = Q K_i^T   (M=128, N=64, K=128; A, B from smem)   -> TMEM S[i%2]
//                 O  += P_i V_i   (M=128, N=128, K=64; A=P from TMEM, B=V from smem) -> TMEM O
//               it polls its K, P and V barriers and issues whichever MMA is
//               ready, so S_{i+1} is computed while the softmax warps work on
//               S_i, and a late K tile holds back no PV (nor a late V tile a QK)
//   warps 2-5   softmax: thread t owns TMEM lane t, i.e. query row t; it reads
//               its 64 scores with one tcgen05.ld, keeps the running max / sum,
//               writes P (bf16) over its scores, and rescales its O row only
//               when the running max grows by more than 2^8 (otherwise the
//               stale max keeps every P <= 256, exact in fp32 accumulation).
// TMEM: S0 cols [0,64), S1 [64,128), O [128,256); P_i aliases S[i%2] cols [0,32).
#include <cooperative_groups.h>

#include <algorithm>

#include "attention_common.cuh"
#include "tcgen05.cuh"

namespace cg = cooperative_groups;

// Tuning (compile-time, so that a sweep can rebuild with -D):
//   TV_TC_SPLIT_FACTOR  key splits are added while units * splits stays within
//                       this many CTAs per SM
//   TV_TC_ONE_PER_SM    1: a grid that fits one wave gets one CTA per SM with
//                       deeper rings; 0: every CTA stays within half an SM's
//                       shared memory, so the next launch's CTAs can become
//                       resident beside it and start streaming early
#ifndef TV_TC_SPLIT_FACTOR
#define TV_TC_SPLIT_FACTOR 2
#endif
#ifndef TV_TC_ONE_PER_SM
#define TV_TC_ONE_PER_SM 1
#endif
// ring depths (K, V) of a CTA that has its SM to itself
//   TV_TC_POLY_EXP_PAIRS  of every 8 pairs of probabilities, how many are
//                       exponentiated on the FMA pipe (the rest on the MUFU)
#ifndef TV_TC_POLY_EXP_PAIRS
#define TV_TC_POLY_EXP_PAIRS 0
#endif
//   TV_TC_FORCE_SOLO    1: one CTA per SM (deep rings) even for grids of
//                       several waves
//   TV_TC_PAIR          1: two query tiles per CTA when a unit has two or more (off:
//                       measured slower)
#ifndef TV_TC_PAIR
#define TV_TC_PAIR 0
#endif
#ifndef TV_TC_FORCE_SOLO
#define TV_TC_FORCE_SOLO 0
#endif
#ifndef TV_TC_K_RING_SOLO
#define TV_TC_K_RING_SOLO 3
#endif
#ifndef TV_TC_V_RING_SOLO
#define TV_TC_V_RING_SOLO 6
#endif
//   TV_TC_PREFETCH_TILES key tiles per CTA warmed in L2 before the grid dependency
//                       (0: measured fastest on B200, the early requests
//                       compete with the launch still running)
//   TV_TC_PREFETCH_Q     1: the CTA's query rows are warmed in L2 before it
//                       (0: measured as fast or faster)
#ifndef TV_TC_PREFETCH_TILES
#define TV_TC_PREFETCH_TILES 0
#endif
#ifndef TV_TC_PREFETCH_Q
#define TV_TC_PREFETCH_Q 0
#endif
// ring depths (K, V) of a CTA that shares its SM with another (up to 5 slots
// fit; 2 + 2 measured faster than 2 + 3 and 3 + 2 on B200: mha7b 17.6 vs
// 18.4 us, b32gqa 151 vs 154 us, stress the same)
#ifndef TV_TC_K_RING_DUO
#define TV_TC_K_RING_DUO 2
#endif
#ifndef TV_TC_V_RING_DUO
#define TV_TC_V_RING_DUO 2
#endif
//   TV_TC_LONGEST_FIRST  1: grids of more than one wave start their (sequence,
//                       kv head) blocks longest prefix first
#ifndef TV_TC_LONGEST_FIRST
#define TV_TC_LONGEST_FIRST 1
#endif
//   TV_TC_Q_TMEM        1: the one-query-tile instance keeps Q in TMEM (the A
//                       operand of S = Q K^T) and a single S buffer, so each
//                       score MMA reads only its K tile from shared memory
#ifndef TV_TC_Q_TMEM
#define TV_TC_Q_TMEM 0
#endif
//   TV_TC_TILE_MAJOR    1: single-wave grids issue their blocks query-tile-major
#ifndef TV_TC_TILE_MAJOR
#define TV_TC_TILE_MAJOR 1
#endif
//   TV_TC_MMA_POLL      1: the MMA thread polls its K, P and V barriers and
//                       issues whichever MMA is ready (no head-of-line wait)
#ifndef TV_TC_MMA_POLL
#define TV_TC_MMA_POLL 1
#endif
//   TV_TC_SPLIT_PRODUCER 1: two producer threads, one per K and V stream
#ifndef TV_TC_SPLIT_PRODUCER
#define TV_TC_SPLIT_PRODUCER 1
#endif
//   TV_TC_EARLY_ROWS    1: grids in row order request the query rows before
//                       the geometry
#ifndef TV_TC_EARLY_ROWS
#define TV_TC_EARLY_ROWS 1
#endif
//   TV_TC_DESC_STEP     1: the polling MMA thread forms each k-step's
//                       shared-memory descriptor as the tile's first one plus a
//                       constant (one add per MMA)
#ifndef TV_TC_DESC_STEP
#define TV_TC_DESC_STEP 1
#endif

namespace tv {
namespace {

constexpr int kRows = 128;
constexpr int kTmemCols = 256;
constexpr int kMaxStages = 8;
constexpr int kQBytes = kRows * 128 * 2;         // 2 boxes of [128 rows][128 B]
constexpr int kTileBytes = kKeyTile * 128 * 2;   // K (or V): 2 boxes of [64 rows][128 B]
constexpr float kRescaleThreshold = 8.0f;        // log2 domain
constexpr int kPrefetchTiles = TV_TC_PREFETCH_TILES;  // key tiles per CTA warmed in L2 before the grid dependency
constexpr int kMaxSplit_tc = 8;                  // portable cluster size

struct TcSmem {
  uint64_t k_full[kMaxStages];
  uint64_t k_empty[kMaxStages];
  uint64_t v_full[kMaxStages];
  uint64_t v_empty[kMaxStages];
  uint64_t s_full[2][2];   // [query pipe][S buffer]
  uint64_t p_full[2][2];   // [query pipe][S buffer]
  uint64_t o_ready[2][2];  // [query pipe][j % 2]: PV_j completes a phase
  uint64_t q_ready;
  uint64_t drain;
  uint32_t tmem_base;
  int timed_out;
};

// The batch row that the `rank`-th (sequence, kv head) block of the grid
// serves, with its cache slot, geometry and status.  Rows are taken longest
// prefix first (ties in row order): the block scheduler starts blocks in grid
// order, so the longest units start first and the last wave is made of short
// ones (longest-processing-time-first list scheduling); in plain row order a
// long sequence that happens to come last leaves most SMs idle at the end.
// For B <= 32 lane i of the calling warp loads row i's slot, kv_len, kv_start
// and status in one round trip, the rows are ranked with shuffles and the
// chosen row's values are shuffled out; every lane gets the same answer.
// Larger batches, and grids that start all at once (LF = false: the order
// cannot matter there), keep row order.  Warp-collective: call with all lanes
// active.
struct RowGeo {
  int b;         // batch row
  int sl;        // cache slot (-1: outside the pool)
  int32_t ks;    // kv_start of the slot (0 when sl < 0)
  int32_t kl;    // kv_len of the slot (0 when sl < 0)
  int32_t st;    // status of the row
  int32_t lane_len;  // this lane's row length (-1 past B or outside the pool; 0 for B > 32)
};

template <bool LF>
__device__ __forceinline__ RowGeo row_of_rank(const AttnParams& p, int rank) {
  RowGeo g;
  if (!LF || p.B > 32) {
    g.b = rank;
    g.sl = cache_slot(p.slot, rank, p.n_slots);
    g.ks = g.sl >= 0 ? __ldcg(p.kv_start + g.sl) : 0;
    g.kl = g.sl >= 0 ? __ldcg(p.kv_len + g.sl) : 0;
    g.st = __ldcg(p.status + rank);
    g.lane_len = 0;
    return g;
  }
  const int lane = threadIdx.x & 31;
  int s = -1;
  int32_t len = -1, ks = 0, st = 0;
  if (lane < p.B) {
    s = cache_slot(p.slot, lane, p.n_slots);
    st = __ldcg(p.status + lane);
    if (s >= 0) {
      len = __ldcg(p.kv_len + s);
      ks = __ldcg(p.kv_start + s);
    }
  }
  // rank of this lane's row: rows that are longer, or as long and earlier
  int r = 0;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const int32_t lj = __shfl_sync(0xffffffffu, len, j);
    r += (j < p.B && (lj > len || (lj == len && j < lane))) ? 1 : 0;
  }
  const unsigned m = __ballot_sync(0xffffffffu, lane < p.B && r == rank);
  const int src = m ? __ffs(m) - 1 : 0;  // (len, -row) is a strict order: exactly one lane matches
  g.b = m ? src : rank;
  g.sl = __shfl_sync(0xffffffffu, s, src);
  g.ks = __shfl_sync(0xffffffffu, ks, src);
  g.kl = __shfl_sync(0xffffffffu, len, src);
  g.st = __shfl_sync(0xffffffffu, st, src);
  if (g.sl < 0) g.ks = g.kl = 0;
  g.lane_len = len;
  return g;
}

// bits [start, start + 64) of an ancestor row (bit t = tree row t); rows outside
// [0, 32 * 8) read as 0, so a window that starts inside the prefix is fine.
__device__ __forceinline__ uint64_t anc_window(const uint32_t (&aw)[kMaxRows / 32], int start) {
  uint64_t r = 0;
#pragma unroll
  for (int q = 0; q < kMaxRows / 32; ++q) {
    const int off = q * 32 - start;  // where bit 0 of word q lands in the window
    const uint64_t w = aw[q];
    if (off >= 0 && off < 64) r |= w << off;
    else if (off < 0 && off > -32) r |= w >> (-off);
  }
  return r;
}

// O_q += P_{q,j} V_j for key tile j and every query pipe q < nq (one thread),
// then release the V stage once every pipe has used it and publish each new
// O.  Pipe q's TMEM block starts at column q * 256: S buffers at +0 / +64 (P_j
// aliases S[j % 2]), O at +128.  Returns false if a P or V never arrived.
// single_s: one S buffer per pipe (P_j at column 0, p_full[q][0] completes one
// phase per tile).
__device__ __forceinline__ bool issue_pv(TcSmem* sh, uint8_t* v_ring, uint32_t tmem, int nq, int j, int v_stages,
                                         uint64_t lim, bool single_s = false) {
  const uint32_t idesc_o = idesc_bf16(128, 128, 1);
  const int sb = single_s ? 0 : (j & 1), s = j % v_stages;
  if (!mbar_wait(&sh->v_full[s], (j / v_stages) & 1, lim)) return false;
  const uint32_t v_addr = smem_u32(v_ring + s * kTileBytes);
  for (int q = 0; q < nq; ++q) {
    if (!mbar_wait(&sh->p_full[q][sb], single_s ? (j & 1) : ((j >> 1) & 1), lim)) return false;
    tc_fence_after();
    const uint32_t t_q = tmem + q * kTmemCols;
#pragma unroll
    for (int kk = 0; kk < kKeyTile / 16; ++kk)
      mma_ts(t_q + 128, t_q + sb * 64 + kk * 8, sw128_desc(v_addr + kk * 16 * 128, kBoxBytes), idesc_o,
             (j > 0 || kk > 0) ? 1u : 0u);
    tc_commit(&sh->o_ready[q][j & 1]);
  }
  tc_commit(&sh->v_empty[s]);
  return true;
}

// NQ query tiles per CTA share every K/V tile (NQ = 2: 8 softmax warps, all 512
// TMEM columns, one CTA per SM); the query tiles of a (sequence, kv head) are
// blockIdx.y * NQ + q.  MW: the grid has more blocks than fit at once.  A
// multi-wave grid is unit-major and, with TV_TC_LONGEST_FIRST, takes its batch
// rows longest prefix first (a separate instance: the ranking code, even when
// skipped at run time, cost single-wave grids about 4 us per launch on B200
// through code generation at the register limit); a single-wave grid is
// query-tile-major with TV_TC_TILE_MAJOR.  The host lays out the grid to match.
template <int NQ, bool MW>
__global__ void __launch_bounds__(64 + 128 * NQ, NQ == 1 ? 2 : 1)
    tree_attn_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                        const __grid_constant__ AttnParams p) {
  // The 128-byte-swizzled tiles need 1024-byte alignment.  The dynamic window
  // starts on such a boundary on this GPU; if it ever did not, every CTA treats
  // its sequence as failed (zero output, TV_SEQ_TIMEOUT) instead of computing.
  // Q in TMEM and one S buffer (one query tile per CTA): TMEM S [0,64),
  // Q [64,128), O [128,256); otherwise S0 [0,64), S1 [64,128), O [128,256)
  constexpr bool kQT = NQ == 1 && TV_TC_Q_TMEM;
  constexpr bool kPoll = NQ == 1 && !kQT && TV_TC_MMA_POLL;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  const bool aligned_ok = (smem_u32(smem_raw) & 1023u) == 0;
  uint8_t* q_s = smem;                              // [NQ][2][128][128 B]
  const int k_stages = p.stages, v_stages = p.v_stages;
  uint8_t* k_ring = smem + NQ * kQBytes;              // [k_stages][2 boxes of 64 rows x 128 B]
  uint8_t* v_ring = k_ring + k_stages * kTileBytes;   // [v_stages][2 boxes]
  TcSmem* sh = reinterpret_cast<TcSmem*>(v_ring + v_stages * kTileBytes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int tiles_q = (p.rows_total + kRows - 1) / kRows;
  // Grids of one wave (MW = false) are query-tile-major, grid (splits, units,
  // query tiles): every unit's first tiles, then its second ones, and the last,
  // often light tile (b32gqa: rows 128, 128, 16) of every unit at the end, so
  // the CTAs that share an SM with another are light ones; every CTA of the
  // wave starts at once, so the tiles of a unit still read its K/V together
  // through L2.  Multi-wave grids stay unit-major, grid (splits, query tiles,
  // units), so that the tiles of a unit run together.
  constexpr bool kTileMajor = !MW && TV_TC_TILE_MAJOR;
  constexpr bool LF = MW && TV_TC_LONGEST_FIRST;
  const int qtile0 = (kTileMajor ? blockIdx.z : blockIdx.y) * NQ;  // first query tile of this CTA
  const int nq = min(NQ, tiles_q - qtile0);            // query tiles present (the last CTA may have fewer)
  const int bh = kTileMajor ? blockIdx.y : blockIdx.z;
  const int hk = bh % p.Hkv;
  const int rank = bh / p.Hkv;  // the block's place in the longest-first row order

  if (threadIdx.x == 0) {
    sh->timed_out = 0;
    for (int s = 0; s < k_stages; ++s) {
      mbar_init(&sh->k_full[s], 1);
      mbar_init(&sh->k_empty[s], 1);
    }
    for (int s = 0; s < v_stages; ++s) {
      mbar_init(&sh->v_full[s], 1);
      mbar_init(&sh->v_empty[s], 1);
    }
    for (int q = 0; q < NQ; ++q)
      for (int s = 0; s < 2; ++s) {
        mbar_init(&sh->s_full[q][s], 1);
        mbar_init(&sh->p_full[q][s], 4);
        mbar_init(&sh->o_ready[q][s], 1);
      }
    mbar_init(&sh->q_ready, 4);  // the four softmax warps, once Q is in TMEM
    mbar_init(&sh->drain, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmk);
    prefetch_tensormap(&tmv);
  }
  // zc_: the tensor-map row block of (cache slot, kv head)
  // one 16 KB box per tile with the 4-D maps, else two 8 KB boxes
  auto load_tile = [&](uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int row, int zc_) {
    mbar_arrive_expect_tx(bar, kTileBytes);
    if (p.kv_4d) {
      tma_load_4d(dst, map, bar, 0, row, 0, zc_);
    } else {
      tma_load_3d(dst, map, bar, 0, row, zc_);
      tma_load_3d(dst + kBoxBytes, map, bar, 64, row, zc_);
    }
  };
  auto issue_k = [&](int i, int32_t ks_, int k_lo_, int zc_) {
    const int s = i % k_stages;
    load_tile(k_ring + s * kTileBytes, &tmk, &sh->k_full[s], ks_ + k_lo_ + i * kKeyTile, zc_);
  };
  auto issue_v = [&](int i, int32_t ks_, int k_lo_, int zc_) {
    const int s = i % v_stages;
    load_tile(v_ring + s * kTileBytes, &tmv, &sh->v_full[s], ks_ + k_lo_ + i * kKeyTile, zc_);
  };
  // This sequence's key tiles are dealt evenly over the splits (ragged batches
  // would otherwise leave short sequences in one split).
  auto split_range = [&](int32_t kl_, int& k_lo_, int& nt_) {
    const int seq_tiles = (kl_ + p.M + 1 + kKeyTile - 1) / kKeyTile;
    const int tps = (seq_tiles + p.nsplit - 1) / p.nsplit;
    k_lo_ = split * tps * kKeyTile;
    nt_ = max(0, min(tps, seq_tiles - split * tps));
  };
  // With programmatic launch this CTA can be resident while the previous kernel
  // is still finishing.
  //  - TV_ATTN_PREFIX_READY: the caller guarantees that the previous launch on
  //    the stream writes neither the geometry, the slot map nor any prefix
  //    column, so the geometry is read now and the first ring's worth of tiles that lie wholly
  //    inside the prefix is requested into shared memory before the grid
  //    dependency resolves.  Tiles reaching the tree rows, the query rows, the
  //    ancestor rows and the status are read only after it.
  //  - otherwise: only warm L2 with the first key tile of this split and with
  //    this CTA's query rows.  A prefetch binds no value: a write of the
  //    previous kernel to the same lines lands in L2, which every later read
  //    goes through, so a stale geometry read here only wastes the prefetch
  //    (issued only for a geometry that fits the cache, so the coordinates stay
  //    inside the tensor).
  const bool prefix_ready = (p.flags & TV_ATTN_PREFIX_READY) != 0;
  // limit of the pipeline waits; the waits that drain copies or MMAs in flight
  // before the CTA exits always keep the full limit
  const uint64_t lim = p.wait_limit_ns;
  // With TV_ATTN_PREFIX_READY (or key tiles to warm in L2), warp 0 reads the
  // row order and the geometry before the grid dependency (one round trip);
  // otherwise every warp reads them after it only.
  RowGeo pre{rank, -1, 0, 0, 0, 0};
  int npre_k = 0, npre_v = 0;  // tiles requested before the grid dependency
  if (warp == 0 && (prefix_ready || kPrefetchTiles > 0)) {
    pre = row_of_rank<LF>(p, rank);
    if (prefix_ready) {
      if (pre.sl >= 0 && aligned_ok && geometry_ok(pre.ks, pre.kl, p.M, p.S_cap)) {
        int k_lo_pre, nt_pre;
        split_range(pre.kl, k_lo_pre, nt_pre);
        const int n_prefix = max(0, min(nt_pre, (pre.kl - k_lo_pre) / kKeyTile));  // tiles wholly inside the prefix
        npre_k = min(n_prefix, k_stages);
        npre_v = min(n_prefix, v_stages);
        if (lane == 0)  // the thread that initialised the barriers
          for (int i = 0; i < max(npre_k, npre_v); ++i) {
            if (i < npre_k) issue_k(i, pre.ks, k_lo_pre, pre.sl * p.Hkv + hk);
            if (i < npre_v) issue_v(i, pre.ks, k_lo_pre, pre.sl * p.Hkv + hk);
          }
      }
    } else if (lane == 0 && pre.sl >= 0 && geometry_ok(pre.ks, pre.kl, p.M, p.S_cap)) {
      int k_lo_h, nt_h;
      split_range(pre.kl, k_lo_h, nt_h);
      const int nt = min(kPrefetchTiles, nt_h);
      for (int i = 0; i < nt; ++i) {
        const int row = pre.ks + k_lo_h + i * kKeyTile;
        if (p.kv_4d) {
          tma_prefetch_4d(&tmk, 0, row, 0, pre.sl * p.Hkv + hk);
          tma_prefetch_4d(&tmv, 0, row, 0, pre.sl * p.Hkv + hk);
        } else {
          tma_prefetch_3d(&tmk, 0, row, pre.sl * p.Hkv + hk);
          tma_prefetch_3d(&tmk, 64, row, pre.sl * p.Hkv + hk);
          tma_prefetch_3d(&tmv, 0, row, pre.sl * p.Hkv + hk);
          tma_prefetch_3d(&tmv, 64, row, pre.sl * p.Hkv + hk);
        }
      }
    }
  }
  // the query rows are warmed in L2 when the row is known without a load
  if (TV_TC_PREFETCH_Q && warp >= 2 && (!LF || p.B > 32)) {
    const int gr_h = (qtile0 + ((warp - 2) >> 2)) * kRows + (warp & 3) * 32 + lane;
    if (gr_h < p.rows_total) {
      const uint16_t* qr =
          p.q + (((int64_t)rank * (p.M + 1) + gr_h / p.G) * p.Hq + hk * p.G + gr_h % p.G) * 128;
      prefetch_l2(qr);
      prefetch_l2(qr + 64);
    }
  }
  pdl_wait_primary();
  pdl_launch_dependents();
  // The row order, the slot and the geometry are read again after the
  // dependency (final values, the same for every warp).  Without
  // TV_ATTN_PREFIX_READY warp 0's early read served only prefetches.  With it,
  // if the caller's promise did not hold (they changed), the sequence is
  // flagged instead of computed; a changed length may also have changed the
  // row order, which CTAs that read early no longer share with the others, so
  // then every row of the batch is flagged.
  const int pipe = warp >= 2 ? (warp - 2) >> 2 : 0;  // query pipe of a softmax warp
  const int qtile = qtile0 + pipe;
  uint8_t* q_pipe = q_s + pipe * kQBytes;
  const uint32_t tq = (uint32_t)(pipe * kTmemCols);  // column offset of this pipe's TMEM block
  const int r = (warp & 3) * 32 + lane;  // TMEM lane == query row of this tile
  const int gr = qtile * kRows + r;
  const bool row_ok = pipe < nq && gr < p.rows_total;
  const int hq = hk * p.G + gr % p.G;
  const int u = min(gr / p.G, p.M);
  // A softmax thread's query row (zero past the tile), its ancestor words and,
  // with TV_ATTN_ROPE, its tree depth.  A grid in row order serves batch row
  // `rank`, known without a load, so these requests go out before the
  // geometry's and the two round trips overlap; the longest-first instance
  // learns its row from the geometry and requests them after it.
  constexpr bool kEarlyRows = !LF && TV_TC_EARLY_ROWS;
  uint4 qv[16];
  uint32_t anc_w[kMaxRows / 32];
  int depth_u = 0;
  auto load_rows = [&](int b_) {
    const int64_t node = (int64_t)b_ * (p.M + 1) + u;
    const uint4* src = reinterpret_cast<const uint4*>(p.q + (node * p.Hq + hq) * 128);
#pragma unroll
    for (int c = 0; c < 16; ++c) qv[c] = row_ok ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
    if ((p.flags & TV_ATTN_ROPE) && row_ok) depth_u = p.depth[node];
#pragma unroll
    for (int w = 0; w < kMaxRows / 32; ++w) anc_w[w] = w < p.W ? __ldg(p.anc + node * p.W + w) : 0u;
  };
  if (kEarlyRows && warp >= 2) load_rows(rank);
  const RowGeo g = row_of_rank<LF>(p, rank);
  const int b = g.b;
  const int sl = g.sl;
  const int32_t ks = g.ks, kl = g.kl;
  bool order_changed = false, broken_promise = false;
  if (prefix_ready) {  // uniform over the CTA
    const bool changed_w = warp == 0 && __any_sync(0xffffffffu, g.lane_len != pre.lane_len);
    order_changed = __syncthreads_or(changed_w) != 0;
    broken_promise = __syncthreads_or(warp == 0 && (changed_w || g.b != pre.b || g.sl != pre.sl ||
                                                    g.ks != pre.ks || g.kl != pre.kl)) != 0;
  }
  const int zc = sl * p.Hkv + hk;  // tensor-map row block of this (slot, kv head)
  const bool valid = aligned_ok && sl >= 0 && !broken_promise && g.st == 0 && geometry_ok(ks, kl, p.M, p.S_cap);
  const int N = kl + p.M + 1;
  int k_lo = 0, nt_geo = 0;
  split_range(kl, k_lo, nt_geo);
  const int ntiles = valid ? nt_geo : 0;

  // The rest of the first ring's worth of K/V tiles and the Q tile are
  // requested before the TMEM allocation barrier, so their memory latency
  // overlaps the set-up.
  // (lane 0 requests the K tiles, lane 1 the V tiles: the copies one thread
  // issues are processed one after another, about 59 GB/s per issuing thread
  // from L2 on B200, so two issuing threads keep K tiles from queueing behind
  // V tiles)
  if (warp == 0 && lane < (TV_TC_SPLIT_PRODUCER ? 2 : 1))
    for (int i = 0; i < min(ntiles, max(k_stages, v_stages)); ++i) {
      if (lane == 0 && i < k_stages && i >= npre_k) issue_k(i, ks, k_lo, zc);
      if (lane == (TV_TC_SPLIT_PRODUCER ? 1 : 0) && i < v_stages && i >= npre_v) issue_v(i, ks, k_lo, zc);
    }
  if (warp >= 2) {
    if (!kEarlyRows) load_rows(b);
    // Q row -> swizzled smem (two 64-column boxes); rows past the tile are zero.
    // With TV_ATTN_ROPE the row is rotated to its tree position kv_len +
    // depth(u) on the way (pairs (i, i + 64) sit in chunks c and c + 8).
    const bool rope = (p.flags & TV_ATTN_ROPE) != 0;
    const int pos = (rope && row_ok) ? kl + depth_u : 0;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint4 lo = qv[c], hi = qv[c + 8];
      if (row_ok && rope) rope_rotate8(lo, hi, pos, p.rope.f, 8 * c);
      *reinterpret_cast<uint4*>(q_pipe + r * 128 + ((c ^ (r & 7)) << 4)) = lo;
      *reinterpret_cast<uint4*>(q_pipe + kRows * 128 + r * 128 + ((c ^ (r & 7)) << 4)) = hi;
    }
    fence_async_smem();  // generic-proxy stores -> visible to the tensor core after the barrier
  }
  if (warp == 1) {
    __syncwarp();  // tcgen05.alloc is warp-collective
    tmem_alloc(&sh->tmem_base, kTmemCols * NQ);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  const uint32_t t_s0 = tmem + tq, t_o = tmem + tq + 128;  // this warp's pipe

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    // K_i waits for S_{i-k_stages} to finish, V_i for PV_{i-v_stages}; each
    // stream completes in the order it is issued, so a wait never blocks early.
    // Lane 0 streams K and lane 1 streams V (with a single producer, lane 0
    // streams both, interleaved).
    constexpr bool kSplit = TV_TC_SPLIT_PRODUCER != 0;
    if (lane < (kSplit ? 2 : 1)) {
      bool to = false;
      for (int st = 0; st < 2; ++st) {
        if (kSplit && st != lane) continue;
        const bool is_k = st == 0;
        const int stages = is_k ? k_stages : v_stages;
        uint64_t* full = is_k ? sh->k_full : sh->v_full;
        uint64_t* empty = is_k ? sh->k_empty : sh->v_empty;
        // the first ring's worth is already requested (or, for a sequence found
        // invalid after the grid dependency, only the tiles requested before it)
        int issued = ntiles > 0 ? min(ntiles, stages) : (is_k ? npre_k : npre_v);
        if (kSplit) {
          for (int i = stages; i < ntiles && !to; ++i) {
            if (!mbar_wait(&empty[i % stages], ((i / stages) - 1) & 1, lim)) {
              to = true;
              break;
            }
            if (is_k)
              issue_k(i, ks, k_lo, zc);
            else
              issue_v(i, ks, k_lo, zc);
            ++issued;
          }
        } else if (is_k) {
          // one thread, K and V interleaved tile by tile
          int v_issued = ntiles > 0 ? min(ntiles, v_stages) : npre_v;
          for (int i = 0; i < ntiles && !to; ++i) {
            if (i >= k_stages) {
              if (!mbar_wait(&sh->k_empty[i % k_stages], ((i / k_stages) - 1) & 1, lim)) {
                to = true;
                break;
              }
              issue_k(i, ks, k_lo, zc);
              ++issued;
            }
            if (i >= v_stages) {
              if (!mbar_wait(&sh->v_empty[i % v_stages], ((i / v_stages) - 1) & 1, lim)) {
                to = true;
                break;
              }
              issue_v(i, ks, k_lo, zc);
              ++v_issued;
            }
          }
          for (int i = max(0, v_issued - v_stages); i < v_issued; ++i)
            mbar_wait(&sh->v_full[i % v_stages], (i / v_stages) & 1);
        }
        // Every copy issued must land before the CTA's shared memory is
        // released, whether or not a consumer waited for it (a consumer that
        // gave up, or a sequence found invalid, leaves copies unconsumed).  The
        // last issued tile of each slot decides, so one wait per slot suffices.
        for (int i = max(0, issued - stages); i < issued; ++i) mbar_wait(&full[i % stages], (i / stages) & 1);
        if (!kSplit) break;  // the single producer handled V above
      }
      if (to) atomicExch(&sh->timed_out, 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (kQT && lane == 0 && ntiles > 0) {
      // S_i = Q K_i^T with Q from TMEM, then O += P_i V_i, tile by tile: S_{i+1}
      // overwrites S_i (and P_i) only after PV_i, which the tensor core runs
      // in issue order; the other CTA on the SM fills the tensor core while this
      // one's softmax works
      const uint32_t idesc_s = idesc_bf16(128, kKeyTile, 0);
      bool to = !mbar_wait(&sh->q_ready, 0, lim);
      tc_fence_after();
      for (int i = 0; i < ntiles && !to; ++i) {
        const int s = i % k_stages;
        if (!mbar_wait(&sh->k_full[s], (i / k_stages) & 1, lim)) {
          to = true;
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(k_ring + s * kTileBytes);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t db = sw128_desc(k_addr + (k >> 2) * kBoxBytes + (k & 3) * 32, 16);
          mma_ts(tmem, tmem + 64 + k * 8, db, idesc_s, k > 0 ? 1u : 0u);
        }
        tc_commit(&sh->s_full[0][0]);
        tc_commit(&sh->k_empty[s]);
        if (!issue_pv(sh, v_ring, tmem, 1, i, v_stages, lim, true)) to = true;
      }
      if (to) atomicExch(&sh->timed_out, 1);
      // Every MMA issued so far retires before TMEM and shared memory are
      // released, also when a softmax warp gave up before reading the last O.
      tc_commit(&sh->drain);
      mbar_wait(&sh->drain, 0);
    } else if (kPoll && lane == 0 && ntiles > 0) {
      // One query tile, two S buffers.  QK_j may go once K_j has landed and
      // PV_{j-2} is issued (it frees S[j % 2], which held P_{j-2}; the tensor
      // core runs MMAs in issue order); PV_j once QK_j is issued and P_j and
      // V_j are ready.  Polling both lets a late K tile hold back no PV and a
      // late V tile no QK.  The wait limit applies to time without progress.
      const uint32_t idesc_s = idesc_bf16(128, kKeyTile, 0);
      const uint32_t idesc_o = idesc_bf16(128, 128, 1);
      constexpr bool kDescStep = TV_TC_DESC_STEP != 0;
      const uint64_t dq0 = sw128_desc(smem_u32(q_s), 16);  // the query tile's first k-step
      int nqk = 0, npv = 0;
      bool to = false;
      uint64_t t_last = globaltimer_ns();
      uint32_t idle = 0;
      while (npv < ntiles) {
        bool progress = false;
        if (nqk < ntiles && nqk < npv + 2 &&
            mbar_test_wait(&sh->k_full[nqk % k_stages], (nqk / k_stages) & 1)) {
          tc_fence_after();
          const int s = nqk % k_stages, sb = nqk & 1;
          const uint32_t k_addr = smem_u32(k_ring + s * kTileBytes);
          if (kDescStep) {
            // the k-steps' descriptors differ from the tile's first one only in
            // the address field (16-byte units, bits 0-13; every address stays
            // below 256 KB, so the sum never carries out of the field): one add
            // per MMA keeps the issuing thread's dependent chain short
            const uint64_t dk0 = sw128_desc(k_addr, 16);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              mma_ss(tmem + sb * 64, dq0 + (uint64_t)((k >> 2) * (kRows * 128 / 16) + (k & 3) * 2),
                     dk0 + (uint64_t)((k >> 2) * (kBoxBytes / 16) + (k & 3) * 2), idesc_s, k > 0 ? 1u : 0u);
          } else {
            const uint32_t q_addr = smem_u32(q_s);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint64_t da = sw128_desc(q_addr + (k >> 2) * (kRows * 128) + (k & 3) * 32, 16);
              const uint64_t db = sw128_desc(k_addr + (k >> 2) * kBoxBytes + (k & 3) * 32, 16);
              mma_ss(tmem + sb * 64, da, db, idesc_s, k > 0 ? 1u : 0u);
            }
          }
          tc_commit(&sh->s_full[0][sb]);
          tc_commit(&sh->k_empty[s]);
          ++nqk;
          progress = true;
        }
        if (npv < nqk && mbar_test_wait(&sh->p_full[0][npv & 1], (npv >> 1) & 1) &&
            mbar_test_wait(&sh->v_full[npv % v_stages], (npv / v_stages) & 1)) {
          tc_fence_after();
          const int s = npv % v_stages, sb = npv & 1;
          const uint32_t v_addr = smem_u32(v_ring + s * kTileBytes);
          if (kDescStep) {
            const uint64_t dv0 = sw128_desc(v_addr, kBoxBytes);
#pragma unroll
            for (int kk = 0; kk < kKeyTile / 16; ++kk)
              mma_ts(tmem + 128, tmem + sb * 64 + kk * 8, dv0 + (uint64_t)(kk * (16 * 128 / 16)), idesc_o,
                     (npv > 0 || kk > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int kk = 0; kk < kKeyTile / 16; ++kk)
              mma_ts(tmem + 128, tmem + sb * 64 + kk * 8, sw128_desc(v_addr + kk * 16 * 128, kBoxBytes), idesc_o,
                     (npv > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(&sh->o_ready[0][npv & 1]);
          tc_commit(&sh->v_empty[s]);
          ++npv;
          progress = true;
        }
        if (progress) {
          idle = 0;
          t_last = globaltimer_ns();
        } else if (++idle >= 64) {
          idle = 0;
          if (globaltimer_ns() - t_last > lim) {
            to = true;
            break;
          }
        }
      }
      if (to) atomicExch(&sh->timed_out, 1);
      // Every MMA issued so far retires before TMEM and shared memory are
      // released, also when a softmax warp gave up before reading the last O.
      tc_commit(&sh->drain);
      mbar_wait(&sh->drain, 0);
    } else if (!kQT && !kPoll && lane == 0 && ntiles > 0) {
      const uint32_t idesc_s = idesc_bf16(128, kKeyTile, 0);
      bool to = false;
      for (int i = 0; i < ntiles && !to; ++i) {
        const int s = i % k_stages, sb = i & 1;
        if (!mbar_wait(&sh->k_full[s], (i / k_stages) & 1, lim)) {
          to = true;
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(k_ring + s * kTileBytes);
        for (int q = 0; q < nq; ++q) {  // S_q = Q_q K^T, every pipe on the same K tile
          const uint32_t q_addr = smem_u32(q_s + q * kQBytes);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint64_t da = sw128_desc(q_addr + (k >> 2) * (kRows * 128) + (k & 3) * 32, 16);
            const uint64_t db = sw128_desc(k_addr + (k >> 2) * kBoxBytes + (k & 3) * 32, 16);
            mma_ss(tmem + q * kTmemCols + sb * 64, da, db, idesc_s, k > 0 ? 1u : 0u);
          }
          tc_commit(&sh->s_full[q][sb]);
        }
        tc_commit(&sh->k_empty[s]);
        if (i >= 1 && !issue_pv(sh, v_ring, tmem, nq, i - 1, v_stages, lim)) to = true;
      }
      if (!to && !issue_pv(sh, v_ring, tmem, nq, ntiles - 1, v_stages, lim)) to = true;
      if (to) atomicExch(&sh->timed_out, 1);
      // Every MMA issued so far retires before TMEM and shared memory are
      // released, also when a softmax warp gave up before reading the last O.
      tc_commit(&sh->drain);
      mbar_wait(&sh->drain, 0);
    }
  }

  // ------------------------------------------------------------------ softmax warps
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  float m = -INFINITY, l = 0.f;
  bool have = false;
  const bool warp_live = __any_sync(0xffffffffu, row_ok);  // some row of this warp is real
  if (kQT && warp >= 2) {
    // this thread's Q row (staged in shared memory before the allocation;
    // zero for padding rows) -> TMEM columns [64, 128) of its lane, as bf16
    // pairs: column j holds elements (2j, 2j+1), the A-operand layout
    uint32_t qr[32];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 v4 = *reinterpret_cast<const uint4*>(q_pipe + h * kRows * 128 + r * 128 + ((c ^ (r & 7)) << 4));
        qr[4 * c] = v4.x;
        qr[4 * c + 1] = v4.y;
        qr[4 * c + 2] = v4.z;
        qr[4 * c + 3] = v4.w;
      }
      tmem_st32(t_s0 + lane_off + 64 + h * 32, qr);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sh->q_ready);
  }
  if (warp >= 2 && pipe < nq) {
    bool to = false;
    for (int i = 0; i < ntiles; ++i) {
      const int sb = kQT ? 0 : (i & 1);
      // every wait that gates a TMEM access is decided for the whole warp: the
      // tcgen05.ld / tcgen05.st that follow are warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(&sh->s_full[pipe][sb], kQT ? (i & 1) : ((i >> 1) & 1), lim))) {
        to = true;
        break;
      }
      tc_fence_after();
      const int key0 = k_lo + i * kKeyTile;
      // a warp made only of padding rows (zero queries, so zero scores and a zero
      // P already in TMEM) has nothing to compute
      if (warp_live) {
        uint32_t sr[2][32];
        tmem_ld32(t_s0 + lane_off + sb * 64, sr[0]);
        tmem_ld32(t_s0 + lane_off + sb * 64 + 32, sr[1]);
        tmem_wait_ld();
        float x[64];  // raw scores; the scale is folded into the exponent's FFMA
#pragma unroll
        for (int j = 0; j < 64; ++j) x[j] = __uint_as_float(sr[j >> 5][j & 31]);
        if (key0 + kKeyTile > kl) {  // tile reaches the tree rows or the end of the range
          const int np = kl - key0;  // prefix keys in this tile
          const uint64_t pre = np >= 64 ? ~0ull : (np <= 0 ? 0ull : ((1ull << np) - 1ull));
          const uint64_t allowed = pre | anc_window(anc_w, key0 - kl);
#pragma unroll
          for (int j = 0; j < 64; ++j)
            if (!((allowed >> j) & 1ull)) x[j] = -INFINITY;
        }
        // row maximum: four chains of three-input maxima over the 64 scores
        float c4[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
        for (int q = 0; q < 30; ++q) c4[q & 3] = fmax3(c4[q & 3], x[4 + 2 * q], x[5 + 2 * q]);
        const float mx = fmaxf(fmax3(c4[0], c4[1], c4[2]), c4[3]) * p.scale_log2;
        // Lazy rescale: a row moves its reference maximum only when the tile's
        // maximum exceeds it by more than the threshold (always on its first
        // finite tile, where m = -inf).  Rescaling O is a TMEM access, which is
        // warp-collective, so the warp rescales when any of its rows needs it,
        // each row by its own factor (1 for a row whose maximum stays, and for
        // a row with no finite score yet, whose O row is still zero).
        const bool grow = mx > m + kRescaleThreshold;
        const bool scale_o = grow && m != -INFINITY;
        if (__any_sync(0xffffffffu, scale_o)) {
          // O holds earlier tiles: rescale once PV_{i-1} has landed
          if (!__all_sync(0xffffffffu, mbar_wait(&sh->o_ready[pipe][(i - 1) & 1], ((i - 1) >> 1) & 1, lim))) {
            to = true;
            break;
          }
          tc_fence_after();
          const float corr = scale_o ? fast_exp2(m - mx) : 1.f;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(t_o + lane_off + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * corr);
            tmem_st32(t_o + lane_off + c * 32, o);
          }
          tmem_wait_st();
          l *= corr;
        }
        if (grow) m = mx;
        const float ms = m == -INFINITY ? 0.f : m;
        // exponent argument and row sum two keys at a time (packed FP32 pairs)
        uint32_t pk[32];
        const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2), nm2 = f2_pack(-ms, -ms);
        uint64_t rs2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const uint64_t arg = f2_fma(f2_pack(x[2 * j], x[2 * j + 1]), sc2, nm2);
          float p0, p1;
          if ((j & 7) < TV_TC_POLY_EXP_PAIRS) {  // a share of the pairs on the FMA pipe
            f2_unpack(f2_exp2_poly(arg), p0, p1);
          } else {
            float a0, a1;
            f2_unpack(arg, a0, a1);
            p0 = fast_exp2(a0);
            p1 = fast_exp2(a1);
          }
          rs2[j & 3] = f2_add(rs2[j & 3], f2_pack(p0, p1));
          pk[j] = pack_bf16x2(p0, p1);
        }
        {
          float s0, s1, s2, s3, s4, s5, s6, s7;
          f2_unpack(rs2[0], s0, s1);
          f2_unpack(rs2[1], s2, s3);
          f2_unpack(rs2[2], s4, s5);
          f2_unpack(rs2[3], s6, s7);
          l += ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7));
        }
        tmem_st32(t_s0 + lane_off + sb * 64, pk);
        tmem_wait_st();
      }
      // past the end of the key range the V rows may hold anything: zero them
      const int kend = N - key0;
      if (kend < kKeyTile && pipe == 0) {  // pipe 0 zeroes; every PV on this tile waits for it
        uint8_t* vt = v_ring + (i % v_stages) * kTileBytes;
        if (!__all_sync(0xffffffffu, mbar_wait(&sh->v_full[i % v_stages], (i / v_stages) & 1, lim))) {
          to = true;  // V_i must have landed before its rows are overwritten
          break;
        }
        const int first = max(kend, 0);
        for (int idx = r; idx < (kKeyTile - first) * 16; idx += kRows) {
          const int row = first + idx / 16, c = idx % 16;
          *reinterpret_cast<uint4*>(vt + (c >> 3) * kBoxBytes + row * 128 + (((c & 7) ^ (row & 7)) << 4)) =
              make_uint4(0, 0, 0, 0);
        }
        fence_async_smem();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->p_full[pipe][sb]);
    }
    if (to) atomicExch(&sh->timed_out, 1);
    have = __all_sync(0xffffffffu, ntiles > 0 && !to && warp_live);
    if (ntiles > 0 && !to) {
      if (!mbar_wait(&sh->o_ready[pipe][(ntiles - 1) & 1], ((ntiles - 1) >> 1) & 1, lim)) {
        atomicExch(&sh->timed_out, 1);
        have = false;
      }
      tc_fence_after();
    }
    have = __all_sync(0xffffffffu, have);  // gates warp-collective TMEM reads
    if (p.nsplit == 1) {
      // normalised bf16 row -> smem (the Q tile is dead once the last MMA is done),
      // then the four warps copy whole rows out with coalesced 16-byte stores
      const float inv = (have && valid && l > 0.f) ? 1.f / l : 0.f;
      uint8_t* ost = q_pipe;  // [128 rows][256 B], 16-byte chunks rotated by row
      if (warp_live) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          if (have) {
            tmem_ld32(t_o + lane_off + c * 32, o);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = 0u;
          }
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[8 * q4 + 0]) * inv, __uint_as_float(o[8 * q4 + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(o[8 * q4 + 2]) * inv, __uint_as_float(o[8 * q4 + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(o[8 * q4 + 4]) * inv, __uint_as_float(o[8 * q4 + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(o[8 * q4 + 6]) * inv, __uint_as_float(o[8 * q4 + 7]) * inv);
            const int chunk = c * 4 + q4;
            *reinterpret_cast<uint4*>(ost + r * 256 + ((chunk ^ (r & 15)) << 4)) = w;
          }
        }
      }
      asm volatile("bar.sync %0, 128;" ::"r"(1 + pipe) : "memory");  // the four softmax warps of this pipe
      const int rows = min(kRows, p.rows_total - qtile * kRows);
      const int t = ((warp - 2) & 3) * 32 + lane;
      for (int idx = t; idx < rows * 16; idx += 128) {
        const int rr = idx >> 4, chunk = idx & 15;
        const int g2 = qtile * kRows + rr;
        const int64_t orow = (((int64_t)b * (p.M + 1) + g2 / p.G) * p.Hq + hk * p.G + g2 % p.G) * 128;
        reinterpret_cast<uint4*>(p.out + orow)[chunk] =
            *reinterpret_cast<const uint4*>(ost + rr * 256 + ((chunk ^ (rr & 15)) << 4));
      }
    }
  }

  if (p.nsplit > 1) {
    // ---------------------------------------------------------------- split merge
    // Each split writes (max, sum, O) of its real rows to the workspace (L2),
    // the cluster barrier orders the writes, and every CTA then merges its
    // share of the rows from the other splits' records.
    cg::cluster_group cluster = cg::this_cluster();
    const int ns = p.nsplit;
    // records per query tile (unit = (sequence, kv head, query tile)); chunk-major
    // ([32 float4 chunks][128 rows]) so that a warp's 32 rows write, and read
    // back, 512 contiguous bytes
    const size_t n_units = (size_t)p.B * p.Hkv * tiles_q;
    auto rec_o = [&](int qt) {
      return reinterpret_cast<float4*>(p.ws) + ((size_t)bh * tiles_q + qt) * ns * 32 * kRows;
    };
    auto rec_ml = [&](int qt) {
      return reinterpret_cast<float2*>(p.ws + n_units * ns * kRows * 128) + ((size_t)bh * tiles_q + qt) * ns * kRows;
    };
    float4* ws_o = rec_o(qtile);
    float2* ws_ml = rec_ml(qtile);
    if (warp >= 2 && warp_live) {
      float4* dst = ws_o + (size_t)split * 32 * kRows + r;
#pragma unroll
      for (int c = 0; c < 4; c += 2) {
        uint32_t o[2][32];
        if (have) {  // warp-uniform: the TMEM reads are warp-collective
          tmem_ld32(t_o + lane_off + c * 32, o[0]);
          tmem_ld32(t_o + lane_off + (c + 1) * 32, o[1]);
          tmem_wait_ld();
        } else {  // an empty split contributes zeros (its weight is 0 as well)
#pragma unroll
          for (int j = 0; j < 32; ++j) o[0][j] = o[1][j] = 0u;
        }
        if (row_ok) {
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              __stcg(dst + ((c + h) * 8 + q4) * kRows,
                     make_float4(__uint_as_float(o[h][4 * q4]), __uint_as_float(o[h][4 * q4 + 1]),
                                 __uint_as_float(o[h][4 * q4 + 2]), __uint_as_float(o[h][4 * q4 + 3])));
        }
      }
      if (row_ok) __stcg(ws_ml + (size_t)split * kRows + r, make_float2(have ? m : -INFINITY, have ? l : 0.f));
    }
    // barrier.cluster.arrive releases and barrier.cluster.wait acquires at
    // cluster scope, which orders the records' global stores for every CTA of
    // the cluster: no separate device-scope fence is needed
    tc_fence_before();
    cluster.sync();  // every split's record is written
    const int rank = (int)cluster.block_rank();
    // rank j merges chunks [q_lo, q_hi) of every real row of every query tile of
    // the CTA; consecutive threads take consecutive rows, so each split's
    // record is read with coalesced loads
    const int q_lo = rank * 32 / ns, q_hi = (rank + 1) * 32 / ns;
    for (int mq = 0; mq < nq; ++mq) {
    const int mtile = qtile0 + mq;
    const int rows = min(kRows, p.rows_total - mtile * kRows);  // real rows of this tile
    const float4* mo = rec_o(mtile);
    const float2* mml = rec_ml(mtile);
    for (int idx = threadIdx.x; idx < (q_hi - q_lo) * rows; idx += blockDim.x) {
      const int rr = idx % rows;
      const int q = q_lo + idx / rows;
      const int g2 = mtile * kRows + rr;
      float2 ml[kMaxSplit_tc];
      float4 oj[kMaxSplit_tc];
#pragma unroll
      for (int j = 0; j < kMaxSplit_tc; ++j) {
        if (j < ns) {
          ml[j] = __ldcg(mml + (size_t)j * kRows + rr);
          oj[j] = __ldcg(mo + ((size_t)j * 32 + q) * kRows + rr);
        } else {
          ml[j] = make_float2(-INFINITY, 0.f);
          oj[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      float mmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < kMaxSplit_tc; ++j) mmax = fmaxf(mmax, ml[j].x);
      const float msafe = mmax == -INFINITY ? 0.f : mmax;
      float L = 0.f;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int j = 0; j < kMaxSplit_tc; ++j) {
        const float w = fast_exp2(ml[j].x - msafe);  // 0 for an empty split
        L += w * ml[j].y;
        a.x += w * oj[j].x;
        a.y += w * oj[j].y;
        a.z += w * oj[j].z;
        a.w += w * oj[j].w;
      }
      const float inv = (valid && L > 0.f) ? 1.f / L : 0.f;
      const int64_t orow = (((int64_t)b * (p.M + 1) + g2 / p.G) * p.Hq + hk * p.G + g2 % p.G) * 128;
      uint2 pk;
      pk.x = pack_bf16x2(a.x * inv, a.y * inv);
      pk.y = pack_bf16x2(a.z * inv, a.w * inv);
      *reinterpret_cast<uint2*>(p.out + orow + q * 4) = pk;
    }
    }
  } else {
    tc_fence_before();
    __syncthreads();
  }
  if (warp == 1) {
    __syncwarp();  // tcgen05.dealloc is warp-collective
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols * NQ);
  }
  if (threadIdx.x == 0 && (sh->timed_out || !aligned_ok)) atomicOr(&p.status[b], kSeqTimeout);
  if (threadIdx.x == 0 && (broken_promise || sl < 0)) atomicOr(&p.status[b], kSeqBadGeometry);
  if (threadIdx.x == 0 && order_changed)
    for (int i = 0; i < p.B; ++i) atomicOr(&p.status[i], kSeqBadGeometry);
}

}  // namespace

tv_status plan_attention_tc(int B, int M, int Hq, int Hkv, int64_t S_cap, TcPlan& lp) {
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda_error(e);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int rows_total = (Hq / Hkv) * (M + 1);
  lp.tiles_q = (rows_total + kRows - 1) / kRows;
  // Two query tiles per CTA (TV_TC_PAIR) when a (sequence, kv head) has two or
  // more: every K/V tile brought into shared memory then serves both, halving
  // the K/V traffic from L2.  Measured slower on B200 (b32gqa 252 vs 162 us,
  // stress 2.41 vs 1.63 ms per launch: one CTA per SM with two pipes loses to
  // two CTAs per SM with one pipe each), so it is off by default.
  lp.nq = (TV_TC_PAIR && lp.tiles_q >= 2) ? 2 : 1;
  const int grid_y = (lp.tiles_q + lp.nq - 1) / lp.nq;
  const int64_t units = (int64_t)B * Hkv * lp.tiles_q;  // query tiles (workspace records)
  const int64_t ctas_per_split = (int64_t)B * Hkv * grid_y;
  const int key_tiles = (int)std::max<int64_t>(1, (S_cap + kKeyTile - 1) / kKeyTile);
  // Split the key range while the query tiles alone leave SMs idle: a split
  // adds a merge, and past the resident CTAs it adds a partial wave.
  const int64_t cap = lp.nq == 2 ? sms : (int64_t)TV_TC_SPLIT_FACTOR * sms;  // CTAs that fit at once
  int ns = ctas_per_split >= sms ? 1
                                 : (int)std::min<int64_t>(kMaxSplit_tc, std::max<int64_t>(1, cap / ctas_per_split));
  ns = std::min(ns, key_tiles);
  lp.tiles_per_split = (key_tiles + ns - 1) / ns;
  lp.nsplit = (key_tiles + lp.tiles_per_split - 1) / lp.tiles_per_split;
  if (lp.nq == 2) {
    // one CTA per SM (all 512 TMEM columns): deep rings
    lp.stages = std::min(4, std::max(2, lp.tiles_per_split));
    lp.v_stages = std::min(5, std::max(2, lp.tiles_per_split));
    lp.smem = 2 * (size_t)kQBytes + (size_t)(lp.stages + lp.v_stages) * kTileBytes + sizeof(TcSmem);
    lp.per_sm = 1;
  } else {
    // Deepest ring that keeps the grid resident: two CTAs per SM when the grid
    // needs it (each then holds 256 of the 512 TMEM columns, so an allocation
    // never waits on a CTA that is itself waiting), else one CTA per SM.
    const int64_t ctas = ctas_per_split * lp.nsplit;
    const bool two_per_sm = !TV_TC_FORCE_SOLO && (!TV_TC_ONE_PER_SM || ctas > sms);
    lp.per_sm = two_per_sm ? 2 : 1;
    // two CTAs per SM: K and V rings of TV_TC_K_RING_DUO / TV_TC_V_RING_DUO slots
    // (Q 32 KB + up to 5 x 16 KB fits twice in an SM);
    // one CTA per SM: deeper rings
    lp.stages = two_per_sm ? TV_TC_K_RING_DUO : std::min(TV_TC_K_RING_SOLO, std::max(2, lp.tiles_per_split));
    lp.v_stages = two_per_sm ? TV_TC_V_RING_DUO : std::min(TV_TC_V_RING_SOLO, std::max(2, lp.tiles_per_split));
    const size_t smem_min = two_per_sm ? 0 : (size_t)120 * 1024;  // > half the SM: one CTA per SM
    lp.smem = std::max(smem_min, kQBytes + (size_t)(lp.stages + lp.v_stages) * kTileBytes + sizeof(TcSmem));
  }
  lp.ws_bytes = lp.nsplit > 1 ? (size_t)units * lp.nsplit * kRows * (128 + 2) * sizeof(float) : 0;
  return TV_OK;
}

tv_status run_attention_tc(const CUtensorMap& tmk, const CUtensorMap& tmv, AttnParams p, const TcPlan& lp,
                           cudaStream_t s) {
  p.tiles_per_split = lp.tiles_per_split;
  p.nsplit = lp.nsplit;
  p.stages = lp.stages;
  p.v_stages = lp.v_stages;
  if ((int64_t)p.B * p.Hkv > 65535 || lp.tiles_q > 65535) return TV_ERR_UNSUPPORTED;
  const int grid_y = (lp.tiles_q + lp.nq - 1) / lp.nq;
  dim3 grid(lp.nsplit, grid_y, p.B * p.Hkv);  // unit-major; query-tile-major below for one wave
  const int threads = 64 + 128 * lp.nq;
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda_error(e);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // The instance: blocks in longest-first order only when not every block
  // starts at once (more blocks than the plan's resident CTAs) and the batch is
  // small enough to rank in one warp.
  auto occupancy = [&](auto kern, int& occ) {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)lp.smem);
    if (err != cudaSuccess) return err;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, threads, lp.smem);
  };
  int occ = 0;
  e = lp.nq == 2 ? occupancy(tree_attn_tc_kernel<2, false>, occ) : occupancy(tree_attn_tc_kernel<1, false>, occ);
  if (e != cudaSuccess) return record_cuda_error(e);
  // multi-wave instance (unit-major, longest first) for one-tile CTAs whose grid
  // exceeds the plan's resident CTAs; the single-wave instance otherwise
  const bool lf = lp.nq == 1 && (int64_t)grid.x * grid.y * grid.z > (int64_t)lp.per_sm * sms;
  if (lf) {
    e = occupancy(tree_attn_tc_kernel<1, true>, occ);
    if (e != cudaSuccess) return record_cuda_error(e);
  }
  // TMEM: 256 columns per query tile; never more CTAs on an SM than 512 columns hold
  if (occ < 1 || occ * lp.nq > 2) return TV_ERR_UNSUPPORTED;
  auto kern = lp.nq == 2 ? tree_attn_tc_kernel<2, false>
                         : (lf ? tree_attn_tc_kernel<1, true> : tree_attn_tc_kernel<1, false>);
  if (!lf && TV_TC_TILE_MAJOR) grid = dim3(lp.nsplit, p.B * p.Hkv, grid_y);
  return launch(kern, grid, dim3(threads), lp.smem, s, lp.nsplit, true, tmk, tmv, p);
}

}  // namespace tv
