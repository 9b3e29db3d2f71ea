/*
 * treeverify.h -- C ABI of the teacher-side verification step of tree
 * speculative decoding, for NVIDIA B200 (sm_100a).
 *
 * The step, as the pages state it:
 *   "EAGLE-Pangu: Accelerator-Safe Tree Speculative Decoding on Ascend NPUs"
 *     methodology B  sentinel-free tree tensors: a dummy root at row 0, every
 *                    parent pointer in [0, M], invariants (in range, acyclic)
 *                    checked before the fused kernels run;
 *     methodology C  one batched teacher pass over all speculative tokens with a
 *                    tree mask: node k attends node j only if j is an ancestor
 *                    of k (itself included);
 *     methodology A  path-index commit: the new cache segment is reordered by
 *                    the accepted path ("fast reorder");
 *     results        accepted length per verification step (greedy agreement).
 *   "Batch Speculative Decoding Done Right"
 *     methodology    EQSPEC unpad-append-repad, keeping rectangular alignment
 *                    (pad + length = batch maximum) and position IDs contiguous
 *                    from 0 over the attended positions.
 *
 * Conventions shared by every call
 *   - Every tensor pointer is a DEVICE pointer owned by the caller.  Nothing is
 *     allocated, nothing is kept between calls.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; 0 = legacy default
 *     stream) and never synchronises.  The return value reports only argument
 *     errors and launch errors, detected synchronously on the host.
 *   - Data-dependent errors are reported on the device, per sequence, in the
 *     int32 `status[B]` array (bit flags below).  A sequence with status != 0
 *     gets zero attention rows, accept_len = -1 with a zero path, and commits
 *     nothing (in left-padded mode it is still shifted to keep the batch
 *     rectangular).
 *   - Indices are int32 and never negative (except accept_len = -1); padding of
 *     index arrays uses 0, the dummy root, so any gather stays in bounds.
 *   - Trees have M+1 rows: row 0 is the dummy root (the last emitted token, not
 *     yet in the cache), rows 1..M are draft nodes, parent[0] = 0 and
 *     0 <= parent[i] < i.
 *   - bf16 tensors are passed as uint16_t bit patterns.
 *   - KV cache of one layer: [B][Hkv][S_cap][D] bf16.  Sequence b's committed
 *     prefix is columns [kv_start[b], kv_start[b] + kv_len[b]); the M+1 tree
 *     rows of the current step sit right behind it, at columns
 *     kv_start[b] + kv_len[b] + r, r = 0..M (written by the caller, or by
 *     tree_kv_write from a [L][B][Hkv][M+1][D] staging buffer).  A sequence whose geometry breaks
 *     0 <= kv_start, 0 <= kv_len, kv_start + kv_len + M + 1 <= S_cap is flagged
 *     TV_SEQ_BAD_GEOMETRY and skipped.
 */
#ifndef TREEVERIFY_H
#define TREEVERIFY_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* cudaStream_t without pulling in the CUDA headers. */
typedef struct CUstream_st* tv_stream_t;

typedef enum {
  TV_OK = 0,
  TV_ERR_INVALID_ARG = 1, /* null pointer, negative size, misaligned pointer, bad combination */
  TV_ERR_UNSUPPORTED = 2, /* valid but outside what the kernels implement (e.g. D not 64/128) */
  TV_ERR_CUDA = 3         /* a CUDA runtime call or launch failed; see tv_last_cuda_error() */
} tv_status;

/* per-sequence device status bits */
#define TV_SEQ_BAD_PARENT 1   /* parent[0] != 0, or parent[i] outside [0, i) */
#define TV_SEQ_TOO_DEEP 2     /* some node deeper than max_depth */
#define TV_SEQ_TIMEOUT 4      /* a bounded device wait gave up (the sequence's outputs are void) */
#define TV_SEQ_BAD_GEOMETRY 8 /* kv_start / kv_len / S_cap inconsistent with M+1 tree rows */

/* Largest tree the kernels take: M + 1 <= TV_MAX_TREE_ROWS. */
#define TV_MAX_TREE_ROWS 256

/*
 * tree_build_mask -- validate sentinel-free parent arrays and expand them into
 * ancestor bitmasks.  [EAGLE-Pangu, methodology B (dummy-root indexing,
 * ancestor tables, invariant checks) and C (tree attention mask).]
 *
 *   parent    int32 [B][M+1]   in
 *   anc_mask  uint32 [B][M+1][W], W = ceil((M+1)/32)   out: bit r of row u is
 *             set iff row r lies on the root..u path, u included
 *   depth     int32 [B][M+1]   out: edges from the root (root = 0)
 *   status    int32 [B]        out: 0, or TV_SEQ_BAD_PARENT / TV_SEQ_TOO_DEEP;
 *             a flagged sequence gets all-zero mask and depth rows
 *   B >= 0, 0 <= M < TV_MAX_TREE_ROWS, max_depth >= 0.
 */
tv_status tree_build_mask(const int32_t* parent, int B, int M, int max_depth, uint32_t* anc_mask,
                          int32_t* depth, int32_t* status, tv_stream_t stream);

/*
 * tree_attention -- tree-masked GQA attention of the M+1 tree queries of every
 * sequence over its committed prefix plus its tree rows.  [EAGLE-Pangu,
 * methodology C: one batched pass over all speculative tokens; node u attends
 * the whole prefix, and inside the tree only rows whose bit is set in
 * anc_mask[b][u].]
 *
 *   q         bf16 [B][M+1][Hq][D]       in (post-RoPE)
 *   k, v      bf16 [B][Hkv][S_cap][D]    in (one layer); 16-byte aligned
 *   kv_start, kv_len  int32 [B]          in
 *   anc_mask  uint32 [B][M+1][W]         in (from tree_build_mask)
 *   status    int32 [B]                  in/out: sequences with status != 0 (or a
 *             bad cache geometry) get zero output rows; a device wait that timed
 *             out ORs in TV_SEQ_TIMEOUT
 *   out       bf16 [B][M+1][Hq][D]       out: softmax(q k^T * scale) v over the
 *             allowed keys, fp32 accumulation
 *   workspace device scratch of at least tree_attention_workspace_size(...)
 *             bytes (16-byte aligned; may be NULL when that size is 0).  It holds
 *             the partial results of the key splits of one call; its contents
 *             need no initialisation and are dead after the call.  Calls that
 *             overlap on the device must not share a workspace.
 *   flags     0 or an OR of TV_ATTN_PREFIX_READY and TV_ATTN_ROPE (below); any
 *             other bit is an argument error
 *   depth     int32 [B][M+1] node depths (from tree_build_mask); read only with
 *             TV_ATTN_ROPE, may be NULL otherwise
 *   rope_theta  rotary base (> 1, e.g. 10000), TV_ATTN_ROPE only
 *   slot, n_slots  optional cache-slot map (see "Slot map" below); slot = NULL
 *             means batch row b uses cache slot b (n_slots is then ignored)
 *   D in {64, 128}; Hq % Hkv == 0 (q head h reads kv head h / (Hq/Hkv));
 *   scale > 0 (normally 1/sqrt(D)).
 * Contract: the K/V rows inside each sequence's key range hold finite values.
 */
size_t tree_attention_workspace_size(int B, int M, int Hq, int Hkv, int D, int64_t S_cap);

/*
 * TV_ATTN_PREFIX_READY -- the caller promises that the kernel launched just
 * before this call on the same stream writes neither kv_start / kv_len nor any
 * K/V column of the committed prefixes (it may write q, the tree rows, the
 * ancestor masks, the depths or the status; not the slot map).  That holds for
 * the attention call of the next layer, and after tree_kv_write or
 * tree_build_mask.  The kernel may then read
 * the geometry and start streaming prefix K/V tiles while that launch is still
 * running; the tree rows, q, the masks and the status are read only after it
 * has finished.  If the geometry turns out to have changed anyway, the affected
 * sequences get zero rows and TV_SEQ_BAD_GEOMETRY instead of a wrong result
 * (every sequence of the batch, when a length changed under a grid of more
 * than one wave, whose blocks are ordered by length).  Never set it right
 * after kv_commit_realign, which rewrites both.  The head dim 64 kernel
 * ignores the flag.  On B200 it measured no faster than a plain launch (0 to
 * 14 % slower: the early tile requests compete with the launch still
 * running), so this library's step drivers leave it off.
 */
#define TV_ATTN_PREFIX_READY 1u

/*
 * TV_ATTN_ROPE -- q is given before its rotary position embedding: each query
 * row of node u is rotated to position kv_len[b] + depth[b][u] while it is
 * staged (the tree positions of "Batch Speculative Decoding Done Right",
 * methodology: position-ID contiguity -- the prefix holds positions 0 ..
 * kv_len-1 and every root-to-node path continues it without a gap).  Rotation:
 * the pair (x[i], x[i + D/2]), i < D/2, turns by pos * rope_theta^(-2i/D)
 * (half-split rotary embedding); the rotated row is rounded to bf16.  The keys
 * are used as stored: write the tree rows with tree_kv_write's rotation.  Head
 * dim 128 only (TV_ERR_UNSUPPORTED for 64).
 */
#define TV_ATTN_ROPE 2u

/*
 * Slot map (tree_attention, tree_kv_write, kv_commit_realign).  With slot !=
 * NULL (int32 [B], device), the cache is a pool of n_slots sequences, each layer
 * bf16 [n_slots][Hkv][S_cap][D], and batch row b uses slot slot[b]; kv_start,
 * kv_len (and attn_mask / pos_ids rows) are indexed by slot, [n_slots], while
 * the step's per-row arrays (q, out, parent, anc_mask, depth, status, path,
 * accept_len, tree rows) stay indexed by batch row.  A batch can so be any set
 * of the pool's sequences without moving their caches (the cross-batch
 * scheduling of "Batch Speculative Decoding Done Right", methodology: EXSPEC
 * groups sequences of equal length).  The slots of one batch must be distinct;
 * a slot outside [0, n_slots) gets TV_SEQ_BAD_GEOMETRY and is skipped.
 */

tv_status tree_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t S_cap,
                         const int32_t* kv_start, const int32_t* kv_len, const uint32_t* anc_mask,
                         int32_t* status, int B, int M, int Hq, int Hkv, int D, float scale,
                         uint16_t* out, void* workspace, size_t workspace_bytes, unsigned flags,
                         const int32_t* depth, float rope_theta, const int32_t* slot, int n_slots,
                         tv_stream_t stream);

/*
 * tree_attention_noalloc -- tree_attention for callers that cannot allocate
 * device memory (for instance a serving process whose memory pool already owns
 * the whole GPU, or a plugin whose host framework gives it no device
 * allocator).  The pages have no counterpart: this is a deployment variant.
 *
 * Same arguments, layouts and results as tree_attention, without the
 * workspace: the key-split partials go to a fixed scratch array of
 * tree_attention_noalloc_max_scratch() bytes (32 MiB) compiled into the
 * library, which every GPU that loads the library holds until the process
 * exits.  A shape whose tree_attention_workspace_size exceeds that maximum is
 * rejected with TV_ERR_UNSUPPORTED; on a 148-SM GPU none does (splits are
 * added only while query tiles x splits stays within 2 CTAs per SM, so the
 * partials stay within 2 x SMs x 128 rows x 130 floats = 19.7 MB on 148 SMs).
 * Nothing is allocated: the first call on a device only looks up the array's
 * device address and caches it (make that first call before any stream
 * capture).  The cache assumes one primary context per device for the life of
 * the process: after a cudaDeviceReset the address is stale, so do not call
 * this entry point on a device that was reset.  All calls share the one array,
 * so calls that overlap on the device race with each other; each call
 * overwrites what it reads, so no clearing is needed between calls.  The
 * launch flags of tree_attention are not offered here (flags = 0).
 */
size_t tree_attention_noalloc_max_scratch(void);

tv_status tree_attention_noalloc(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t S_cap,
                                 const int32_t* kv_start, const int32_t* kv_len, const uint32_t* anc_mask,
                                 int32_t* status, int B, int M, int Hq, int Hkv, int D, float scale,
                                 uint16_t* out, tv_stream_t stream);

/*
 * tree_accept -- per-node greedy argmax of the teacher logits fused with
 * longest accepted path selection.  [EAGLE-Pangu, results: accepted length per
 * verification step.]  Node i is accepted iff its parent is accepted and
 * draft[i] == argmax[parent[i]]; the root is always accepted.  The committed
 * endpoint e is the deepest accepted node, lowest row index on ties.
 *
 *   logits     fp32 [B][M+1][V]   in (row u predicts the children of node u)
 *   draft      int32 [B][M+1]     in (draft token of node i; row 0 ignored)
 *   parent, depth  int32 [B][M+1], anc_mask uint32 [B][M+1][W]   in
 *   status     int32 [B]          in/out: non-zero -> sequence rejected
 *   argmax     int32 [B][M+1]     out: first index of the row maximum
 *   accept_len int32 [B]          out: depth of e (accepted draft tokens), -1 if rejected
 *   path       int32 [B][max_depth+1]  out: path[j] = row of depth j on root..e, 0-padded
 *   bonus      int32 [B]          out: argmax[e] (the teacher's next token), 0 if rejected
 *   V >= 1; max_depth must be the value given to tree_build_mask.
 * Contract: logits are finite (NaN ordering is unspecified).
 */
tv_status tree_accept(const float* logits, const int32_t* draft, const int32_t* parent,
                      const int32_t* depth, const uint32_t* anc_mask, int32_t* status, int B, int M,
                      int V, int max_depth, int32_t* argmax, int32_t* accept_len, int32_t* path,
                      int32_t* bonus, tv_stream_t stream);

/*
 * tree_accept_lm_head -- tree_accept with the teacher's LM head fused in: the
 * logits logit[b][u][v] = sum_h hidden[b][u][h] * w_lm[v][h] are formed tile by
 * tile on the tensor cores and reduced to their first maximum on the spot, so
 * the [B][M+1][V] logits are never written; the acceptance walk then runs as in
 * tree_accept.  [EAGLE-Pangu, methodology C: one batched teacher pass over all
 * speculative tokens, whose greedy choice at each node is the argmax of its
 * logits; results: accepted length per verification step.]
 *
 *   hidden     bf16 [B][M+1][H]   in (final hidden state of every tree node),
 *              16-byte aligned
 *   w_lm       bf16 [V][H]        in (LM-head weights), 16-byte aligned
 *   draft, parent, depth, anc_mask, status, argmax, accept_len, path, bonus:
 *              as for tree_accept (argmax = first index of the row maximum of
 *              the fp32-accumulated logits)
 *   workspace  device scratch of tree_accept_lm_head_workspace_size(B, M) bytes,
 *              8-byte aligned; no initialisation needed, dead after the call
 *   H a multiple of 64; V >= 1.
 * A tile whose pipeline wait gave up marks its rows' sequences TV_SEQ_TIMEOUT.
 */
size_t tree_accept_lm_head_workspace_size(int B, int M);

tv_status tree_accept_lm_head(const uint16_t* hidden, const uint16_t* w_lm, const int32_t* draft,
                              const int32_t* parent, const int32_t* depth, const uint32_t* anc_mask,
                              int32_t* status, int B, int M, int H, int V, int max_depth, int32_t* argmax,
                              int32_t* accept_len, int32_t* path, int32_t* bonus, void* workspace,
                              size_t workspace_bytes, tv_stream_t stream);

/*
 * kv_commit_realign -- commit the accepted path into the KV cache of every
 * layer and, in left-padded mode, repad the batch.  [EAGLE-Pangu, methodology A:
 * path-index commit; Batch Speculative Decoding Done Right, methodology:
 * EQSPEC unpad-append-repad and its two invariants.]
 *
 * For sequence b with n_b = accept_len[b] + 1 committed rows (0 if rejected):
 *   new content = old content ++ { tail row path[b][j] : j < n_b }, where the
 *   tail is the M+1 tree rows behind the content; kv_len[b] += n_b.
 *   realign = 0  per-sequence lengths: content stays at kv_start[b] (with a
 *                slot map, b's slot).
 *   realign = 1  left-padded: with Lmax' = max_b kv_len'[b], content moves to
 *                [Lmax' - kv_len'[b], Lmax'); kv_start'[b] = Lmax' - kv_len'[b].
 * All sources are read before they are overwritten (moves are in place).
 *
 *   k_layers, v_layers  DEVICE arrays of L device pointers, each to a
 *             bf16 [B][Hkv][S_cap][D] layer (16-byte aligned)
 *   path, accept_len, status   in (from tree_accept); status gains
 *             TV_SEQ_BAD_GEOMETRY for skipped sequences
 *   kv_start, kv_len  int32 [B]   in/out
 *   max_len   int32 [1]           out: max_b kv_start'[b] + kv_len'[b] over
 *             sequences with a valid geometry (Lmax' in left-padded mode)
 *   attn_mask uint8 [B][S_cap], pos_ids int32 [B][S_cap]   out, may be NULL:
 *             mask = 1 on the new content columns, pos = column - kv_start',
 *             0 elsewhere
 *   slot, n_slots  optional slot map (see tree_attention); with a map the
 *             repad is over the batch's sequences only and Lmax' is theirs
 */
tv_status kv_commit_realign(uint16_t* const* k_layers, uint16_t* const* v_layers, int L, int B,
                            int Hkv, int D, int64_t S_cap, int M, const int32_t* path,
                            const int32_t* accept_len, int32_t* status, int max_depth,
                            int32_t* kv_start, int32_t* kv_len, int32_t* max_len, int realign,
                            uint8_t* attn_mask, int32_t* pos_ids, const int32_t* slot, int n_slots,
                            tv_stream_t stream);

/*
 * tree_kv_write -- place the K and V rows of the current step's M+1 tree nodes
 * behind each sequence's committed prefix, in every layer: the cache layout
 * that tree_attention and kv_commit_realign read.  The pages have no separate
 * step for it (their branch caches are written by the model's own forward);
 * it is the append that this library's cache layout needs, offered so that a
 * caller holding the new rows in one staging buffer needs no per-sequence
 * copies and no host copy of the geometry.
 *
 *   k_layers, v_layers  DEVICE arrays of L device pointers to bf16
 *             [B][Hkv][S_cap][D] layers (16-byte aligned), written
 *   tree_k, tree_v  bf16 [L][B][Hkv][M+1][D] in (16-byte aligned)
 *   kv_start, kv_len  int32 [B] in: row r of sequence b goes to column
 *             kv_start[b] + kv_len[b] + r
 *   depth     int32 [B][M+1] or NULL: with depths, each K row r is rotated to
 *             position kv_len[b] + depth[b][r] (the rotation of TV_ATTN_ROPE,
 *             base rope_theta > 1) and stored as bf16; V rows are copied as they
 *             are.  NULL: K and V are copied as they are (rope_theta ignored).
 *   slot, n_slots  optional slot map (see tree_attention)
 *   D in {64, 128}; 0 <= M < 256.
 * A sequence whose geometry breaks 0 <= kv_start, 0 <= kv_len,
 * kv_start + kv_len + M + 1 <= S_cap is left untouched (tree_attention then
 * gives it zero rows and kv_commit_realign flags it TV_SEQ_BAD_GEOMETRY).
 */
tv_status tree_kv_write(uint16_t* const* k_layers, uint16_t* const* v_layers, const uint16_t* tree_k,
                        const uint16_t* tree_v, int L, int B, int Hkv, int D, int64_t S_cap, int M,
                        const int32_t* kv_start, const int32_t* kv_len, const int32_t* depth, float rope_theta,
                        const int32_t* slot, int n_slots, tv_stream_t stream);

/* Human-readable name of a tv_status. */
const char* tv_status_string(tv_status s);

/* The cudaError_t of the most recent TV_ERR_CUDA returned on this thread (0 if none). */
int tv_last_cuda_error(void);

/* ABI version (major * 100 + minor). */
int tv_version(void);

/*
 * tv_set_wait_limit_ns -- testing hook for the timeout path of tree_attention
 * (the pages have no counterpart).  Every device wait of the tensor-core
 * attention kernel is bounded; this sets, for the launches that follow in this
 * process, the limit of the pipeline waits (a stage that waits for the previous
 * one: scores, probabilities, output, K/V tiles).  A wait that runs out makes
 * the kernel give up on that sequence: its rows are zero and TV_SEQ_TIMEOUT is
 * OR-ed into its status.  The waits that drain copies and MMAs still in flight
 * before a CTA exits keep the full 1 s limit, so a short limit never leaves work
 * behind.  ns = 0 restores the default (1 s); larger values are clamped to it.
 * Not thread-safe with respect to launches on other threads.
 */
void tv_set_wait_limit_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif

#endif /* TREEVERIFY_H */
