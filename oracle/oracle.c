/*
 * oracle.c -- plain, slow, obviously-correct CPU reference for the teacher-side
 * verification step of tree speculative decoding.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or load
 * this file: only the tests, the smoke check and the benchmark's CPU-baseline /
 * reference arm do.  It shares no code, header, table or helper with the CUDA
 * library; it includes only the C standard library.
 *
 * Sources (web pages summarising two papers):
 *   [EP]  "EAGLE-Pangu: Accelerator-Safe Tree Speculative Decoding on Ascend NPUs"
 *         technical summary, section 2 (methodology):
 *           A  branchable KV cache, commit modes (length-based, path-index based)
 *           B  accelerator-safe tree tensors (dummy root row 0, parents in [0,M],
 *              ancestor tables, invariant checks before fused kernels)
 *           C  fused tree-masked teacher execution (node k may attend node j only
 *              if j is an ancestor of k)
 *         section 4 (results): accepted length per verification step.
 *   [BSD] "Batch Speculative Decoding Done Right", section 2 (methodology):
 *           synchronization invariants (rectangular alignment, position-ID
 *           contiguity) and EQSPEC unpad-append-repad.
 *
 * Precision: attention is evaluated in double precision from exactly-converted
 * bf16 inputs (the pages fix no precision); argmax compares the fp32 logits
 * themselves (no arithmetic, so the decision is exact in any precision).
 *
 * Every function below has at least one pin in the CPU test-suite (closed forms,
 * reductions to a library routine, brute force on tiny inputs, invariants).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* per-sequence status bits (shared *meaning* with the library's header, not code) */
#define OR_BAD_PARENT 1
#define OR_TOO_DEEP 2
#define OR_BAD_GEOMETRY 8

/* ---------------------------------------------------------------------------
 * Tree validation and ancestor sets.
 * [EP] 2.B: row 0 is the dummy root; every parent pointer lies in [0, M]; the
 * structure is acyclic and in range (checked before any kernel runs).  With the
 * reading parent[0] = 0 and parent[i] < i for i >= 1, acyclicity is implied.
 * ------------------------------------------------------------------------- */

/* Returns the status bits for one tree; fills depth[0..M] when the tree is valid. */
static int validate_tree(const int32_t* par, int M, int max_depth, int32_t* depth) {
  int st = 0;
  if (par[0] != 0) st |= OR_BAD_PARENT;
  for (int i = 1; i <= M; ++i)
    if (par[i] < 0 || par[i] >= i) st |= OR_BAD_PARENT;
  if (st) return st;
  for (int u = 0; u <= M; ++u) {
    int d = 0, x = u;
    while (x != 0) { /* terminates: par[x] < x */
      x = par[x];
      ++d;
    }
    depth[u] = d;
    if (d > max_depth) st |= OR_TOO_DEEP;
  }
  return st;
}

/* Ancestor bitmask, built by walking parent pointers from u up to the root.
 * anc_mask is [B][M+1][W] uint32, W = ceil((M+1)/32); bit r of row u is set iff
 * tree row r lies on the root..u path (u itself included).  Invalid trees get
 * all-zero mask and depth rows. */
int oracle_tree_build_mask(const int32_t* parent, int B, int M, int max_depth,
                           uint32_t* anc_mask, int32_t* depth, int32_t* status) {
  if (B < 0 || M < 0) return -1;
  const int n = M + 1, W = (M + 1 + 31) / 32;
  for (int b = 0; b < B; ++b) {
    const int32_t* par = parent + (int64_t)b * n;
    int32_t* dep = depth + (int64_t)b * n;
    uint32_t* msk = anc_mask + (int64_t)b * n * W;
    memset(msk, 0, sizeof(uint32_t) * (size_t)n * W);
    memset(dep, 0, sizeof(int32_t) * (size_t)n);
    int st = validate_tree(par, M, max_depth, dep);
    status[b] = st;
    if (st) {
      memset(dep, 0, sizeof(int32_t) * (size_t)n);
      continue;
    }
    for (int u = 0; u < n; ++u) {
      uint32_t* row = msk + (int64_t)u * W;
      int x = u;
      for (;;) {
        row[x / 32] |= 1u << (x % 32);
        if (x == 0) break;
        x = par[x];
      }
    }
  }
  return 0;
}

/* ---------------------------------------------------------------------------
 * Tree-masked attention.
 * [EP] 2.C: one batched teacher pass over all speculative tokens; query node u
 * sees the whole committed prefix and, inside the tree, only its ancestors and
 * itself.  Reading adopted: scale 1/sqrt(D) is passed in; GQA maps q-head h to
 * kv-head h / (Hq/Hkv).
 * Layouts: q, out [B][M+1][Hq][D]; k, v [B][Hkv][S_cap][D] (bf16 bits);
 * the prefix of b is columns [kv_start, kv_start+kv_len); tree row r lives at
 * column kv_start+kv_len+r.
 * ------------------------------------------------------------------------- */

static double bf16_to_double(uint16_t h) {
  uint32_t bits = (uint32_t)h << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

static int geometry_ok(int32_t ks, int32_t kl, int M, int64_t S_cap) {
  return ks >= 0 && kl >= 0 && (int64_t)ks + kl + M + 1 <= S_cap;
}

/* ---------------------------------------------------------------------------
 * Rotary position embedding of the tree rows.
 * [BSD] 2, position-ID contiguity: position IDs run from 0 without gaps over the
 * attended columns (the condition a rotary embedding needs).  Reading adopted
 * for a tree: the committed prefix holds positions 0 .. kv_len-1 and node u sits
 * at position kv_len + depth(u), so every root-to-node path continues the prefix
 * without a gap (siblings share a position).  The rotation is the published
 * rotary embedding (RoFormer, Su et al.) in the half-split arrangement: the pair
 * (x[i], x[i + D/2]), i < D/2, is turned by the angle pos * base^(-2i/D).
 * ------------------------------------------------------------------------- */
static void rope_rotate(double* x, int D, double pos, double base) {
  const int h = D / 2;
  for (int i = 0; i < h; ++i) {
    const double th = pos * pow(base, -2.0 * i / D);
    const double c = cos(th), s = sin(th);
    const double a = x[i], b = x[i + h];
    x[i] = a * c - b * s;
    x[i + h] = b * c + a * s;
  }
}

/* rows x [rows][D] rotated in place, row i by the angle set of position pos[i]. */
int oracle_rope_rows(double* x, const double* pos, int64_t rows, int D, double base) {
  if (D <= 0 || D % 2 != 0 || !(base > 0.0)) return -1;
  for (int64_t i = 0; i < rows; ++i) rope_rotate(x + i * D, D, pos[i], base);
  return 0;
}

/* Round a double to the nearest bf16 (ties to even), in one rounding: scale the
 * significand to 8 bits, round it with rint (round-to-nearest-even mode), scale
 * back; 8 significant bits are exact in a float, whose upper 16 bits are the
 * bf16 pattern.  Finite values of ordinary range only (no subnormal care). */
static uint16_t double_to_bf16(double v) {
  if (v != v) return 0x7FC0;
  if (v == 0.0) return signbit(v) ? 0x8000 : 0;
  int e;
  const double m = frexp(v, &e); /* v = m * 2^e, 0.5 <= |m| < 1 */
  const double r = ldexp(rint(ldexp(m, 8)), e - 8);
  const float f = (float)r;
  uint32_t bits;
  memcpy(&bits, &f, sizeof bits);
  return (uint16_t)(bits >> 16);
}

/* One output row: sequence b, node u, query head h.  Key set is the prefix in
 * column order followed by the walked ancestor rows in ascending row order. */
static void attend_one(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t S_cap,
                       int32_t ks, int32_t kl, const int32_t* par, int b, int u, int h, int M,
                       int Hq, int Hkv, int D, double scale, double rope_base, double* o) {
  const int G = Hq / Hkv, hk = h / G, n = M + 1;
  const uint16_t* qr = q + (((int64_t)b * n + u) * Hq + h) * D;
  const uint16_t* kb = k + ((int64_t)b * Hkv + hk) * S_cap * D;
  const uint16_t* vb = v + ((int64_t)b * Hkv + hk) * S_cap * D;
  /* the query row, rotated to its position when a rotary base is given (the
   * keys are used as stored: tree rows are rotated when they are written) */
  double* qd = (double*)malloc(sizeof(double) * (size_t)D);
  for (int d = 0; d < D; ++d) qd[d] = bf16_to_double(qr[d]);
  if (rope_base > 0.0) {
    int depth_u = 0;
    for (int x = u; x != 0; x = par[x]) ++depth_u;
    rope_rotate(qd, D, (double)kl + depth_u, rope_base);
  }

  /* explicit key list: prefix columns, then ancestor tree rows ascending */
  char* is_anc = (char*)calloc((size_t)n, 1);
  for (int x = u;;) {
    is_anc[x] = 1;
    if (x == 0) break;
    x = par[x];
  }
  int64_t nkeys = kl;
  for (int r = 0; r < n; ++r) nkeys += is_anc[r];
  int64_t* cols = (int64_t*)malloc(sizeof(int64_t) * (size_t)nkeys);
  double* s = (double*)malloc(sizeof(double) * (size_t)nkeys);
  int64_t t = 0;
  for (int64_t c = 0; c < kl; ++c) cols[t++] = (int64_t)ks + c;
  for (int r = 0; r < n; ++r)
    if (is_anc[r]) cols[t++] = (int64_t)ks + kl + r;

  double mx = -INFINITY;
  for (t = 0; t < nkeys; ++t) {
    const uint16_t* kr = kb + cols[t] * D;
    double acc = 0.0;
    for (int d = 0; d < D; ++d) acc += qd[d] * bf16_to_double(kr[d]);
    s[t] = acc * scale;
    if (s[t] > mx) mx = s[t];
  }
  double l = 0.0;
  for (int d = 0; d < D; ++d) o[d] = 0.0;
  for (t = 0; t < nkeys; ++t) {
    double p = exp(s[t] - mx);
    l += p;
    const uint16_t* vr = vb + cols[t] * D;
    for (int d = 0; d < D; ++d) o[d] += p * bf16_to_double(vr[d]);
  }
  for (int d = 0; d < D; ++d) o[d] /= l;
  free(qd);
  free(s);
  free(cols);
  free(is_anc);
}

/* One row of sequence b, or zeros if the sequence is invalid (status != 0 or
 * a bad cache geometry). */
static void attend_row_or_zero(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t S_cap,
                               const int32_t* kv_start, const int32_t* kv_len, const int32_t* parent,
                               const int32_t* status, int b, int u, int h, int M, int Hq, int Hkv, int D,
                               double scale, double rope_base, double* o) {
  if (status[b] != 0 || !geometry_ok(kv_start[b], kv_len[b], M, S_cap)) {
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    return;
  }
  attend_one(q, k, v, S_cap, kv_start[b], kv_len[b], parent + (int64_t)b * (M + 1), b, u, h, M, Hq, Hkv, D,
             scale, rope_base, o);
}

/* Selected rows: sel is [nsel][3] = (b, u, h); out is [nsel][D].  Rows of an
 * invalid sequence (status != 0 or bad cache geometry) are zero.  rope_base > 0
 * rotates each query row to position kv_len + depth(u) first (0: q is used as
 * given).  (Rows are independent; the OpenMP pragmas only take effect in the
 * benchmark's all-cores build.) */
int oracle_tree_attention_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t S_cap,
                               const int32_t* kv_start, const int32_t* kv_len, const int32_t* parent,
                               const int32_t* status, int B, int M, int Hq, int Hkv, int D,
                               double scale, double rope_base, const int32_t* sel, int64_t nsel, double* out) {
  if (Hkv <= 0 || Hq % Hkv != 0) return -1;
  for (int64_t i = 0; i < nsel; ++i) {
    int b = sel[3 * i], u = sel[3 * i + 1], h = sel[3 * i + 2];
    if (b < 0 || b >= B || u < 0 || u > M || h < 0 || h >= Hq) return -2;
  }
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < nsel; ++i)
    attend_row_or_zero(q, k, v, S_cap, kv_start, kv_len, parent, status, sel[3 * i], sel[3 * i + 1],
                       sel[3 * i + 2], M, Hq, Hkv, D, scale, rope_base, out + i * D);
  return 0;
}

/* All rows: out is [B][M+1][Hq][D]. */
int oracle_tree_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t S_cap,
                          const int32_t* kv_start, const int32_t* kv_len, const int32_t* parent,
                          const int32_t* status, int B, int M, int Hq, int Hkv, int D, double scale,
                          double rope_base, double* out) {
  if (Hkv <= 0 || Hq % Hkv != 0) return -1;
  const int64_t rows = (int64_t)B * (M + 1) * Hq;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < rows; ++i) {
    const int h = (int)(i % Hq), u = (int)((i / Hq) % (M + 1)), b = (int)(i / ((int64_t)Hq * (M + 1)));
    attend_row_or_zero(q, k, v, S_cap, kv_start, kv_len, parent, status, b, u, h, M, Hq, Hkv, D, scale,
                       rope_base, out + i * D);
  }
  return 0;
}

/* ---------------------------------------------------------------------------
 * Greedy acceptance.
 * [EP] section 4: the accepted length is the number of speculative tokens the
 * teacher's greedy choice agrees with in one verification step.  For a tree:
 * node i is accepted iff its parent is accepted and its draft token equals the
 * teacher's argmax at the parent; the committed branch is the deepest accepted
 * node (lowest row index on ties) and the teacher's argmax there is the bonus.
 * ------------------------------------------------------------------------- */

/* First maximum wins (strict '>'). */
int oracle_argmax_rows(const float* logits, int64_t rows, int V, int32_t* out) {
#pragma omp parallel for
  for (int64_t r = 0; r < rows; ++r) {
    const float* x = logits + r * V;
    int best = 0;
    float bv = x[0];
    for (int j = 1; j < V; ++j)
      if (x[j] > bv) {
        bv = x[j];
        best = j;
      }
    out[r] = best;
  }
  return 0;
}

/* ---------------------------------------------------------------------------
 * Teacher logits from the final hidden states.
 * [EP] 2.C: the teacher evaluates every speculative token in one batched pass;
 * its greedy choice at node u is the argmax over the vocabulary of the LM-head
 * logits, logit[u][v] = sum_h hidden[u][h] * W[v][h] (W: [V][H], bf16 inputs).
 * The sum is taken in double precision: every bf16 product is exact in double,
 * so the only rounding is that of the double accumulation.
 * rows: nsel row indices into hidden [R][H]; out [nsel][V] double.
 * ------------------------------------------------------------------------- */
int oracle_lm_head_logits(const uint16_t* hidden, const uint16_t* w, const int32_t* rows, int64_t nsel, int H,
                          int V, double* out) {
  if (H <= 0 || V <= 0) return -1;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < nsel; ++i) {
    const uint16_t* x = hidden + (int64_t)rows[i] * H;
    double* o = out + i * V;
    for (int v = 0; v < V; ++v) {
      const uint16_t* wr = w + (int64_t)v * H;
      double acc = 0.0;
      for (int h = 0; h < H; ++h) acc += bf16_to_double(x[h]) * bf16_to_double(wr[h]);
      o[v] = acc;
    }
  }
  return 0;
}

/* First maximum of each double row (strict '>'), as for the fp32 logits. */
int oracle_argmax_rows_f64(const double* x, int64_t rows, int V, int32_t* out) {
  for (int64_t r = 0; r < rows; ++r) {
    const double* a = x + r * V;
    int best = 0;
    for (int j = 1; j < V; ++j)
      if (a[j] > a[best]) best = j;
    out[r] = best;
  }
  return 0;
}

/* Brute force: every root-to-leaf path, its longest accepted prefix. */
static void brute_force_best(const int32_t* par, const int32_t* draft, const int32_t* am, int M,
                             int* best_len, int* best_end) {
  const int n = M + 1;
  char* has_child = (char*)calloc((size_t)n, 1);
  int* chain = (int*)malloc(sizeof(int) * (size_t)n);
  for (int i = 1; i < n; ++i) has_child[par[i]] = 1;
  *best_len = -1;
  *best_end = 0;
  for (int leaf = 0; leaf < n; ++leaf) {
    if (has_child[leaf]) continue;
    int len = 0;
    for (int x = leaf;; x = par[x]) { /* collect leaf..root */
      chain[len++] = x;
      if (x == 0) break;
    }
    /* chain[len-1] is the root; walk downwards */
    int acc = 0, end = 0;
    for (int j = len - 2; j >= 0; --j) {
      int node = chain[j], p = chain[j + 1];
      if (draft[node] != am[p]) break;
      acc += 1;
      end = node;
    }
    if (acc > *best_len || (acc == *best_len && end < *best_end)) {
      *best_len = acc;
      *best_end = end;
    }
  }
  free(chain);
  free(has_child);
}

/* Returns 0 on success, -3 if the recurrence and brute force disagree. */
int oracle_tree_accept(const float* logits, const int32_t* draft, const int32_t* parent,
                       const int32_t* status, int B, int M, int V, int max_depth, int32_t* argmax,
                       int32_t* accept_len, int32_t* path, int32_t* bonus) {
  const int n = M + 1;
  int32_t* dep = (int32_t*)malloc(sizeof(int32_t) * (size_t)n);
  char* acc = (char*)malloc((size_t)n);
  int rc = 0;
  oracle_argmax_rows(logits, (int64_t)B * n, V, argmax);
  for (int b = 0; b < B; ++b) {
    const int32_t* par = parent + (int64_t)b * n;
    const int32_t* dr = draft + (int64_t)b * n;
    const int32_t* am = argmax + (int64_t)b * n;
    int32_t* pth = path + (int64_t)b * (max_depth + 1);
    for (int j = 0; j <= max_depth; ++j) pth[j] = 0;
    if (status[b] != 0 || validate_tree(par, M, max_depth, dep) != 0) {
      accept_len[b] = -1;
      bonus[b] = 0;
      continue;
    }
    acc[0] = 1;
    for (int i = 1; i < n; ++i) acc[i] = acc[par[i]] && dr[i] == am[par[i]];
    int e = 0;
    for (int i = 1; i < n; ++i)
      if (acc[i] && dep[i] > dep[e]) e = i; /* strict: lowest index kept on ties */
    int bl, be;
    brute_force_best(par, dr, am, M, &bl, &be);
    if (bl != dep[e] || be != e) rc = -3;
    accept_len[b] = dep[e];
    bonus[b] = am[e];
    for (int x = e;; x = par[x]) {
      pth[dep[x]] = x;
      if (x == 0) break;
    }
  }
  free(acc);
  free(dep);
  return rc;
}

/* ---------------------------------------------------------------------------
 * KV commit and EQSPEC realignment.
 * [EP] 2.A: path-index commit -- after acceptance the new cache segment is
 * reordered by the accepted path; the committed prefix keeps its order.
 * [BSD] 2: unpad-append-repad keeps (i) rectangular alignment: pad_b + len_b is
 * the batch maximum for every b, (ii) position IDs contiguous from 0 over the
 * attended (mask = 1) positions.
 * Reading adopted: the committed rows are the root row plus the accepted nodes
 * (a+1 rows, root first); a sequence with status != 0, or whose path points
 * outside the tree, commits nothing; a sequence with an out-of-range cache
 * geometry is left untouched and flagged in status.
 * k_layers / v_layers are host arrays of L host pointers to [B][Hkv][S_cap][D].
 * realign = 0: per-sequence lengths (content stays at kv_start).
 * realign = 1: left-padded; content is repadded to end at the new batch maximum.
 * ------------------------------------------------------------------------- */
int oracle_kv_commit_realign(uint16_t* const* k_layers, uint16_t* const* v_layers, int L, int B,
                             int Hkv, int D, int64_t S_cap, int M, const int32_t* path,
                             const int32_t* accept_len, int32_t* status, int max_depth,
                             int32_t* kv_start, int32_t* kv_len, int32_t* max_len, int realign,
                             uint8_t* attn_mask, int32_t* pos_ids) {
  int32_t* nb = (int32_t*)calloc((size_t)(B > 0 ? B : 1), sizeof(int32_t));
  int32_t* good = (int32_t*)calloc((size_t)(B > 0 ? B : 1), sizeof(int32_t));
  int32_t* new_start = (int32_t*)calloc((size_t)(B > 0 ? B : 1), sizeof(int32_t));
  int64_t lmax = 0;
  for (int b = 0; b < B; ++b) {
    good[b] = geometry_ok(kv_start[b], kv_len[b], M, S_cap);
    int a = accept_len[b];
    nb[b] = (good[b] && status[b] == 0 && a >= 0 && a <= max_depth && a <= M) ? a + 1 : 0;
    /* a path row outside [0, M] would gather outside the tree: commit nothing */
    for (int j = 0; j < nb[b]; ++j) {
      int r = path[(int64_t)b * (max_depth + 1) + j];
      if (r < 0 || r > M) nb[b] = 0;
    }
    if (good[b]) {
      int64_t nl = (int64_t)kv_len[b] + nb[b];
      int64_t end = realign ? nl : (int64_t)kv_start[b] + nl;
      if (end > lmax) lmax = end;
    }
  }
  for (int b = 0; b < B; ++b) {
    if (!good[b]) {
      new_start[b] = kv_start[b];
      continue;
    }
    new_start[b] = realign ? (int32_t)(lmax - (kv_len[b] + nb[b])) : kv_start[b];
  }
  const size_t row = (size_t)D * sizeof(uint16_t);
  for (int l = 0; l < L; ++l)
    for (int kvsel = 0; kvsel < 2; ++kvsel) {
      uint16_t* base = kvsel ? v_layers[l] : k_layers[l];
      for (int b = 0; b < B; ++b) {
        if (!good[b]) continue;
        for (int h = 0; h < Hkv; ++h) {
          uint16_t* c = base + ((int64_t)b * Hkv + h) * S_cap * D;
          const int64_t len = kv_len[b], ks = kv_start[b], n_new = len + nb[b];
          /* unpad + append: new content = old content ++ tail rows picked by path */
          uint16_t* tmp = (uint16_t*)malloc(row * (size_t)(n_new > 0 ? n_new : 1));
          for (int64_t i = 0; i < len; ++i) memcpy(tmp + i * D, c + (ks + i) * D, row);
          for (int j = 0; j < nb[b]; ++j) {
            int r = path[(int64_t)b * (max_depth + 1) + j];
            memcpy(tmp + (len + j) * D, c + (ks + len + r) * D, row);
          }
          /* repad: write it back starting at the new start column */
          for (int64_t i = 0; i < n_new; ++i) memcpy(c + (new_start[b] + i) * D, tmp + i * D, row);
          free(tmp);
        }
      }
    }
  for (int b = 0; b < B; ++b) {
    if (good[b]) {
      kv_len[b] += nb[b];
      kv_start[b] = new_start[b];
    } else {
      status[b] |= OR_BAD_GEOMETRY;
    }
    if (attn_mask || pos_ids)
      for (int64_t t = 0; t < S_cap; ++t) {
        int in = good[b] && t >= kv_start[b] && t < (int64_t)kv_start[b] + kv_len[b];
        if (attn_mask) attn_mask[(int64_t)b * S_cap + t] = (uint8_t)in;
        if (pos_ids) pos_ids[(int64_t)b * S_cap + t] = in ? (int32_t)(t - kv_start[b]) : 0;
      }
  }
  *max_len = (int32_t)lmax;
  free(new_start);
  free(good);
  free(nb);
  return 0;
}

/* ---------------------------------------------------------------------------
 * Appending the step's tree rows to the cache.
 * [EP] 2.C evaluates all speculative tokens in one teacher pass against the
 * cached prefix; in this layout the M+1 tree rows of sequence b sit right
 * behind its prefix, row r at column kv_start[b] + kv_len[b] + r, in every
 * layer.  tree_k / tree_v are [L][B][Hkv][M+1][D]; a sequence whose rows would
 * not fit the cache (or whose geometry is negative) is left untouched.
 * ------------------------------------------------------------------------- */
/* depth [B][M+1] and rope_base > 0: each K row r is rotated to position
 * kv_len + depth[b][r] (the rotary embedding above) and stored as the nearest
 * bf16; V rows are copied as they are.  depth NULL or rope_base <= 0: plain copy. */
int oracle_tree_kv_write(uint16_t* const* k_layers, uint16_t* const* v_layers, const uint16_t* tree_k,
                         const uint16_t* tree_v, int L, int B, int Hkv, int D, int64_t S_cap, int M,
                         const int32_t* kv_start, const int32_t* kv_len, const int32_t* depth,
                         double rope_base) {
  const int n = M + 1;
  const int rope = depth != NULL && rope_base > 0.0;
  double* row = (double*)malloc(sizeof(double) * (size_t)D);
  for (int l = 0; l < L; ++l)
    for (int b = 0; b < B; ++b) {
      if (!geometry_ok(kv_start[b], kv_len[b], M, S_cap)) continue;
      for (int h = 0; h < Hkv; ++h)
        for (int r = 0; r < n; ++r) {
          const int64_t src = ((((int64_t)l * B + b) * Hkv + h) * n + r) * D;
          const int64_t col = (int64_t)kv_start[b] + kv_len[b] + r;
          const int64_t dst = (((int64_t)b * Hkv + h) * S_cap + col) * D;
          if (rope) {
            for (int d = 0; d < D; ++d) row[d] = bf16_to_double(tree_k[src + d]);
            rope_rotate(row, D, (double)kv_len[b] + depth[(int64_t)b * n + r], rope_base);
            for (int d = 0; d < D; ++d) k_layers[l][dst + d] = double_to_bf16(row[d]);
          } else {
            for (int d = 0; d < D; ++d) k_layers[l][dst + d] = tree_k[src + d];
          }
          for (int d = 0; d < D; ++d) v_layers[l][dst + d] = tree_v[src + d];
        }
    }
  free(row);
  return 0;
}

/* Nearest bf16 of each double (exported for its pins). */
int oracle_round_bf16(const double* x, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = double_to_bf16(x[i]);
  return 0;
}
