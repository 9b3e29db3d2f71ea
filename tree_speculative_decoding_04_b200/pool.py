"""Cross-batch scheduling of a pool of sequences (EXSPEC).

"Batch Speculative Decoding Done Right", methodology: instead of keeping one
fixed batch, EXSPEC keeps a SequencePool and batches together sequences of
equal length, which need no realignment; only when no such group is available
does it fall back to EQSPEC's unpad-append-repad.

Here every sequence of the pool owns a cache slot (each layer of the cache is
[n_slots][Hkv][S_cap][D]) with its own geometry (kv_start, kv_len per slot), and
the four calls take a slot map, so a batch is any set of slots and forming it
moves no KV.  ``SequencePool`` is the host-side scheduler (pure bookkeeping of
lengths and waiting times); ``PoolVerifier`` runs one verification step of a
batch of slots on the GPU through the C ABI: equal-length batches commit in
per-sequence-length mode (appends only), fallback batches commit with the
EQSPEC repad.
"""
from __future__ import annotations

import torch

from . import _lib as tv

GROUPED = "grouped"    # every sequence of the batch has the same length: no realignment
FALLBACK = "fallback"  # lengths differ: EQSPEC unpad-append-repad


class SequencePool:
    """Which slots form the next batch.

    lengths: committed length of every slot's sequence.  batch: largest batch.
    min_group: smallest equal-length group worth a grouped batch (default 2).
    max_wait: a sequence left out for more than this many rounds is scheduled in
    the next batch (a fallback batch of the longest-waiting sequences), so no
    sequence starves (default: enough rounds to visit every slot twice).
    """

    def __init__(self, lengths, batch: int, min_group: int = 2, max_wait: int | None = None):
        self.length = [int(x) for x in lengths]
        self.n = len(self.length)
        if batch < 1 or self.n < 1:
            raise ValueError("empty pool or batch")
        self.batch = int(batch)
        self.min_group = max(1, int(min_group))
        self.max_wait = int(max_wait) if max_wait is not None else max(2, 2 * -(-self.n // self.batch))
        self.active = [True] * self.n
        self.last = [-1] * self.n  # round each slot was last scheduled
        self.round = 0

    def _waited(self, s):
        return self.round - self.last[s]

    def next_batch(self):
        """(slots, mode): the next batch and how it commits (GROUPED: per-sequence
        lengths, no realignment; FALLBACK: EQSPEC repad)."""
        live = [s for s in range(self.n) if self.active[s]]
        if not live:
            return [], GROUPED
        by_wait = sorted(live, key=lambda s: (-self._waited(s), s))
        if self._waited(by_wait[0]) > self.max_wait:
            return self._as_batch(by_wait[:self.batch])
        groups = {}
        for s in live:
            groups.setdefault(self.length[s], []).append(s)
        # the largest group; ties go to the shorter length
        best_len = min(groups, key=lambda ln: (-len(groups[ln]), ln))
        group = groups[best_len]
        if len(group) >= self.min_group:
            group = sorted(group, key=lambda s: (-self._waited(s), s))[:self.batch]
            return sorted(group), GROUPED
        return self._as_batch(by_wait[:self.batch])

    def _as_batch(self, slots):
        slots = sorted(slots)
        same = len({self.length[s] for s in slots}) == 1
        return slots, GROUPED if same else FALLBACK

    def commit(self, slots, accept_len):
        """Record one finished step: accept_len[i] draft tokens accepted by slot
        slots[i] (-1: rejected, nothing committed)."""
        for s, a in zip(slots, accept_len):
            a = int(a)
            self.length[s] += a + 1 if a >= 0 else 0
            self.last[s] = self.round
        self.round += 1

    def retire(self, slot):
        self.active[slot] = False


class PoolVerifier:
    """One verification step of a batch of pool slots, through the C ABI.

    The pool cache (L layers of [n_slots][Hkv][S_cap][D]) and the per-slot
    geometry live here; the step's inputs are per batch row: parent, draft,
    logits, q [L][B][M+1][Hq][D], tree_k / tree_v [L][B][Hkv][M+1][D].  Batches
    may be smaller than B (the first rows are used)."""

    def __init__(self, n_slots, B, M, Hq, Hkv, D, V, L, S_cap, max_depth, device="cuda", k_layers=None,
                 v_layers=None, with_mask_outputs=True):
        self.n_slots, self.B, self.M, self.Hq, self.Hkv, self.D, self.V, self.L = n_slots, B, M, Hq, Hkv, D, V, L
        self.S_cap, self.max_depth = S_cap, max_depth
        n = M + 1
        self.n = n
        dev = torch.device(device)
        self.device = dev
        i32 = dict(dtype=torch.int32, device=dev)
        bf = dict(dtype=torch.bfloat16, device=dev)
        self.k = k_layers if k_layers is not None else [torch.zeros((n_slots, Hkv, S_cap, D), **bf) for _ in range(L)]
        self.v = v_layers if v_layers is not None else [torch.zeros((n_slots, Hkv, S_cap, D), **bf) for _ in range(L)]
        self.k_ptrs = tv.layer_pointers(self.k, dev)
        self.v_ptrs = tv.layer_pointers(self.v, dev)
        self.kv_start = torch.zeros((n_slots,), **i32)
        self.kv_len = torch.zeros((n_slots,), **i32)
        self.max_len = torch.zeros((1,), **i32)
        self.attn_mask = torch.zeros((n_slots, S_cap), dtype=torch.uint8, device=dev) if with_mask_outputs else None
        self.pos_ids = torch.zeros((n_slots, S_cap), **i32) if with_mask_outputs else None
        # per batch row
        self.slot = torch.zeros((B,), **i32)
        self._slot_host = torch.zeros((B,), dtype=torch.int32, pin_memory=True)
        self.parent = torch.zeros((B, n), **i32)
        self.draft = torch.zeros((B, n), **i32)
        self.logits = torch.zeros((B, n, V), dtype=torch.float32, device=dev)
        self.q = torch.zeros((L, B, n, Hq, D), **bf)
        self.tree_k = torch.zeros((L, B, Hkv, n, D), **bf)
        self.tree_v = torch.zeros((L, B, Hkv, n, D), **bf)
        self.out = torch.zeros((L, B, n, Hq, D), **bf)
        self.anc = torch.zeros((B, n, (n + 31) // 32), **i32)
        self.depth = torch.zeros((B, n), **i32)
        self.status = torch.zeros((B,), **i32)
        self.argmax = torch.zeros((B, n), **i32)
        self.accept_len = torch.zeros((B,), **i32)
        self.path = torch.zeros((B, max_depth + 1), **i32)
        self.bonus = torch.zeros((B,), **i32)
        self.workspace = {}
        self._graphs = {}

    def _ws(self, Bb):
        if Bb not in self.workspace:
            self.workspace[Bb] = tv.attention_workspace(Bb, self.M, self.Hq, self.Hkv, self.D, self.S_cap, self.device)
        return self.workspace[Bb]

    def set_slots(self, slots, stream=None):
        """The batch's slots -> the device slot map (one small asynchronous copy)."""
        Bb = len(slots)
        if not 0 < Bb <= self.B or len(set(slots)) != Bb:
            raise ValueError("a batch holds 1..B distinct slots")
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        # the previous copy out of the pinned buffer must have been consumed
        s.synchronize()
        self._slot_host[:Bb] = torch.as_tensor(slots, dtype=torch.int32)
        with torch.cuda.stream(s):
            self.slot[:Bb].copy_(self._slot_host[:Bb], non_blocking=True)

    def step(self, Bb, realign, stream=None, before_commit=None):
        """One verification step of the first Bb batch rows (slots set by
        set_slots); asynchronous on `stream`.  before_commit: optional callable
        run (on the host) between the accept and the commit launches, e.g. to
        record a CUDA event."""
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        self._step_main(Bb, s)
        if before_commit is not None:
            before_commit()
        self._step_commit(Bb, realign, s)

    def _step_main(self, Bb, s):
        """mask, per layer tree_kv_write + attention, accept"""
        sl = self.slot[:Bb]
        tv.tree_build_mask(self.parent[:Bb], self.max_depth, self.anc[:Bb], self.depth[:Bb], self.status[:Bb], s)
        for layer in range(self.L):
            tv.tree_kv_write(self.k_ptrs[layer:layer + 1], self.v_ptrs[layer:layer + 1],
                             self.tree_k[layer:layer + 1, :Bb], self.tree_v[layer:layer + 1, :Bb], self.S_cap,
                             self.kv_start, self.kv_len, s, slot=sl)
            tv.tree_attention(self.q[layer, :Bb], self.k[layer], self.v[layer], self.kv_start, self.kv_len,
                              self.anc[:Bb], self.status[:Bb], self.out[layer, :Bb], self._ws(Bb), stream=s, slot=sl)
        tv.tree_accept(self.logits[:Bb], self.draft[:Bb], self.parent[:Bb], self.depth[:Bb], self.anc[:Bb],
                       self.status[:Bb], self.max_depth, self.argmax[:Bb], self.accept_len[:Bb], self.path[:Bb],
                       self.bonus[:Bb], s)

    def _step_commit(self, Bb, realign, s):
        sl = self.slot[:Bb]
        tv.kv_commit_realign(self.k_ptrs, self.v_ptrs, Bb, self.Hkv, self.D, self.S_cap, self.M, self.path[:Bb],
                             self.accept_len[:Bb], self.status[:Bb], self.max_depth, self.kv_start, self.kv_len,
                             self.max_len, int(realign), self.attn_mask, self.pos_ids, s, slot=sl)

    def graphs(self, Bb, realign, stream):
        """CUDA graphs of one step of the first Bb batch rows, captured once per
        (Bb, realign) and replayed: (everything up to the accept, the commit).
        The slot map and the per-slot geometry are read on the device, so one
        pair of graphs serves every batch of that size and mode; set_slots
        before each replay."""
        key = (int(Bb), int(realign))
        if key not in self._graphs:
            s = stream
            self._ws(Bb)  # allocated outside the capture
            g_main, g_commit = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
            # two graphs: the launches before the commit, then the commit
            with torch.cuda.graph(g_main, stream=s):
                self._step_main(Bb, s)
            with torch.cuda.graph(g_commit, stream=s):
                self._step_commit(Bb, realign, s)
            self._graphs[key] = (g_main, g_commit)
        return self._graphs[key]

    def step_graphed(self, Bb, realign, stream=None, between=None):
        """step() through the captured graphs (asynchronous on `stream`, which
        must be a side stream, not the default one); between: optional callable
        run on the host between the two replays, e.g. to record a CUDA event."""
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        g_main, g_commit = self.graphs(Bb, realign, s)
        with torch.cuda.stream(s):
            g_main.replay()
            if between is not None:
                between()
            g_commit.replay()

    def launches_per_step(self) -> int:
        """mask 1, per layer tree_kv_write 1 + attention 1, accept 2, commit 2."""
        return 1 + 2 * self.L + 2 + 2
