"""Host-side driver of one whole verification step.

``TreeVerifier`` owns the device buffers of one workload shape and chains the
four C-ABI calls on one CUDA stream:

    tree_build_mask -> tree_attention (every layer) -> tree_accept -> kv_commit_realign

``step()`` works on inputs already resident on the GPU, with the tree rows'
K/V already in the cache (and can be captured in a CUDA graph).
``step_from_host()`` is the end-to-end entry point for callers that hold the
step's inputs in host memory: one pinned staging buffer mirrors the device
input buffer byte for byte, so the inputs cross in one copy for the tree
section and one per layer (q, tree K, tree V together) on a copy stream, while
the compute stream starts each layer as soon as its copy has landed; the tree
rows reach the cache through ``tree_kv_write`` and the accept results come
back in one copy.  Nothing here computes: it allocates, copies and calls.
"""
from __future__ import annotations

import dataclasses

import torch

from . import _lib as tv

_ALIGN = 256


def _align(x: int) -> int:
    return (x + _ALIGN - 1) // _ALIGN * _ALIGN


class _InputLayout:
    """Byte layout shared by the device input buffer and the pinned host staging
    buffer: [parent | draft] [logits] then, per layer, [q | tree K | tree V]."""

    def __init__(self, B, n, Hq, Hkv, D, V, L):
        self.B, self.n, self.Hq, self.Hkv, self.D, self.V, self.L = B, n, Hq, Hkv, D, V, L
        self.parent_off = 0
        self.draft_off = B * n * 4
        self.meta_bytes = 2 * B * n * 4
        self.logits_off = _align(self.meta_bytes)
        self.logits_bytes = B * n * V * 4
        self.q_bytes = B * n * Hq * D * 2
        self.rows_bytes = B * Hkv * n * D * 2
        self.layer_bytes = _align(self.q_bytes + 2 * self.rows_bytes)
        self.layers_off = _align(self.logits_off + self.logits_bytes)
        self.nbytes = self.layers_off + L * self.layer_bytes

    def layer_off(self, layer):
        return self.layers_off + layer * self.layer_bytes

    def views(self, buf: torch.Tensor):
        """Typed views of a uint8 buffer of this layout."""
        B, n, Hq, Hkv, D, V, L = self.B, self.n, self.Hq, self.Hkv, self.D, self.V, self.L
        i32 = buf.view(torch.int32)
        f32 = buf.view(torch.float32)
        b16 = buf.view(torch.bfloat16)
        le = self.layer_bytes // 2
        return dict(
            parent=i32[self.parent_off // 4:self.parent_off // 4 + B * n].view(B, n),
            draft=i32[self.draft_off // 4:self.draft_off // 4 + B * n].view(B, n),
            logits=f32[self.logits_off // 4:self.logits_off // 4 + B * n * V].view(B, n, V),
            q=b16.as_strided((L, B, n, Hq, D), (le, n * Hq * D, Hq * D, D, 1), self.layers_off // 2),
            tree_k=b16.as_strided((L, B, Hkv, n, D), (le, Hkv * n * D, n * D, D, 1),
                                  (self.layers_off + self.q_bytes) // 2),
            tree_v=b16.as_strided((L, B, Hkv, n, D), (le, Hkv * n * D, n * D, D, 1),
                                  (self.layers_off + self.q_bytes + self.rows_bytes) // 2),
        )


@dataclasses.dataclass
class StepResult:
    accept_len: torch.Tensor  # [B] int32
    path: torch.Tensor  # [B][max_depth+1] int32
    bonus: torch.Tensor  # [B] int32


class TreeVerifier:
    def __init__(self, B, M, Hq, Hkv, D, V, L, S_cap, max_depth, realign=False, device="cuda",
                 k_layers=None, v_layers=None, with_mask_outputs=None, commit_layers=None, rope_theta=0.0):
        """k_layers / v_layers: the L per-layer caches (default: allocated here).
        commit_layers: the indices of the layers kv_commit_realign moves (default
        all); a caller whose layer list repeats a buffer commits each buffer once.
        rope_theta > 0: q and the tree rows' K are given before their rotary
        embedding; the kernels rotate them to the tree positions kv_len + depth
        (tree_kv_write for K, tree_attention's query staging for q)."""
        self.B, self.M, self.Hq, self.Hkv, self.D, self.V, self.L = B, M, Hq, Hkv, D, V, L
        self.S_cap, self.max_depth, self.realign = S_cap, max_depth, bool(realign)
        self.rope_theta = float(rope_theta)
        self.n = M + 1
        self.W = (self.n + 31) // 32
        dev = torch.device(device)
        self.device = dev
        i32 = dict(dtype=torch.int32, device=dev)
        bf = dict(dtype=torch.bfloat16, device=dev)
        # the step's inputs: one device buffer laid out like the pinned staging buffer
        self.layout = _InputLayout(B, self.n, Hq, Hkv, D, V, L)
        self._inputs = torch.zeros(self.layout.nbytes, dtype=torch.uint8, device=dev)
        views = self.layout.views(self._inputs)
        self.parent, self.draft, self.logits = views["parent"], views["draft"], views["logits"]
        self.q = [views["q"][layer] for layer in range(L)]
        self.tree_k, self.tree_v = views["tree_k"], views["tree_v"]  # [L][B][Hkv][M+1][D]
        self.anc = torch.zeros((B, self.n, self.W), **i32)
        self.depth = torch.zeros((B, self.n), **i32)
        self.status = torch.zeros((B,), **i32)
        self.kv_start = torch.zeros((B,), **i32)
        self.kv_len = torch.zeros((B,), **i32)
        self.max_len = torch.zeros((1,), **i32)
        self.out = [torch.zeros((B, self.n, Hq, D), **bf) for _ in range(L)]
        self.k = k_layers if k_layers is not None else [torch.zeros((B, Hkv, S_cap, D), **bf) for _ in range(L)]
        self.v = v_layers if v_layers is not None else [torch.zeros((B, Hkv, S_cap, D), **bf) for _ in range(L)]
        self.k_ptrs = tv.layer_pointers(self.k, dev)
        self.v_ptrs = tv.layer_pointers(self.v, dev)
        ids = list(range(L)) if commit_layers is None else list(commit_layers)
        self.k_commit_ptrs = tv.layer_pointers([self.k[i] for i in ids], dev)
        self.v_commit_ptrs = tv.layer_pointers([self.v[i] for i in ids], dev)
        self.workspace = tv.attention_workspace(B, M, Hq, Hkv, D, S_cap, dev)
        self.argmax = torch.zeros((B, self.n), **i32)
        # accept results side by side, so that they come back in one copy
        nres = B + B * (max_depth + 1) + B
        self._results = torch.zeros((nres,), **i32)
        self.accept_len = self._results[:B]
        self.path = self._results[B:B + B * (max_depth + 1)].view(B, max_depth + 1)
        self.bonus = self._results[B + B * (max_depth + 1):]
        want_mask = self.realign if with_mask_outputs is None else with_mask_outputs
        self.attn_mask = torch.zeros((B, S_cap), dtype=torch.uint8, device=dev) if want_mask else None
        self.pos_ids = torch.zeros((B, S_cap), **i32) if want_mask else None
        self._host = None
        self._copy_stream = None
        self._events = None

    # ------------------------------------------------------------------ device path
    def launches_per_step(self) -> int:
        """Kernels this library launches per step(): mask 1, attention 1 per layer,
        accept 2, commit 2 (step_from_host adds one tree_kv_write per layer)."""
        return 1 + self.L + 2 + 2

    def build_mask(self, stream=None):
        tv.tree_build_mask(self.parent, self.max_depth, self.anc, self.depth, self.status, stream)

    def attention(self, layer, stream=None, prefix_ready=False):
        """tree_attention of one layer.  prefix_ready: the kernel launched just
        before on `stream` writes neither the geometry nor any prefix K/V column
        (true after tree_build_mask, tree_kv_write and the attention of another
        layer; false after kv_commit_realign), so prefix tiles may stream while
        it finishes.  Off by default: on B200 it measured no faster."""
        flags = (tv.ATTN_PREFIX_READY if prefix_ready else 0) | (tv.ATTN_ROPE if self.rope_theta > 0 else 0)
        tv.tree_attention(self.q[layer], self.k[layer], self.v[layer], self.kv_start, self.kv_len, self.anc,
                          self.status, self.out[layer], self.workspace, stream=stream, flags=flags,
                          depth=self.depth, rope_theta=self.rope_theta)

    def write_tree_rows(self, layer, stream=None):
        """tree_k / tree_v of one layer -> the cache, behind each sequence's prefix."""
        tv.tree_kv_write(self.k_ptrs[layer:layer + 1], self.v_ptrs[layer:layer + 1],
                         self.tree_k[layer].unsqueeze(0), self.tree_v[layer].unsqueeze(0), self.S_cap,
                         self.kv_start, self.kv_len, stream,
                         depth=self.depth if self.rope_theta > 0 else None, rope_theta=self.rope_theta)

    def accept(self, stream=None):
        tv.tree_accept(self.logits, self.draft, self.parent, self.depth, self.anc, self.status, self.max_depth,
                       self.argmax, self.accept_len, self.path, self.bonus, stream)

    def commit(self, stream=None):
        tv.kv_commit_realign(self.k_commit_ptrs, self.v_commit_ptrs, self.B, self.Hkv, self.D, self.S_cap, self.M,
                             self.path,
                             self.accept_len, self.status, self.max_depth, self.kv_start, self.kv_len,
                             self.max_len, int(self.realign), self.attn_mask, self.pos_ids, stream)

    def step(self, stream=None) -> StepResult:
        """One verification step on device-resident inputs (asynchronous); the tree
        rows' K/V must already be in the cache."""
        self.build_mask(stream)
        for layer in range(self.L):
            self.attention(layer, stream)
        self.accept(stream)
        self.commit(stream)
        return StepResult(self.accept_len, self.path, self.bonus)

    # ------------------------------------------------------------------ host path
    def tree_row_views(self, layer):
        """Per-sequence device views of the M+1 tree rows behind each prefix
        (columns kv_start + kv_len + r) of one layer, for K and V."""
        ks = self.kv_start.tolist()
        kl = self.kv_len.tolist()
        views = []
        for b in range(self.B):
            c0 = ks[b] + kl[b]
            views.append((self.k[layer][b, :, c0:c0 + self.n], self.v[layer][b, :, c0:c0 + self.n]))
        return views

    def pinned_inputs(self):
        """Pinned host staging buffers (allocated once): parent, draft, logits,
        q [L][B][M+1][Hq][D], tree_k / tree_v [L][B][Hkv][M+1][D] for the inputs;
        accept_len, path, bonus for the results."""
        if self._host is None:
            buf = torch.zeros(self.layout.nbytes, dtype=torch.uint8, pin_memory=True)
            res = torch.zeros(self._results.shape, dtype=torch.int32, pin_memory=True)
            B, md = self.B, self.max_depth
            h = self.layout.views(buf)
            h.update(_buf=buf, _res=res, accept_len=res[:B], path=res[B:B + B * (md + 1)].view(B, md + 1),
                     bonus=res[B + B * (md + 1):])
            self._host = h
        return self._host

    def h2d_bytes(self) -> int:
        lay = self.layout
        return lay.meta_bytes + lay.logits_bytes + lay.L * (lay.q_bytes + 2 * lay.rows_bytes)

    def d2h_bytes(self) -> int:
        return self._results.numel() * 4

    def step_from_host(self, host=None, stream=None):
        """End-to-end step: the inputs in the pinned staging buffers (see
        pinned_inputs()) are copied in on a copy stream, a section at a time; each
        layer's tree rows are written into the cache and its attention runs as
        soon as that layer's section has landed; accept_len / path / bonus come
        back into the pinned result buffers.  Asynchronous: synchronise on
        `stream` before reading the results, and before rewriting the staging
        buffer for the next step (its copies may still be in flight)."""
        h = host if host is not None else self.pinned_inputs()
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        if self._copy_stream is None:
            self._copy_stream = torch.cuda.Stream(self.device)
            self._events = [torch.cuda.Event() for _ in range(self.L + 3)]
            self._events[-1].record(s)
        cs, ev = self._copy_stream, self._events
        lay, src, dst = self.layout, h["_buf"], self._inputs
        cs.wait_event(ev[-1])  # the previous step has finished reading the device inputs
        with torch.cuda.stream(cs):
            dst[:lay.meta_bytes].copy_(src[:lay.meta_bytes], non_blocking=True)
            ev[0].record(cs)
            for layer in range(self.L):
                o = lay.layer_off(layer)
                dst[o:o + lay.layer_bytes].copy_(src[o:o + lay.layer_bytes], non_blocking=True)
                ev[1 + layer].record(cs)
            o = lay.logits_off
            dst[o:o + lay.logits_bytes].copy_(src[o:o + lay.logits_bytes], non_blocking=True)
            ev[1 + self.L].record(cs)
        with torch.cuda.stream(s):
            s.wait_event(ev[0])
            self.build_mask(s)
            for layer in range(self.L):
                s.wait_event(ev[1 + layer])
                self.write_tree_rows(layer, s)
                self.attention(layer, s)
            s.wait_event(ev[1 + self.L])
            self.accept(s)
            self.commit(s)
            h["_res"].copy_(self._results, non_blocking=True)
            ev[-1].record(s)
        return StepResult(h["accept_len"], h["path"], h["bonus"])
