"""Host-side driver of one whole verification step.

``TreeVerifier`` owns the device buffers of one workload shape and chains the
four C-ABI calls on one CUDA stream:

    tree_build_mask -> tree_attention (every layer) -> tree_accept -> kv_commit_realign

``step()`` works on inputs already resident on the GPU (and can be captured in
a CUDA graph).  ``step_from_host()`` is the end-to-end entry point for callers
that hold the step's inputs in host memory: it copies them to the device,
runs ``step()`` and copies the accept results back.  Nothing here computes: it
allocates, copies and calls.
"""
from __future__ import annotations

import dataclasses

import torch

from . import _lib as tv


@dataclasses.dataclass
class StepResult:
    accept_len: torch.Tensor  # [B] int32
    path: torch.Tensor  # [B][max_depth+1] int32
    bonus: torch.Tensor  # [B] int32


class TreeVerifier:
    def __init__(self, B, M, Hq, Hkv, D, V, L, S_cap, max_depth, realign=False, device="cuda",
                 k_layers=None, v_layers=None, with_mask_outputs=None):
        self.B, self.M, self.Hq, self.Hkv, self.D, self.V, self.L = B, M, Hq, Hkv, D, V, L
        self.S_cap, self.max_depth, self.realign = S_cap, max_depth, bool(realign)
        self.n = M + 1
        self.W = (self.n + 31) // 32
        dev = torch.device(device)
        self.device = dev
        i32 = dict(dtype=torch.int32, device=dev)
        bf = dict(dtype=torch.bfloat16, device=dev)
        self.parent = torch.zeros((B, self.n), **i32)
        self.draft = torch.zeros((B, self.n), **i32)
        self.anc = torch.zeros((B, self.n, self.W), **i32)
        self.depth = torch.zeros((B, self.n), **i32)
        self.status = torch.zeros((B,), **i32)
        self.kv_start = torch.zeros((B,), **i32)
        self.kv_len = torch.zeros((B,), **i32)
        self.max_len = torch.zeros((1,), **i32)
        self.q = [torch.zeros((B, self.n, Hq, D), **bf) for _ in range(L)]
        self.out = [torch.zeros((B, self.n, Hq, D), **bf) for _ in range(L)]
        self.k = k_layers if k_layers is not None else [torch.zeros((B, Hkv, S_cap, D), **bf) for _ in range(L)]
        self.v = v_layers if v_layers is not None else [torch.zeros((B, Hkv, S_cap, D), **bf) for _ in range(L)]
        self.k_ptrs = tv.layer_pointers(self.k, dev)
        self.v_ptrs = tv.layer_pointers(self.v, dev)
        self.workspace = tv.attention_workspace(B, M, Hq, Hkv, D, S_cap, dev)
        self.logits = torch.zeros((B, self.n, V), dtype=torch.float32, device=dev)
        self.argmax = torch.zeros((B, self.n), **i32)
        self.accept_len = torch.zeros((B,), **i32)
        self.path = torch.zeros((B, max_depth + 1), **i32)
        self.bonus = torch.zeros((B,), **i32)
        want_mask = self.realign if with_mask_outputs is None else with_mask_outputs
        self.attn_mask = torch.zeros((B, S_cap), dtype=torch.uint8, device=dev) if want_mask else None
        self.pos_ids = torch.zeros((B, S_cap), **i32) if want_mask else None
        self._host = None

    # ------------------------------------------------------------------ device path
    def launches_per_step(self) -> int:
        """Kernels this library launches per step: mask 1, attention 1 per layer,
        accept 2, commit 2."""
        return 1 + self.L + 2 + 2

    def build_mask(self, stream=None):
        tv.tree_build_mask(self.parent, self.max_depth, self.anc, self.depth, self.status, stream)

    def attention(self, layer, stream=None):
        tv.tree_attention(self.q[layer], self.k[layer], self.v[layer], self.kv_start, self.kv_len, self.anc,
                          self.status, self.out[layer], self.workspace, stream=stream)

    def accept(self, stream=None):
        tv.tree_accept(self.logits, self.draft, self.parent, self.depth, self.anc, self.status, self.max_depth,
                       self.argmax, self.accept_len, self.path, self.bonus, stream)

    def commit(self, stream=None):
        tv.kv_commit_realign(self.k_ptrs, self.v_ptrs, self.B, self.Hkv, self.D, self.S_cap, self.M, self.path,
                             self.accept_len, self.status, self.max_depth, self.kv_start, self.kv_len,
                             self.max_len, int(self.realign), self.attn_mask, self.pos_ids, stream)

    def step(self, stream=None) -> StepResult:
        """One verification step on device-resident inputs (asynchronous)."""
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
        """Pinned host buffers for the per-step inputs (allocated once)."""
        if self._host is None:
            B, n, L = self.B, self.n, self.L
            pin = dict(pin_memory=True)
            self._host = dict(
                parent=torch.zeros((B, n), dtype=torch.int32, **pin),
                draft=torch.zeros((B, n), dtype=torch.int32, **pin),
                q=torch.zeros((L, B, n, self.Hq, self.D), dtype=torch.bfloat16, **pin),
                tree_k=torch.zeros((L, B, self.Hkv, n, self.D), dtype=torch.bfloat16, **pin),
                tree_v=torch.zeros((L, B, self.Hkv, n, self.D), dtype=torch.bfloat16, **pin),
                logits=torch.zeros((B, n, self.V), dtype=torch.float32, **pin),
                accept_len=torch.zeros((B,), dtype=torch.int32, **pin),
                path=torch.zeros((B, self.max_depth + 1), dtype=torch.int32, **pin),
                bonus=torch.zeros((B,), dtype=torch.int32, **pin),
            )
        return self._host

    def h2d_bytes(self) -> int:
        h = self.pinned_inputs()
        return sum(h[k].numel() * h[k].element_size() for k in ("parent", "draft", "q", "tree_k", "tree_v", "logits"))

    def d2h_bytes(self) -> int:
        h = self.pinned_inputs()
        return sum(h[k].numel() * h[k].element_size() for k in ("accept_len", "path", "bonus"))

    def step_from_host(self, host=None, geometry=None, stream=None):
        """End-to-end step: copy the step's inputs from pinned host memory, run the
        four calls, copy accept_len / path / bonus back.  ``geometry`` is the host
        (kv_start, kv_len) the tree rows are written behind; it defaults to a
        device read of the current values."""
        h = host if host is not None else self.pinned_inputs()
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        with torch.cuda.stream(s):
            self.parent.copy_(h["parent"], non_blocking=True)
            self.draft.copy_(h["draft"], non_blocking=True)
            self.logits.copy_(h["logits"], non_blocking=True)
            if geometry is None:
                ks, kl = self.kv_start.tolist(), self.kv_len.tolist()
            else:
                ks, kl = geometry
            for layer in range(self.L):
                self.q[layer].copy_(h["q"][layer], non_blocking=True)
                for b in range(self.B):
                    c0 = ks[b] + kl[b]
                    self.k[layer][b, :, c0:c0 + self.n].copy_(h["tree_k"][layer, b], non_blocking=True)
                    self.v[layer][b, :, c0:c0 + self.n].copy_(h["tree_v"][layer, b], non_blocking=True)
            self.step(s)
            h["accept_len"].copy_(self.accept_len, non_blocking=True)
            h["path"].copy_(self.path, non_blocking=True)
            h["bonus"].copy_(self.bonus, non_blocking=True)
        return StepResult(h["accept_len"], h["path"], h["bonus"])
