"""Device-resident driver of one Orthrus dual-view decode step (hot path only).

One step, per the technical summary of "Orthrus: Memory-Efficient Parallel
Token Generation via Dual-View Diffusion" (gist.science), section 2.3:

    write_block(DIFF)  -> attention(DIFF) for every layer   (parallel projection)
    write_block(AR)    -> attention(AR)   for every layer   (structural verification)
    consensus(AR logits, proposals)                          (consensus)
    kv_commit(accepted prefix)                               (commitment / truncation)

The projections, MLPs and LM heads that sit between these calls need trained
weights and are not part of this path: their outputs (queries, block K/V,
logits, proposals) are seeded synthetic tensors resident on the device.  The
"cold" order (all DIFF layers, then all AR layers) is the model's real order,
so each view re-reads every layer's cache from HBM; "interleaved" runs DIFF
then AR per layer (the AR pass may then hit L2).

Every kernel launched here is liborthrus's, through its C ABI; the only other
device work is a 4-byte-per-sequence copy that restores ctx_lens between
benchmark steps so every step sees the same workload.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import numpy as np
import torch

from . import binding as ob
from . import workloads as wl



def layer_groups(L: int, chunk) -> list:
    """Consecutive layer ranges covering [0, L): groups of ``chunk`` layers, or
    of the sizes in ``chunk`` (a sequence; its last size repeats)."""
    sizes = [int(chunk)] if isinstance(chunk, int) else [int(c) for c in chunk]
    out, c, k = [], 0, 0
    while c < L:
        n = max(1, sizes[min(k, len(sizes) - 1)])
        out.append(range(c, min(c + n, L)))
        c += n
        k += 1
    return out

@dataclass
class StepResult:
    accepted: np.ndarray
    next_token: np.ndarray
    ctx_after: np.ndarray


class DecodeStep:
    def __init__(self, w: wl.Workload, layers: Optional[int] = None, order: str = "cold",
                 device: Optional[torch.device] = None, project: bool = False):
        assert order in ("cold", "interleaved", "fused")
        self.w = w
        self.L = w.layers if layers is None else layers
        self.order = order
        self.dev = device or torch.device("cuda", torch.cuda.current_device())
        self.dtype = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        B, K, Hq, Hkv, D, S = w.B, w.K, w.Hq, w.Hkv, w.D, w.S_max
        dev, dt = self.dev, self.dtype
        self.ctx0 = torch.from_numpy(w.ctx_lens()).to(dev)
        self.ctx = self.ctx0.clone()
        # per-layer caches (context rows seeded; block rows installed per view)
        self.k_cache: List[torch.Tensor] = []
        self.v_cache: List[torch.Tensor] = []
        for layer in range(self.L):
            kc, vc = wl.context_cache(w, layer, poison=False)
            self.k_cache.append(torch.from_numpy(kc).to(dev, dt))
            self.v_cache.append(torch.from_numpy(vc).to(dev, dt))
        # per-step inputs, one contiguous buffer each so a host copy is one transfer
        self.q_all = torch.empty((2, self.L, B, K, Hq, D), dtype=dt, device=dev)
        self.kb_all = torch.empty((2, self.L, B, K, Hkv, D), dtype=dt, device=dev)
        self.vb_all = torch.empty((2, self.L, B, K, Hkv, D), dtype=dt, device=dev)
        for view in (ob.DIFF, ob.AR):
            for layer in range(self.L):
                q, kb, vb = wl.block_inputs(w, layer, view)
                self.q_all[view, layer].copy_(torch.from_numpy(q))
                self.kb_all[view, layer].copy_(torch.from_numpy(kb))
                self.vb_all[view, layer].copy_(torch.from_numpy(vb))
        ci = wl.consensus_inputs(w)
        self.consensus_in = ci
        self.logits = torch.from_numpy(ci.logits).to(dev)
        self.proposed = torch.from_numpy(ci.proposed).to(dev)
        self.out = [torch.empty((B, K, Hq, D), dtype=torch.float32, device=dev) for _ in range(2)]
        self.accepted = torch.empty(B, dtype=torch.int32, device=dev)
        self.next_token = torch.empty(B, dtype=torch.int32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.attn_ws = torch.zeros(ob.orthrus_attn_workspace_size(B, Hq, Hkv, D, K, dt),
                                   dtype=torch.uint8, device=dev)
        self.cons_ws = torch.empty(ob.orthrus_consensus_workspace_size(B, K, w.vocab),
                                   dtype=torch.uint8, device=dev)
        self.graphs = None
        self.whole = None
        self.tc_path = ob.orthrus_attn_path(B, Hq, Hkv, D, K, dt) == 1
        self.project = False
        if project:
            self.enable_projection()

    def enable_projection(self):
        """The fused layer step: each view's block hidden states x and every
        layer's projection weights (random, N(0, 1/hidden)), drawn on the device
        from a seeded generator; orthrus_qkv_project writes q_all and the cache
        tail, replacing the block install."""
        if self.project:
            return
        w, dev, dt = self.w, self.dev, self.dtype
        B, K, Hq, Hkv, D, Hd = w.B, w.K, w.Hq, w.Hkv, w.D, w.hidden
        g = torch.Generator(device=dev)
        g.manual_seed(1000 * w.cid + 95)
        self.x_all = torch.randn((2, self.L, B, K, Hd), generator=g, device=dev).to(dt)
        sc = 1.0 / Hd ** 0.5
        self.w_qkv = []
        for _ in range(self.L):
            self.w_qkv.append(tuple(
                (torch.randn((n * D, Hd), generator=g, device=dev) * sc).to(dt)
                for n in (Hq, Hkv, Hkv)))
        self.qkv_ws = torch.zeros(ob.orthrus_qkv_workspace_size(B, K, Hd, Hq, Hkv, D), dtype=torch.uint8,
                                  device=dev)
        self.project = True

    # -- the hot path, as launch sequences ---------------------------------
    def _write_block(self, view, layers=None):
        layers = range(self.L) if layers is None else layers
        ob.orthrus_write_block(self.ctx, [self.k_cache[l] for l in layers], [self.v_cache[l] for l in layers],
                               [self.kb_all[view, l] for l in layers],
                               [self.vb_all[view, l] for l in layers], status=self.status)

    def _attn(self, view, layer):
        ob.orthrus_attn(view, self.q_all[view, layer], self.k_cache[layer], self.v_cache[layer],
                        self.ctx, self.out[view], self.attn_ws, status=self.status)

    def _attn_view(self, view):
        for layer in range(self.L):
            self._attn(view, layer)

    def _project(self, view, layer):
        wq, wk, wv = self.w_qkv[layer]
        ob.orthrus_qkv_project(self.x_all[view, layer], wq, wk, wv, self.ctx, self.q_all[view, layer],
                               self.k_cache[layer], self.v_cache[layer], self.qkv_ws, status=self.status)

    def _fused_view(self, view):
        for layer in range(self.L):
            self._project(view, layer)
            self._attn(view, layer)

    def _project_view(self, view):
        for layer in range(self.L):
            self._project(view, layer)

    def _tail(self):
        w = self.w
        ob.orthrus_consensus(self.logits, self.proposed, self.accepted, self.next_token,
                             self.cons_ws, status=self.status)
        ob.orthrus_kv_commit(self.ctx, self.accepted, K=w.K, Hkv=w.Hkv, D=w.D, S_max=w.S_max,
                             dtype=self.dtype, num_layers=self.L, status=self.status)

    def segments(self, chunk: int = 0, order: Optional[str] = None):
        """The step as ordered launch segments (timed separately by the bench).

        With ``chunk`` (cold order: a group size, or a sequence of group sizes
        with the last repeated to cover the layers, or a dict of either per
        view, keys "diff" and "ar") each view runs as layer groups, block
        install then attention per group: the same launches' work in smaller
        segments, so that a caller feeding the step from the host can start
        each group once its inputs have arrived.
        """
        order = self.order if order is None else order
        if order == "fused":
            # per layer: QKV projection (q + cache tail) -> attention, per view
            return [("fused_diff", lambda: self._fused_view(ob.DIFF)),
                    ("fused_ar", lambda: self._fused_view(ob.AR)),
                    ("consensus_commit", self._tail)]
        if order == "project_only":
            return [("project_diff", lambda: self._project_view(ob.DIFF)),
                    ("project_ar", lambda: self._project_view(ob.AR))]
        if order == "cold" and chunk:
            segs = []
            for view, vn in ((ob.DIFF, "diff"), (ob.AR, "ar")):
                for layers in layer_groups(self.L, chunk[vn] if isinstance(chunk, dict) else chunk):
                    c = layers.start
                    segs.append((f"write_block_{vn}_{c}", lambda v=view, ls=layers: self._write_block(v, ls)))
                    segs.append((f"attn_{vn}_{c}", lambda v=view, ls=layers: [self._attn(v, l) for l in ls]))
            segs.append(("consensus_commit", self._tail))
            return segs
        if order == "cold":
            return [("write_block_diff", lambda: self._write_block(ob.DIFF)),
                    ("attn_diff", lambda: self._attn_view(ob.DIFF)),
                    ("write_block_ar", lambda: self._write_block(ob.AR)),
                    ("attn_ar", lambda: self._attn_view(ob.AR)),
                    ("consensus_commit", self._tail)]
        # interleaved: per-layer DIFF then AR (block install for one layer at a time)
        def inter():
            for layer in range(self.L):
                for view in (ob.DIFF, ob.AR):
                    ob.orthrus_write_block(self.ctx, [self.k_cache[layer]], [self.v_cache[layer]],
                                           [self.kb_all[view, layer]], [self.vb_all[view, layer]],
                                           status=self.status)
                    self._attn(view, layer)
        return [("attn_interleaved", inter), ("consensus_commit", self._tail)]

    def reset(self):
        self.ctx.copy_(self.ctx0, non_blocking=True)

    def run_eager(self, chunk: int = 0):
        self.reset()
        for _, fn in self.segments(chunk):
            fn()

    def capture(self, stream: torch.cuda.Stream, chunk: int = 0, order: Optional[str] = None):
        """CUDA graphs of the reset and of every segment (captured on ``stream``)."""
        self.reset()
        for _, fn in self.segments(chunk, order):   # warm: attributes set, plans cached
            fn()
        torch.cuda.synchronize()
        graphs = []
        with torch.cuda.stream(stream):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                self.reset()
            graphs.append(("reset", g))
            for name, fn in self.segments(chunk, order):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    fn()
                graphs.append((name, g))
        torch.cuda.synchronize()
        self.graphs = graphs
        return graphs

    def capture_whole(self, stream: torch.cuda.Stream, order: Optional[str] = None) -> torch.cuda.CUDAGraph:
        """One CUDA graph of the whole step: the reset and every segment."""
        self.reset()
        for _, fn in self.segments(0, order):      # warm: attributes set, plans cached
            fn()
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                self.reset()
                for _, fn in self.segments(0, order):
                    fn()
        torch.cuda.synchronize()
        self.whole = g
        return g

    def result(self) -> StepResult:
        torch.cuda.synchronize()
        return StepResult(self.accepted.cpu().numpy(), self.next_token.cpu().numpy(),
                          self.ctx.cpu().numpy())

    def tokens_per_step(self) -> int:
        """Verified tokens one step commits: sum_b min(a_b + 1, K) (planted a)."""
        a = self.consensus_in.planted_accept
        return int(np.minimum(a + 1, self.w.K).sum())

    def tokens_per_step_expected(self) -> float:
        """The same count's expectation under the workload's acceptance law."""
        return wl.expected_tokens_per_step(self.w)

    def kv_bytes_per_attn_call(self) -> int:
        return self.w.kv_bytes_per_view_layer()
