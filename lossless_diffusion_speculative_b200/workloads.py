"""Seeded synthetic workloads for the Orthrus dual-view decode step.

This module only draws inputs.  It holds none of the method's arithmetic (no
attention, no argmax, no prefix match): the tests feed what it returns both to
the CPU oracle and to the CUDA library, and the benchmark uploads it.

Shapes follow the five Qwen3-shaped workloads of the decode step (the pages
name the Qwen3 1.7B / 4B / 8B family and K = 32; head counts, head_dim and
layer counts are those models' published shapes).  Values are drawn on the host
with numpy's PCG64, rounded to bf16 with round-to-nearest-even where the
workload is bf16, and returned as float32 arrays that hold those values exactly.
Seeds are ``1000*config + 10*layer + tensor_id``.

The public benchmarks the pages evaluate on (MATH-500, GSM8K, AIME, HumanEval,
MBPP) are not used; planted acceptance lengths stand in for their acceptance
statistics: every logits row gets a planted unique argmax (row max + 1.0) and
the proposals match it on exactly the first ``a`` slots.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Tuple

import numpy as np

# tensor ids inside one layer's seed block
T_K_CTX, T_V_CTX = 1, 2
T_Q = {0: 3, 1: 6}          # view -> query tensor id (0 = DIFF, 1 = AR)
T_K_BLK = {0: 4, 1: 7}
T_V_BLK = {0: 5, 1: 8}
T_LOGITS, T_PLANT = 9, 10   # consensus inputs (layer index 99)
T_HIDDEN, T_LMHEAD, T_LMPLANT = 11, 12, 13   # fused LM-head inputs (layer index 97)


@dataclass(frozen=True)
class Workload:
    """One decode-step workload.  ``ctx`` is the per-sequence committed length."""
    cid: int
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    K: int
    layers: int
    dtype: str                 # "f32" or "bf16"
    vocab: int
    logit_sigma: float
    plant: str                 # "fixed:a", "geom:p", "uniform", "half"
    ctx_lo: int
    ctx_hi: int                # ctx_b = ctx_lo when lo == hi, else U[lo, hi]
    value_scale: float         # Q/K/V ~ N(0,1) * value_scale
    extra_rows: int = -1       # cache rows beyond max(ctx)+K (default: K)
    note: str = ""
    hidden: int = 4096         # model width (the AR LM head's input size)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def ctx_lens(self) -> np.ndarray:
        if self.ctx_lo == self.ctx_hi:
            return np.full(self.B, self.ctx_lo, dtype=np.int32)
        rng = np.random.Generator(np.random.PCG64(1000 * self.cid + 7))
        return rng.integers(self.ctx_lo, self.ctx_hi + 1, size=self.B).astype(np.int32)

    @property
    def S_max(self) -> int:
        extra = self.K if self.extra_rows < 0 else self.extra_rows
        s = int(self.ctx_lens().max()) + self.K + extra
        return (s + 7) // 8 * 8

    def kv_bytes_per_view_layer(self) -> int:
        """Algorithmic K+V bytes one view reads for one layer."""
        esz = 4 if self.dtype == "f32" else 2
        return int(self.Hkv * (self.ctx_lens().astype(np.int64) + self.K).sum()
                   * self.D * esz * 2)

    def attn_flops_per_view_layer(self) -> int:
        return int(4 * self.Hq * self.K * self.D
                   * (self.ctx_lens().astype(np.int64) + self.K).sum())

    def with_(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


_INV_SQRT_128 = 1.0 / np.sqrt(128.0)

WORKLOADS = {
    "tiny_f32": Workload(1, "tiny_f32", B=1, Hq=4, Hkv=2, D=64, K=8, layers=1,
                         dtype="f32", vocab=1000, logit_sigma=1.0, plant="fixed:3",
                         ctx_lo=256, ctx_hi=256, value_scale=1.0, hidden=256,
                         note="tiny single step, fp32, 1 layer"),
    "qwen3_1p7b_layer": Workload(2, "qwen3_1p7b_layer", B=1, Hq=16, Hkv=8, D=128, K=32,
                                 layers=1, dtype="bf16", vocab=151936, logit_sigma=2.0,
                                 plant="geom:0.14285714285714285", ctx_lo=4096,
                                 ctx_hi=4096, value_scale=_INV_SQRT_128, hidden=2048,
                                 note="Qwen3-1.7B-shaped single layer"),
    "qwen3_8b_step": Workload(3, "qwen3_8b_step", B=1, Hq=32, Hkv=8, D=128, K=32,
                              layers=36, dtype="bf16", vocab=151936, logit_sigma=2.0,
                              plant="uniform", ctx_lo=8192, ctx_hi=8192,
                              value_scale=_INV_SQRT_128,
                              note="Qwen3-8B-shaped decode step, 36 layers"),
    "qwen3_4b_ragged": Workload(4, "qwen3_4b_ragged", B=16, Hq=32, Hkv=8, D=128, K=32,
                                layers=1, dtype="bf16", vocab=151936, logit_sigma=2.0,
                                plant="geom:0.1111111111111111", ctx_lo=2048,
                                ctx_hi=16384, value_scale=_INV_SQRT_128, hidden=2560,
                                note="Qwen3-4B-shaped ragged batch of 16"),
    "qwen3_8b_long_k8": Workload(5, "qwen3_8b_long_k8", B=4, Hq=32, Hkv=8, D=128, K=8,
                                 layers=1, dtype="bf16", vocab=151936, logit_sigma=2.0,
                                 plant="half", ctx_lo=32768, ctx_hi=32768,
                                 value_scale=_INV_SQRT_128, note="long context, K=8"),
    "qwen3_8b_long_k16": Workload(5, "qwen3_8b_long_k16", B=4, Hq=32, Hkv=8, D=128, K=16,
                                  layers=1, dtype="bf16", vocab=151936, logit_sigma=2.0,
                                  plant="half", ctx_lo=32768, ctx_hi=32768,
                                  value_scale=_INV_SQRT_128, note="long context, K=16"),
    "qwen3_8b_long_k32": Workload(5, "qwen3_8b_long_k32", B=4, Hq=32, Hkv=8, D=128, K=32,
                                  layers=1, dtype="bf16", vocab=151936, logit_sigma=2.0,
                                  plant="half", ctx_lo=32768, ctx_hi=32768,
                                  value_scale=_INV_SQRT_128, note="long context, K=32"),
}


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32.

    Input quantisation only: the workloads are bf16 tensors.  Values are finite.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    r = ((u + bias) >> np.uint32(16)) << np.uint32(16)
    return r.astype(np.uint32).view(np.float32)


def _rng(w: Workload, layer: int, tensor_id: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(1000 * w.cid + 10 * layer + tensor_id))


def _normal(w: Workload, layer: int, tid: int, shape) -> np.ndarray:
    x = _rng(w, layer, tid).standard_normal(size=shape, dtype=np.float32)
    x *= np.float32(w.value_scale)
    return round_to_bf16(x) if w.dtype == "bf16" else x


@dataclass
class LayerInputs:
    """Host copies of one layer's inputs for one view (float32, exact values)."""
    q: np.ndarray             # [B, K, Hq, D]
    k_cache: np.ndarray       # [B, Hkv, S_max, D]; block rows already installed
    v_cache: np.ndarray
    k_blk: np.ndarray         # [B, K, Hkv, D]  this view's block keys
    v_blk: np.ndarray
    ctx_lens: np.ndarray      # [B] int32


def context_cache(w: Workload, layer: int, poison: bool = True) -> Tuple[np.ndarray, np.ndarray]:
    """K and V caches [B,Hkv,S_max,D] with the committed context rows filled.

    Rows at and beyond ctx_b hold NaN when ``poison`` (nothing may read them
    before the block is installed); otherwise zeros.  Sequence b's rows are
    drawn in order b = 0..B-1 from one stream per tensor.
    """
    ctx = w.ctx_lens()
    S = w.S_max
    fill = np.float32(np.nan if poison else 0.0)
    kc = np.empty((w.B, w.Hkv, S, w.D), dtype=np.float32)
    vc = np.empty((w.B, w.Hkv, S, w.D), dtype=np.float32)
    rk, rv = _rng(w, layer, T_K_CTX), _rng(w, layer, T_V_CTX)
    for b in range(w.B):
        c = int(ctx[b])
        for dst, rng in ((kc, rk), (vc, rv)):
            x = rng.standard_normal(size=(w.Hkv, c, w.D), dtype=np.float32)
            x *= np.float32(w.value_scale)
            dst[b, :, :c] = round_to_bf16(x) if w.dtype == "bf16" else x
            dst[b, :, c:] = fill
    return kc, vc


def block_inputs(w: Workload, layer: int, view: int):
    """(q [B,K,Hq,D], k_blk [B,K,Hkv,D], v_blk [B,K,Hkv,D]) of one view."""
    q = _normal(w, layer, T_Q[view], (w.B, w.K, w.Hq, w.D))
    kb = _normal(w, layer, T_K_BLK[view], (w.B, w.K, w.Hkv, w.D))
    vb = _normal(w, layer, T_V_BLK[view], (w.B, w.K, w.Hkv, w.D))
    return q, kb, vb


def install_block(k_cache: np.ndarray, v_cache: np.ndarray, k_blk: np.ndarray,
                  v_blk: np.ndarray, ctx_lens: np.ndarray) -> None:
    """Write block slot s of sequence b into cache row ctx_b + s (caller's job
    in a real model: the view's K/V projection writes the block's rows)."""
    B, K = k_blk.shape[:2]
    for b in range(B):
        c = int(ctx_lens[b])
        k_cache[b, :, c:c + K] = k_blk[b].transpose(1, 0, 2)
        v_cache[b, :, c:c + K] = v_blk[b].transpose(1, 0, 2)


def layer_inputs(w: Workload, layer: int, view: int, poison: bool = True) -> LayerInputs:
    kc, vc = context_cache(w, layer, poison=poison)
    q, kb, vb = block_inputs(w, layer, view)
    ctx = w.ctx_lens()
    install_block(kc, vc, kb, vb, ctx)
    return LayerInputs(q, kc, vc, kb, vb, ctx)


@dataclass
class ConsensusInputs:
    logits: np.ndarray        # [B, K, V] float32
    proposed: np.ndarray      # [B, K] int32
    planted_argmax: np.ndarray  # [B, K] int32, the unique maximum of each row
    planted_accept: np.ndarray  # [B] int32
    planted_next: np.ndarray    # [B] int32


def planted_accept_lengths(w: Workload) -> np.ndarray:
    rng = _rng(w, 99, T_PLANT)
    kind, _, arg = w.plant.partition(":")
    if kind == "fixed":
        a = np.full(w.B, int(arg))
    elif kind == "geom":
        a = rng.geometric(float(arg), size=w.B) - 1
    elif kind == "uniform":
        a = rng.integers(0, w.K + 1, size=w.B)
    elif kind == "half":
        a = np.full(w.B, w.K // 2)
    else:
        raise ValueError(w.plant)
    return np.minimum(a, w.K).astype(np.int32)


def expected_tokens_per_step(w: Workload) -> float:
    """E[sum_b min(a_b + 1, K)] under the workload's planted acceptance law
    (the seeded draw gives one sample of it; the kernels' time does not depend
    on it).  Per sequence:
      fixed:a   min(a + 1, K)
      geom:p    a = min(X - 1, K), X ~ Geometric(p) on {1, 2, ...}:
                E[min(X, K)] = sum_{j=1..K} P(X >= j) = (1 - (1 - p)^K) / p
      uniform   a ~ U{0..K}: (sum_{a<K} (a + 1) + K) / (K + 1)
      half      a = K // 2: min(K // 2 + 1, K)
    """
    K = w.K
    kind, _, arg = w.plant.partition(":")
    if kind == "fixed":
        per = min(int(arg) + 1, K)
    elif kind == "geom":
        p = float(arg)
        per = (1.0 - (1.0 - p) ** K) / p
    elif kind == "uniform":
        per = (K * (K + 1) / 2 + K) / (K + 1)
    elif kind == "half":
        per = min(K // 2 + 1, K)
    else:
        raise ValueError(w.plant)
    return float(w.B * per)


def consensus_inputs(w: Workload, accept: Optional[np.ndarray] = None,
                     B: Optional[int] = None) -> ConsensusInputs:
    """Logits ~ N(0, sigma) with a planted unique argmax per row (margin 1.0)
    and proposals matching it on exactly the first a_b slots."""
    B = w.B if B is None else B
    K, V = w.K, w.vocab
    rng = _rng(w, 99, T_LOGITS)
    logits = rng.standard_normal(size=(B, K, V), dtype=np.float32)
    logits *= np.float32(w.logit_sigma)
    r = rng.integers(0, V, size=(B, K)).astype(np.int32)
    top = logits.max(axis=2)
    bi, ki = np.meshgrid(np.arange(B), np.arange(K), indexing="ij")
    logits[bi, ki, r] = top + np.float32(1.0)
    a = planted_accept_lengths(w)[:B] if accept is None else np.asarray(accept, np.int32)
    prop = rng.integers(0, V, size=(B, K)).astype(np.int32)
    for b in range(B):
        prop[b, :a[b]] = r[b, :a[b]]
        if a[b] < K:
            prop[b, a[b]] = (r[b, a[b]] + 1 + rng.integers(0, V - 1)) % V
    nxt = r[np.arange(B), np.minimum(a, K - 1)].astype(np.int32)
    return ConsensusInputs(logits, prop, r, a.astype(np.int32), nxt)


@dataclass
class LMHeadInputs:
    hidden: np.ndarray          # [B, K, Hd] float32 holding bf16 values
    lm_head: np.ndarray         # [V, Hd] float32 holding bf16 values
    proposed: np.ndarray        # [B, K] int32
    planted_argmax: np.ndarray  # [B, K] int32
    planted_accept: np.ndarray  # [B] int32
    planted_next: np.ndarray    # [B] int32


def lm_head_inputs(w: Workload, Hd: Optional[int] = None, V: Optional[int] = None,
                   accept: Optional[np.ndarray] = None, plant: bool = True) -> LMHeadInputs:
    """Inputs of the fused AR LM head + consensus: the AR view's final hidden
    states h [B, K, Hd] ~ N(0, 1) and a weight W [V, Hd] ~ N(0, 1/Hd), both
    rounded to bf16 (random logits ~ N(0, 1)).

    With ``plant``, every token row t gets its own planted token r_t (distinct)
    whose weight row is W[r_t] = 12 h_t / |h_t|^2: its logit is 12, far above
    the random ones (max ~ 4.6 over 151936) and the other planted rows' cross
    terms (~ 12 / sqrt(Hd) std), so the argmax is known; the proposals match it
    on exactly the first a_b slots (the workload's acceptance law)."""
    Hd = w.hidden if Hd is None else Hd
    V = w.vocab if V is None else V
    B, K = w.B, w.K
    rng = _rng(w, 97, T_HIDDEN)
    h = round_to_bf16(rng.standard_normal((B, K, Hd), dtype=np.float32))
    W = _rng(w, 97, T_LMHEAD).standard_normal((V, Hd), dtype=np.float32)
    W *= np.float32(1.0 / np.sqrt(Hd))
    W = round_to_bf16(W)
    prng = _rng(w, 97, T_LMPLANT)
    r = prng.choice(V, size=B * K, replace=False).astype(np.int32) if plant else \
        np.zeros(B * K, np.int32)
    if plant:
        hf = h.reshape(B * K, Hd).astype(np.float64)
        rows = 12.0 * hf / (hf * hf).sum(axis=1, keepdims=True)
        W[r] = round_to_bf16(rows.astype(np.float32))
    r = r.reshape(B, K)
    a = planted_accept_lengths(w) if accept is None else np.asarray(accept, np.int32)
    prop = prng.integers(0, V, size=(B, K)).astype(np.int32)
    for b in range(B):
        prop[b, :a[b]] = r[b, :a[b]]
        if a[b] < K:
            prop[b, a[b]] = (r[b, a[b]] + 1 + prng.integers(0, V - 1)) % V
    nxt = r[np.arange(B), np.minimum(a, K - 1)].astype(np.int32)
    return LMHeadInputs(h, W, prop, r, a.astype(np.int32), nxt)
