"""CPU oracle for the Orthrus dual-view decode step.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``.  The product library never imports,
links or calls it, and it shares no code with the CUDA path.

The attention, consensus and commit arithmetic lives in ``orthrus_oracle.c``
(plain C, double precision, OpenMP over output rows); this module compiles it
with gcc and marshals numpy arrays through ctypes.  The fused LM-head consensus
(``lm_head_consensus``) is numpy in float64: one library matrix product for the
logits, then the argmax and the prefix walk written out here.  Each function follows the technical summary of
"Orthrus: Memory-Efficient Parallel Token Generation via Dual-View Diffusion"
(gist.science page), sections 2.2 (mask M_diff) and 2.3 (verification,
consensus and commitment); see the C file's header for the readings taken
where the pages are silent.

Parity pins (tests/test_oracle_pins.py): K=1 reduction to causal decode, DIFF
permutation invariance, AR view = K sequential decodes, explicit-mask brute
force, a library SDPA cross-check, closed forms, planted consensus, hand cases
and the lossless toy decode loop.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "orthrus_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

DIFF = 0
AR = 1

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle.so`` (gcc, -O2, OpenMP)."""
    stale = (not os.path.exists(_LIB_PATH)) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i32p = ctypes.POINTER(ctypes.c_int32)
        f32p = ctypes.POINTER(ctypes.c_float)
        f64p = ctypes.POINTER(ctypes.c_double)
        lib.oracle_attn.restype = ctypes.c_int
        lib.oracle_attn.argtypes = [
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, i32p, f32p, f32p, f32p, ctypes.c_double,
            ctypes.c_int, i32p, f64p, ctypes.c_int]
        lib.oracle_consensus.restype = None
        lib.oracle_consensus.argtypes = [
            ctypes.c_int, ctypes.c_int, ctypes.c_int, f32p, i32p, i32p, i32p, i32p]
        lib.oracle_kv_commit.restype = ctypes.c_int
        lib.oracle_kv_commit.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            i32p, i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_num_threads.argtypes = []
        _lib = lib
    return _lib


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def attention(view: int, q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
              ctx_lens: np.ndarray, scale: float = 0.0, rows=None,
              n_threads: int = 0) -> np.ndarray:
    """fp64 masked softmax attention of the DIFF (M_diff) or AR (causal) view.

    q [B,K,Hq,D], caches [B,Hkv,S_max,D] (values exact in float32), ctx_lens [B].
    Returns float64 [B,K,Hq,D], or [len(rows), D] when ``rows`` lists (b,i,h).
    """
    B, K, Hq, D = q.shape
    _, Hkv, S_max, D2 = k_cache.shape
    assert D2 == D and v_cache.shape == k_cache.shape
    q = np.ascontiguousarray(q, dtype=np.float32)
    k_cache = np.ascontiguousarray(k_cache, dtype=np.float32)
    v_cache = np.ascontiguousarray(v_cache, dtype=np.float32)
    ctx = np.ascontiguousarray(ctx_lens, dtype=np.int32)
    if rows is None:
        out = np.empty((B, K, Hq, D), dtype=np.float64)
        rp, n_rows = None, 0
    else:
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 3))
        n_rows = rows.shape[0]
        out = np.empty((n_rows, D), dtype=np.float64)
        rp = _ptr(rows, ctypes.c_int32)
    rc = _load().oracle_attn(
        int(view), B, Hq, Hkv, D, S_max, K, _ptr(ctx, ctypes.c_int32),
        _ptr(q, ctypes.c_float), _ptr(k_cache, ctypes.c_float),
        _ptr(v_cache, ctypes.c_float), float(scale), n_rows, rp,
        _ptr(out, ctypes.c_double), int(n_threads))
    if rc != 0:
        raise ValueError("oracle_attn: bad argument or capacity violation")
    return out


def consensus(logits: np.ndarray, proposed: np.ndarray):
    """Greedy consensus.  Returns (accepted_len [B], next_token [B], argmax [B,K])."""
    B, K, V = logits.shape
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    proposed = np.ascontiguousarray(proposed, dtype=np.int32)
    acc = np.empty(B, dtype=np.int32)
    nxt = np.empty(B, dtype=np.int32)
    am = np.empty((B, K), dtype=np.int32)
    _load().oracle_consensus(B, K, V, _ptr(logits, ctypes.c_float),
                             _ptr(proposed, ctypes.c_int32),
                             _ptr(acc, ctypes.c_int32), _ptr(nxt, ctypes.c_int32),
                             _ptr(am, ctypes.c_int32))
    return acc, nxt, am


def kv_commit(k_cache: np.ndarray, v_cache: np.ndarray, k_blk, v_blk,
              ctx_lens: np.ndarray, accepted: np.ndarray, K: int,
              advance: bool = True) -> None:
    """In-place commit of one layer: copy block slots 0..n-1 (if given), advance ctx.

    Caches [B,Hkv,S_max,D] and blocks [B,K,Hkv,D] of any fixed-size dtype; the
    copy is byte-exact.  ctx_lens (int32) is updated in place when ``advance``.
    """
    B, Hkv, S_max, D = k_cache.shape
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    assert ctx_lens.dtype == np.int32 and ctx_lens.flags.c_contiguous
    acc = np.ascontiguousarray(accepted, dtype=np.int32)
    kb = vb = None
    if k_blk is not None:
        assert k_blk.shape == (B, K, Hkv, D) and k_blk.dtype == k_cache.dtype
        k_blk = np.ascontiguousarray(k_blk)
        v_blk = np.ascontiguousarray(v_blk)
        kb, vb = k_blk.ctypes.data, v_blk.ctypes.data
    rc = _load().oracle_kv_commit(
        k_cache.ctypes.data, v_cache.ctypes.data, kb, vb,
        _ptr(ctx_lens, ctypes.c_int32), _ptr(acc, ctypes.c_int32),
        B, Hkv, D, S_max, K, k_cache.dtype.itemsize, 1 if advance else 0)
    if rc != 0:
        raise ValueError("oracle_kv_commit: bad argument or capacity violation")


def lm_head_logits(hidden: np.ndarray, lm_head: np.ndarray) -> np.ndarray:
    """float64 logits[t, v] = <hidden[t], lm_head[v]> for token rows t = b*K + i.

    The AR head scores every block position in one pass ("Orthrus: Memory-
    Efficient Parallel Token Generation via Dual-View Diffusion", gist.science
    technical summary, section 2.3 "structural verification").  hidden
    [B, K, Hd] and lm_head [V, Hd] hold bf16 values exactly (float32 arrays);
    the product is taken in float64 (a library matmul), so every logit is
    within ~1e-16 relative of the exact dot product.
    """
    B, K, Hd = hidden.shape
    V, Hd2 = lm_head.shape
    assert Hd2 == Hd
    h = np.asarray(hidden, np.float64).reshape(B * K, Hd)
    return h @ np.asarray(lm_head, np.float64).T


def lm_head_consensus(hidden: np.ndarray, lm_head: np.ndarray, proposed: np.ndarray):
    """Greedy consensus on the AR head's logits, never materialised on the GPU.

    r[b, i] = argmax_v logits[b*K + i, v] (lowest index wins ties), then the
    left-to-right prefix walk of section 2.3 "consensus and commitment": a =
    number of leading i with proposed[b, i] == r[b, i]; next = r[b, min(a, K-1)].

    Returns (accepted [B], next [B], argmax [B, K], gap [B, K], absdot [B, K])
    where gap is the float64 difference between each row's largest and second
    largest logit and absdot = max_v sum_d |hidden[t, d] * lm_head[v, d]|, the
    scale of the rounding error of a float32 accumulation of that row.
    """
    B, K, Hd = hidden.shape
    logits = lm_head_logits(hidden, lm_head)
    r = np.argmax(logits, axis=1)                       # first maximum = lowest index
    top2 = np.partition(logits, logits.shape[1] - 2, axis=1)[:, -2:] if logits.shape[1] > 1 else None
    gap = (top2[:, 1] - top2[:, 0]) if top2 is not None else np.full(B * K, np.inf)
    absdot = (np.abs(np.asarray(hidden, np.float64).reshape(B * K, Hd))
              @ np.abs(np.asarray(lm_head, np.float64)).T).max(axis=1)
    r = r.reshape(B, K).astype(np.int32)
    acc = np.empty(B, np.int32)
    nxt = np.empty(B, np.int32)
    for b in range(B):
        a = 0
        while a < K and int(proposed[b, a]) == int(r[b, a]):
            a += 1
        acc[b] = a
        nxt[b] = r[b, min(a, K - 1)]
    return acc, nxt, r, gap.reshape(B, K), absdot.reshape(B, K)


def fp32_dot_error_bound(n: int, absdot) -> np.ndarray:
    """Rigorous bound on |fl32(sum) - sum| for a float32 accumulation of n
    exact products (bf16 x bf16 products are exact in float32) in any order,
    with rounding to nearest or toward zero: gamma_n * sum |x_d y_d|, gamma_n =
    n*u / (1 - n*u), u = 2^-23 (the toward-zero unit, twice round-to-nearest's).
    """
    u = 2.0 ** -23
    return n * u / (1.0 - n * u) * np.asarray(absdot, np.float64)


def _softmax64(x: np.ndarray, temperature: float) -> np.ndarray:
    z = np.asarray(x, np.float64) / float(temperature)
    z = z - z.max()
    e = np.exp(z)
    return e / e.sum()


def rejection_verify(ar_logits: np.ndarray, draft_logits: np.ndarray, proposed: np.ndarray,
                     u_accept: np.ndarray, u_resample: np.ndarray, temperature: float):
    """Lossless verification of the block at temperature T > 0 (the pages
    evaluate "greedy and rejection sampling" -- Orthrus-Qwen3, agentlenshq.com,
    "limitations"; results "depending on task and temperature" -- gist.science
    technical summary, section 4 -- without a formula; this is the standard
    speculative-sampling rule, which keeps the AR head's distribution exactly).

    For sequence b, left to right over block slots i, with p = softmax(AR
    logits / T) and q = softmax(draft logits / T) of row i and x = proposed[b, i]:
      accept x  iff  u_accept[b, i] * q(x) < p(x)      (probability min(1, p/q));
    at the first rejection (slot a) the next token is drawn from the residual
    r(v) = max(0, p(v) - q(v)) by inverse CDF: the smallest v whose cumulative
    residual exceeds u_resample[b] * sum_v r(v) (from p itself if the residual
    is empty).  With all K accepted the next token is the last proposal (the AR
    view has not scored a token after the block).  Everything in float64.

    Returns (accepted [B], next [B], acc_margin [B, K], cdf_margin [B]): the
    relative margin of every accept decision taken, |u q(x) - p(x)| /
    max(p(x), u q(x)) (inf where not taken), and the distance of the resampling
    target from the nearest cumulative-residual boundary relative to the total
    residual (inf when nothing was resampled).
    """
    B, K, V = ar_logits.shape
    acc = np.zeros(B, np.int32)
    nxt = np.zeros(B, np.int32)
    acc_margin = np.full((B, K), np.inf)
    cdf_margin = np.full(B, np.inf)
    for b in range(B):
        a = 0
        p = q = None
        while a < K:
            p = _softmax64(ar_logits[b, a], temperature)
            q = _softmax64(draft_logits[b, a], temperature)
            x = int(proposed[b, a])
            lhs = float(u_accept[b, a]) * q[x]
            den = max(p[x], lhs)
            acc_margin[b, a] = abs(lhs - p[x]) / den if den > 0 else np.inf
            if not lhs < p[x]:
                break
            a += 1
        acc[b] = a
        if a == K:
            nxt[b] = int(proposed[b, K - 1])
            continue
        r = np.maximum(p - q, 0.0)
        if r.sum() <= 0.0:
            r = p
        cdf = np.cumsum(r)
        R = cdf[-1]
        target = float(u_resample[b]) * R
        v = int(np.searchsorted(cdf, target, side="right"))
        v = min(v, V - 1)
        while v > 0 and r[v] == 0.0:                  # (a zero-mass tail is never drawn)
            v -= 1
        nxt[b] = v
        lo = cdf[v - 1] if v > 0 else 0.0
        cdf_margin[b] = min(target - lo, cdf[v] - target) / R
    return acc, nxt, acc_margin, cdf_margin


def residual_cdf(ar_row: np.ndarray, draft_row: np.ndarray, temperature: float) -> np.ndarray:
    """float64 cumulative residual max(0, p - q) of one row (of p itself when
    the residual is empty), the distribution rejection_verify draws from."""
    p = _softmax64(ar_row, temperature)
    q = _softmax64(draft_row, temperature)
    r = np.maximum(p - q, 0.0)
    if r.sum() <= 0.0:
        r = p
    return np.cumsum(r)


def qkv_project(x: np.ndarray, w_q: np.ndarray, w_k: np.ndarray, w_v: np.ndarray, D: int):
    """float64 projections of a view's block ("Orthrus: Memory-Efficient
    Parallel Token Generation via Dual-View Diffusion", gist.science technical
    summary, section 2.3 "parallel projection" / "structural verification";
    section 2.1: the block's keys and values join the one shared cache).

    x [B, K, hidden]; w_q [Hq*D, hidden]; w_k, w_v [Hkv*D, hidden] (exact bf16
    values in float32).  Returns q [B, K, Hq, D], k [B, K, Hkv, D], v [B, K,
    Hkv, D] in float64 (one library matrix product each) and, for each output,
    sum_d |x_d w_d|, the scale of a float32 accumulation's rounding error.
    """
    B, K, hidden = x.shape
    xf = np.asarray(x, np.float64).reshape(B * K, hidden)
    xa = np.abs(xf)
    outs = []
    for w in (w_q, w_k, w_v):
        wf = np.asarray(w, np.float64)
        H = wf.shape[0] // D
        outs.append(((xf @ wf.T).reshape(B, K, H, D), (xa @ np.abs(wf).T).reshape(B, K, H, D)))
    (q, qa), (k, ka), (v, va) = outs
    return q, k, v, qa, ka, va


def install_block_rows(k_cache: np.ndarray, v_cache: np.ndarray, k_blk: np.ndarray, v_blk: np.ndarray,
                       ctx_lens: np.ndarray, S_max: int) -> None:
    """Cache rows [ctx_b, ctx_b + K) of every KV head take the block's keys and
    values (in place); a sequence without room (ctx_b < 0 or ctx_b + K > S_max)
    is left untouched."""
    B, K = k_blk.shape[:2]
    for b in range(B):
        c = int(ctx_lens[b])
        if c < 0 or c + K > S_max:
            continue
        k_cache[b, :, c:c + K] = np.transpose(k_blk[b], (1, 0, 2))
        v_cache[b, :, c:c + K] = np.transpose(v_blk[b], (1, 0, 2))
