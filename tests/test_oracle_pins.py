"""Pins for the CPU oracle: each check ties it to something other than itself.

Sources: "Orthrus: Memory-Efficient Parallel Token Generation via Dual-View
Diffusion" (gist.science technical summary) section 2.2 (mask M_diff: block
queries see the clean context causally and the block bidirectionally), section
2.3 (the AR head verifies the filled block causally; consensus and commitment);
Orthrus-Qwen3 (agentlenshq.com blog) for K = 32 and the ~4.5 MiB O(1) KV overhead.

A plausible mistake in the oracle (a dropped scale, an off-by-one in the AR
limit, DIFF made causal, the wrong KV head for a query head, a transposed
operand, argmax tie order, prefix-match off by one) fails at least one test
here.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from lossless_diffusion_speculative_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_case(seed, B=2, K=4, Hq=4, Hkv=2, D=16, ctx=(5, 9), extra=3, scale=1.0):
    rng = np.random.default_rng(seed)
    ctx = np.asarray(ctx[:B], dtype=np.int32)
    S = int(ctx.max()) + K + extra
    q = rng.standard_normal((B, K, Hq, D)).astype(np.float32) * scale
    kc = rng.standard_normal((B, Hkv, S, D)).astype(np.float32) * scale
    vc = rng.standard_normal((B, Hkv, S, D)).astype(np.float32)
    return q, kc, vc, ctx


def _sdpa(q, k, v, mask=None):
    """torch CPU fp64 scaled_dot_product_attention (a library routine)."""
    qt = torch.from_numpy(np.asarray(q, np.float64))
    kt = torch.from_numpy(np.asarray(k, np.float64))
    vt = torch.from_numpy(np.asarray(v, np.float64))
    m = None if mask is None else torch.from_numpy(mask)
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m).numpy()


# --------------------------------------------------------------------------- attention

@pytest.mark.parametrize("view", [oracle.DIFF, oracle.AR])
def test_k1_reduces_to_causal_decode_library(view):
    """K=1: both views are plain single-token decode over C+1 keys (library SDPA)."""
    q, kc, vc, ctx = _rand_case(1, B=2, K=1, ctx=(7, 12))
    out = oracle.attention(view, q, kc, vc, ctx)
    G = q.shape[2] // kc.shape[1]
    for b in range(2):
        n = int(ctx[b]) + 1
        for h in range(q.shape[2]):
            ref = _sdpa(q[b, 0, h][None], kc[b, h // G, :n], vc[b, h // G, :n])
            np.testing.assert_allclose(out[b, 0, h], ref[0], rtol=1e-12, atol=1e-12)


def test_k1_views_agree():
    q, kc, vc, ctx = _rand_case(2, K=1)
    np.testing.assert_array_equal(oracle.attention(oracle.DIFF, q, kc, vc, ctx),
                                  oracle.attention(oracle.AR, q, kc, vc, ctx))


def _explicit_mask(view, C, K):
    """Full (C+K)x(C+K) boolean mask over positions [0, C+K): causal context rows,
    then the block rows (M_diff for DIFF, causal for AR).  True = may attend."""
    n = C + K
    m = np.tril(np.ones((n, n), dtype=bool))
    if view == oracle.DIFF:
        m[C:, :] = True            # block rows: whole context + whole block
    return m


@pytest.mark.parametrize("view", [oracle.DIFF, oracle.AR])
@pytest.mark.parametrize("seed", [3, 4])
def test_bruteforce_explicit_mask_library(view, seed):
    """Dense attention with the explicit mask matrix (library SDPA) = oracle."""
    q, kc, vc, ctx = _rand_case(seed, B=2, K=5, Hq=6, Hkv=2, D=8, ctx=(0, 11))
    out = oracle.attention(view, q, kc, vc, ctx)
    G = 3
    for b in range(2):
        C, K = int(ctx[b]), 5
        mask = _explicit_mask(view, C, K)
        for h in range(6):
            g = h // G
            # queries for context positions are arbitrary; only the last K rows are used
            qq = np.concatenate([kc[b, g, :C], q[b, :, h]], axis=0)
            ref = _sdpa(qq, kc[b, g, :C + K], vc[b, g, :C + K], mask)[C:]
            np.testing.assert_allclose(out[b, :, h], ref, rtol=1e-11, atol=1e-12)


def test_numpy_bruteforce_tiny():
    """Second brute force: explicit mask, numpy softmax of the full score matrix."""
    q, kc, vc, ctx = _rand_case(5, B=1, K=3, Hq=2, Hkv=1, D=4, ctx=(4,))
    for view in (oracle.DIFF, oracle.AR):
        out = oracle.attention(view, q, kc, vc, ctx)
        C, K = 4, 3
        mask = _explicit_mask(view, C, K)[C:]
        for h in range(2):
            s = (q[0, :, h].astype(np.float64) @ kc[0, 0, :C + K].astype(np.float64).T) / 2.0
            s = np.where(mask, s, -np.inf)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            np.testing.assert_allclose(out[0, :, h], p @ vc[0, 0, :C + K], rtol=1e-12)


def test_diff_query_permutation():
    """M_diff: permuting the block's query rows permutes the outputs."""
    q, kc, vc, ctx = _rand_case(6, K=6)
    out = oracle.attention(oracle.DIFF, q, kc, vc, ctx)
    perm = np.array([3, 0, 5, 1, 4, 2])
    outp = oracle.attention(oracle.DIFF, q[:, perm], kc, vc, ctx)
    np.testing.assert_allclose(outp, out[:, perm], rtol=1e-13, atol=1e-14)


def test_diff_block_key_permutation_invariance():
    """M_diff is bidirectional inside the block: permuting the block's K/V rows
    leaves every DIFF output unchanged, while the AR view does change."""
    q, kc, vc, ctx = _rand_case(7, K=6)
    out = oracle.attention(oracle.DIFF, q, kc, vc, ctx)
    out_ar = oracle.attention(oracle.AR, q, kc, vc, ctx)
    perm = np.array([5, 2, 0, 4, 1, 3])
    kc2, vc2 = kc.copy(), vc.copy()
    for b, c in enumerate(ctx):
        kc2[b, :, c:c + 6] = kc[b][:, c + perm]
        vc2[b, :, c:c + 6] = vc[b][:, c + perm]
    np.testing.assert_allclose(oracle.attention(oracle.DIFF, q, kc2, vc2, ctx), out,
                               rtol=1e-12, atol=1e-13)
    assert not np.allclose(oracle.attention(oracle.AR, q, kc2, vc2, ctx), out_ar)


def test_ar_equals_sequential_decodes():
    """AR view slot i == a one-token decode whose context is C+i (K=1 call)."""
    q, kc, vc, ctx = _rand_case(8, K=5)
    out = oracle.attention(oracle.AR, q, kc, vc, ctx)
    for i in range(5):
        one = oracle.attention(oracle.DIFF, q[:, i:i + 1], kc, vc, ctx + i)
        np.testing.assert_allclose(out[:, i], one[:, 0], rtol=1e-13, atol=1e-14)


def test_closed_form_equal_keys_mean_of_visible_values():
    """All keys equal -> uniform weights -> output = mean of the visible V rows."""
    q, kc, vc, ctx = _rand_case(9, B=1, K=4, ctx=(6,))
    kc[:] = kc[:, :, :1]
    for view in (oracle.DIFF, oracle.AR):
        out = oracle.attention(view, q, kc, vc, ctx)
        G = q.shape[2] // kc.shape[1]
        for i in range(4):
            n = 6 + 4 if view == oracle.DIFF else 6 + i + 1
            for h in range(q.shape[2]):
                ref = vc[0, h // G, :n].astype(np.float64).mean(axis=0)
                np.testing.assert_allclose(out[0, i, h], ref, rtol=1e-12, atol=1e-13)


def test_closed_form_dominant_key_and_gqa_mapping():
    """One key aligned with the query with a huge score -> output = its V row.
    The dominant key sits in KV head h//G only, pinning the GQA mapping."""
    B, K, Hq, Hkv, D, C = 1, 3, 4, 2, 8, 5
    S = C + K
    q = np.zeros((B, K, Hq, D), np.float32)
    kc = np.zeros((B, Hkv, S, D), np.float32)
    vc = np.random.default_rng(10).standard_normal((B, Hkv, S, D)).astype(np.float32)
    q[..., 0] = 60.0
    kc[0, 1, 2, 0] = 60.0          # only KV head 1, context row 2
    for view in (oracle.DIFF, oracle.AR):
        out = oracle.attention(view, q, kc, vc, np.array([C], np.int32))
        for h in range(Hq):
            if h // 2 == 1:
                np.testing.assert_allclose(out[0, :, h], np.tile(vc[0, 1, 2], (K, 1)), atol=1e-12)
            else:   # head group 0 sees all-zero keys: uniform weights
                for i in range(K):
                    n = C + K if view == oracle.DIFF else C + i + 1
                    ref = vc[0, 0, :n].astype(np.float64).mean(0)
                    np.testing.assert_allclose(out[0, i, h], ref, atol=1e-12)


def test_default_scale_is_inverse_sqrt_d():
    q, kc, vc, ctx = _rand_case(11, D=16)
    a = oracle.attention(oracle.DIFF, q, kc, vc, ctx)
    b = oracle.attention(oracle.DIFF, q, kc, vc, ctx, scale=0.25)
    np.testing.assert_array_equal(a, b)
    c = oracle.attention(oracle.DIFF, q, kc, vc, ctx, scale=0.5)
    assert not np.allclose(a, c)


def test_rows_subset_matches_full():
    q, kc, vc, ctx = _rand_case(12, B=2, K=4)
    full = oracle.attention(oracle.AR, q, kc, vc, ctx)
    rows = [(1, 3, 2), (0, 0, 0), (1, 0, 3)]
    sub = oracle.attention(oracle.AR, q, kc, vc, ctx, rows=rows)
    for r, (b, i, h) in enumerate(rows):
        np.testing.assert_array_equal(sub[r], full[b, i, h])


def test_rows_past_the_block_are_never_read():
    """Cache rows at and beyond ctx+K (NaN-poisoned by the generator) never leak."""
    w = wl.WORKLOADS["tiny_f32"].with_(ctx_lo=40, ctx_hi=40)
    li = wl.layer_inputs(w, 0, oracle.AR, poison=True)
    assert np.isnan(li.k_cache[0, 0, 40 + w.K:]).all()
    out = oracle.attention(oracle.AR, li.q, li.k_cache, li.v_cache, li.ctx_lens)
    assert np.isfinite(out).all()


def test_capacity_violation_raises():
    q, kc, vc, ctx = _rand_case(13, B=1, K=4, ctx=(5,), extra=0)
    with pytest.raises(ValueError):
        oracle.attention(oracle.DIFF, q, kc, vc, ctx + 1)


# --------------------------------------------------------------------------- consensus

def _parse(x):
    return float(x) if isinstance(x, str) else x


def test_consensus_golden_cases():
    with open(os.path.join(GOLDEN, "consensus_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        logits = np.array([[_parse(v) for v in row] for row in c["logits"]], np.float32)[None]
        prop = np.array(c["proposed"], np.int32)[None]
        acc, nxt, am = oracle.consensus(logits, prop)
        assert acc[0] == c["accepted"], c["name"]
        assert nxt[0] == c["next"], c["name"]
        assert list(am[0]) == c["argmax"], c["name"]


def test_consensus_argmax_matches_numpy_without_nan():
    rng = np.random.default_rng(14)
    logits = rng.integers(-3, 4, size=(3, 8, 50)).astype(np.float32)   # many ties
    prop = rng.integers(0, 50, size=(3, 8)).astype(np.int32)
    _, _, am = oracle.consensus(logits, prop)
    np.testing.assert_array_equal(am, logits.argmax(axis=2))           # first max wins


def test_consensus_argmax_matches_torch_with_nan():
    rng = np.random.default_rng(15)
    logits = rng.standard_normal((2, 8, 40)).astype(np.float32)
    logits[rng.random(logits.shape) < 0.05] = np.nan
    prop = np.zeros((2, 8), np.int32)
    _, _, am = oracle.consensus(logits, prop)
    np.testing.assert_array_equal(am, torch.from_numpy(logits).argmax(dim=2).numpy())


@pytest.mark.parametrize("name", list(wl.WORKLOADS))
def test_consensus_recovers_plant(name):
    w = wl.WORKLOADS[name]
    B = min(w.B, 4)
    ci = wl.consensus_inputs(w.with_(vocab=min(w.vocab, 5000)), B=B)
    acc, nxt, am = oracle.consensus(ci.logits, ci.proposed)
    np.testing.assert_array_equal(am, ci.planted_argmax)
    np.testing.assert_array_equal(acc, ci.planted_accept)
    np.testing.assert_array_equal(nxt, ci.planted_next)


@pytest.mark.parametrize("a", [0, 1, 7, 8])
def test_consensus_extremes(a):
    w = wl.WORKLOADS["tiny_f32"]
    ci = wl.consensus_inputs(w, accept=np.array([a]))
    acc, nxt, _ = oracle.consensus(ci.logits, ci.proposed)
    assert acc[0] == a
    assert nxt[0] == ci.planted_argmax[0, min(a, w.K - 1)]


# --------------------------------------------------------------------------- commit

def test_commit_copies_prefix_and_advances():
    rng = np.random.default_rng(16)
    B, Hkv, D, K, S = 3, 2, 4, 5, 24
    kc = rng.standard_normal((B, Hkv, S, D)).astype(np.float32)
    vc = rng.standard_normal((B, Hkv, S, D)).astype(np.float32)
    kb = rng.standard_normal((B, K, Hkv, D)).astype(np.float32)
    vb = rng.standard_normal((B, K, Hkv, D)).astype(np.float32)
    ctx = np.array([3, 10, 0], np.int32)
    acc = np.array([0, 5, 2], np.int32)
    k0, v0, c0 = kc.copy(), vc.copy(), ctx.copy()
    oracle.kv_commit(kc, vc, kb, vb, ctx, acc, K)
    n = np.minimum(acc + 1, K)
    np.testing.assert_array_equal(ctx, c0 + n)
    for b in range(B):
        lo, hi = c0[b], c0[b] + n[b]
        np.testing.assert_array_equal(kc[b, :, lo:hi], kb[b, :n[b]].transpose(1, 0, 2))
        np.testing.assert_array_equal(vc[b, :, lo:hi], vb[b, :n[b]].transpose(1, 0, 2))
        np.testing.assert_array_equal(kc[b, :, :lo], k0[b, :, :lo])
        np.testing.assert_array_equal(kc[b, :, hi:], k0[b, :, hi:])


def test_commit_without_copy_only_advances():
    kc = np.zeros((1, 1, 16, 4), np.float32)
    vc = kc.copy()
    ctx = np.array([4], np.int32)
    oracle.kv_commit(kc, vc, None, None, ctx, np.array([2], np.int32), 8)
    assert ctx[0] == 7 and not kc.any()


def test_tail_is_the_pages_4p5_mib():
    """Committing a full block (a = K = 32) of a Qwen3-8B-shaped bf16 cache over all
    layers writes exactly the O(1) overhead the pages quote: 4.5 MiB."""
    with open(os.path.join(GOLDEN, "tail_overhead.json")) as f:
        g = json.load(f)
    L, Hkv, D, K = g["layers"], g["kv_heads"], g["head_dim"], g["K"]
    B, S = 1, K + 8
    written = 0
    ctx_all = np.zeros(1, np.int32)
    for layer in range(L):
        kc = np.zeros((B, Hkv, S, D), np.uint16)
        vc = np.zeros((B, Hkv, S, D), np.uint16)
        kb = np.full((B, K, Hkv, D), 0x3F80, np.uint16)   # bf16 1.0
        vb = kb.copy()
        ctx = np.zeros(1, np.int32)
        oracle.kv_commit(kc, vc, kb, vb, ctx, np.array([K], np.int32), K,
                         advance=(layer == L - 1))
        written += int((kc != 0).sum() + (vc != 0).sum()) * g["elem_bytes"]
        if layer == L - 1:
            ctx_all = ctx
    assert written == g["block_bytes"]
    assert written / 2 ** 20 == g["block_mib"]
    assert ctx_all[0] == K


# --------------------------------------------------------------------------- lossless

def _toy_model_logits(tokens, V, seed=17):
    """A deterministic toy 'frozen AR model': next-token logits from a hash of the
    whole prefix.  Stands in for the LM head; only argmax matters here."""
    h = 1469598103934665603
    for t in tokens:
        h = ((h ^ int(t)) * 1099511628211) & 0xFFFFFFFFFFFFFFFF
    return np.random.default_rng([seed, h & 0xFFFFFFFF, h >> 32]).standard_normal(V).astype(np.float32)


@pytest.mark.parametrize("mode", ["adversarial", "oracle_draft", "mixed"])
def test_lossless_toy_loop_equals_greedy(mode):
    """The dual-view loop (proposals -> AR logits -> consensus -> commit) emits
    exactly the base model's greedy sequence, whatever the proposals are."""
    V, K, steps_tokens = 37, 6, 40
    prompt = [3, 1, 4]
    greedy = list(prompt)
    while len(greedy) < len(prompt) + steps_tokens:
        greedy.append(int(np.argmax(_toy_model_logits(greedy, V))))

    rng = np.random.default_rng(18)
    seq = list(prompt[:-1])
    anchor = prompt[-1]
    while len(seq) + 1 < len(prompt) + steps_tokens:
        ctx = seq + [anchor]
        # proposals p_1..p_K for positions after the anchor
        if mode == "adversarial":
            prop = list(rng.integers(0, V, size=K))
        else:
            prop, t = [], list(ctx)
            for _ in range(K):
                nxt = int(np.argmax(_toy_model_logits(t, V)))
                if mode == "mixed" and rng.random() < 0.3:
                    nxt = (nxt + 1) % V
                prop.append(nxt)
                t.append(nxt)
        # AR view over [anchor, p_1..p_{K-1}]: row i predicts the token after slot i
        logits = np.stack([_toy_model_logits(ctx + prop[:i], V) for i in range(K)])[None]
        acc, nxt, _ = oracle.consensus(logits, np.array([prop], np.int32))
        a = int(acc[0])
        n = min(a + 1, K)
        block = [anchor] + prop[:K - 1]
        seq = seq + block[:n]                  # commit slots 0..n-1
        anchor = int(nxt[0])                   # next anchor = AR token
        if mode == "oracle_draft":
            assert a == K
    out = (seq + [anchor])[:len(prompt) + steps_tokens]
    assert out == greedy[:len(out)]


# --------------------------------------------------------------------------- fused LM head

def _lm_case(seed, B=2, K=4, Hd=32, V=50):
    rng = np.random.default_rng(seed)
    h = wl.round_to_bf16(rng.standard_normal((B, K, Hd), dtype=np.float32))
    W = wl.round_to_bf16(rng.standard_normal((V, Hd), dtype=np.float32) / np.float32(np.sqrt(Hd)))
    return h, W


def test_lm_head_bruteforce_tiny():
    """Explicit loops: dot products, first maximum, left-to-right prefix walk."""
    h, W = _lm_case(40)
    B, K, Hd = h.shape
    V = W.shape[0]
    rng = np.random.default_rng(41)
    prop = rng.integers(0, V, (B, K)).astype(np.int32)
    r_bf = np.zeros((B, K), np.int32)
    for b in range(B):
        for i in range(K):
            best, arg = -math.inf, -1
            for v in range(V):
                dot = math.fsum(float(h[b, i, d]) * float(W[v, d]) for d in range(Hd))
                if dot > best:
                    best, arg = dot, v
            r_bf[b, i] = arg
    prop[0, :2] = r_bf[0, :2]                     # sequence 0 accepts 2, sequence 1 all K
    prop[0, 2] = (r_bf[0, 2] + 1) % V
    prop[1, :] = r_bf[1, :]
    acc, nxt, r, _, _ = oracle.lm_head_consensus(h, W, prop)
    assert (r == r_bf).all()
    assert acc[0] == 2 and nxt[0] == r_bf[0, 2]
    assert acc[1] == K and nxt[1] == r_bf[1, K - 1]


@pytest.mark.parametrize("a", [0, 5, 32])
def test_lm_head_recovers_plant(a):
    w = wl.WORKLOADS["qwen3_8b_step"].with_(vocab=3000)
    li = wl.lm_head_inputs(w, Hd=128, accept=np.array([a], np.int32))
    acc, nxt, r, gap, _ = oracle.lm_head_consensus(li.hidden, li.lm_head, li.proposed)
    assert (r == li.planted_argmax).all()
    assert acc[0] == a and nxt[0] == li.planted_next[0]
    assert gap.min() > 1.0


def test_lm_head_matches_materialised_consensus():
    """The fused definition and the C consensus over materialised (float32)
    logits agree wherever the top-2 gap dwarfs float32 rounding."""
    w = wl.WORKLOADS["qwen3_4b_ragged"].with_(B=3, vocab=2000)
    li = wl.lm_head_inputs(w, Hd=96)
    acc, nxt, r, gap, _ = oracle.lm_head_consensus(li.hidden, li.lm_head, li.proposed)
    logits = oracle.lm_head_logits(li.hidden, li.lm_head).astype(np.float32).reshape(3, w.K, -1)
    acc2, nxt2, r2 = oracle.consensus(logits, li.proposed)
    assert gap.min() > 1e-3
    assert (acc == acc2).all() and (nxt == nxt2).all() and (r == r2).all()


def test_lm_head_ties_go_to_the_lowest_index():
    h, W = _lm_case(42, B=1, K=2, Hd=16, V=20)
    W[7] = W[3] = h[0, 0] * 4                     # two equal maxima for row 0
    prop = np.array([[3, 0]], np.int32)
    acc, nxt, r, gap, _ = oracle.lm_head_consensus(h, W, prop)
    assert r[0, 0] == 3 and gap[0, 0] == 0.0 and acc[0] >= 1


def test_fp32_accumulation_stays_within_the_stated_bound():
    """float32 sums of the exact products in several orders never leave the
    bound the GPU parity tests use to decide which argmaxes are unique."""
    rng = np.random.default_rng(43)
    for n in (64, 1000, 4096):
        x = wl.round_to_bf16(rng.standard_normal(n, dtype=np.float32))
        y = wl.round_to_bf16(rng.standard_normal(n, dtype=np.float32) * np.float32(3))
        prod = (x.astype(np.float64) * y.astype(np.float64))
        exact = math.fsum(prod)
        bound = float(oracle.fp32_dot_error_bound(n, np.abs(prod).sum()))
        p32 = prod.astype(np.float32)                 # exact: bf16 x bf16 fits in float32
        assert (p32.astype(np.float64) == prod).all()
        for order in (p32, p32[::-1], np.sort(p32), rng.permutation(p32)):
            acc = np.float32(0)
            for v in order:
                acc = np.float32(acc + v)
            assert abs(float(acc) - exact) <= bound
        assert abs(float(np.sum(p32, dtype=np.float32)) - exact) <= bound


# --------------------------------------------------------------------------- rejection sampling

def test_rejection_is_lossless_monte_carlo():
    """Proposals drawn from q, verified against p: the emitted token of a
    one-slot block is distributed as p (chi-square over 6 tokens)."""
    rng = np.random.default_rng(50)
    V, N, T = 6, 60000, 0.8
    ar = rng.standard_normal(V) * 1.5
    dr = rng.standard_normal(V) * 1.5
    p = np.exp(ar / T) / np.exp(ar / T).sum()
    q = np.exp(dr / T) / np.exp(dr / T).sum()
    x = rng.choice(V, size=N, p=q).astype(np.int32)
    acc, nxt, _, _ = oracle.rejection_verify(np.broadcast_to(ar, (N, 1, V)), np.broadcast_to(dr, (N, 1, V)),
                                             x[:, None], rng.random((N, 1)), rng.random(N), T)
    emitted = np.where(acc == 1, x, nxt)
    counts = np.bincount(emitted, minlength=V)
    chi2 = float((((counts - N * p) ** 2) / (N * p)).sum())
    assert chi2 < 30.0, (chi2, counts, N * p)          # 5 dof: P(chi2 > 30) ~ 1.5e-5


def test_rejection_at_low_temperature_is_greedy():
    """T -> 0 with argmax-q proposals: the rule reduces to the greedy
    consensus (the independent C oracle) on the AR logits."""
    w = wl.WORKLOADS["qwen3_4b_ragged"].with_(B=4, K=8, vocab=300)
    ci = wl.consensus_inputs(w)
    rng = np.random.default_rng(51)
    draft = rng.standard_normal(ci.logits.shape).astype(np.float32)
    draft[np.arange(4)[:, None], np.arange(8)[None, :], ci.proposed] += 20.0   # q peaks at the proposal
    acc, nxt, _, _ = oracle.rejection_verify(ci.logits, draft, ci.proposed, rng.random((4, 8)),
                                             rng.random(4), 1e-3)
    gacc, gnxt, _ = oracle.consensus(ci.logits, ci.proposed)
    assert (acc == gacc).all() and (nxt == gnxt).all()


def test_rejection_identical_views_accept_everything():
    rng = np.random.default_rng(52)
    lg = rng.standard_normal((3, 5, 40))
    prop = rng.integers(0, 40, (3, 5)).astype(np.int32)
    acc, nxt, _, _ = oracle.rejection_verify(lg, lg, prop, rng.random((3, 5)) * 0.999, rng.random(3), 1.3)
    assert (acc == 5).all() and (nxt == prop[:, 4]).all()


def test_rejection_hand_cases():
    """p = (.5, .3, .2), q = (.2, .3, .5) at T = 1: x = 2 is kept with
    probability .4 and the residual (.3, 0, 0) always yields token 0; x = 0
    (ratio 2.5) is always kept.  A two-token residual splits at its midpoint."""
    ar = np.log(np.array([[[0.5, 0.3, 0.2]]]))
    dr = np.log(np.array([[[0.2, 0.3, 0.5]]]))
    for u, a, n in ((0.5, 0, 0), (0.3, 1, 2), (0.399, 1, 2), (0.401, 0, 0)):
        acc, nxt, _, _ = oracle.rejection_verify(ar, dr, np.array([[2]], np.int32), np.array([[u]]),
                                                 np.array([0.77]), 1.0)
        assert (acc[0], nxt[0]) == (a, n), (u, acc, nxt)
    acc, _, _, _ = oracle.rejection_verify(ar, dr, np.array([[0]], np.int32), np.array([[0.999]]),
                                           np.array([0.5]), 1.0)
    assert acc[0] == 1
    ar2 = np.log(np.array([[[0.5, 0.5, 1e-12]]]))
    dr2 = np.log(np.array([[[0.1, 0.1, 0.8]]]))            # residual (.4, .4, 0)
    for up, n in ((0.3, 0), (0.6, 1), (0.49, 0), (0.51, 1)):
        acc, nxt, _, cm = oracle.rejection_verify(ar2, dr2, np.array([[2]], np.int32), np.array([[0.9]]),
                                                  np.array([up]), 1.0)
        assert acc[0] == 0 and nxt[0] == n, (up, nxt)


# --------------------------------------------------------------------------- QKV projection

def test_qkv_project_bruteforce_tiny():
    rng = np.random.default_rng(80)
    B, K, hidden, Hq, Hkv, D = 2, 3, 16, 4, 2, 4
    x = wl.round_to_bf16(rng.standard_normal((B, K, hidden), dtype=np.float32))
    wq = wl.round_to_bf16(rng.standard_normal((Hq * D, hidden), dtype=np.float32))
    wk = wl.round_to_bf16(rng.standard_normal((Hkv * D, hidden), dtype=np.float32))
    wv = wl.round_to_bf16(rng.standard_normal((Hkv * D, hidden), dtype=np.float32))
    q, k, v, qa, ka, va = oracle.qkv_project(x, wq, wk, wv, D)
    for b in range(B):
        for i in range(K):
            for w, out, H in ((wq, q, Hq), (wk, k, Hkv), (wv, v, Hkv)):
                for h in range(H):
                    for d in range(D):
                        row = w[h * D + d]
                        exact = math.fsum(float(x[b, i, j]) * float(row[j]) for j in range(hidden))
                        assert abs(out[b, i, h, d] - exact) < 1e-12
    assert qa.shape == q.shape and (qa >= np.abs(q) - 1e-12).all()


def test_qkv_project_feature_mapping_one_hot():
    """One-hot weight rows: output feature h*D + d of a projection copies input
    dimension (h*D + d) mod hidden, so the head and dim indices of q, k, v are
    pinned to the weight rows."""
    rng = np.random.default_rng(81)
    B, K, hidden, Hq, Hkv, D = 2, 2, 40, 4, 2, 8
    x = wl.round_to_bf16(rng.standard_normal((B, K, hidden), dtype=np.float32))
    eye = lambda n: np.eye(hidden, dtype=np.float32)[np.arange(n) % hidden]
    q, k, v, _, _, _ = oracle.qkv_project(x, eye(Hq * D), eye(Hkv * D) * 2, eye(Hkv * D) * 3, D)
    for h in range(Hq):
        for d in range(D):
            assert (q[:, :, h, d] == x[:, :, (h * D + d) % hidden]).all()
    for g in range(Hkv):
        for d in range(D):
            assert (k[:, :, g, d] == 2 * x[:, :, (g * D + d) % hidden]).all()
            assert (v[:, :, g, d] == 3 * x[:, :, (g * D + d) % hidden]).all()


def test_install_block_rows_places_the_tail_only():
    rng = np.random.default_rng(82)
    B, K, Hkv, D, S = 3, 4, 2, 5, 20
    kc = rng.standard_normal((B, Hkv, S, D))
    vc = rng.standard_normal((B, Hkv, S, D))
    kb = rng.standard_normal((B, K, Hkv, D))
    vb = rng.standard_normal((B, K, Hkv, D))
    ctx = np.array([0, 9, S - K + 1], np.int32)            # the last has no room
    k2, v2 = kc.copy(), vc.copy()
    oracle.install_block_rows(k2, v2, kb, vb, ctx, S)
    for b in range(2):
        c = int(ctx[b])
        for g in range(Hkv):
            assert (k2[b, g, c:c + K] == kb[b, :, g]).all() and (v2[b, g, c:c + K] == vb[b, :, g]).all()
            keep = np.r_[0:c, c + K:S]
            assert (k2[b, g, keep] == kc[b, g, keep]).all() and (v2[b, g, keep] == vc[b, g, keep]).all()
    assert (k2[2] == kc[2]).all() and (v2[2] == vc[2]).all()


# --------------------------------------------------------------------------- prefill

def test_ar_view_at_empty_context_is_causal_prefill_library():
    """Causal prefill over S prompt tokens is the AR view with no committed
    context and K = S: it matches the library's causal SDPA (torch, fp64)."""
    rng = np.random.default_rng(60)
    B, S, Hq, Hkv, D = 2, 11, 4, 2, 8
    q = rng.standard_normal((B, S, Hq, D)).astype(np.float32)
    kc = rng.standard_normal((B, Hkv, S + 3, D)).astype(np.float32)
    vc = rng.standard_normal((B, Hkv, S + 3, D)).astype(np.float32)
    out = oracle.attention(oracle.AR, q, kc, vc, np.zeros(B, np.int32))
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            qt = torch.from_numpy(q[b, :, h].astype(np.float64))[None]
            kt = torch.from_numpy(kc[b, h // G, :S].astype(np.float64))[None]
            vt = torch.from_numpy(vc[b, h // G, :S].astype(np.float64))[None]
            ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)[0].numpy()
            np.testing.assert_allclose(out[b, :, h], ref, rtol=1e-12, atol=1e-12)
