"""GPU parity of orthrus_rejection_verify (temperature > 0) against the fp64
oracle, and the lossless property on the GPU itself.

Accept decisions are compared where the oracle's margin exceeds 1e-4
relative: the kernel's probabilities carry a relative error of ~1e-6 (fp32
sums of at most a few hundred terms per thread plus a log-depth tree, and
ex2.approx with ~2^-22 relative error), so 1e-4 leaves a factor of ~100.  The
inverse-CDF draw is compared exactly where the target lies more than 2e-5 of
the residual's total from every cumulative boundary (the kernel's cumulative
sums carry ~2e-6 of it: ~5e-7 from the probabilities, ~1.2e-6 from about 20
rounding levels of tile, run and block sums); closer than that -- common at a
151936-token vocabulary, where one token holds ~1e-5 of the mass -- the drawn
token's cumulative interval must contain the target within that tolerance.
"""
import numpy as np
import pytest
import torch

import oracle
from lossless_diffusion_speculative_b200 import binding as ob
from lossless_diffusion_speculative_b200 import workloads as wl

pytestmark = pytest.mark.gpu

TOL = 1e-4
CDF_TOL = 2e-5


def _gpu(ar, dr, prop, ua, ur, T):
    B, K, V = ar.shape
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    acc = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    nxt = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    ws = torch.zeros(ob.orthrus_rejection_workspace_size(B, K, V), dtype=torch.uint8, device="cuda")
    ob.orthrus_rejection_verify(dev(ar.astype(np.float32)), dev(dr.astype(np.float32)),
                                dev(prop.astype(np.int32)), dev(ua.astype(np.float32)),
                                dev(ur.astype(np.float32)), T, acc, nxt, ws)
    torch.cuda.synchronize()
    assert int(ws[:4 * B].count_nonzero().item()) == 0, "per-sequence counters not left zero"
    return acc.cpu().numpy(), nxt.cpu().numpy()


def _compare(ar, dr, prop, ua, ur, T):
    acc, nxt = _gpu(ar, dr, prop, ua, ur, T)
    racc, rnxt, am, cm = oracle.rejection_verify(ar.astype(np.float32), dr.astype(np.float32), prop,
                                                 ua.astype(np.float32), ur.astype(np.float32), T)
    B, K = prop.shape
    checked = 0
    for b in range(B):
        taken = am[b][np.isfinite(am[b])]
        if (taken < TOL).any():
            continue                                   # an accept decision too close to call
        checked += 1
        assert acc[b] == racc[b], (b, acc[b], racc[b])
        if acc[b] == K or cm[b] > CDF_TOL:
            assert nxt[b] == rnxt[b], (b, nxt[b], rnxt[b])
        else:                                          # a valid draw: its interval holds the target
            a = int(acc[b])
            cdf = oracle.residual_cdf(ar[b, a].astype(np.float32), dr[b, a].astype(np.float32), T)
            v, R = int(nxt[b]), cdf[-1]
            target = float(np.float32(ur[b])) * R
            lo = cdf[v - 1] if v > 0 else 0.0
            assert lo - CDF_TOL * R <= target <= cdf[v] + CDF_TOL * R, (b, v, lo, cdf[v], target)
    return checked


def _inputs(seed, B, K, V, sigma=2.0, draft_noise=1.0):
    """AR logits N(0, sigma); draft logits = AR + N(0, draft_noise) (a drafter
    close to the target); proposals drawn from q; uniform draws."""
    rng = np.random.default_rng(seed)
    ar = (rng.standard_normal((B, K, V)) * sigma).astype(np.float32)
    dr = (ar + rng.standard_normal((B, K, V)) * draft_noise).astype(np.float32)
    return ar, dr, rng


@pytest.mark.parametrize("T", [0.5, 1.0, 1.7])
@pytest.mark.parametrize("V", [1000, 1003, 7])
def test_rejection_matches_oracle(T, V):
    B, K = 6, 8
    ar, dr, rng = _inputs(int(T * 10) + V, B, K, V)
    q = np.exp(dr.astype(np.float64) / T)
    q /= q.sum(axis=2, keepdims=True)
    prop = np.array([[rng.choice(V, p=q[b, i]) for i in range(K)] for b in range(B)], np.int32)
    ua, ur = rng.random((B, K)), rng.random(B)
    assert _compare(ar, dr, prop, ua, ur, T) >= B - 1


def test_rejection_is_lossless_on_the_gpu():
    """Proposals drawn from q and verified against p on the GPU: the emitted
    token of a one-slot block follows p (chi-square over 6 tokens, 60000
    sequences in one call)."""
    rng = np.random.default_rng(70)
    V, N, T = 6, 60000, 0.9
    ar = (rng.standard_normal(V) * 1.5).astype(np.float32)
    dr = (rng.standard_normal(V) * 1.5).astype(np.float32)
    p = np.exp(ar.astype(np.float64) / T)
    p /= p.sum()
    q = np.exp(dr.astype(np.float64) / T)
    q /= q.sum()
    x = rng.choice(V, size=N, p=q).astype(np.int32)
    acc, nxt = _gpu(np.broadcast_to(ar, (N, 1, V)), np.broadcast_to(dr, (N, 1, V)), x[:, None],
                    rng.random((N, 1)), rng.random(N), T)
    emitted = np.where(acc == 1, x, nxt)
    counts = np.bincount(emitted, minlength=V)
    chi2 = float((((counts - N * p) ** 2) / (N * p)).sum())
    assert chi2 < 30.0, (chi2, counts, N * p)


def test_rejection_edge_cases():
    """Identical views keep every proposal (next = the last one); a proposal
    outside the vocabulary is never kept; an empty residual (the rejected
    token has no mass under either view) draws from p."""
    B, K, V = 3, 5, 50
    ar, _, rng = _inputs(71, B, K, V)
    prop = rng.integers(0, V, (B, K)).astype(np.int32)
    acc, nxt = _gpu(ar, ar, prop, rng.random((B, K)) * 0.999, rng.random(B), 1.2)
    assert (acc == K).all() and (nxt == prop[:, K - 1]).all()
    prop2 = prop.copy()
    prop2[1, 2] = V + 3
    prop2[2, 0] = -1
    acc, _ = _gpu(ar, ar, prop2, rng.random((B, K)) * 0.999, rng.random(B), 1.2)
    assert acc[0] == K and acc[1] == 2 and acc[2] == 0
    ar3 = ar.copy()
    ar3[0, 1, prop[0, 1]] = -1e4                       # no mass under either (identical) view
    ua, ur = rng.random((B, K)) * 0.999, rng.random(B)
    acc, nxt = _gpu(ar3, ar3, prop, ua, ur, 1.2)
    racc, rnxt, _, cm = oracle.rejection_verify(ar3, ar3, prop, ua.astype(np.float32),
                                                ur.astype(np.float32), 1.2)
    assert acc[0] == 1 and racc[0] == 1
    if cm[0] > TOL:
        assert nxt[0] == rnxt[0]


@pytest.mark.parametrize("name", ["qwen3_8b_step", "qwen3_4b_ragged"])
def test_rejection_full_vocabulary(name):
    """Full Qwen3 vocabulary and the workload's batch, in the benchmark's
    launch configuration."""
    w = wl.WORKLOADS[name]
    B, K, V = w.B, w.K, w.vocab
    ar, dr, rng = _inputs(72 + w.cid, B, K, V)
    prop = np.argmax(dr, axis=2).astype(np.int32)        # the draft's favourite token
    ua, ur = rng.random((B, K)), rng.random(B)
    assert _compare(ar, dr, prop, ua, ur, 1.0) >= B - 1
