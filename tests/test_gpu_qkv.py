"""GPU parity of orthrus_qkv_project (the block's QKV projection written into
the query buffer and the cache tail) against the fp64 oracle, and of the fused
layer step projection -> attention.

Tolerance per output element: 2^-8 |exact| (the bf16 rounding of the result,
half an ulp of 8 significant bits) + 2 * gamma_n * sum_d |x_d w_d| (the fp32
accumulation bound, oracle.fp32_dot_error_bound).  Every cache byte outside
rows [ctx_b, ctx_b + K) must be unchanged.
"""
import numpy as np
import pytest
import torch

import oracle
from lossless_diffusion_speculative_b200 import binding as ob
from lossless_diffusion_speculative_b200 import workloads as wl
from gpu_util import assert_attn_close

pytestmark = pytest.mark.gpu


def _case(seed, B, K, hidden, Hq, Hkv, D, ctx, extra=8):
    rng = np.random.default_rng(seed)
    ctx = np.asarray(ctx, np.int32)
    S = int(max(int(ctx.max()) + K, K)) + extra
    bf = wl.round_to_bf16
    x = bf(rng.standard_normal((B, K, hidden), dtype=np.float32))
    sc = np.float32(1 / np.sqrt(hidden))
    wq = bf(rng.standard_normal((Hq * D, hidden), dtype=np.float32) * sc)
    wk = bf(rng.standard_normal((Hkv * D, hidden), dtype=np.float32) * sc)
    wv = bf(rng.standard_normal((Hkv * D, hidden), dtype=np.float32) * sc)
    kc = bf(rng.standard_normal((B, Hkv, S, D), dtype=np.float32) * np.float32(0.1))
    vc = bf(rng.standard_normal((B, Hkv, S, D), dtype=np.float32) * np.float32(0.1))
    return x, wq, wk, wv, kc, vc, ctx


def _gpu(x, wq, wk, wv, kc, vc, ctx, status=None):
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(torch.bfloat16)
    B, K, _ = x.shape
    Hq = wq.shape[0] // kc.shape[3]
    q = torch.full((B, K, Hq, kc.shape[3]), float("nan"), dtype=torch.bfloat16, device="cuda")
    tk, tv = dev(kc), dev(vc)
    own = status is None
    if own:
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.zeros(ob.orthrus_qkv_workspace_size(B, K, x.shape[2], Hq, kc.shape[1], kc.shape[3]),
                     dtype=torch.uint8, device="cuda")
    for _ in range(2):                               # (the second call reuses the workspace)
        ob.orthrus_qkv_project(dev(x), dev(wq), dev(wk), dev(wv), torch.from_numpy(ctx).cuda(), q, tk, tv,
                               ws, status=status)
    torch.cuda.synchronize()
    assert int(ws.count_nonzero().item()) == 0 or ob.orthrus_qkv_workspace_size(
        B, K, x.shape[2], Hq, kc.shape[1], kc.shape[3]) > 4096   # (partials may stay)
    torch.cuda.synchronize()
    if own:
        assert int(status.item()) == 0
    f = lambda t: t.float().cpu().numpy()
    return f(q), f(tk), f(tv), (q, tk, tv)


def _check(got, exact, absdot, hidden, what):
    tol = 2.0 ** -8 * np.abs(exact) + 2 * oracle.fp32_dot_error_bound(hidden, absdot)
    err = np.abs(got.astype(np.float64) - exact)
    assert (err <= tol).all(), f"{what}: worst {float((err - tol).max()):.3e} over tolerance"


CASES = {   # name: (B, K, hidden, Hq, Hkv, D, ctx)
    "small_ragged": (3, 8, 512, 8, 2, 64, [5, 700, 0]),
    "k1_one_token": (2, 1, 256, 4, 4, 128, [17, 300]),
    "rows_not_16": (3, 5, 192, 8, 2, 128, [40, 9, 123]),
    "qwen3_8b_layer": (1, 32, 4096, 32, 8, 128, [8192]),
    "qwen3_4b_batch": (16, 32, 2560, 32, 8, 128, list(range(100, 1700, 100))),
}


@pytest.mark.parametrize("name", list(CASES))
def test_qkv_project_matches_oracle(name):
    B, K, hidden, Hq, Hkv, D, ctx = CASES[name]
    x, wq, wk, wv, kc, vc, ctx = _case(90 + list(CASES).index(name), B, K, hidden, Hq, Hkv, D, ctx)
    gq, gk, gv, _ = _gpu(x, wq, wk, wv, kc, vc, ctx)
    q, k, v, qa, ka, va = oracle.qkv_project(x, wq, wk, wv, D)
    _check(gq, q, qa, hidden, "q")
    S = kc.shape[2]
    for b in range(B):
        c = int(ctx[b])
        _check(np.transpose(gk[b, :, c:c + K], (1, 0, 2)), k[b], ka[b], hidden, f"k seq {b}")
        _check(np.transpose(gv[b, :, c:c + K], (1, 0, 2)), v[b], va[b], hidden, f"v seq {b}")
        keep = np.r_[0:c, c + K:S]
        assert (gk[b][:, keep] == kc[b][:, keep]).all() and (gv[b][:, keep] == vc[b][:, keep]).all()


def test_qkv_project_capacity_leaves_the_sequence_untouched():
    x, wq, wk, wv, kc, vc, ctx = _case(97, 3, 8, 256, 8, 2, 64, [10, 20, 30], extra=0)
    S = kc.shape[2]
    ctx = np.array([10, S - 8 + 1, 30 - 30], np.int32)                  # sequence 1 has no room
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gq, gk, gv, _ = _gpu(x, wq, wk, wv, kc, vc, ctx, status=status)
    assert int(status.item()) & ob.STATUS_CAPACITY
    assert (gk[1] == kc[1]).all() and (gv[1] == vc[1]).all()
    q, k, _, qa, ka, _ = oracle.qkv_project(x, wq, wk, wv, 64)
    _check(gq, q, qa, 256, "q")
    _check(np.transpose(gk[0, :, 10:18], (1, 0, 2)), k[0], ka[0], 256, "k seq 0")


def test_fused_layer_projection_then_attention():
    """projection -> attention on the same stream: the attention sees the
    projected block in the cache tail (checked against the oracle attention
    over the GPU's own projected query and cache, read back)."""
    B, K, hidden, Hq, Hkv, D = 2, 32, 1024, 32, 8, 128
    x, wq, wk, wv, kc, vc, ctx = _case(98, B, K, hidden, Hq, Hkv, D, [3000, 517])
    _, _, _, (q, tk, tv) = _gpu(x, wq, wk, wv, kc, vc, ctx)
    c = torch.from_numpy(ctx).cuda()
    for view in (ob.DIFF, ob.AR):
        out = torch.empty((B, K, Hq, D), dtype=torch.float32, device="cuda")
        ws = torch.zeros(ob.orthrus_attn_workspace_size(B, Hq, Hkv, D, K, torch.bfloat16),
                         dtype=torch.uint8, device="cuda")
        ob.orthrus_attn(view, q, tk, tv, c, out, ws)
        torch.cuda.synchronize()
        f = lambda t: t.float().cpu().numpy()
        ref = oracle.attention(view, f(q), f(tk), f(tv), ctx)
        assert_attn_close(out.cpu().numpy(), ref, f"fused view {view}")
