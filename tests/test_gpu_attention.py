"""GPU parity of orthrus_attn (both views) against the fp64 oracle.

Tolerance (both paths): max |gpu - oracle| <= 2e-3 * RMS(oracle output).
Every workload is compared element by element over every output row, the
full-size ones (one layer of the Qwen3-8B step, the ragged batch of 16 and the
long-context batch at K = 8, 16, 32) in the launch configuration the benchmark
times, so every split segment and every CTA that straddles two segments is
covered.
"""
import functools

import numpy as np
import pytest
import torch

import oracle
from lossless_diffusion_speculative_b200 import binding as ob
from lossless_diffusion_speculative_b200 import workloads as wl
from gpu_util import assert_attn_close, run_attn, tdtype, to_dev

pytestmark = pytest.mark.gpu

# the workspace's leading block of split-merge flags and counters: 3 x 160 int32
SYNC_BYTES = 3 * 160 * 4


@functools.lru_cache(maxsize=2)
def _inputs(name, layer, view):
    return wl.layer_inputs(wl.WORKLOADS[name], layer, view, poison=True)


def _gpu(w, li, view, status=None):
    dt = tdtype(w)
    out = run_attn(view, to_dev(li.q, dt), to_dev(li.k_cache, dt), to_dev(li.v_cache, dt),
                   torch.from_numpy(li.ctx_lens).cuda(), dt, status=status)
    return out.cpu().numpy()


@pytest.mark.parametrize("view", [ob.DIFF, ob.AR])
@pytest.mark.parametrize("name", ["tiny_f32", "qwen3_1p7b_layer"])
def test_attention_full_compare(name, view):
    w = wl.WORKLOADS[name]
    li = _inputs(name, 0, view)
    got = _gpu(w, li, view)
    ref = oracle.attention(view, li.q, li.k_cache, li.v_cache, li.ctx_lens)
    assert_attn_close(got, ref, f"{name}/{view}")


@pytest.mark.parametrize("view", [ob.DIFF, ob.AR])
@pytest.mark.parametrize("name", ["qwen3_8b_step", "qwen3_4b_ragged", "qwen3_8b_long_k8",
                                  "qwen3_8b_long_k16", "qwen3_8b_long_k32"])
def test_attention_full_size_every_row(name, view):
    w = wl.WORKLOADS[name]
    li = _inputs(name, 0, view)
    got = _gpu(w, li, view)
    ref = oracle.attention(view, li.q, li.k_cache, li.v_cache, li.ctx_lens)
    assert_attn_close(got, ref, f"{name}/{view}")


def _custom(seed, B, Hq, Hkv, D, K, ctx, dtype="bf16", extra=0, scale=1 / np.sqrt(128)):
    """Seeded edge-case inputs: rows past ctx+K poisoned with NaN."""
    rng = np.random.default_rng(seed)
    ctx = np.asarray(ctx, np.int32)
    S = int(ctx.max()) + K + extra
    S = (S + 7) // 8 * 8 if dtype == "bf16" else S
    f = (lambda x: wl.round_to_bf16(x)) if dtype == "bf16" else (lambda x: x)
    q = f(rng.standard_normal((B, K, Hq, D), dtype=np.float32) * np.float32(scale))
    kc = np.full((B, Hkv, S, D), np.nan, np.float32)
    vc = np.full((B, Hkv, S, D), np.nan, np.float32)
    for b in range(B):
        n = int(ctx[b]) + K
        kc[b, :, :n] = f(rng.standard_normal((Hkv, n, D), dtype=np.float32) * np.float32(scale))
        vc[b, :, :n] = f(rng.standard_normal((Hkv, n, D), dtype=np.float32) * np.float32(scale))
    return q, kc, vc, ctx


EDGE_CASES = {
    # name: (B, Hq, Hkv, D, K, ctx list, dtype)
    "block_only_C0": (1, 32, 8, 128, 32, [0], "bf16"),
    "ragged_tile_edges": (9, 32, 8, 128, 32, [0, 1, 63, 64, 65, 127, 128, 129, 5003], "bf16"),
    "K1_decode": (2, 32, 8, 128, 1, [777, 4096], "bf16"),
    "K8": (2, 32, 8, 128, 8, [1000, 3], "bf16"),
    "K16_G2": (3, 16, 8, 128, 16, [2222, 17, 640], "bf16"),
    "K2_G1_mha": (2, 8, 8, 128, 2, [300, 1], "bf16"),
    "G4_K20_odd": (2, 32, 8, 128, 20, [999, 1501], "bf16"),
    "rows_over_128_simt": (1, 16, 2, 128, 32, [700], "bf16"),
    "D64_bf16_simt": (2, 8, 2, 64, 8, [300, 45], "bf16"),
    "D256_bf16_simt": (1, 4, 1, 256, 4, [129], "bf16"),
    "f32_D128": (2, 8, 2, 128, 8, [200, 13], "f32"),
}


@pytest.mark.parametrize("view", [ob.DIFF, ob.AR])
@pytest.mark.parametrize("case", list(EDGE_CASES))
def test_attention_edge_cases(case, view):
    B, Hq, Hkv, D, K, ctx, dt = EDGE_CASES[case]
    q, kc, vc, ctx = _custom(100 + list(EDGE_CASES).index(case), B, Hq, Hkv, D, K, ctx, dt)
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    got = run_attn(view, to_dev(q, tdt), to_dev(kc, tdt), to_dev(vc, tdt),
                   torch.from_numpy(ctx).cuda(), tdt).cpu().numpy()
    ref = oracle.attention(view, q, kc, vc, ctx)
    assert_attn_close(got, ref, case)


def test_exact_capacity_and_overflow_status():
    """ctx + K == S_max is valid; a sequence with ctx + K > S_max sets the status
    bit (no fault) and the other sequences are still exact."""
    B, Hq, Hkv, D, K = 3, 32, 8, 128, 32
    q, kc, vc, ctx = _custom(5, B, Hq, Hkv, D, K, [1000, 400, 64], extra=0)
    S = kc.shape[2]
    ctx_dev = ctx.copy()
    ctx_dev[0] = S - K                      # exactly full
    ctx_dev[2] = S - K + 1                  # one row over capacity
    kc2, vc2 = kc.copy(), vc.copy()
    rng = np.random.default_rng(6)
    kc2[0, :, :S] = wl.round_to_bf16(rng.standard_normal((Hkv, S, D), dtype=np.float32) / 11.3)
    vc2[0, :, :S] = wl.round_to_bf16(rng.standard_normal((Hkv, S, D), dtype=np.float32) / 11.3)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for view in (ob.DIFF, ob.AR):
        got = run_attn(view, to_dev(q, torch.bfloat16), to_dev(kc2, torch.bfloat16),
                       to_dev(vc2, torch.bfloat16), torch.from_numpy(ctx_dev).cuda(),
                       torch.bfloat16, status=status).cpu().numpy()
        ok = ctx_dev.copy()
        ok[2] = 0
        ref = oracle.attention(view, q[:2], kc2[:2], vc2[:2], ok[:2])
        assert_attn_close(got[:2], ref, "capacity")
    assert int(status.item()) & ob.STATUS_CAPACITY


def test_negative_ctx_sets_status():
    q, kc, vc, ctx = _custom(7, 2, 32, 8, 128, 8, [100, 50])
    ctx[1] = -5
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = run_attn(ob.AR, to_dev(q, torch.bfloat16), to_dev(kc, torch.bfloat16),
                   to_dev(vc, torch.bfloat16), torch.from_numpy(ctx).cuda(), torch.bfloat16,
                   status=status).cpu().numpy()
    assert int(status.item()) == ob.STATUS_CAPACITY
    ref = oracle.attention(ob.AR, q[:1], kc[:1], vc[:1], ctx[:1])
    assert_attn_close(got[:1], ref, "negative ctx")


def test_custom_scale():
    q, kc, vc, ctx = _custom(8, 1, 32, 8, 128, 32, [900])
    got = run_attn(ob.DIFF, to_dev(q, torch.bfloat16), to_dev(kc, torch.bfloat16),
                   to_dev(vc, torch.bfloat16), torch.from_numpy(ctx).cuda(), torch.bfloat16,
                   scale=0.3).cpu().numpy()
    assert_attn_close(got, oracle.attention(ob.DIFF, q, kc, vc, ctx, scale=0.3), "scale")


def test_workspace_too_small_is_rejected():
    q, kc, vc, ctx = _custom(9, 1, 32, 8, 128, 32, [100])
    tq, tk, tv = (to_dev(x, torch.bfloat16) for x in (q, kc, vc))
    out = torch.empty((1, 32, 32, 128), dtype=torch.float32, device="cuda")
    need = ob.orthrus_attn_workspace_size(1, 32, 8, 128, 32, torch.bfloat16)
    ws = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(ob.OrthrusError) as ei:
        ob.orthrus_attn(ob.DIFF, tq, tk, tv, torch.from_numpy(ctx).cuda(), out, ws)
    assert ei.value.code == ob.ERR_WORKSPACE


def test_repeatable_bitwise():
    """Same inputs, same launch configuration -> bitwise identical output."""
    q, kc, vc, ctx = _custom(10, 2, 32, 8, 128, 32, [3000, 700])
    args = [to_dev(x, torch.bfloat16) for x in (q, kc, vc)]
    c = torch.from_numpy(ctx).cuda()
    a = run_attn(ob.AR, *args, c, torch.bfloat16)
    b = run_attn(ob.AR, *args, c, torch.bfloat16)
    assert torch.equal(a, b)


def test_workspace_reused_across_calls_and_shapes():
    """One workspace, zero-filled once, serves consecutive calls of different
    context lengths, views and batch shapes: every call matches the oracle and
    leaves the split-merge flag and counter block (the workspace's first 1920
    bytes)
    zero again."""
    cases = [(11, 1, [5000]), (12, 2, [3000, 700]), (13, 3, [1, 2500, 129]), (14, 1, [200])]
    need = max(ob.orthrus_attn_workspace_size(B, 32, 8, 128, 32, torch.bfloat16) for _, B, _ in cases)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for seed, B, lens in cases:
        q, kc, vc, ctx = _custom(seed, B, 32, 8, 128, 32, lens)
        for view in (ob.DIFF, ob.AR):
            out = torch.full((B, 32, 32, 128), float("nan"), dtype=torch.float32, device="cuda")
            status = torch.zeros(1, dtype=torch.int32, device="cuda")
            ob.orthrus_attn(view, to_dev(q, torch.bfloat16), to_dev(kc, torch.bfloat16),
                            to_dev(vc, torch.bfloat16), torch.from_numpy(ctx).cuda(), out, ws,
                            status=status)
            torch.cuda.synchronize()
            assert int(status.item()) == 0
            assert int(ws[:SYNC_BYTES].count_nonzero().item()) == 0, "split-merge flags left set"
            assert_attn_close(out.cpu().numpy(), oracle.attention(view, q, kc, vc, ctx),
                              f"reuse B={B} view={view}")


def test_merge_wait_gives_up_on_counters_that_never_complete():
    """A workspace whose split-merge flags were not zeroed (documented misuse):
    every split segment's merge waits for a publish flag that can never reach
    one, gives up after its bound, and the call sets ORTHRUS_STATUS_TIMEOUT
    instead of hanging or faulting; the context stays usable and the next call
    on a zeroed workspace is exact."""
    q, kc, vc, ctx = _custom(15, 1, 32, 8, 128, 32, [5000])     # every segment split
    args = [to_dev(x, torch.bfloat16) for x in (q, kc, vc)]
    c = torch.from_numpy(ctx).cuda()
    need = ob.orthrus_attn_workspace_size(1, 32, 8, 128, 32, torch.bfloat16)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    ws[:2 * SYNC_BYTES // 3].view(torch.int32).fill_(-1_000_000)   # publish flags
    out = torch.empty((1, 32, 32, 128), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ob.orthrus_attn(ob.DIFF, *args, c, out, ws, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & ob.STATUS_TIMEOUT
    ws.zero_()
    status.zero_()
    ob.orthrus_attn(ob.DIFF, *args, c, out, ws, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert_attn_close(out.cpu().numpy(), oracle.attention(ob.DIFF, q, kc, vc, ctx), "after timeout")


def test_parity_while_another_stream_holds_sms():
    """A bounded matmul on another stream holds SMs while the attention runs:
    the cooperative launch keeps every CTA of the split merge resident, so the
    call is exact and no bounded wait gives up."""
    q, kc, vc, ctx = _custom(16, 1, 32, 8, 128, 32, [8192])
    args = [to_dev(x, torch.bfloat16) for x in (q, kc, vc)]
    c = torch.from_numpy(ctx).cuda()
    ws = torch.zeros(ob.orthrus_attn_workspace_size(1, 32, 8, 128, 32, torch.bfloat16),
                     dtype=torch.uint8, device="cuda")
    a = torch.randn(4096, 4096, device="cuda", dtype=torch.bfloat16)
    other, mine = torch.cuda.Stream(), torch.cuda.Stream()
    outs = []
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    for rep in range(8):
        with torch.cuda.stream(other):
            for _ in range(4):                   # ~1 ms of tensor-core work
                a = (a @ a) * (1.0 / 64)
        with torch.cuda.stream(mine):
            out = torch.empty((1, 32, 32, 128), dtype=torch.float32, device="cuda")
            ob.orthrus_attn(rep % 2, *args, c, out, ws, status=status, stream=mine)
            outs.append((rep % 2, out))
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"device status {int(status.item()):#x}"
    refs = {v: oracle.attention(v, q, kc, vc, ctx) for v in (ob.DIFF, ob.AR)}
    for view, out in outs:
        assert_attn_close(out.cpu().numpy(), refs[view], f"concurrent view {view}")


_TWO_THREADS = r"""
import sys, threading
import numpy as np, torch
sys.path.insert(0, {root!r})
from lossless_diffusion_speculative_b200 import binding as ob
torch.cuda.init()
rng = np.random.default_rng(3)
B, Hq, Hkv, D, K, C = 1, 32, 8, 128, 32, 3000
S = C + K
q = torch.from_numpy(rng.standard_normal((B, K, Hq, D), dtype=np.float32) / 11.3).cuda().bfloat16()
kc = torch.from_numpy(rng.standard_normal((B, Hkv, S, D), dtype=np.float32) / 11.3).cuda().bfloat16()
vc = torch.from_numpy(rng.standard_normal((B, Hkv, S, D), dtype=np.float32) / 11.3).cuda().bfloat16()
ctx = torch.tensor([C], dtype=torch.int32, device="cuda")
need = ob.lib().orthrus_attn_workspace_size(B, Hq, Hkv, D, K, ob.BF16)
res = {{}}
go = threading.Barrier(2)
def worker(t):
    torch.cuda.set_device(0)
    s = torch.cuda.Stream()
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    out = torch.empty((B, K, Hq, D), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    go.wait()
    try:
        ob.orthrus_attn(t % 2, q, kc, vc, ctx, out, ws, stream=s)
        s.synchronize()
        res[t] = out.cpu()
    except Exception as e:
        res[t] = e
ts = [threading.Thread(target=worker, args=(t,)) for t in range(2)]
[t.start() for t in ts]; [t.join() for t in ts]
for t in range(2):
    assert isinstance(res[t], torch.Tensor), res[t]
    assert torch.isfinite(res[t]).all()
np.save(sys.argv[1], np.stack([res[0].numpy(), res[1].numpy()]))
print("ok")
"""


def test_first_calls_from_two_threads(tmp_path):
    """The first orthrus_attn calls of a fresh process, made from two host
    threads at once, both succeed (the library's one-time set-up is
    thread-safe) and are exact."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    script = tmp_path / "two_threads.py"
    script.write_text(_TWO_THREADS.format(root=root))
    out = tmp_path / "out.npy"
    r = subprocess.run([sys.executable, str(script), str(out)], capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout + r.stderr
    got = np.load(out)
    rng = np.random.default_rng(3)
    B, Hq, Hkv, D, K, C = 1, 32, 8, 128, 32, 3000
    S = C + K
    bf = wl.round_to_bf16
    q = bf(rng.standard_normal((B, K, Hq, D), dtype=np.float32) / np.float32(11.3))
    kc = bf(rng.standard_normal((B, Hkv, S, D), dtype=np.float32) / np.float32(11.3))
    vc = bf(rng.standard_normal((B, Hkv, S, D), dtype=np.float32) / np.float32(11.3))
    ctx = np.array([C], np.int32)
    for t in range(2):
        assert_attn_close(got[t], oracle.attention(t % 2, q, kc, vc, ctx), f"thread {t}")
