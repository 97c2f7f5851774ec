"""GPU parity of orthrus_consensus and orthrus_kv_commit: bit-exact against the
oracle (and the plant), on every workload's full vocabulary and batch, on the
hand-made golden cases, on tie/NaN-heavy rows, and through a lossless decode
loop whose consensus and commit run on the device."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from lossless_diffusion_speculative_b200 import binding as ob
from lossless_diffusion_speculative_b200 import workloads as wl

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _gpu_consensus(logits: np.ndarray, proposed: np.ndarray, status=None):
    B, K, V = logits.shape
    lg = torch.from_numpy(np.ascontiguousarray(logits, np.float32)).cuda()
    pr = torch.from_numpy(np.ascontiguousarray(proposed, np.int32)).cuda()
    acc = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    nxt = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    am = torch.full((B, K), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(ob.orthrus_consensus_workspace_size(B, K, V), dtype=torch.uint8,
                     device="cuda")
    ob.orthrus_consensus(lg, pr, acc, nxt, ws, argmax_out=am, status=status)
    torch.cuda.synchronize()
    return acc.cpu().numpy(), nxt.cpu().numpy(), am.cpu().numpy()


@pytest.mark.parametrize("name", list(wl.WORKLOADS))
def test_consensus_planted_full_vocab(name):
    w = wl.WORKLOADS[name]
    ci = wl.consensus_inputs(w)
    acc, nxt, am = _gpu_consensus(ci.logits, ci.proposed)
    oacc, onxt, oam = oracle.consensus(ci.logits, ci.proposed)
    np.testing.assert_array_equal(am, oam)
    np.testing.assert_array_equal(acc, oacc)
    np.testing.assert_array_equal(nxt, onxt)
    np.testing.assert_array_equal(acc, ci.planted_accept)
    np.testing.assert_array_equal(nxt, ci.planted_next)


@pytest.mark.parametrize("a", [0, 1, 16, 31, 32])
def test_consensus_extremes_qwen_vocab(a):
    w = wl.WORKLOADS["qwen3_8b_step"]
    ci = wl.consensus_inputs(w, accept=np.array([a]))
    acc, nxt, _ = _gpu_consensus(ci.logits, ci.proposed)
    assert acc[0] == a and nxt[0] == ci.planted_argmax[0, min(a, 31)]


def test_consensus_golden_cases():
    cases = json.load(open(os.path.join(GOLDEN, "consensus_cases.json")))["cases"]
    for c in cases:
        logits = np.array([[float(v) if isinstance(v, str) else v for v in row]
                           for row in c["logits"]], np.float32)[None]
        acc, nxt, am = _gpu_consensus(logits, np.array(c["proposed"], np.int32)[None])
        assert acc[0] == c["accepted"] and nxt[0] == c["next"], c["name"]
        assert list(am[0]) == c["argmax"], c["name"]


@pytest.mark.parametrize("V", [1, 3, 4, 999, 1000, 4097, 151936])
def test_consensus_ties_nan_and_odd_vocab(V):
    """Quantised logits (many ties), scattered NaN, -0.0 and infinities; V not a
    multiple of 4 takes the scalar path.  Bit-exact against the oracle."""
    rng = np.random.default_rng(V)
    B, K = 3, 32
    logits = rng.integers(-4, 5, size=(B, K, V)).astype(np.float32)
    logits[rng.random(logits.shape) < 0.01] = -0.0
    if V > 10:
        logits[0, 3, rng.integers(V, size=3)] = np.nan
        logits[1, 5, rng.integers(V, size=2)] = np.inf
        logits[2, 7] = -np.inf
    prop = rng.integers(0, V, size=(B, K)).astype(np.int32)
    _, _, oam = oracle.consensus(logits, prop)
    prop[:, :20] = oam[:, :20]               # long accepted prefixes
    oacc, onxt, oam = oracle.consensus(logits, prop)
    acc, nxt, am = _gpu_consensus(logits, prop)
    np.testing.assert_array_equal(am, oam)
    np.testing.assert_array_equal(acc, oacc)
    np.testing.assert_array_equal(nxt, onxt)


# ----------------------------------------------------------------------------- commit

def _bits(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns of float32 values that are exact in bf16."""
    return (np.ascontiguousarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


@pytest.mark.parametrize("layers", [1, 3, 36])
def test_kv_commit_copy_bit_exact(layers):
    rng = np.random.default_rng(20 + layers)
    B, Hkv, D, K = 4, 8, 128, 32
    ctx = np.array([0, 100, 4000, 17], np.int32)
    acc = np.array([0, 32, 7, 31], np.int32)
    S = int(ctx.max()) + 2 * K
    kcs, vcs, kbs, vbs = [], [], [], []
    for _ in range(layers):
        kcs.append(rng.integers(0, 2 ** 16, size=(B, Hkv, S, D), dtype=np.uint16))
        vcs.append(rng.integers(0, 2 ** 16, size=(B, Hkv, S, D), dtype=np.uint16))
        kbs.append(rng.integers(0, 2 ** 16, size=(B, K, Hkv, D), dtype=np.uint16))
        vbs.append(rng.integers(0, 2 ** 16, size=(B, K, Hkv, D), dtype=np.uint16))
    dev = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    dk, dv, dkb, dvb = ([dev(a) for a in arrs] for arrs in (kcs, vcs, kbs, vbs))
    dctx = torch.from_numpy(ctx).cuda()
    dacc = torch.from_numpy(acc).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ob.orthrus_kv_commit(dctx, dacc, K=K, Hkv=Hkv, D=D, S_max=S, k_caches=dk, v_caches=dv,
                         k_blks=dkb, v_blks=dvb, status=status)
    torch.cuda.synchronize()
    octx = ctx.copy()
    for l in range(layers):
        oracle.kv_commit(kcs[l], vcs[l], kbs[l], vbs[l], octx, acc, K, advance=(l == layers - 1))
        got_k = dk[l].view(torch.int16).cpu().numpy().view(np.uint16)
        got_v = dv[l].view(torch.int16).cpu().numpy().view(np.uint16)
        np.testing.assert_array_equal(got_k, kcs[l])
        np.testing.assert_array_equal(got_v, vcs[l])
    np.testing.assert_array_equal(dctx.cpu().numpy(), octx)
    assert int(status.item()) == 0


def test_kv_commit_advance_only_and_status():
    ctx = np.array([10, 20, 30, 40, 50], np.int32)
    acc = np.array([0, 31, 32, 33, -1], np.int32)
    S, K = 70, 32
    dctx = torch.from_numpy(ctx).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ob.orthrus_kv_commit(dctx, torch.from_numpy(acc).cuda(), K=K, Hkv=8, D=128, S_max=S,
                         status=status)
    torch.cuda.synchronize()
    # b=3,4: accepted out of range (flagged, untouched); b=4 also ctx 50+32 > 70
    np.testing.assert_array_equal(dctx.cpu().numpy(), [11, 52, 62, 40, 50])
    assert int(status.item()) & ob.STATUS_ACCEPT
    ctx2 = torch.tensor([50], dtype=torch.int32, device="cuda")
    status.zero_()
    ob.orthrus_kv_commit(ctx2, torch.tensor([3], dtype=torch.int32, device="cuda"), K=K, Hkv=8,
                         D=128, S_max=S, status=status)
    torch.cuda.synchronize()
    assert int(ctx2.item()) == 50 and int(status.item()) == ob.STATUS_CAPACITY


def _toy_logits(tokens, V, seed=17):
    h = 1469598103934665603
    for t in tokens:
        h = ((h ^ int(t)) * 1099511628211) & 0xFFFFFFFFFFFFFFFF
    return np.random.default_rng([seed, h & 0xFFFFFFFF, h >> 32]).standard_normal(V).astype(np.float32)


def test_lossless_loop_on_device():
    """Consensus and commit on the GPU inside the dual-view loop (toy frozen
    model on the host): the emitted stream equals greedy decoding, and the
    device ctx_lens tracks the committed length."""
    V, K, target = 64, 8, 60
    prompt = [5, 9, 2]
    greedy = list(prompt)
    while len(greedy) < target:
        greedy.append(int(np.argmax(_toy_logits(greedy, V))))
    rng = np.random.default_rng(30)
    seq, anchor = list(prompt[:-1]), prompt[-1]
    dctx = torch.tensor([len(seq)], dtype=torch.int32, device="cuda")
    while len(seq) + 1 < target:
        ctx = seq + [anchor]
        prop, t = [], list(ctx)
        for _ in range(K):
            nx = int(np.argmax(_toy_logits(t, V)))
            if rng.random() < 0.25:
                nx = int(rng.integers(V))
            prop.append(nx)
            t.append(nx)
        logits = np.stack([_toy_logits(ctx + prop[:i], V) for i in range(K)])[None]
        acc, nxt, _ = _gpu_consensus(logits, np.array([prop], np.int32))
        ob.orthrus_kv_commit(dctx, torch.from_numpy(acc).cuda(), K=K, Hkv=1, D=128,
                             S_max=4096)
        n = min(int(acc[0]) + 1, K)
        seq = seq + ([anchor] + prop[:K - 1])[:n]
        anchor = int(nxt[0])
        torch.cuda.synchronize()
        assert int(dctx.item()) == len(seq)
    out = (seq + [anchor])[:target]
    assert out == greedy[:len(out)]


def test_write_block_installs_every_slot_without_advancing():
    rng = np.random.default_rng(40)
    B, Hkv, D, K, layers = 3, 8, 128, 32, 4
    ctx = np.array([0, 250, 1000], np.int32)
    S = int(ctx.max()) + K
    kcs = [rng.integers(0, 2 ** 16, size=(B, Hkv, S, D), dtype=np.uint16) for _ in range(layers)]
    vcs = [rng.integers(0, 2 ** 16, size=(B, Hkv, S, D), dtype=np.uint16) for _ in range(layers)]
    kbs = [rng.integers(0, 2 ** 16, size=(B, K, Hkv, D), dtype=np.uint16) for _ in range(layers)]
    vbs = [rng.integers(0, 2 ** 16, size=(B, K, Hkv, D), dtype=np.uint16) for _ in range(layers)]
    dev = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    dk, dv, dkb, dvb = ([dev(a) for a in arrs] for arrs in (kcs, vcs, kbs, vbs))
    dctx = torch.from_numpy(ctx).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ob.orthrus_write_block(dctx, dk, dv, dkb, dvb, status=status)
    torch.cuda.synchronize()
    for l in range(layers):
        # oracle commit with a = K copies all K slots; no advance
        oracle.kv_commit(kcs[l], vcs[l], kbs[l], vbs[l], ctx.copy(), np.full(B, K, np.int32), K,
                         advance=False)
        np.testing.assert_array_equal(dk[l].view(torch.int16).cpu().numpy().view(np.uint16), kcs[l])
        np.testing.assert_array_equal(dv[l].view(torch.int16).cpu().numpy().view(np.uint16), vcs[l])
    np.testing.assert_array_equal(dctx.cpu().numpy(), ctx)
    assert int(status.item()) == 0
    # a sequence without room is flagged and skipped
    dctx2 = torch.tensor([0, S - K + 1, 5], dtype=torch.int32, device="cuda")
    ob.orthrus_write_block(dctx2, dk[:1], dv[:1], dkb[:1], dvb[:1], status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == ob.STATUS_CAPACITY


def test_tensor_core_path_is_selected_for_bf16_d128():
    assert ob.orthrus_attn_path(1, 32, 8, 128, 32, torch.bfloat16) == 1
    assert ob.orthrus_attn_path(4, 32, 8, 128, 8, torch.bfloat16) == 1
    assert ob.orthrus_attn_path(1, 16, 8, 128, 32, torch.bfloat16) == 1
    assert ob.orthrus_attn_path(1, 16, 2, 128, 32, torch.bfloat16) == 0   # G*K = 256
    assert ob.orthrus_attn_path(1, 4, 2, 64, 8, torch.float32) == 0
