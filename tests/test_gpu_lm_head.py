"""GPU parity of orthrus_lm_head_consensus (fused AR LM head + argmax +
consensus) against the fp64 oracle.

The kernel sums exact bf16 products in fp32 on the tensor cores; the oracle in
fp64.  Where a row's two largest fp64 logits differ by more than twice the
rigorous fp32 accumulation bound (oracle.fp32_dot_error_bound) the argmax is
unique under any rounding and must match exactly; elsewhere the GPU's choice
must be a valid maximum (its exact logit within twice the bound of the row
maximum).  On planted inputs (margin ~7 against bounds < 0.4) accepted lengths,
next tokens and every argmax are bit-exact against the oracle and the plant.
"""
import numpy as np
import pytest
import torch

import oracle
from lossless_diffusion_speculative_b200 import binding as ob
from lossless_diffusion_speculative_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _run(li, ws=None, status=None):
    B, K, Hd = li.hidden.shape
    h = torch.from_numpy(li.hidden).cuda().to(torch.bfloat16)
    W = torch.from_numpy(li.lm_head).cuda().to(torch.bfloat16)
    prop = torch.from_numpy(li.proposed).cuda()
    acc = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    nxt = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    am = torch.full((B, K), -7, dtype=torch.int32, device="cuda")
    if ws is None:
        ws = torch.zeros(ob.orthrus_lm_head_workspace_size(B, K), dtype=torch.uint8, device="cuda")
    own = status is None
    if own:
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ob.orthrus_lm_head_consensus(h, W, prop, acc, nxt, ws, argmax_out=am, status=status)
    torch.cuda.synchronize()
    if own:
        assert int(status.item()) == 0
    assert int(ws.count_nonzero().item()) == 0, "workspace not left zero"
    return acc.cpu().numpy(), nxt.cpu().numpy(), am.cpu().numpy()


SHAPES = {   # name: (B, K, Hd, V)
    "one_row_tiny_vocab": (1, 1, 64, 2),
    "k8_vocab_not_16": (1, 8, 64, 1000),
    "rows_not_16": (3, 5, 128, 5003),
    "vocab_under_a_tile": (2, 4, 192, 100),
    "many_ctas_partial_tiles": (1, 32, 256, 20011),
    "two_mma_halves": (16, 32, 128, 3001),
    "rows_300": (10, 30, 64, 777),
    "two_tile_passes_128_rows": (4, 32, 192, 40009),      # 270 vocabulary rows per CTA
    "two_tile_passes_90_rows": (3, 30, 128, 30011),       # 203: a pair with a short second half
    "two_tile_passes_vocab_under_a_pair": (2, 40, 64, 200),
}


@pytest.mark.parametrize("name", list(SHAPES))
def test_lm_head_planted_bit_exact(name):
    B, K, Hd, V = SHAPES[name]
    w = wl.WORKLOADS["qwen3_4b_ragged"].with_(B=B, K=K, vocab=V)
    plant = V >= B * K
    li = wl.lm_head_inputs(w, Hd=Hd, plant=plant)
    acc, nxt, am = _run(li)
    racc, rnxt, ram, gap, absdot = oracle.lm_head_consensus(li.hidden, li.lm_head, li.proposed)
    bound = oracle.fp32_dot_error_bound(Hd, absdot)
    unique = gap > 2 * bound
    assert (am[unique] == ram[unique]).all()
    if plant:
        assert unique.all()
        assert (am == li.planted_argmax).all()
        assert (acc == li.planted_accept).all() and (nxt == li.planted_next).all()
    if unique.all():
        assert (acc == racc).all() and (nxt == rnxt).all()


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_lm_head_unplanted_matches_where_unique(seed):
    """Random logits (no plant): exact argmax wherever the fp64 top-2 gap beats
    the fp32 rounding bound, a valid maximum elsewhere; the prefix walk over
    the GPU's argmax is the consensus rule."""
    B, K, Hd, V = 2, 16, 512, 30011
    w = wl.WORKLOADS["qwen3_4b_ragged"].with_(B=B, K=K, vocab=V, cid=60 + seed)
    li = wl.lm_head_inputs(w, Hd=Hd, plant=False)
    logits = oracle.lm_head_logits(li.hidden, li.lm_head).reshape(B, K, V)
    li.proposed[:] = np.argmax(logits, axis=2)[:, :]          # let every proposal match...
    li.proposed[1, 7] = (li.proposed[1, 7] + 1) % V           # ...but one
    acc, nxt, am = _run(li)
    racc, rnxt, ram, gap, absdot = oracle.lm_head_consensus(li.hidden, li.lm_head, li.proposed)
    bound = oracle.fp32_dot_error_bound(Hd, absdot)
    unique = gap > 2 * bound
    assert unique.mean() > 0.9
    assert (am[unique] == ram[unique]).all()
    rowmax = logits.max(axis=2)
    picked = np.take_along_axis(logits, am[..., None].astype(np.int64), axis=2)[..., 0]
    assert (rowmax - picked <= 2 * bound).all()
    for b in range(B):                                        # the rule on the GPU's argmax
        a = 0
        while a < K and li.proposed[b, a] == am[b, a]:
            a += 1
        assert acc[b] == a and nxt[b] == am[b, min(a, K - 1)]


def test_lm_head_ties_lowest_index_and_workspace_reuse():
    """Identical weight rows tie exactly in any rounding order: the lowest
    index wins.  The same workspace serves consecutive calls."""
    w = wl.WORKLOADS["qwen3_8b_step"].with_(vocab=4000)
    li = wl.lm_head_inputs(w, Hd=128)
    r = li.planted_argmax[0]
    free = np.setdiff1d(np.arange(4000), r)
    dup = np.random.default_rng(5).choice(free, size=r.size, replace=False)
    lo = np.minimum(r, dup)
    li.lm_head[dup] = li.lm_head[r]                            # exact copies
    ws = torch.zeros(ob.orthrus_lm_head_workspace_size(1, 32), dtype=torch.uint8, device="cuda")
    for _ in range(2):
        acc, nxt, am = _run(li, ws=ws)
        assert (am[0] == lo).all()
    _, _, ram, _, _ = oracle.lm_head_consensus(li.hidden, li.lm_head, li.proposed)
    assert (ram[0] == lo).all()


@pytest.mark.parametrize("name", ["qwen3_8b_step", "qwen3_4b_ragged", "qwen3_1p7b_layer", "qwen3_8b_long_k32"])
def test_lm_head_full_size_planted(name):
    """Full Qwen3 vocabulary and width, in the benchmark's launch configuration:
    the planted argmax (margin ~7 against an fp32 bound < 0.4) is recovered
    exactly for every token row, and the consensus equals the plant."""
    w = wl.WORKLOADS[name]
    li = wl.lm_head_inputs(w)
    acc, nxt, am = _run(li)
    assert (am == li.planted_argmax).all()
    assert (acc == li.planted_accept).all() and (nxt == li.planted_next).all()


def test_lm_head_rejects_bad_arguments():
    h = torch.zeros((1, 8, 100), dtype=torch.bfloat16, device="cuda")     # Hd not a multiple of 64
    W = torch.zeros((50, 100), dtype=torch.bfloat16, device="cuda")
    prop = torch.zeros((1, 8), dtype=torch.int32, device="cuda")
    out = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    with pytest.raises(ob.OrthrusError) as ei:
        ob.orthrus_lm_head_consensus(h, W, prop, out, out, ws)
    assert ei.value.code == ob.ERR_UNSUPPORTED
    h = torch.zeros((1, 8, 64), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((50, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ob.OrthrusError) as ei:
        ob.orthrus_lm_head_consensus(h, W, prop, out, out, ws[:8])
    assert ei.value.code == ob.ERR_WORKSPACE
