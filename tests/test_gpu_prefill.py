"""GPU parity of orthrus_prefill_attn (causal attention over the prompt, run as
chunked AR-view attention) against the fp64 oracle: the AR view with no
committed context and K = S (pinned to the library's causal SDPA).
Tolerance: max |gpu - oracle| <= 2e-3 * RMS(oracle output)."""
import numpy as np
import pytest
import torch

import oracle
from lossless_diffusion_speculative_b200 import binding as ob
from lossless_diffusion_speculative_b200 import workloads as wl
from gpu_util import assert_attn_close

pytestmark = pytest.mark.gpu


def _case(seed, B, S, Hq, Hkv, D, dtype="bf16", extra=16):
    rng = np.random.default_rng(seed)
    f = wl.round_to_bf16 if dtype == "bf16" else (lambda x: x)
    sc = np.float32(1 / np.sqrt(D))
    q = f(rng.standard_normal((B, S, Hq, D), dtype=np.float32) * sc)
    Smax = S + extra
    kc = np.full((B, Hkv, Smax, D), np.nan, np.float32)          # rows past the prompt: never read
    vc = np.full((B, Hkv, Smax, D), np.nan, np.float32)
    kc[:, :, :S] = f(rng.standard_normal((B, Hkv, S, D), dtype=np.float32) * sc)
    vc[:, :, :S] = f(rng.standard_normal((B, Hkv, S, D), dtype=np.float32) * sc)
    return q, kc, vc


def _gpu(q, kc, vc, dtype):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda().to(tdt)
    B, S, Hq, D = q.shape
    Hkv = kc.shape[1]
    out = torch.full((B, S, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.zeros(ob.orthrus_prefill_workspace_size(B, S, Hq, Hkv, D, tdt), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ob.orthrus_prefill_attn(dev(q), dev(kc), dev(vc), out, ws, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return out.cpu().numpy()


CASES = {   # name: (B, S, Hq, Hkv, D, dtype)
    "qwen3_8b_prompt_4096": (1, 4096, 32, 8, 128, "bf16"),
    "batch_ragged_tail": (2, 1000, 32, 8, 128, "bf16"),
    "shorter_than_a_chunk": (3, 20, 32, 8, 128, "bf16"),
    "one_token": (2, 1, 32, 8, 128, "bf16"),
    "mha_g1": (1, 300, 8, 8, 128, "bf16"),
    "g2_chunks_of_64": (2, 257, 16, 8, 128, "bf16"),
    "fp32_cuda_core": (1, 130, 4, 2, 64, "f32"),
    "d64_cuda_core": (2, 77, 8, 2, 64, "bf16"),
}


@pytest.mark.parametrize("name", list(CASES))
def test_prefill_matches_causal_oracle(name):
    B, S, Hq, Hkv, D, dt = CASES[name]
    q, kc, vc = _case(300 + list(CASES).index(name), B, S, Hq, Hkv, D, dt)
    got = _gpu(q, kc, vc, dt)
    ref = oracle.attention(oracle.AR, q, kc, vc, np.zeros(B, np.int32))
    assert_attn_close(got, ref, name)
