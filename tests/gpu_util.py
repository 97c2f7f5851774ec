"""Shared helpers of the GPU tests: upload seeded inputs, run the library through
its C ABI, compare with the oracle at the stated tolerance."""
from __future__ import annotations

import numpy as np
import torch

from lossless_diffusion_speculative_b200 import binding as ob

# Attention tolerance: max |gpu - oracle| <= ATOL_REL_RMS * RMS(oracle output)
# (bf16 or fp32 inputs, fp32 accumulation, fp32 output).
ATOL_REL_RMS = 2e-3


def tdtype(w):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def to_dev(x: np.ndarray, dtype) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to(dtype).cuda()


def run_attn(view: int, q, kc, vc, ctx, dtype, status=None, scale=0.0):
    """Device tensors in, fp32 output tensor out (after a synchronise).  Without
    a caller status word, the call must leave the device status at zero."""
    B, K, Hq, D = q.shape
    Hkv = kc.shape[1]
    out = torch.full((B, K, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.zeros(ob.orthrus_attn_workspace_size(B, Hq, Hkv, D, K, dtype),
                     dtype=torch.uint8, device="cuda")
    own = status is None
    if own:
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ob.orthrus_attn(view, q, kc, vc, ctx, out, ws, status=status, scale=scale)
    torch.cuda.synchronize()
    if own:
        assert int(status.item()) == 0, f"device status {int(status.item()):#x}"
    return out


def assert_attn_close(got: np.ndarray, ref: np.ndarray, what: str = ""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite GPU output"
    rms = float(np.sqrt(np.mean(ref * ref)))
    err = float(np.max(np.abs(got - ref)))
    assert err <= ATOL_REL_RMS * rms, f"{what}: max|err| {err:.3e} > {ATOL_REL_RMS} * rms {rms:.3e}"
    return err / rms
