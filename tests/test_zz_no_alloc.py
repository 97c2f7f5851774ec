"""orthrus_attn_static: attention for callers that cannot allocate device
memory (an engine whose memory plan is frozen after warm-up, a plugin that only
receives input and output pointers, a runtime whose allocator belongs to
another framework).  It uses the library's built-in scratch array instead of a
caller workspace; its results must match the fp64 oracle and orthrus_attn's on
consecutive calls (the shared scratch keeps the previous call's contents), and
warm calls must not change the device's free memory.

This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from lossless_diffusion_speculative_b200 import binding as ob
from lossless_diffusion_speculative_b200 import workloads as wl
from gpu_util import assert_attn_close, run_attn, to_dev

pytestmark = pytest.mark.gpu


def _static_fn():
    L = ob.lib()
    f = L.orthrus_attn_static
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    f.restype = i32
    f.argtypes = [i32, i32, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, ctypes.c_float, vp,
                  vp, vp]
    return f


def _call_static(view, q, kc, vc, ctx, dtype_code):
    B, K, Hq, D = q.shape
    Hkv, S = kc.shape[1], kc.shape[2]
    out = torch.full((B, K, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = _static_fn()(view, dtype_code, q.data_ptr(), kc.data_ptr(), vc.data_ptr(),
                      ctx.data_ptr(), B, Hq, Hkv, D, S, K, 0.0, out.data_ptr(),
                      status.data_ptr(), stream)
    torch.cuda.synchronize()
    assert rc == 0, ob.lib().orthrus_error_string(rc).decode()
    assert int(status.item()) == 0
    return out


def _host_inputs(seed, B, Hq, Hkv, D, K, ctx, dtype):
    """Seeded inputs as float32 arrays holding exactly the values uploaded."""
    rng = np.random.default_rng(seed)
    ctx = np.asarray(ctx, np.int32)
    S = int(ctx.max()) + K
    sc = np.float32(1 / np.sqrt(128))
    f = wl.round_to_bf16 if dtype == torch.bfloat16 else (lambda x: x)
    q = f(rng.standard_normal((B, K, Hq, D), dtype=np.float32) * sc)
    kc = f(rng.standard_normal((B, Hkv, S, D), dtype=np.float32) * sc)
    vc = f(rng.standard_normal((B, Hkv, S, D), dtype=np.float32) * sc)
    return q, kc, vc, ctx


def _inputs(seed, B, Hq, Hkv, D, K, ctx, dtype):
    q, kc, vc, ctx = _host_inputs(seed, B, Hq, Hkv, D, K, ctx, dtype)
    return (to_dev(q, dtype), to_dev(kc, dtype), to_dev(vc, dtype),
            torch.from_numpy(ctx).cuda())


SHAPES = {   # (B, Hq, Hkv, D, K, ctx) of two consecutive calls
    "bf16_tensor_core": [(2, 32, 8, 128, 32, [3000, 517]), (3, 32, 8, 128, 16, [64, 9000, 1])],
    "f32_cuda_core": [(1, 4, 2, 64, 8, [256]), (2, 4, 2, 64, 8, [40, 700])],
}


@pytest.mark.parametrize("name,dtype,code", [("bf16_tensor_core", torch.bfloat16, ob.BF16),
                                             ("f32_cuda_core", torch.float32, ob.F32)])
def test_static_scratch_matches_workspace_call_twice(name, dtype, code):
    cases = [(view, shape, _inputs(10 + view, *shape, dtype))      # two calls in a row
             for view, shape in zip((ob.DIFF, ob.AR), SHAPES[name])]
    for view, shape, (q, kc, vc, ctx) in cases:
        got = _call_static(view, q, kc, vc, ctx, code).cpu().numpy()
        ref = run_attn(view, q, kc, vc, ctx, dtype)
        assert_attn_close(got, ref.cpu().numpy(), "static scratch vs orthrus_attn")
        hq, hk, hv, hc = _host_inputs(10 + view, *shape, dtype)
        assert_attn_close(got, oracle.attention(view, hq, hk, hv, hc), "static scratch vs oracle")


def test_static_scratch_calls_allocate_nothing():
    """After a warm call (which loads the library's device code, scratch array
    included), further calls leave the device's free memory unchanged."""
    q, kc, vc, ctx = _inputs(21, 2, 32, 8, 128, 32, [5000, 300], torch.bfloat16)
    _call_static(ob.DIFF, q, kc, vc, ctx, ob.BF16)
    B, K, Hq, D = q.shape
    out = torch.empty((B, K, Hq, D), dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    f = _static_fn()
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for rep in range(6):
        rc = f(rep % 2, ob.BF16, q.data_ptr(), kc.data_ptr(), vc.data_ptr(), ctx.data_ptr(),
               B, Hq, 8, D, kc.shape[2], K, 0.0, out.data_ptr(), None, stream)
        assert rc == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, (free0, free1)


def test_static_scratch_rejects_oversized_problems():
    q, kc, vc, ctx = _inputs(3, 1, 32, 8, 128, 32, [100], torch.bfloat16)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    out = torch.empty((1, 32, 32, 128), dtype=torch.float32, device="cuda")
    # B = 4096 sequences need far more split scratch than the built-in array holds
    rc = _static_fn()(ob.DIFF, ob.BF16, q.data_ptr(), kc.data_ptr(), vc.data_ptr(),
                      ctx.data_ptr(), 4096, 32, 8, 128, kc.shape[2], 32, 0.0, out.data_ptr(),
                      None, stream)
    assert rc == ob.ERR_WORKSPACE
