"""Thin ctypes binding of liborthrus.so (argument marshalling only).

Every function here has the name of the C entry point it wraps and does nothing
but read shapes and device pointers off torch tensors and forward them; all
arithmetic runs in the library's CUDA kernels.  There is no CPU fallback: if the
library is missing or the device cannot run it, the call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

from .build import LIB

DIFF, AR = 0, 1
BF16, F32 = 0, 1

ERR_ARG, ERR_UNSUPPORTED, ERR_ALIGN, ERR_WORKSPACE, ERR_LAUNCH, ERR_DEVICE = -1, -2, -3, -4, -5, -6
STATUS_CAPACITY, STATUS_ACCEPT, STATUS_TIMEOUT = 0x1, 0x2, 0x4

EXPORTED = ("orthrus_attn_workspace_size", "orthrus_attn", "orthrus_attn_path",
            "orthrus_consensus_workspace_size", "orthrus_consensus",
            "orthrus_kv_commit", "orthrus_write_block", "orthrus_error_string",
            "orthrus_version", "orthrus_lm_head_workspace_size",
            "orthrus_lm_head_consensus", "orthrus_rejection_workspace_size",
            "orthrus_rejection_verify", "orthrus_qkv_workspace_size", "orthrus_qkv_project",
            "orthrus_prefill_workspace_size",
            "orthrus_prefill_attn")


class OrthrusError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed: {msg} (code {code})")
        self.code = code


_lib = None


def lib():
    """Load liborthrus.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise RuntimeError(
                f"liborthrus.so not found at {LIB}; build it with "
                "`python -m lossless_diffusion_speculative_b200.build`")
        L = ctypes.CDLL(LIB)
        vp, sz, i32, f32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
        L.orthrus_attn_workspace_size.restype = sz
        L.orthrus_attn_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32]
        L.orthrus_attn.restype = i32
        L.orthrus_attn.argtypes = [i32, i32, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                   f32, vp, vp, sz, vp, vp]
        L.orthrus_consensus_workspace_size.restype = sz
        L.orthrus_consensus_workspace_size.argtypes = [i32, i32, i32]
        L.orthrus_consensus.restype = i32
        L.orthrus_consensus.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp, vp, sz, vp, vp]
        L.orthrus_kv_commit.restype = i32
        L.orthrus_kv_commit.argtypes = [i32, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                        i32, vp, vp]
        L.orthrus_write_block.restype = i32
        L.orthrus_write_block.argtypes = [i32, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                          i32, vp, vp]
        L.orthrus_attn_path.restype = i32
        L.orthrus_attn_path.argtypes = [i32, i32, i32, i32, i32, i32]
        L.orthrus_lm_head_workspace_size.restype = sz
        L.orthrus_lm_head_workspace_size.argtypes = [i32, i32]
        L.orthrus_lm_head_consensus.restype = i32
        L.orthrus_lm_head_consensus.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, sz,
                                                vp, vp]
        L.orthrus_rejection_workspace_size.restype = sz
        L.orthrus_rejection_workspace_size.argtypes = [i32, i32, i32]
        L.orthrus_rejection_verify.restype = i32
        L.orthrus_rejection_verify.argtypes = [vp, vp, vp, vp, vp, f32, i32, i32, i32, vp, vp, vp, sz,
                                               vp, vp]
        L.orthrus_qkv_workspace_size.restype = sz
        L.orthrus_qkv_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32]
        L.orthrus_qkv_project.restype = i32
        L.orthrus_qkv_project.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, vp, vp,
                                          vp, vp, sz, vp, vp]
        L.orthrus_prefill_workspace_size.restype = sz
        L.orthrus_prefill_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32]
        L.orthrus_prefill_attn.restype = i32
        L.orthrus_prefill_attn.argtypes = [i32, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, vp, vp, sz,
                                           vp, vp]
        L.orthrus_error_string.restype = ctypes.c_char_p
        L.orthrus_error_string.argtypes = [i32]
        L.orthrus_version.restype = i32
        L.orthrus_version.argtypes = []
        _lib = L
    return _lib


def _check(fn: str, rc: int) -> None:
    if rc != 0:
        raise OrthrusError(fn, rc, lib().orthrus_error_string(rc).decode())


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("liborthrus takes device tensors")
    if not t.is_contiguous():
        raise ValueError("liborthrus takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return BF16
    if dt == torch.float32:
        return F32
    raise ValueError(f"unsupported dtype {dt}")


def orthrus_version() -> int:
    return int(lib().orthrus_version())


def orthrus_attn_workspace_size(B: int, Hq: int, Hkv: int, D: int, K: int,
                                dtype: torch.dtype = torch.bfloat16) -> int:
    return int(lib().orthrus_attn_workspace_size(B, Hq, Hkv, D, K, _dtype_code(dtype)))


def orthrus_attn(view: int, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                 ctx_lens: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor,
                 status: Optional[torch.Tensor] = None, scale: float = 0.0,
                 stream=None) -> None:
    """q [B,K,Hq,D], caches [B,Hkv,S_max,D] (bf16 or fp32), ctx_lens [B] int32,
    out [B,K,Hq,D] fp32, workspace uint8 of orthrus_attn_workspace_size bytes."""
    B, K, Hq, D = q.shape
    _, Hkv, S_max, _ = k_cache.shape
    assert ctx_lens.dtype == torch.int32 and out.dtype == torch.float32
    rc = lib().orthrus_attn(int(view), _dtype_code(q.dtype), _ptr(q), _ptr(k_cache),
                            _ptr(v_cache), _ptr(ctx_lens), B, Hq, Hkv, D, S_max, K,
                            float(scale), _ptr(out), _ptr(workspace),
                            workspace.numel() * workspace.element_size(), _ptr(status),
                            _stream(stream))
    _check("orthrus_attn", rc)


def orthrus_consensus_workspace_size(B: int, K: int, V: int) -> int:
    return int(lib().orthrus_consensus_workspace_size(B, K, V))


def orthrus_consensus(logits: torch.Tensor, proposed: torch.Tensor, accepted_len: torch.Tensor,
                      next_token: torch.Tensor, workspace: torch.Tensor,
                      argmax_out: Optional[torch.Tensor] = None,
                      status: Optional[torch.Tensor] = None, stream=None) -> None:
    """logits [B,K,V] fp32, proposed [B,K] int32 -> accepted_len [B], next_token [B]."""
    B, K, V = logits.shape
    assert logits.dtype == torch.float32 and proposed.dtype == torch.int32
    rc = lib().orthrus_consensus(_ptr(logits), _ptr(proposed), B, K, V, _ptr(accepted_len),
                                 _ptr(next_token), _ptr(argmax_out), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(),
                                 _ptr(status), _stream(stream))
    _check("orthrus_consensus", rc)


def _ptr_array(ts):
    """(void*, keep-alive) for a host array of device pointers, or (None, None)."""
    if ts is None:
        return None, None
    a = (ctypes.c_void_p * len(ts))(*[t.data_ptr() for t in ts])
    return ctypes.cast(a, ctypes.c_void_p), a


def orthrus_attn_path(B: int, Hq: int, Hkv: int, D: int, K: int,
                      dtype: torch.dtype = torch.bfloat16) -> int:
    """1 = tensor-core path, 0 = CUDA-core path (negative: error code)."""
    return int(lib().orthrus_attn_path(B, Hq, Hkv, D, K, _dtype_code(dtype)))


def orthrus_write_block(ctx_lens: torch.Tensor, k_caches: Sequence[torch.Tensor],
                        v_caches: Sequence[torch.Tensor], k_blks: Sequence[torch.Tensor],
                        v_blks: Sequence[torch.Tensor], status: Optional[torch.Tensor] = None,
                        stream=None) -> None:
    """Copy each layer's block K/V [B,K,Hkv,D] into cache rows [ctx, ctx+K)."""
    B, Hkv, S_max, D = k_caches[0].shape
    K = k_blks[0].shape[1]
    packs = [_ptr_array(x) for x in (k_caches, v_caches, k_blks, v_blks)]
    rc = lib().orthrus_write_block(len(k_caches), *[p[0] for p in packs], _ptr(ctx_lens), B, Hkv,
                                   D, S_max, K, _dtype_code(k_caches[0].dtype), _ptr(status),
                                   _stream(stream))
    _check("orthrus_write_block", rc)


def orthrus_kv_commit(ctx_lens: torch.Tensor, accepted_len: torch.Tensor, *, K: int, Hkv: int,
                      D: int, S_max: int, dtype: torch.dtype = torch.bfloat16,
                      num_layers: int = 1,
                      k_caches: Optional[Sequence[torch.Tensor]] = None,
                      v_caches: Optional[Sequence[torch.Tensor]] = None,
                      k_blks: Optional[Sequence[torch.Tensor]] = None,
                      v_blks: Optional[Sequence[torch.Tensor]] = None,
                      status: Optional[torch.Tensor] = None, stream=None) -> None:
    """Commit min(a+1, K) block slots (copying from staging when k_blks is given)
    and advance ctx_lens once."""
    B = ctx_lens.shape[0]
    packs = [_ptr_array(x) for x in (k_caches, v_caches, k_blks, v_blks)]
    if k_blks is not None:
        num_layers = len(k_blks)
    rc = lib().orthrus_kv_commit(num_layers, *[p[0] for p in packs],
                                 _ptr(ctx_lens), _ptr(accepted_len), B, Hkv, D, S_max, K,
                                 _dtype_code(dtype), _ptr(status), _stream(stream))
    _check("orthrus_kv_commit", rc)


def orthrus_lm_head_workspace_size(B: int, K: int) -> int:
    return int(lib().orthrus_lm_head_workspace_size(B, K))


def orthrus_lm_head_consensus(hidden: torch.Tensor, lm_head: torch.Tensor, proposed: torch.Tensor,
                              accepted_len: torch.Tensor, next_token: torch.Tensor,
                              workspace: torch.Tensor, argmax_out: Optional[torch.Tensor] = None,
                              status: Optional[torch.Tensor] = None, stream=None) -> None:
    """hidden [B,K,Hd] bf16, lm_head [V,Hd] bf16, proposed [B,K] int32 ->
    accepted_len [B], next_token [B] (the logits are never materialised)."""
    B, K, Hd = hidden.shape
    V = lm_head.shape[0]
    assert hidden.dtype == torch.bfloat16 and lm_head.dtype == torch.bfloat16
    assert proposed.dtype == torch.int32 and lm_head.shape[1] == Hd
    rc = lib().orthrus_lm_head_consensus(_ptr(hidden), _ptr(lm_head), _ptr(proposed), B, K, V, Hd,
                                         _ptr(accepted_len), _ptr(next_token), _ptr(argmax_out),
                                         _ptr(workspace), workspace.numel() * workspace.element_size(),
                                         _ptr(status), _stream(stream))
    _check("orthrus_lm_head_consensus", rc)


def orthrus_rejection_workspace_size(B: int, K: int, V: int) -> int:
    return int(lib().orthrus_rejection_workspace_size(B, K, V))


def orthrus_rejection_verify(ar_logits: torch.Tensor, draft_logits: torch.Tensor,
                             proposed: torch.Tensor, u_accept: torch.Tensor, u_resample: torch.Tensor,
                             temperature: float, accepted_len: torch.Tensor, next_token: torch.Tensor,
                             workspace: torch.Tensor, status: Optional[torch.Tensor] = None,
                             stream=None) -> None:
    """Logits [B,K,V] fp32 of both views, proposals [B,K] int32, uniform draws
    u_accept [B,K] and u_resample [B] fp32 -> accepted_len [B], next_token [B]."""
    B, K, V = ar_logits.shape
    assert ar_logits.dtype == torch.float32 and draft_logits.dtype == torch.float32
    assert draft_logits.shape == ar_logits.shape and proposed.dtype == torch.int32
    assert u_accept.dtype == torch.float32 and u_resample.dtype == torch.float32
    rc = lib().orthrus_rejection_verify(_ptr(ar_logits), _ptr(draft_logits), _ptr(proposed),
                                        _ptr(u_accept), _ptr(u_resample), float(temperature), B, K, V,
                                        _ptr(accepted_len), _ptr(next_token), _ptr(workspace),
                                        workspace.numel() * workspace.element_size(), _ptr(status),
                                        _stream(stream))
    _check("orthrus_rejection_verify", rc)


def orthrus_qkv_workspace_size(B: int, K: int, hidden: int, Hq: int, Hkv: int, D: int) -> int:
    return int(lib().orthrus_qkv_workspace_size(B, K, hidden, Hq, Hkv, D))


def orthrus_qkv_project(x: torch.Tensor, w_q: torch.Tensor, w_k: torch.Tensor, w_v: torch.Tensor,
                        ctx_lens: torch.Tensor, q_out: torch.Tensor, k_cache: torch.Tensor,
                        v_cache: torch.Tensor, workspace: torch.Tensor,
                        status: Optional[torch.Tensor] = None, stream=None) -> None:
    """x [B,K,hidden] bf16, weights [features, hidden] bf16 -> q_out [B,K,Hq,D]
    and cache rows [ctx, ctx+K) of k_cache / v_cache [B,Hkv,S_max,D] (bf16)."""
    B, K, hidden = x.shape
    _, Hkv, S_max, D = k_cache.shape
    Hq = q_out.shape[2]
    for t in (x, w_q, w_k, w_v, q_out, k_cache, v_cache):
        assert t.dtype == torch.bfloat16
    assert ctx_lens.dtype == torch.int32 and w_q.shape == (Hq * D, hidden)
    assert w_k.shape == (Hkv * D, hidden) and w_v.shape == (Hkv * D, hidden)
    rc = lib().orthrus_qkv_project(_ptr(x), _ptr(w_q), _ptr(w_k), _ptr(w_v), _ptr(ctx_lens), B, K,
                                   hidden, Hq, Hkv, D, S_max, _ptr(q_out), _ptr(k_cache),
                                   _ptr(v_cache), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _ptr(status),
                                   _stream(stream))
    _check("orthrus_qkv_project", rc)


def orthrus_prefill_workspace_size(B: int, S: int, Hq: int, Hkv: int, D: int,
                                   dtype: torch.dtype = torch.bfloat16) -> int:
    return int(lib().orthrus_prefill_workspace_size(B, S, Hq, Hkv, D, _dtype_code(dtype)))


def orthrus_prefill_attn(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                         out: torch.Tensor, workspace: torch.Tensor, status: Optional[torch.Tensor] = None,
                         scale: float = 0.0, stream=None) -> None:
    """Causal attention over the prompt: q [B,S,Hq,D], caches [B,Hkv,S_max,D]
    (rows [0, S) = the prompt) -> out [B,S,Hq,D] fp32."""
    B, S, Hq, D = q.shape
    _, Hkv, S_max, _ = k_cache.shape
    assert out.dtype == torch.float32 and out.shape == q.shape
    rc = lib().orthrus_prefill_attn(_dtype_code(q.dtype), _ptr(q), _ptr(k_cache), _ptr(v_cache), B, S, Hq,
                                    Hkv, D, S_max, float(scale), _ptr(out), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _ptr(status),
                                    _stream(stream))
    _check("orthrus_prefill_attn", rc)
