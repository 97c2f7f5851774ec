"""The C-ABI library loads without a GPU and exports exactly what
include/orthrus.h declares; host-side argument checks reject bad calls before
touching the device."""
import ctypes
import os
import re

import pytest

from lossless_diffusion_speculative_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"ORTHRUS_API\s+[\w\s\*]*?\b(orthrus_\w+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.lib()


def test_header_declares_the_entry_points():
    assert set(binding.EXPORTED) <= _declared()


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_no_internal_symbols_leak():
    out = os.popen(f"nm -D --defined-only {build.LIB}").read()
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert exported == _declared()


def test_version_and_error_strings(lib):
    assert binding.orthrus_version() >> 16 == 1
    for code in (0, -1, -2, -3, -4, -5, -6, -99):
        assert lib.orthrus_error_string(code)


def test_host_checks_reject_bad_arguments_without_a_device(lib):
    vp = ctypes.c_void_p
    # NULL q
    assert lib.orthrus_attn(0, 0, None, vp(16), vp(16), vp(16), 1, 4, 2, 128, 64, 8, 0.0,
                            vp(16), vp(16), 1 << 20, None, None) == binding.ERR_ARG
    # bad view
    assert lib.orthrus_attn(7, 0, vp(16), vp(16), vp(16), vp(16), 1, 4, 2, 128, 64, 8, 0.0,
                            vp(16), vp(16), 1 << 20, None, None) == binding.ERR_ARG
    # Hq not a multiple of Hkv
    assert lib.orthrus_attn(0, 0, vp(16), vp(16), vp(16), vp(16), 1, 5, 2, 128, 64, 8, 0.0,
                            vp(16), vp(16), 1 << 20, None, None) == binding.ERR_ARG
    # K > S_max
    assert lib.orthrus_attn(0, 0, vp(16), vp(16), vp(16), vp(16), 1, 4, 2, 128, 4, 8, 0.0,
                            vp(16), vp(16), 1 << 20, None, None) == binding.ERR_ARG
    # head_dim not a multiple of 32
    assert lib.orthrus_attn(0, 0, vp(16), vp(16), vp(16), vp(16), 1, 4, 2, 100, 64, 8, 0.0,
                            vp(16), vp(16), 1 << 20, None, None) == binding.ERR_UNSUPPORTED
    # misaligned q
    assert lib.orthrus_attn(0, 0, vp(18), vp(16), vp(16), vp(16), 1, 4, 2, 128, 64, 8, 0.0,
                            vp(16), vp(16), 1 << 20, None, None) == binding.ERR_ALIGN
    # consensus: K too large, NULL logits
    assert lib.orthrus_consensus(vp(16), vp(16), 1, 1000, 10, vp(16), vp(16), None, vp(16),
                                 1 << 20, None, None) == binding.ERR_UNSUPPORTED
    assert lib.orthrus_consensus(None, vp(16), 1, 8, 10, vp(16), vp(16), None, vp(16),
                                 1 << 20, None, None) == binding.ERR_ARG
    # commit: too many layers, NULL ctx
    assert lib.orthrus_kv_commit(1000, None, None, None, None, vp(16), vp(16), 1, 8, 128, 64,
                                 8, 0, None, None) == binding.ERR_UNSUPPORTED
    assert lib.orthrus_kv_commit(1, None, None, None, None, None, vp(16), 1, 8, 128, 64, 8, 0,
                                 None, None) == binding.ERR_ARG


def test_host_checks_of_the_next_rows_without_a_device(lib):
    """The fused LM head, rejection verification, QKV projection and prefill
    reject bad arguments on the host, before any device call."""
    vp = ctypes.c_void_p
    ok = vp(16)
    # LM head: NULL hidden; hidden size not a multiple of 64; more than 512 token rows;
    # misaligned weight; workspace too small
    assert lib.orthrus_lm_head_consensus(None, ok, ok, 1, 8, 100, 64, ok, ok, None, ok, 1 << 20,
                                         None, None) == binding.ERR_ARG
    assert lib.orthrus_lm_head_consensus(ok, ok, ok, 1, 8, 100, 100, ok, ok, None, ok, 1 << 20,
                                         None, None) == binding.ERR_UNSUPPORTED
    assert lib.orthrus_lm_head_consensus(ok, ok, ok, 32, 32, 100, 64, ok, ok, None, ok, 1 << 20,
                                         None, None) == binding.ERR_UNSUPPORTED
    assert lib.orthrus_lm_head_consensus(ok, vp(24), ok, 1, 8, 100, 64, ok, ok, None, ok, 1 << 20,
                                         None, None) == binding.ERR_ALIGN
    assert lib.orthrus_lm_head_consensus(ok, ok, ok, 1, 8, 100, 64, ok, ok, None, ok, 8,
                                         None, None) == binding.ERR_WORKSPACE
    assert lib.orthrus_lm_head_workspace_size(1, 32) >= 32 * 8 + 4
    assert lib.orthrus_lm_head_workspace_size(0, 32) == 0 and lib.orthrus_lm_head_workspace_size(32, 32) == 0
    # rejection: NULL draws; temperature <= 0; K above the block limit; misaligned logits
    assert lib.orthrus_rejection_verify(ok, ok, ok, None, ok, 1.0, 1, 8, 100, ok, ok, ok, 1 << 20,
                                        None, None) == binding.ERR_ARG
    assert lib.orthrus_rejection_verify(ok, ok, ok, ok, ok, 0.0, 1, 8, 100, ok, ok, ok, 1 << 20,
                                        None, None) == binding.ERR_ARG
    assert lib.orthrus_rejection_verify(ok, ok, ok, ok, ok, 1.0, 1, 200, 100, ok, ok, ok, 1 << 20,
                                        None, None) == binding.ERR_UNSUPPORTED
    assert lib.orthrus_rejection_verify(vp(20), ok, ok, ok, ok, 1.0, 1, 8, 100, ok, ok, ok, 1 << 20,
                                        None, None) == binding.ERR_ALIGN
    assert lib.orthrus_rejection_workspace_size(1, 200, 100) == 0
    # QKV projection: NULL cache; hidden not a multiple of 64; D not a multiple of 16;
    # Hq not a multiple of Hkv; misaligned x
    assert lib.orthrus_qkv_project(ok, ok, ok, ok, ok, 1, 8, 256, 8, 2, 128, 64, ok, None, ok, ok,
                                   1 << 20, None, None) == binding.ERR_ARG
    assert lib.orthrus_qkv_project(ok, ok, ok, ok, ok, 1, 8, 250, 8, 2, 128, 64, ok, ok, ok, ok,
                                   1 << 20, None, None) == binding.ERR_UNSUPPORTED
    assert lib.orthrus_qkv_project(ok, ok, ok, ok, ok, 1, 8, 256, 8, 2, 100, 64, ok, ok, ok, ok,
                                   1 << 20, None, None) == binding.ERR_UNSUPPORTED
    assert lib.orthrus_qkv_project(ok, ok, ok, ok, ok, 1, 8, 256, 9, 2, 128, 64, ok, ok, ok, ok,
                                   1 << 20, None, None) == binding.ERR_UNSUPPORTED
    assert lib.orthrus_qkv_project(vp(18), ok, ok, ok, ok, 1, 8, 256, 8, 2, 128, 64, ok, ok, ok, ok,
                                   1 << 20, None, None) == binding.ERR_ALIGN
    assert lib.orthrus_qkv_workspace_size(1, 8, 250, 8, 2, 128) == 0
    # prefill: NULL q; prompt longer than the cache; Hq not a multiple of Hkv
    assert lib.orthrus_prefill_attn(0, None, ok, ok, 1, 64, 8, 2, 128, 128, 0.0, ok, ok, 1 << 20,
                                    None, None) == binding.ERR_ARG
    assert lib.orthrus_prefill_attn(0, ok, ok, ok, 1, 200, 8, 2, 128, 128, 0.0, ok, ok, 1 << 20,
                                    None, None) == binding.ERR_ARG
    assert lib.orthrus_prefill_attn(0, ok, ok, ok, 1, 64, 9, 2, 128, 128, 0.0, ok, ok, 1 << 20,
                                    None, None) == binding.ERR_ARG
    assert lib.orthrus_prefill_workspace_size(1, 64, 9, 2, 128, 0) == 0


def test_device_status_is_a_per_call_word():
    """Every entry point that enqueues device work takes the caller's status
    word; the library keeps no global status (there is no get-status call),
    and no entry point takes a host-side context-length hint (the work split
    is computed on the device from ctx_lens)."""
    src = open(os.path.join(ROOT, "include", "orthrus.h")).read()
    decls = dict(re.findall(r"ORTHRUS_API\s+[\w\s\*]*?\b(orthrus_\w+)\s*\(([^;]*)\);", src))
    for name in ("orthrus_attn", "orthrus_attn_static", "orthrus_consensus",
                 "orthrus_kv_commit", "orthrus_write_block", "orthrus_lm_head_consensus",
                 "orthrus_rejection_verify", "orthrus_qkv_project", "orthrus_prefill_attn"):
        assert re.search(r"int32_t\s*\*\s*status", decls[name]), name
        assert "hint" not in decls[name], name
    assert not any("status" in n for n in decls), sorted(decls)
