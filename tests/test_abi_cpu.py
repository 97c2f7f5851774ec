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


def test_device_status_is_a_per_call_word():
    """Every entry point that enqueues device work takes the caller's status
    word; the library keeps no global status (there is no get-status call),
    and no entry point takes a host-side context-length hint (the work split
    is computed on the device from ctx_lens)."""
    src = open(os.path.join(ROOT, "include", "orthrus.h")).read()
    decls = dict(re.findall(r"ORTHRUS_API\s+[\w\s\*]*?\b(orthrus_\w+)\s*\(([^;]*)\);", src))
    for name in ("orthrus_attn", "orthrus_attn_static", "orthrus_consensus",
                 "orthrus_kv_commit", "orthrus_write_block"):
        assert re.search(r"int32_t\s*\*\s*status", decls[name]), name
        assert "hint" not in decls[name], name
    assert not any("status" in n for n in decls), sorted(decls)
