"""B200-native (sm_100a) hot path of the Orthrus dual-view diffusion decode step.

The compute lives in ``liborthrus.so`` (C ABI, include/orthrus.h); this package
holds its ctypes binding (``binding``), the in-tree build (``build``), the
seeded synthetic workloads (``workloads``) and a device-resident decode-step
driver (``step``).
"""
from .binding import (AR, BF16, DIFF, F32, OrthrusError, orthrus_attn,  # noqa: F401
                      orthrus_attn_path, orthrus_attn_workspace_size, orthrus_consensus,
                      orthrus_consensus_workspace_size, orthrus_kv_commit,
                      orthrus_version, orthrus_write_block)
