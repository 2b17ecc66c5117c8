"""B200 (sm_100a) VSA tile-sparse attention layer for reference-to-video.

The compute path lives in ``libvsa.so`` (C ABI, ``include/vsa.h``); this
package holds its ctypes binding (``vsa``), the in-tree build (``build``) and
the seeded synthetic workloads (``inputs``).
"""
from .vsa import (EXPORTS, Layer, Plan, VsaError, lib, vsa_coarse_topk,  # noqa: F401
                  vsa_gate_combine, vsa_permute, vsa_plan, vsa_sparse_attn, vsa_sparse_attn_combine,
                  vsa_sync_status,
                  vsa_unpermute)
