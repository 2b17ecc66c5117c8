"""fp64 CPU oracle for the VSA tile-sparse attention layer.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, the smoke check and the
benchmark's CPU-baseline leg, never by the product package.
"""
from .vsa_oracle import (Plan, plan, keep_count, permute, unpermute, pool,  # noqa: F401
                         coarse_attention, select_topk, key_tiles, fine_tile, fine,
                         sigmoid, gate_combine, project, layer)
