"""fp64 CPU oracle for the VSA tile-sparse attention layer.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, the smoke check and the
benchmark's CPU-baseline leg, never by the product package.
"""
from .vsa_oracle import (Plan, plan, keep_count, keep_count_ref, permute, unpermute,  # noqa: F401
                         pool, coarse_attention, select_topk, select_topk_ref, key_tiles,
                         fine_tile, fine,
                         sigmoid, gate_combine, project, layer,
                         gate_combine_backward, softmax_backward, fine_tile_backward,
                         fine_backward, coarse_attention_backward, pool_backward, layer_backward)
