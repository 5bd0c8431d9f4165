"""CPU fp64 oracle of Thinformer / Thinformer Express attention.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU legs of ``bench.py``.  The CUDA library never imports it and the
two share no code.
"""
from .thin_oracle import (  # noqa: F401
    NEAR_TIE_REL, HalvingOut, OracleOut, Stats, compress_sizes, exact_attention, express, express_a,
    express_a_layout, express_a_sizes, express_layout, kappa_att, kernel_halving, kh_compress, philox4x32_10, philox_uniform,
    philox_word, round_batch, round_merge, round_noncausal, round_subsample, snapshot_nodes,
    subsample_indices, thinformer, weighted_attention)
