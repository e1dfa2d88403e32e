"""Test infrastructure only: the plain fp64 CPU oracle for trellis-coded quantization.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never does: the product
path fails loudly when its extension is missing instead of falling back here.
"""
from .tcq_oracle import (  # noqa: F401
    oracle_bcjr,
    build_oracle,
    oracle_decode,
    oracle_encode,
    oracle_encode_vec,
    oracle_decode_vec,
    oracle_feedback_targets,
    oracle_gemv,
    oracle_greedy,
    oracle_ldlq,
    oracle_mad_codebook,
    oracle_path_cost,
    oracle_ub8_decode,
    oracle_ub8_encode,
    oracle_words_per_block,
)
