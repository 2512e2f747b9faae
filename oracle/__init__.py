"""CPU oracle for the weight-quantised GEMM (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs may import this package. The CUDA library never does.
"""
from .qgemm_oracle import *  # noqa: F401,F403
from .qgemm_oracle import (  # noqa: F401
    pack_ref, unpack_codes, pack_codes, dequant_ref, dequant_ref_bits, wq_exact,
    qgemm_ref, qgemm_ref_bf16w, qgemm_ref_rows, dense_ref, fp16_rn, bf16_rn_bits,
    bf16_bits_to_f64, rel_frobenius, max_abs_rel, cosine, within_tolerance,
    REL_FROB_TOL, MAX_ABS_TOL, code_bit_position, codes_per_word, format_bytes,
)
