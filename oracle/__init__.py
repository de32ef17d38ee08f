"""CPU oracle for the Sparse-BitLinear forward (test infrastructure only).

Imported by the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg; never by the library itself.
"""
from .sbl_oracle import *  # noqa: F401,F403
from .sbl_oracle import (SUPPORTED_NM, acc_entries, dequant, global_scale, int_contract, linear,  # noqa: F401
                         mask_monitor, nm_mask,
                         pack_codes, pack_mask_bits, prepare_weights, quant_act, rms_sumsq, rmsnorm,
                         rmsnorm_quant_act, round_to_bf16, row_scale, ste_backward, ternarise, unpack_codes)
