"""B200 (sm_100a) library for the GuidedQuant + LNQ hot path: guided Fisher blocks and per-row
layer-wise non-uniform quantisation, behind the C ABI in include/lnq.h."""
from .binding import (LNQ_OP_BUILD_FISHER, LNQ_OP_INIT_CODEBOOK, LNQ_OP_OBJECTIVE,  # noqa: F401
                      LNQ_OP_QUANTIZE_ROWS, LnqError, lnq_build_fisher, lnq_init_codebook,
                      lnq_objective, lnq_quantize_rows, lnq_set_wait_limit, lnq_status_string,
                      lnq_workspace_check, lnq_workspace_size, lnq_packed_words,
                      lnq_pack_codes, lnq_lut_gemv, lnq_quantize_rows_diag,
                      lnq_sweep_counters, lnq_fp32_probe, lnq_build_fisher_noalloc,
                      lnq_noalloc_check, lnq_ganq_rows, LNQ_OP_GANQ_ROWS, LNQ_ROW_NOT_PD)
