"""B200-native (sm_100a) Stem block-sparse prefill: OAM scoring, TPD selection, block-sparse
causal attention.  The kernels and the C ABI live in libbsa.so (``build.build()`` compiles
it in-tree); this package exposes the ABI's entry points through ``binding``."""
from .binding import (BSA_BF16, BSA_FP8_E4M3, BSA_FP32, BSA_METRIC_OAM, BSA_METRIC_OAM_MUL, BSA_METRIC_SAM,
                      BsaError, block_mask_buffer, bsa_check_device_error, bsa_mask_to_lists,
                      bsa_mask_workspace_bytes, bsa_prefill, bsa_prefill_group, bsa_prefill_mask, bsa_prefill_paged,
                      bsa_prefill_paged_group,
                      bsa_prefill_skip,
                      bsa_score_group_workspace_bytes, bsa_score_workspace_bytes, bsa_selftest_wait_timeout,
                      bsa_score_select_workspace_bytes, bsa_tpd_budget, bsa_validate_lists, stem_score, stem_score_group,
                      stem_score_noalloc, stem_score_select,
                      stem_select)

__all__ = ["stem_score", "stem_select", "stem_score_select", "bsa_score_select_workspace_bytes", "bsa_prefill", "bsa_prefill_paged", "bsa_prefill_paged_group", "bsa_prefill_mask",
           "stem_score_group", "bsa_prefill_group", "bsa_score_group_workspace_bytes", "bsa_prefill_skip",
           "bsa_mask_to_lists", "bsa_mask_workspace_bytes", "block_mask_buffer", "bsa_validate_lists", "bsa_tpd_budget",
           "bsa_score_workspace_bytes", "bsa_check_device_error", "bsa_selftest_wait_timeout", "stem_score_noalloc",
           "BsaError", "BSA_BF16", "BSA_FP8_E4M3",
           "BSA_FP32", "BSA_METRIC_OAM", "BSA_METRIC_SAM", "BSA_METRIC_OAM_MUL"]
