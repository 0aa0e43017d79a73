"""libgdn: the Gated DeltaNet gated delta rule (prefill + decode) and the QSA compressed
indexer on one B200.

The compute lives in libgdn.so (CUDA C++ for sm_100a behind the C ABI in
include/gdn.h); this package is its ctypes binding plus the seeded input
generators used by the tests and the bench.
"""
from ._binding import (GDN_BF16, GDN_ERR_CUDA, GDN_ERR_INVALID_ARG, GDN_ERR_TIMEOUT,
                       GDN_ERR_UNSUPPORTED, GDN_F32, GDN_FLAG_FORCE_CUDA_CORE,
                       GDN_FLAG_GATE_LOGITS, GDN_FLAG_QK_L2NORM, GDN_OK, EXPORTED, GdnError, gdn_backward, gdn_decode_multi,
                       gdn_decode_step,
                       gdn_get_device_error, gdn_prefill, gdn_prefill_static_scratch,
                       gdn_prefill_workspace_size, gdn_set_prefill_segment_tokens,
                       gdn_set_wait_budget, gdn_prefill_schedule,
                       gdn_status_string, lib, prefill_workspace, gdn_qsa_compress,
                       gdn_qsa_index_decode, gdn_qsa_index_workspace_size, qsa_index_workspace,
                       gdn_qsa_index_multi, gdn_qsa_index_multi_workspace_size,
                       qsa_index_multi_workspace)

__all__ = [
    "gdn_prefill", "gdn_prefill_static_scratch", "gdn_decode_step", "gdn_decode_multi", "gdn_backward", "gdn_get_device_error", "gdn_prefill_workspace_size",
    "gdn_status_string", "prefill_workspace", "GdnError", "lib", "EXPORTED", "GDN_OK",
    "GDN_ERR_INVALID_ARG", "GDN_ERR_UNSUPPORTED", "GDN_ERR_CUDA", "GDN_ERR_TIMEOUT", "GDN_F32",
    "GDN_BF16", "GDN_FLAG_QK_L2NORM", "GDN_FLAG_FORCE_CUDA_CORE", "GDN_FLAG_GATE_LOGITS",
    "gdn_qsa_compress", "gdn_qsa_index_decode", "gdn_qsa_index_workspace_size",
    "qsa_index_workspace", "gdn_qsa_index_multi", "gdn_qsa_index_multi_workspace_size",
    "qsa_index_multi_workspace", "gdn_set_prefill_segment_tokens", "gdn_set_wait_budget",
    "gdn_prefill_schedule",
]
