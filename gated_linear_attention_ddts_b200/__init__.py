"""B200-native DDTS-gated linear-attention recurrence (Rodimus).

    alpha_t = exp(-g_t*tau_t), alpha_hat_t = g_t^tau_t
    S_t = diag(alpha_t) S_{t-1} + (alpha_hat_t*k_t)(beta_hat_t*v_t)^T,  o_t = S_t^T q_t

The computation lives in librdm_ddts.so (CUDA, sm_100a; C ABI in
include/rdm_ddts.h).  This package is its Python binding: same entry-point
names, torch tensors for device memory and streams.
"""
from ._binding import (IMPL, RDM_BF16, RDM_ERR_CUDA, RDM_ERR_INVALID_ARG, RDM_ERR_TIMEOUT,
                       RDM_ERR_UNSUPPORTED, RDM_ERR_WORKSPACE, RDM_F32, RDM_OK, RdmError,
                       rdm_ddts_bwd, rdm_ddts_bwd_noalloc, rdm_ddts_bwd_workspace_size, rdm_ddts_decode, rdm_ddts_decode_step,
                       rdm_ddts_fwd, rdm_ddts_fwd_workspace_size, rdm_ddts_saved_states_size,
                       rdm_ddts_set_test_hooks, rdm_ddts_sync_status,
                       rdm_ddts_version, rdm_shortconv_bwd, rdm_shortconv_bwd_many, rdm_shortconv_fwd,
                       rdm_shortconv_fwd_many, rdm_ska_decode, rdm_ska_fwd, rdm_status_string)

__all__ = ["rdm_ddts_fwd", "rdm_ddts_fwd_workspace_size", "rdm_ddts_bwd", "rdm_ddts_bwd_noalloc", "rdm_ddts_bwd_workspace_size",
           "rdm_ddts_saved_states_size", "rdm_ddts_decode", "rdm_ddts_decode_step", "rdm_ddts_sync_status",
           "rdm_status_string", "rdm_ddts_set_test_hooks", "rdm_ddts_version", "rdm_shortconv_fwd",
           "rdm_shortconv_bwd", "rdm_shortconv_fwd_many", "rdm_shortconv_bwd_many", "rdm_ska_fwd",
           "rdm_ska_decode", "RdmError", "IMPL", "RDM_OK",
           "RDM_ERR_INVALID_ARG", "RDM_ERR_UNSUPPORTED", "RDM_ERR_CUDA", "RDM_ERR_TIMEOUT",
           "RDM_ERR_WORKSPACE", "RDM_F32", "RDM_BF16"]
