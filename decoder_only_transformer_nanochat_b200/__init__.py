"""B200-native forward + backward of the nanochat decoder behind a C ABI.

`libnanochat_b200.so` (built from csrc/ by `build.py`) holds every kernel;
this package is its thin Python binding.  `Model` adds PyTorch-owned device
memory and streams on top.
"""
from ._binding import (NC_BF16, NC_EALIGN, NC_ECUDA, NC_EINVAL, NC_ENOMEM,  # noqa: F401
                       NC_ENONFINITE, NC_ERANGE, NC_ESHAPE, NC_ETIMEOUT, NC_EUNSUPPORTED, NC_F32,
                       NC_OK, LIB_PATH, NcError, load_library, nc_destroy, nc_fwd, nc_fwd_bwd,
                       nc_get_dims, nc_init, nc_param_layout, nc_strerror, nc_sync_status,
                       nc_workspace_bytes, nc_gemm, nc_attention_fwd, nc_attention_bwd,
                       NC_EPI_STORE, NC_EPI_STORE_F32, NC_EPI_ADD, NC_EPI_RELU2, NC_EPI_DRELU2,
                       NC_EPI_SOFTCAP, nc_profile, nc_profile_read,
                       nc_attention_bwd_noalloc, NC_ATTN_BWD_NOALLOC_MAX_ROWS, nc_ops_status,
                       nc_check_wait_expiry, nc_softcap_ce, nc_init_ex, nc_layer_window,
                       nc_param_count, nc_fwd_bwd_ex, nc_grad_buckets, nc_set_grad_events,
                       NC_ACCUMULATE, nc_kv_cache_bytes, nc_prefill, nc_decode, nc_optim_state_bytes,
                       nc_optim_workspace_bytes, nc_optim_init, nc_optim_step, nc_rmsnorm, nc_rmsnorm_bwd,
                       nc_rope_qknorm, nc_rope_qknorm_bwd, nc_attention_bwd_scratch_bytes, nc_attention_bwd_ex,
                       nc_set_attention_ctas)


def __getattr__(name):
    if name == "Model":
        from .model import Model
        return Model
    raise AttributeError(name)
