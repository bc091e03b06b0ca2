"""ctypes binding of libnanochat_b200.so, one Python function per C entry point.

Argument marshalling only: every step of the decoder computation runs in the
library's CUDA kernels.  Device buffers are passed as integer addresses and the
stream as an integer cudaStream_t.  If the shared library has not been built
the first call raises, naming the build step; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnanochat_b200.so")

NC_OK = 0
NC_EINVAL = 1
NC_ESHAPE = 2
NC_ENOMEM = 3
NC_EUNSUPPORTED = 4
NC_ECUDA = 5
NC_ERANGE = 6
NC_ENONFINITE = 7
NC_ETIMEOUT = 8
NC_EALIGN = 9

NC_F32 = 0
NC_BF16 = 1

NC_ACCUMULATE = 1


class NcError(RuntimeError):
    def __init__(self, code: int, where: str = ""):
        self.code = code
        super().__init__(f"{where}: {nc_strerror(code)} (status {code})")


class nc_dims(ctypes.Structure):
    _fields_ = [("depth", ctypes.c_int), ("width", ctypes.c_int), ("n_head", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("hidden", ctypes.c_int), ("vocab", ctypes.c_int),
                ("seq", ctypes.c_int), ("dtype", ctypes.c_int), ("n_params", ctypes.c_int64)]


class nc_param(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 24), ("offset", ctypes.c_int64),
                ("rows", ctypes.c_int), ("cols", ctypes.c_int)]


class nc_kernel_stat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 24), ("launches", ctypes.c_int64), ("ms", ctypes.c_double),
                ("flops", ctypes.c_double), ("bytes", ctypes.c_double)]


_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_SIGS = {
    "nc_init": (_I, [_I, _I, _I, _I, ctypes.POINTER(_P)]),
    "nc_get_dims": (_I, [_P, ctypes.POINTER(nc_dims)]),
    "nc_param_layout": (_I, [_P, _I, ctypes.POINTER(nc_param)]),
    "nc_workspace_bytes": (_I, [_P, _I, _I, ctypes.POINTER(ctypes.c_size_t)]),
    "nc_fwd_bwd": (_I, [_P, _P, _P, _P, _I, _I, _P, ctypes.c_size_t, _P, _P, _P, _P]),
    "nc_fwd": (_I, [_P, _P, _P, _I, _I, _P, ctypes.c_size_t, _P, _P]),
    "nc_sync_status": (_I, [_P, _P, _I]),
    "nc_strerror": (ctypes.c_char_p, [_I]),
    "nc_destroy": (None, [_P]),
    "nc_attention_bwd_noalloc": (_I, [_P, ctypes.c_int64, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "nc_profile": (_I, [_P, _I]),
    "nc_profile_read": (_I, [_P, ctypes.POINTER(nc_kernel_stat), _I, ctypes.POINTER(_I)]),
    "nc_gemm": (_I, [_P, ctypes.c_int64, _I, _P, ctypes.c_int64, _I, _P, ctypes.c_int64, _I, _I, _I,
                     _I, _I, _I, _P]),
    "nc_attention_fwd": (_I, [_P, ctypes.c_int64, _P, _P, _I, _I, _I, _I, _I, _I, _P]),
    "nc_attention_bwd": (_I, [_P, ctypes.c_int64, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P]),
    "nc_init_ex": (_I, [_I, _I, _I, _I, _P, ctypes.POINTER(_P)]),
    "nc_layer_window": (_I, [_P, _I, ctypes.POINTER(_I)]),
    "nc_param_count": (_I, [_P, ctypes.POINTER(_I)]),
    "nc_fwd_bwd_ex": (_I, [_P, _P, _P, _P, _I, _I, _P, ctypes.c_size_t, _P, _P, _P, _I, _P]),
    "nc_grad_bucket_count": (_I, [_P, ctypes.POINTER(_I)]),
    "nc_grad_bucket": (_I, [_P, _I, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64)]),
    "nc_set_grad_events": (_I, [_P, ctypes.POINTER(_P), _I]),
    "nc_kv_cache_bytes": (_I, [_P, _I, _I, ctypes.POINTER(ctypes.c_size_t)]),
    "nc_optim_state_bytes": (_I, [_P, ctypes.POINTER(ctypes.c_size_t)]),
    "nc_optim_workspace_bytes": (_I, [_P, ctypes.POINTER(ctypes.c_size_t)]),
    "nc_optim_init": (_I, [_P, _P, _P, _P]),
    "nc_optim_step": (_I, [_P, _P, _P, _P, _I, _P, _P, ctypes.c_size_t, _P]),
    "nc_prefill": (_I, [_P, _P, _P, _I, _I, _P, _I, _P, _P, ctypes.c_size_t, _P, _P]),
    "nc_decode": (_I, [_P, _P, _P, _I, _P, _I, _P, _P, ctypes.c_size_t, _P, _P]),
    "nc_ops_status": (_I, [_P, _I]),
    "nc_softcap_ce": (_I, [_P, ctypes.c_int64, _P, _P, _I, _I, ctypes.c_float, _I, _P]),
    "nc_check_wait_expiry": (_I, [_I, _P]),
    "nc_attention_bwd_scratch_bytes": (_I, [_I, _I, _I, _I, ctypes.POINTER(ctypes.c_size_t)]),
    "nc_attention_bwd_ex": (_I, [_P, ctypes.c_int64, _P, _P, _P, _P, _P, ctypes.c_size_t, _P, _I, _I, _I, _I,
                                 _I, _I, _P]),
    "nc_set_attention_ctas": (_I, [_I]),
    "nc_rmsnorm": (_I, [_P, _P, _P, _I, _I, _I, _P]),
    "nc_rmsnorm_bwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "nc_rope_qknorm": (_I, [_P, _P, ctypes.c_int64, _P, _P, _I, _I, _P]),
    "nc_rope_qknorm_bwd": (_I, [_P, _P, _P, ctypes.c_int64, _P, _P, _I, _I, _P]),
}

NC_EPI_STORE = 0
NC_EPI_STORE_F32 = 1
NC_EPI_ADD = 2
NC_EPI_RELU2 = 3
NC_EPI_DRELU2 = 4
NC_EPI_SOFTCAP = 5


def load_library(path: str = LIB_PATH):
    """Load the CUDA library once; raise if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise OSError(f"{path} is missing: build it with "
                      "`python -m decoder_only_transformer_nanochat_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def nc_init(depth: int, vocab: int, seq: int, dtype: int):
    """Returns (status, handle)."""
    h = _P()
    rc = load_library().nc_init(depth, vocab, seq, dtype, ctypes.byref(h))
    return rc, h.value


class nc_block_opts(ctypes.Structure):
    _fields_ = [("window", ctypes.c_int), ("value_embeds", ctypes.c_int), ("resid_scalars", ctypes.c_int)]


def nc_init_ex(depth: int, vocab: int, seq: int, dtype: int, window: int = 0, value_embeds: bool = False,
               resid_scalars: bool = False):
    """Returns (status, handle) of a model with the full block's options."""
    h = _P()
    o = nc_block_opts(window, int(value_embeds), int(resid_scalars))
    rc = load_library().nc_init_ex(depth, vocab, seq, dtype, ctypes.byref(o), ctypes.byref(h))
    return rc, h.value


def nc_layer_window(handle, layer: int):
    w = _I()
    rc = load_library().nc_layer_window(handle, layer, ctypes.byref(w))
    return rc, w.value


def nc_param_count(handle):
    n = _I()
    rc = load_library().nc_param_count(handle, ctypes.byref(n))
    return rc, n.value


def nc_get_dims(handle):
    d = nc_dims()
    rc = load_library().nc_get_dims(handle, ctypes.byref(d))
    return rc, {f: getattr(d, f) for f, _ in nc_dims._fields_}


def nc_param_layout(handle, index: int):
    p = nc_param()
    rc = load_library().nc_param_layout(handle, index, ctypes.byref(p))
    return rc, (p.name.decode(), p.offset, p.rows, p.cols)


def nc_workspace_bytes(handle, B: int, T: int):
    n = ctypes.c_size_t()
    rc = load_library().nc_workspace_bytes(handle, B, T, ctypes.byref(n))
    return rc, n.value


def nc_fwd_bwd(handle, weights, tokens, targets, B, T, workspace, ws_bytes, loss, token_loss,
               grads, stream):
    return load_library().nc_fwd_bwd(handle, weights, tokens, targets, B, T, workspace, ws_bytes,
                                     loss, token_loss, grads, stream)


def nc_fwd_bwd_ex(handle, weights, tokens, targets, B, T, workspace, ws_bytes, loss, token_loss,
                  grads, flags, stream):
    return load_library().nc_fwd_bwd_ex(handle, weights, tokens, targets, B, T, workspace, ws_bytes,
                                        loss, token_loss, grads, flags, stream)


def nc_grad_buckets(handle):
    """Returns (status, [(offset, count), ...]) in the order the backward finishes them."""
    lib = load_library()
    n = _I()
    rc = lib.nc_grad_bucket_count(handle, ctypes.byref(n))
    if rc != NC_OK:
        return rc, []
    out = []
    for k in range(n.value):
        o, c = ctypes.c_int64(), ctypes.c_int64()
        rc = lib.nc_grad_bucket(handle, k, ctypes.byref(o), ctypes.byref(c))
        if rc != NC_OK:
            return rc, []
        out.append((o.value, c.value))
    return NC_OK, out


def nc_set_grad_events(handle, events) -> int:
    """events: raw cudaEvent_t handles (ints), one per bucket (or fewer)."""
    arr = (_P * max(1, len(events)))(*[_P(e) for e in events])
    return load_library().nc_set_grad_events(handle, arr, len(events))


class nc_optim_opts(ctypes.Structure):
    _fields_ = [("lr_matrix", ctypes.c_float), ("lr_embed", ctypes.c_float), ("lr_head", ctypes.c_float),
                ("lr_scalar", ctypes.c_float), ("weight_decay", ctypes.c_float),
                ("muon_momentum", ctypes.c_float), ("ns_steps", ctypes.c_int), ("beta1", ctypes.c_float),
                ("beta2", ctypes.c_float), ("eps", ctypes.c_float)]


def nc_optim_state_bytes(handle):
    n = ctypes.c_size_t()
    rc = load_library().nc_optim_state_bytes(handle, ctypes.byref(n))
    return rc, n.value


def nc_optim_workspace_bytes(handle):
    n = ctypes.c_size_t()
    rc = load_library().nc_optim_workspace_bytes(handle, ctypes.byref(n))
    return rc, n.value


def nc_optim_init(handle, weights, state, stream) -> int:
    return load_library().nc_optim_init(handle, weights, state, stream)


def nc_optim_step(handle, weights, grads, state, step, opts: dict, workspace, ws_bytes, stream) -> int:
    o = nc_optim_opts(**opts)
    return load_library().nc_optim_step(handle, weights, grads, state, step, ctypes.byref(o), workspace,
                                        ws_bytes, stream)


def nc_kv_cache_bytes(handle, B: int, T_max: int):
    n = ctypes.c_size_t()
    rc = load_library().nc_kv_cache_bytes(handle, B, T_max, ctypes.byref(n))
    return rc, n.value


def nc_prefill(handle, weights, tokens, B, T, cache, T_max, seqlens, workspace, ws_bytes, logits, stream) -> int:
    return load_library().nc_prefill(handle, weights, tokens, B, T, cache, T_max, seqlens, workspace, ws_bytes,
                                     logits, stream)


def nc_decode(handle, weights, tokens, B, cache, T_max, seqlens, workspace, ws_bytes, logits, stream) -> int:
    return load_library().nc_decode(handle, weights, tokens, B, cache, T_max, seqlens, workspace, ws_bytes,
                                    logits, stream)


def nc_fwd(handle, weights, tokens, B, T, workspace, ws_bytes, logits, stream):
    return load_library().nc_fwd(handle, weights, tokens, B, T, workspace, ws_bytes, logits, stream)


def nc_sync_status(handle, stream, timeout_ms: int) -> int:
    return load_library().nc_sync_status(handle, stream, timeout_ms)


def nc_strerror(code: int) -> str:
    try:
        return load_library().nc_strerror(code).decode()
    except OSError:
        return f"status {code}"


def nc_destroy(handle) -> None:
    if handle:
        load_library().nc_destroy(handle)


def nc_gemm(A, lda, a_mn, B, ldb, b_mn, D, ldd, M, N, K, dtype, epilogue, engine, stream) -> int:
    return load_library().nc_gemm(A, lda, a_mn, B, ldb, b_mn, D, ldd, M, N, K, dtype, epilogue,
                                  engine, stream)


def nc_attention_fwd(qkv, ld, O, lse, B, T, H, dtype, engine, stream, window: int = 0) -> int:
    return load_library().nc_attention_fwd(qkv, ld, O, lse, B, T, H, window, dtype, engine, stream)


def nc_attention_bwd(qkv, ld, O, dO, lse, Drow, dqkv, B, T, H, dtype, engine, stream, window: int = 0) -> int:
    return load_library().nc_attention_bwd(qkv, ld, O, dO, lse, Drow, dqkv, B, T, H, window, dtype, engine,
                                           stream)


def nc_softcap_ce(z, ldz, targets, token_loss, M, V, grad_scale, dtype, stream) -> int:
    return load_library().nc_softcap_ce(z, ldz, targets, token_loss, M, V, grad_scale, dtype, stream)


def nc_attention_bwd_scratch_bytes(B, T, H, window: int = 0):
    n = ctypes.c_size_t(0)
    rc = load_library().nc_attention_bwd_scratch_bytes(B, T, H, window, ctypes.byref(n))
    return rc, n.value


def nc_attention_bwd_ex(qkv, ld, O, dO, lse, Drow, scratch, scratch_bytes, dqkv, B, T, H, dtype, engine, stream,
                        window: int = 0) -> int:
    return load_library().nc_attention_bwd_ex(qkv, ld, O, dO, lse, Drow, scratch, scratch_bytes, dqkv, B, T, H,
                                              window, dtype, engine, stream)


def nc_set_attention_ctas(ctas: int) -> int:
    """Cap on the CTAs of the persistent attention kernels (0: one per SM)."""
    return load_library().nc_set_attention_ctas(ctas)


def nc_rmsnorm(x, y, r, M, C, dtype, stream) -> int:
    return load_library().nc_rmsnorm(x, y, r, M, C, dtype, stream)


def nc_rmsnorm_bwd(dy, y, r, dx, dx_t, M, C, accumulate, dtype, stream) -> int:
    return load_library().nc_rmsnorm_bwd(dy, y, r, dx, dx_t, M, C, accumulate, dtype, stream)


def nc_rope_qknorm(handle, qkv, ld, rq, rk, B, T, stream) -> int:
    return load_library().nc_rope_qknorm(handle, qkv, ld, rq, rk, B, T, stream)


def nc_rope_qknorm_bwd(handle, dqkv, qkv, ld, rq, rk, B, T, stream) -> int:
    return load_library().nc_rope_qknorm_bwd(handle, dqkv, qkv, ld, rq, rk, B, T, stream)


def nc_ops_status(stream, timeout_ms: int) -> int:
    """Status of the op-level calls (no model handle): read and clear."""
    return load_library().nc_ops_status(stream, timeout_ms)


def nc_check_wait_expiry(wait_us: int, stream) -> int:
    """Enqueue a wait that runs out after wait_us and records a timeout."""
    return load_library().nc_check_wait_expiry(wait_us, stream)


def nc_profile(handle, enable: int) -> int:
    return load_library().nc_profile(handle, enable)


def nc_profile_read(handle, max_classes: int = 32):
    """Returns (status, [ {name, launches, ms, flops, bytes}, ... ])."""
    arr = (nc_kernel_stat * max_classes)()
    n = _I()
    rc = load_library().nc_profile_read(handle, arr, max_classes, ctypes.byref(n))
    out = [dict(name=arr[i].name.decode(), launches=arr[i].launches, ms=arr[i].ms,
                flops=arr[i].flops, bytes=arr[i].bytes) for i in range(n.value)]
    return rc, out


NC_ATTN_BWD_NOALLOC_MAX_ROWS = 1 << 20


def nc_attention_bwd_noalloc(qkv, ld, O, dO, lse, dqkv, B, T, H, dtype, engine, stream) -> int:
    """nc_attention_bwd without the Drow scratch argument: the library's fixed
    device scratch is used instead, for callers that cannot allocate."""
    return load_library().nc_attention_bwd_noalloc(qkv, ld, O, dO, lse, dqkv, B, T, H, dtype, engine,
                                                   stream)
