"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point declared in include/*.h, and rejects bad arguments."""
import ctypes
import glob
import os
import re

import pytest

import decoder_only_transformer_nanochat_b200 as nc
from decoder_only_transformer_nanochat_b200 import build as nc_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(re.findall(r"^\s*(?:const\s+)?\w+\s*\**\s*(nc_\w+)\s*\(", src, flags=re.M))
    return names


@pytest.fixture(scope="module")
def lib():
    nc_build.build()
    return nc.load_library()


def test_header_declares_entry_points():
    names = _declared()
    for n in ["nc_init", "nc_fwd_bwd", "nc_fwd", "nc_sync_status", "nc_strerror", "nc_destroy",
              "nc_get_dims", "nc_param_layout", "nc_workspace_bytes"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in _declared():
        assert hasattr(lib, n), n
        assert ctypes.cast(getattr(lib, n), ctypes.c_void_p).value


def test_strerror_covers_codes(lib):
    seen = set()
    for code in range(0, 10):
        s = nc.nc_strerror(code)
        assert s and s != "unknown status"
        seen.add(s)
    assert len(seen) == 10
    assert nc.nc_strerror(1234) == "unknown status"


def test_init_rejects_bad_arguments(lib):
    assert nc.nc_init(0, 65536, 2048, nc.NC_BF16)[0] == nc.NC_EINVAL
    assert nc.nc_init(4, 1, 2048, nc.NC_BF16)[0] == nc.NC_EINVAL
    assert nc.nc_init(4, 65536, 0, nc.NC_BF16)[0] == nc.NC_EINVAL
    assert nc.nc_init(4, 65536, 2048, 7)[0] == nc.NC_EUNSUPPORTED
    assert nc.nc_init(200, 65536, 2048, nc.NC_BF16)[0] == nc.NC_EINVAL  # wider than 4096
    assert lib.nc_init(4, 65536, 2048, 0, None) == nc.NC_EINVAL


def test_null_handle_is_rejected(lib):
    assert nc.nc_get_dims(None)[0] == nc.NC_EINVAL
    assert nc.nc_param_layout(None, 0)[0] == nc.NC_EINVAL
    assert nc.nc_workspace_bytes(None, 1, 1)[0] == nc.NC_EINVAL
    assert nc.nc_fwd_bwd(None, 1, 1, 1, 1, 1, 1, 1, 1, None, 1, None) == nc.NC_EINVAL
    assert nc.nc_fwd(None, 1, 1, 1, 1, 1, 1, 1, None) == nc.NC_EINVAL
    assert nc.nc_sync_status(None, None, 10) == nc.NC_EINVAL
    nc.nc_destroy(None)


def test_init_without_a_b200_fails_cleanly(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    rc, h = nc.nc_init(4, 65536, 256, nc.NC_F32)
    assert rc in (nc.NC_ECUDA, nc.NC_EUNSUPPORTED) and h is None


def test_op_entry_points_reject_bad_arguments_on_the_host(lib):
    # every check below returns before any device work or CUDA call
    BF16 = nc.NC_BF16
    H, B, T = 2, 1, 64
    ld = 128 * (H + 2)
    # strides beyond INT_MAX are a shape error, not a silent 32-bit truncation
    big = (1 << 31) + 8
    assert nc.nc_attention_fwd(16, big, 16, 16, B, T, H, BF16, 0, None) == nc.NC_ESHAPE
    assert nc.nc_attention_bwd(16, big, 16, 16, 16, 16, 16, B, T, H, BF16, 0, None) == nc.NC_ESHAPE
    assert nc.nc_attention_bwd_noalloc(16, big, 16, 16, 16, 16, B, T, H, BF16, 0, None) == nc.NC_ESHAPE
    assert nc.nc_attention_fwd(16, ld - 8, 16, 16, B, T, H, BF16, 0, None) == nc.NC_ESHAPE
    # the tensor-core engines take 16-byte aligned operands only: no slower fallback
    assert nc.nc_attention_fwd(24, ld, 16, 16, B, T, H, BF16, 0, None) == nc.NC_EALIGN
    assert nc.nc_attention_fwd(16, ld + 4, 16, 16, B, T, H, BF16, 0, None) == nc.NC_EALIGN
    assert nc.nc_attention_bwd(16, ld, 16, 24, 16, 16, 16, B, T, H, BF16, 0, None) == nc.NC_EALIGN
    assert nc.nc_attention_bwd_noalloc(16, ld, 16, 16, 16, 40, B, T, H, BF16, 0, None) == nc.NC_EALIGN
    # attention forward engines: 0 (model path), 1 (CUDA cores), 2 and 3 (the other
    # tcgen05 kernel); backward engines: 0 and 1
    assert nc.nc_attention_fwd(16, ld, 16, 16, B, T, H, BF16, 4, None) == nc.NC_EINVAL
    assert nc.nc_attention_bwd(16, ld, 16, 16, 16, 16, 16, B, T, H, BF16, 2, None) == nc.NC_EINVAL
    # the backward with dK/dV scratch: same argument checks, and a misaligned scratch
    assert nc.nc_attention_bwd_ex(16, big, 16, 16, 16, 16, 16, 1 << 20, 16, B, T, H, BF16, 0, None) == nc.NC_ESHAPE
    assert nc.nc_attention_bwd_ex(16, ld, 16, 16, 16, 16, 16, 1 << 20, 16, B, T, H, BF16, 2, None) == nc.NC_EINVAL
    assert nc.nc_attention_bwd_ex(16, ld, 16, 16, 16, 16, 20, 1 << 20, 16, B, T, H, BF16, 0, None) == nc.NC_EALIGN
    assert nc.nc_attention_bwd_ex(0, ld, 16, 16, 16, 16, 16, 1 << 20, 16, B, T, H, BF16, 0, None) == nc.NC_EINVAL
    assert nc.nc_attention_bwd_scratch_bytes(0, T, H, 0)[0] == nc.NC_ESHAPE
    assert nc.nc_attention_bwd_scratch_bytes(B, T, H, -1)[0] == nc.NC_EINVAL
    assert nc.nc_set_attention_ctas(-1) == nc.NC_EINVAL
    # GEMM: a bf16 stride that is not a multiple of 8 on a tensor-core engine
    assert nc.nc_gemm(16, 100, 0, 16, 128, 0, 16, 128, 64, 64, 100, BF16, nc.NC_EPI_STORE, 0,
                      None) == nc.NC_EALIGN
    assert nc.nc_gemm(16, 128, 0, 16, 128, 0, 24, 128, 64, 64, 128, BF16, nc.NC_EPI_STORE, 2,
                      None) == nc.NC_EALIGN
    assert nc.nc_gemm(16, 128, 0, 16, 128, 0, 16, 128, 64, 64, 128, BF16, nc.NC_EPI_STORE, 3,
                      None) == nc.NC_EINVAL
    # the wait-expiry self-check takes 0..1 s only
    assert nc.nc_check_wait_expiry(-1, None) == nc.NC_EINVAL
    assert nc.nc_check_wait_expiry(1000001, None) == nc.NC_EINVAL


def test_op_status_without_a_gpu_fails_cleanly(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert nc.nc_ops_status(None, 10) == nc.NC_ECUDA


def test_init_ex_rejects_bad_options(lib):
    # checked on the host before any device call
    assert nc.nc_init_ex(4, 65536, 2048, nc.NC_BF16, window=-1)[0] == nc.NC_EINVAL
    assert nc.nc_init_ex(0, 65536, 2048, nc.NC_BF16, window=64)[0] == nc.NC_EINVAL
    assert nc.nc_layer_window(None, 0)[0] == nc.NC_EINVAL
    assert nc.nc_param_count(None)[0] == nc.NC_EINVAL
