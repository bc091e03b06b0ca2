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
