"""nc_attention_bwd_noalloc: the attention backward for callers that cannot
allocate device memory (their device memory is fixed by their own allocator,
or they cannot afford the synchronisation that cudaMalloc/cudaFree bring), so
they cannot hand the library the B*H*T scratch nc_attention_bwd takes.  It
uses a fixed scratch array inside the library instead.

Checked through the C ABI against nc_attention_bwd (which takes a caller
scratch buffer) on the same inputs: the results must be bit-identical, on
two calls in a row with different shapes (the second call starts with the
first call's data left in the shared scratch), and again after a call that
leaves NaN in the scratch; plus the size limit.
"""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nc():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from decoder_only_transformer_nanochat_b200 import build
    build.build()
    import decoder_only_transformer_nanochat_b200 as m
    return m


def _bf16(x):
    return synth.bf16_bits_to_f64(synth.f32_to_bf16_bits(x.astype(np.float32)))


def _dev(x):
    import torch
    bits = synth.f32_to_bf16_bits(np.ascontiguousarray(x, dtype=np.float32))
    return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)


def _case(nc, B, T, H, seed):
    """Forward outputs plus the reference backward from nc_attention_bwd."""
    import torch
    ld = 128 * (H + 2)
    q, _ = oracle.rmsnorm(synth.normal(seed, 1, B * T * H * 128).reshape(B * T, H, 128))
    k, _ = oracle.rmsnorm(synth.normal(seed, 2, B * T * 128).reshape(B * T, 128))
    v = synth.normal(seed, 3, B * T * 128).reshape(B * T, 128)
    qkv = _dev(_bf16(np.concatenate([q.reshape(B * T, -1), k, v], 1)))
    dO = _dev(_bf16(synth.normal(seed, 4, B * T * H * 128)))
    st = torch.cuda.current_stream().cuda_stream
    O = torch.empty(B * T * H * 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B * H * T, dtype=torch.float32, device="cuda")
    assert nc.nc_attention_fwd(qkv.data_ptr(), ld, O.data_ptr(), lse.data_ptr(), B, T, H, nc.NC_BF16, 0, st) == 0
    Drow = torch.empty(B * H * T, dtype=torch.float32, device="cuda")
    ref = torch.zeros(B * T * ld, dtype=torch.bfloat16, device="cuda")
    assert nc.nc_attention_bwd(qkv.data_ptr(), ld, O.data_ptr(), dO.data_ptr(), lse.data_ptr(), Drow.data_ptr(),
                               ref.data_ptr(), B, T, H, nc.NC_BF16, 0, st) == 0
    return dict(qkv=qkv, dO=dO, O=O, lse=lse, ref=ref, ld=ld, st=st)


def _run_noalloc(nc, c, B, T, H):
    import torch
    out = torch.full_like(c["ref"], float("nan"))
    rc = nc.nc_attention_bwd_noalloc(c["qkv"].data_ptr(), c["ld"], c["O"].data_ptr(), c["dO"].data_ptr(),
                                     c["lse"].data_ptr(), out.data_ptr(), B, T, H, nc.NC_BF16, 0, c["st"])
    assert rc == 0
    torch.cuda.synchronize()
    return out


def _compare(got, ref):
    # the same deterministic kernels (no atomics in dQ or dK/dV) on the same
    # inputs: only the scratch of rowsum(dO * O) differs, so the results are
    # bit-identical, and a stale or partly written scratch would show
    assert torch_equal(got, ref)


def torch_equal(a, b):
    import torch
    return bool(torch.equal(a.view(torch.int16), b.view(torch.int16)))


def test_noalloc_matches_attention_bwd_twice(nc):
    import torch
    # first call: B=2, T=256, H=2 fills part of the shared scratch
    c1 = _case(nc, 2, 256, 2, 31)
    _compare(_run_noalloc(nc, c1, 2, 256, 2), c1["ref"])
    # second call: another shape reads only what it writes
    c2 = _case(nc, 1, 515, 3, 32)
    _compare(_run_noalloc(nc, c2, 1, 515, 3), c2["ref"])
    # a call whose rowsums are all NaN (dO = NaN) leaves NaN behind in the
    # scratch; the next call must overwrite every entry it reads
    bad = dict(c1)
    bad["dO"] = torch.full_like(c1["dO"], float("nan"))
    out = _run_noalloc(nc, bad, 2, 256, 2)
    assert torch.isnan(out.float()).any()
    _compare(_run_noalloc(nc, c1, 2, 256, 2), c1["ref"])
    assert nc.nc_ops_status(c1["st"], 60000) == nc.NC_OK


def test_noalloc_rejects_sizes_beyond_its_scratch(nc):
    import torch
    H, T = 16, 2048
    B = nc.NC_ATTN_BWD_NOALLOC_MAX_ROWS // (H * T) + 1
    st = torch.cuda.current_stream().cuda_stream
    # rejected on the host before any pointer is touched
    rc = nc.nc_attention_bwd_noalloc(16, 128 * (H + 2), 16, 16, 16, 16, B, T, H, nc.NC_BF16, 0, st)
    assert rc == nc.NC_ENOMEM
