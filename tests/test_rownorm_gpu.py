"""The row kernels of the block (nc_rmsnorm, nc_rmsnorm_bwd, nc_rope_qknorm,
nc_rope_qknorm_bwd) element by element against the fp64 oracle's rmsnorm,
rmsnorm_bwd, rope and rope_bwd on the same inputs (the inputs rounded to the
kernel's dtype first, so both sides start from identical values).

Sizes span several 8-row blocks with a ragged tail (M = 3 x 77) and widths of
every vector count the dispatch takes at the model's sizes.

Tolerances, from the arithmetic:
  * the kernels accumulate in fp32: sums of C <= 4096 squares or products
    carry a relative error below C 2^-24 < 2.5e-4 of the sum of absolute
    values, which for a mean taken once and applied by one multiply keeps
    every output within 1e-5 of max|out| (fp32 outputs);
  * bf16 outputs add their own rounding: half a unit in the 8th bit,
    |d| <= 2^-9 |out| (taken as 2^-8 |out| + 1e-5 max|out|).
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


def _dev(a, dtype):
    """(device tensor, the exact values it holds as fp64)."""
    import torch
    if dtype == "bf16":
        bits = synth.f32_to_bf16_bits(a.astype(np.float32))
        t = torch.from_numpy(bits.view(np.int16).copy()).cuda().view(torch.bfloat16)
        return t, synth.bf16_bits_to_f64(bits)
    f = a.astype(np.float32)
    return torch.from_numpy(f.copy()).cuda(), f.astype(np.float64)


def _host(t):
    return t.float().cpu().numpy().astype(np.float64)


def _check(got, ref, dtype, what):
    scale = np.abs(ref).max()
    rtol = 2.0 ** -8 if dtype == "bf16" else 0.0
    bad = np.abs(got - ref) > rtol * np.abs(ref) + 1e-5 * scale
    assert not bad.any(), (what, np.argwhere(bad)[:4], got[bad][:4], ref[bad][:4])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("C", [256, 768, 1280, 2048, 4096])
def test_rmsnorm_forward_and_backward(nc, dtype, C):
    import torch
    M = 3 * 77
    code = nc.NC_BF16 if dtype == "bf16" else nc.NC_F32
    st = torch.cuda.current_stream().cuda_stream
    x = synth.normal(C, 1, M * C).reshape(M, C) * 2.0
    x[5] *= 1e-3  # a row far below unit rms
    xd, xs = _dev(x, dtype)
    yd = torch.empty_like(xd)
    r = torch.empty(M, dtype=torch.float32, device="cuda")
    assert nc.nc_rmsnorm(xd.data_ptr(), yd.data_ptr(), r.data_ptr(), M, C, code, st) == 0
    y_ref, r_ref = oracle.rmsnorm(xs)
    np.testing.assert_allclose(r.cpu().numpy(), r_ref[:, 0], rtol=1e-5)
    y = _host(yd)
    _check(y, y_ref, dtype, "y")
    # the output's rms is sqrt(ms / (ms + eps)) per row: 1 up to eps (0.986 for
    # the row far below unit rms)
    ms = np.mean(xs * xs, axis=1)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=1)), np.sqrt(ms / (ms + oracle.model.EPS)),
                               atol=4e-3 if dtype == "bf16" else 1e-5)

    dy = synth.normal(C, 2, M * C).reshape(M, C)
    dyd, dys = _dev(dy, dtype)
    old = synth.normal(C, 3, M * C).reshape(M, C).astype(np.float32)
    for acc in (0, 1):
        dx = torch.from_numpy(old.copy()).cuda()
        dx_t = torch.empty_like(xd)
        assert nc.nc_rmsnorm_bwd(dyd.data_ptr(), yd.data_ptr(), r.data_ptr(), dx.data_ptr(), dx_t.data_ptr(),
                                 M, C, acc, code, st) == 0
        ys = y  # the kernel's saved y, as the backward reads it
        g = oracle.rmsnorm_bwd(dys, ys, r.cpu().numpy().astype(np.float64)[:, None])
        ref = g + (old.astype(np.float64) if acc else 0.0)
        got = dx.cpu().numpy().astype(np.float64)
        _check(got, ref, "f32", f"dx acc={acc}")
        _check(_host(dx_t), got, dtype, f"dx_t acc={acc}")
    torch.cuda.synchronize()


@pytest.mark.parametrize("dtype,depth", [("bf16", 20), ("bf16", 4), ("f32", 4)])
def test_rope_qknorm_forward_and_backward(nc, dtype, depth):
    import torch
    from decoder_only_transformer_nanochat_b200 import Model
    Bsz, T = 3, 77
    M = Bsz * T
    model = Model(depth=depth, vocab=1024, seq=T + 5, dtype=dtype)
    H = model.dims["n_head"]
    ld = 128 * (H + 2)
    st = torch.cuda.current_stream().cuda_stream
    qkv = synth.normal(depth, 4, M * ld).reshape(M, ld) * 1.5
    qd, qs = _dev(qkv, dtype)
    rq = torch.empty(M * H, dtype=torch.float32, device="cuda")
    rk = torch.empty(M, dtype=torch.float32, device="cuda")
    assert nc.nc_rope_qknorm(model.handle, qd.data_ptr(), ld, rq.data_ptr(), rk.data_ptr(), Bsz, T, st) == 0
    cos, sin = oracle.rope_tables(T)
    cos = np.tile(cos, (Bsz, 1))[:, None, :]
    sin = np.tile(sin, (Bsz, 1))[:, None, :]
    heads = qs[:, :128 * (H + 1)].reshape(M, H + 1, 128)
    y_ref, r_ref = oracle.rmsnorm(oracle.rope(heads, cos, sin))
    out = _host(qd)
    _check(out[:, :128 * (H + 1)].reshape(M, H + 1, 128), y_ref, dtype, "q,k")
    assert np.array_equal(out[:, 128 * (H + 1):], qs[:, 128 * (H + 1):]), "v must stay untouched"
    np.testing.assert_allclose(rq.cpu().numpy().reshape(M, H), r_ref[:, :H, 0], rtol=1e-5)
    np.testing.assert_allclose(rk.cpu().numpy(), r_ref[:, H, 0], rtol=1e-5)

    dy = synth.normal(depth, 5, M * ld).reshape(M, ld)
    dd, ds = _dev(dy, dtype)
    assert nc.nc_rope_qknorm_bwd(model.handle, dd.data_ptr(), qd.data_ptr(), ld, rq.data_ptr(), rk.data_ptr(),
                                 Bsz, T, st) == 0
    ys = out[:, :128 * (H + 1)].reshape(M, H + 1, 128)
    r_all = np.concatenate([rq.cpu().numpy().reshape(M, H), rk.cpu().numpy()[:, None]], axis=1)[..., None]
    g = oracle.rmsnorm_bwd(ds[:, :128 * (H + 1)].reshape(M, H + 1, 128), ys, r_all.astype(np.float64))
    ref = oracle.rope_bwd(g, cos, sin)
    got = _host(dd)
    _check(got[:, :128 * (H + 1)].reshape(M, H + 1, 128), ref, dtype, "dq,dk")
    assert np.array_equal(got[:, 128 * (H + 1):], ds[:, 128 * (H + 1):]), "dv must stay untouched"
    torch.cuda.synchronize()
    del model


def test_row_ops_reject_bad_shapes(nc):
    import torch
    st = torch.cuda.current_stream().cuda_stream
    x = torch.zeros(64 * 1288, dtype=torch.bfloat16, device="cuda")
    r = torch.zeros(64, dtype=torch.float32, device="cuda")
    assert nc.nc_rmsnorm(x.data_ptr(), x.data_ptr(), r.data_ptr(), 64, 1284, nc.NC_BF16, st) == nc.NC_ESHAPE
    assert nc.nc_rmsnorm(x.data_ptr(), x.data_ptr(), r.data_ptr(), 64, 8192, nc.NC_BF16, st) == nc.NC_ESHAPE
    assert nc.nc_rmsnorm(x.data_ptr() + 2, x.data_ptr(), r.data_ptr(), 8, 1280, nc.NC_BF16, st) == nc.NC_EALIGN
