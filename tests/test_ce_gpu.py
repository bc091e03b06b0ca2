"""Softcap + cross-entropy (nc_softcap_ce) element by element against the
fp64 oracle's head (oracle.head_loss_row / head_backward_row) on the same
logits: per-token losses and every entry of dz = dloss/dz.

Rows cover what the method makes delicate: logits deep in tanh saturation
(|z| 30..60, where 1 - (s/15)^2 is ~1e-3 and below), targets at ids 0 and
V - 1 and at the row's argmax, a target that takes almost all of the
probability (1 - p ~ 1e-11), and rows whose logits are all equal.

Tolerances, from the arithmetic of each path:
  * bf16 model (persistent kernel, V = 65,536, and the general kernel):
    s is formed to ~4e-7 absolute in t (so ~6e-6 in s), the exponentials to
    ~2^-22 relative; w = e (1 - t^2) is held as fp16 (unit roundoff 2^-11,
    or 2^-25 absolute below fp16's normal range) and dz is rounded to bf16
    (unit roundoff 2^-8: 8 significant bits).  Hence
    |d dz| <= (2^-8 + 2^-10) |dz| + 2^-24 g per entry and |d loss| <= 5e-5
    per token.
  * fp32 model: library expf and a correctly rounded division, fp32 storage:
    |d dz| <= 1e-5 |dz| + 1e-12 g and |d loss| <= 2e-5.
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


def _rows(V, M, seed):
    z = synth.normal(seed, 1, M * V).reshape(M, V) * 3.0
    tgt = (synth.uniform01(seed, 2, M) * V).astype(np.int64)
    u = synth.uniform01(seed, 3, V)
    sign = np.where(synth.uniform01(seed, 4, V) < 0.5, -1.0, 1.0)
    z[1] = (30.0 + 30.0 * u) * sign          # deep saturation
    tgt[1] = int(np.argmax(z[1]))
    z[2] = (30.0 + 30.0 * u) * sign
    tgt[2] = int(np.argmin(z[2]))            # target at the row's minimum
    tgt[3] = 0
    tgt[4] = V - 1
    z[5, :] = 0.5                            # all equal: uniform softmax
    tgt[5] = V // 2
    z[6, :] = 40.0                           # all equal and saturated
    tgt[6] = 3
    z[7] = -20.0 + synth.normal(seed, 5, V)  # one dominant target: 1 - p ~ 1e-11
    tgt[7] = V // 3
    z[7, tgt[7]] = 45.0
    z[8] = synth.normal(seed, 6, V) * 0.01   # near zero: loss ~ ln V
    z[9, 11] = 60.0                          # the argmax is not the target
    z[9, 12] = -60.0
    tgt[9] = 12
    return z, tgt.astype(np.int32)


def _oracle(z, tgt, g):
    s = 15.0 * np.tanh(z / 15.0)
    loss, lse = oracle.head_loss_row(s, tgt)
    return loss, oracle.head_backward_row(s, lse, tgt, g)


def _run(nc, z, tgt, dtype, pad, g):
    import torch
    M, V = z.shape
    ldz = V + pad
    if dtype == "bf16":
        zs = synth.bf16_bits_to_f64(synth.f32_to_bf16_bits(z.astype(np.float32)))
        store = np.zeros((M, ldz), dtype=np.float32)
        store[:, :V] = zs
        store[:, V:] = 7.0
        bits = synth.f32_to_bf16_bits(store)
        zd = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
        code = nc.NC_BF16
    else:
        zs = z.astype(np.float32).astype(np.float64)
        store = np.full((M, ldz), 7.0, dtype=np.float32)
        store[:, :V] = zs
        zd = torch.from_numpy(store).cuda()
        code = nc.NC_F32
    t = torch.from_numpy(tgt).cuda()
    tl = torch.zeros(M, dtype=torch.float32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert nc.nc_softcap_ce(zd.data_ptr(), ldz, t.data_ptr(), tl.data_ptr(), M, V, g, code, st) == 0
    assert nc.nc_ops_status(st, 60000) == nc.NC_OK
    out = zd.float().cpu().numpy().astype(np.float64)
    assert np.all(out[:, V:] == 7.0), "entries past V must stay untouched"
    return zs, tl.cpu().numpy().astype(np.float64), out[:, :V]


CASES = [
    # V, M, dtype, row padding: the model path (persistent), then the general kernel
    (65536, 12, "bf16", 64),
    (65536, 10, "bf16", 0),
    (65536, 451, "bf16", 0),    # 3 x 148 + 7 rows: every CTA of the persistent kernel walks 3-4 rows
    (1000, 12, "bf16", 8),      # V % 8 == 0, small: persistent kernel with idle threads
    (1003, 12, "bf16", 5),      # ragged: the general kernel
    (65536, 12, "f32", 64),
    (1003, 12, "f32", 3),
]


@pytest.mark.parametrize("V,M,dtype,pad", CASES)
def test_softcap_ce_matches_oracle_elementwise(nc, V, M, dtype, pad):
    g = 1.0 / 4096
    z, tgt = _rows(V, M, 40 + V % 97 + M)
    zs, tl, dz = _run(nc, z, tgt, dtype, pad, g)
    loss_ref, dz_ref = _oracle(zs, tgt, g)
    if dtype == "bf16":
        rtol, atol, ltol = 2.0 ** -8 + 2.0 ** -10, 2.0 ** -24 * g, 5e-5
    else:
        rtol, atol, ltol = 1e-5, 1e-12 * g, 2e-5
    np.testing.assert_allclose(tl, loss_ref, rtol=0, atol=ltol)
    err = np.abs(dz - dz_ref)
    bad = err > rtol * np.abs(dz_ref) + atol
    assert not bad.any(), (np.argwhere(bad)[:5], dz[bad][:5], dz_ref[bad][:5])
    # the saturated row's gradient is small but resolved, not flushed
    assert np.abs(dz[1]).max() > 0
    # the dominant target's 1 - p ~ 1e-11 comes out with its relative
    # precision (no cancellation against p ~ 1), below the absolute floor above
    t7 = tgt[7]
    assert abs(dz[7, t7] - dz_ref[7, t7]) <= (rtol + 1e-4) * abs(dz_ref[7, t7])


def test_softcap_ce_closed_forms(nc):
    # all logits equal: loss = ln V exactly, dz = (1/V - [v = t]) (1 - (s/15)^2) g
    V, M, g = 65536, 2, 0.5
    z = np.full((M, V), 0.0)
    tgt = np.array([0, V - 1], dtype=np.int32)
    _, tl, dz = _run(nc, z, tgt, "bf16", 0, g)
    np.testing.assert_allclose(tl, np.log(V), rtol=0, atol=2e-6)
    ref = np.full((M, V), g / V)
    ref[0, 0] -= g
    ref[1, V - 1] -= g
    np.testing.assert_allclose(dz, ref, rtol=2.0 ** -8 + 2.0 ** -10, atol=0)
    # every row of dz sums to zero (softmax minus a one-hot, times a factor
    # that is 1 here)
    assert np.all(np.abs(dz.sum(axis=1)) <= 1e-3 * g)


def test_softcap_ce_flags_out_of_range_targets(nc):
    V, M = 65536, 2
    z, _ = _rows(V, 12, 9)
    z = z[:M]
    import torch
    bits = synth.f32_to_bf16_bits(z.astype(np.float32))
    zd = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    t = torch.tensor([V, 5], dtype=torch.int32, device="cuda")
    tl = torch.zeros(M, dtype=torch.float32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert nc.nc_softcap_ce(zd.data_ptr(), V, t.data_ptr(), tl.data_ptr(), M, V, 1.0, nc.NC_BF16, st) == 0
    assert nc.nc_ops_status(st, 60000) == nc.NC_ERANGE
    assert nc.nc_ops_status(st, 60000) == nc.NC_OK
