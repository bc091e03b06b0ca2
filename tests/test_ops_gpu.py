"""Kernel-level parity through the op entry points (nanochat_b200_ops.h):
the GEMM with every operand layout and fused epilogue, and causal MQA
attention forward / backward, each against a float64 CPU reference computed
from the same (bf16-rounded) inputs."""
import math

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


def _dev(x, dtype):
    import torch
    if dtype == "bf16":
        bits = synth.f32_to_bf16_bits(np.ascontiguousarray(x, dtype=np.float32))
        return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def _stored(logical, mn, pad):
    """Storage of a logical [rows, K] operand: K-major rows (ld = K + pad) or
    MN-major [K, rows] (ld = rows + pad)."""
    rows, K = logical.shape
    if not mn:
        s = np.zeros((rows, K + pad))
        s[:, :K] = logical
        return s, K + pad
    s = np.zeros((K, rows + pad))
    s[:, :rows] = logical.T
    return s, rows + pad


EPIS = ["STORE", "STORE_F32", "ADD", "RELU2", "DRELU2", "SOFTCAP"]

GEMM_CASES = [
    # M, N, K, a_mn, b_mn, pad
    (256, 512, 128, 0, 0, 0),
    (300, 520, 200, 0, 0, 8),      # ragged M, N, K (zero-filled tails)
    (384, 1280, 1280, 0, 1, 0),    # input-gradient layout
    (1280, 768, 640, 1, 1, 0),     # weight-gradient layout
    (200, 264, 72, 1, 1, 8),       # ragged weight-gradient layout
    (130, 300, 96, 1, 0, 8),
    (256, 256, 8192, 1, 1, 0),     # few tiles, long K: split-K path for fp32 output
    (520, 392, 136, 0, 1, 8),      # M not a multiple of 256: the second CTA of a pair is partly empty
    (1280, 5120, 256, 1, 1, 0),    # weight-gradient shape with a full second CTA
    # several tiles per CTA pair whose N tiles alternate two half tiles and one
    # (the epilogue's staging tiles alternate by half tile across tiles)
    (20480, 320, 128, 0, 0, 0),
    (20480, 392, 64, 0, 1, 8),     # ... and a last half tile of 8 columns
]


@pytest.mark.parametrize("M,N,K,a_mn,b_mn,pad", GEMM_CASES)
@pytest.mark.parametrize("epi", EPIS)
@pytest.mark.parametrize("engine", [0, 1, 2])
def test_gemm_bf16(nc, M, N, K, a_mn, b_mn, pad, epi, engine):
    # engine 0: pairs of CTAs on 256 x 256 tiles when M >= 256; 2: one CTA per tile; 1: CUDA cores
    import torch
    if engine == 1 and K > 2048 and epi != "STORE_F32":
        pytest.skip("covered by the tensor-core engine")
    seed = M * 7 + N * 3 + K + a_mn * 11 + b_mn * 13
    A = _bf16(synth.normal(seed, 1, M * K).reshape(M, K))
    B = _bf16(synth.normal(seed, 2, N * K).reshape(N, K))
    As, lda = _stored(A, a_mn, pad)
    Bs, ldb = _stored(B, b_mn, pad)
    A_dev = _dev(As / math.sqrt(K), "bf16")
    A_used = _bf16(As / math.sqrt(K))
    A_log = A_used[:, :K] if not a_mn else A_used[:, :M].T
    acc = A_log @ B.T
    ldd = N + pad
    code = getattr(nc, "NC_EPI_" + epi)
    if epi == "STORE_F32":
        D = torch.zeros(M, ldd, dtype=torch.float32, device="cuda")
        ref = acc
    else:
        D0 = _bf16(synth.normal(seed, 3, M * ldd).reshape(M, ldd))
        if epi == "DRELU2":
            D0 = _bf16(np.maximum(D0, 0) ** 2)
        D = _dev(D0, "bf16")
        old = D0[:, :N]
        ref = {"STORE": lambda: acc, "ADD": lambda: old + acc,
               "RELU2": lambda: np.maximum(acc, 0) ** 2,
               "DRELU2": lambda: acc * 2 * np.sqrt(old),
               "SOFTCAP": lambda: 15 * np.tanh(acc / 15)}[epi]()
    B_dev = _dev(Bs, "bf16")
    rc = nc.nc_gemm(A_dev.data_ptr(), lda, a_mn, B_dev.data_ptr(), ldb, b_mn, D.data_ptr(), ldd,
                    M, N, K, nc.NC_BF16, code, engine, torch.cuda.current_stream().cuda_stream)
    if engine != 1 and (lda % 8 or ldb % 8 or (ldd % (4 if epi == "STORE_F32" else 8))):
        # the tensor-core engines take 16-byte row strides only: an error, not a slower path
        assert rc == nc.NC_EALIGN
        return
    assert rc == 0
    torch.cuda.synchronize()
    got = D.float().cpu().numpy().astype(np.float64)
    scale = np.abs(ref).max()
    if epi == "STORE_F32":
        np.testing.assert_allclose(got[:, :N], ref, rtol=0, atol=2e-5 * scale)
    else:
        # one bf16 rounding of the output (plus the input rounding of D)
        err = np.abs(got[:, :N] - ref)
        assert np.all(err <= 2 ** -8 * np.abs(ref) + 2e-3 * scale), float(err.max())
    if pad and epi != "STORE_F32":
        np.testing.assert_array_equal(got[:, N:], D0[:, N:])  # nothing written past N


@pytest.mark.parametrize("M,N,K", [(129, 70, 33), (64, 257, 300)])
def test_gemm_f32(nc, M, N, K):
    import torch
    A = synth.normal(M + N, 1, M * K).reshape(M, K).astype(np.float32).astype(np.float64)
    B = synth.normal(M + N, 2, N * K).reshape(N, K).astype(np.float32).astype(np.float64)
    for a_mn in (0, 1):
        for b_mn in (0, 1):
            As, lda = _stored(A, a_mn, 0)
            Bs, ldb = _stored(B, b_mn, 0)
            D = torch.zeros(M, N, dtype=torch.float32, device="cuda")
            Ad, Bd = _dev(As, "f32"), _dev(Bs, "f32")
            rc = nc.nc_gemm(Ad.data_ptr(), lda, a_mn, Bd.data_ptr(), ldb, b_mn, D.data_ptr(), N,
                            M, N, K, nc.NC_F32, nc.NC_EPI_STORE, 0,
                            torch.cuda.current_stream().cuda_stream)
            assert rc == 0
            got = D.cpu().numpy().astype(np.float64)
            ref = A @ B.T
            np.testing.assert_allclose(got, ref, rtol=0, atol=1e-5 * np.abs(ref).max())


def _attn_inputs(B, T, H, seed, dtype):
    """q, k normalised per head (as after QK-norm), v plain."""
    ld = 128 * (H + 2)
    q = synth.normal(seed, 1, B * T * H * 128).reshape(B, T, H, 128)
    k = synth.normal(seed, 2, B * T * 128).reshape(B, T, 128)
    v = synth.normal(seed, 3, B * T * 128).reshape(B, T, 128)
    q, _ = oracle.rmsnorm(q)
    k, _ = oracle.rmsnorm(k)
    qkv = np.concatenate([q.reshape(B * T, H * 128), k.reshape(B * T, 128), v.reshape(B * T, 128)], 1)
    if dtype == "bf16":
        qkv = _bf16(qkv)
    else:
        qkv = qkv.astype(np.float32).astype(np.float64)
    q = qkv[:, :H * 128].reshape(B, T, H, 128)
    k = qkv[:, H * 128:H * 128 + 128].reshape(B, T, 128)
    v = qkv[:, H * 128 + 128:].reshape(B, T, 128)
    return qkv, ld, q, k, v


ATTN_CASES = [(1, 1, 1), (2, 9, 2), (1, 130, 3), (2, 256, 2), (1, 515, 10)]


@pytest.mark.parametrize("B,T,H", ATTN_CASES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("engine", [0, 1, 2, 3])
def test_attention_fwd_bwd(nc, B, T, H, dtype, engine):
    # engines 2 and 3: the other tcgen05 forward kernel, and the model's kernel
    # with one CTA per query tile; their O and lse then feed the backward
    import torch
    code = nc.NC_BF16 if dtype == "bf16" else nc.NC_F32
    qkv, ld, q, k, v = _attn_inputs(B, T, H, 100 + T + H, dtype)
    st = torch.cuda.current_stream().cuda_stream
    qkv_d = _dev(qkv, dtype)
    O = torch.zeros(B * T, H * 128, dtype=qkv_d.dtype, device="cuda")
    lse = torch.zeros(B, H, T, dtype=torch.float32, device="cuda")
    assert nc.nc_attention_fwd(qkv_d.data_ptr(), ld, O.data_ptr(), lse.data_ptr(), B, T, H, code,
                               engine, st) == 0
    O_ref = np.empty((B, T, H, 128))
    lse_ref = np.empty((B, H, T))
    for b in range(B):
        O_ref[b], lse_ref[b] = oracle.attention(q[b], k[b], v[b])
    got_O = O.float().cpu().numpy().reshape(B, T, H, 128)
    got_lse = lse.cpu().numpy()
    tolO = 1e-5 if dtype == "f32" else 1.5e-2
    np.testing.assert_allclose(got_O, O_ref, rtol=0, atol=tolO * np.abs(O_ref).max())
    np.testing.assert_allclose(got_lse, lse_ref, rtol=0, atol=1e-5 if dtype == "f32" else 2e-3)
    # backward with a random upstream gradient, using the kernel's own O
    dO = synth.normal(7 + T, 4, B * T * H * 128).reshape(B * T, H * 128)
    dO = _bf16(dO) if dtype == "bf16" else dO.astype(np.float32).astype(np.float64)
    dO_d = _dev(dO, dtype)
    Drow = torch.zeros(B, H, T, dtype=torch.float32, device="cuda")
    dqkv = torch.zeros(B * T, ld, dtype=qkv_d.dtype, device="cuda")
    assert nc.nc_attention_bwd(qkv_d.data_ptr(), ld, O.data_ptr(), dO_d.data_ptr(), lse.data_ptr(),
                               Drow.data_ptr(), dqkv.data_ptr(), B, T, H, code, engine % 2, st) == 0
    assert nc.nc_ops_status(st, 60000) == nc.NC_OK
    got = dqkv.float().cpu().numpy().astype(np.float64)
    dq_ref = np.empty((B, T, H, 128))
    dk_ref = np.empty((B, T, 128))
    dv_ref = np.empty((B, T, 128))
    for b in range(B):
        dq_ref[b], dk_ref[b], dv_ref[b] = oracle.attention_bwd(dO.reshape(B, T, H, 128)[b], q[b], k[b], v[b])
    parts = [(got[:, :H * 128], dq_ref.reshape(B * T, -1)), (got[:, H * 128:H * 128 + 128], dk_ref.reshape(B * T, -1)),
             (got[:, H * 128 + 128:], dv_ref.reshape(B * T, -1))]
    for g, r in parts:
        scale = np.abs(r).max()
        if T == 1 and r is not parts[2][1]:
            # one key: the softmax is constant, dq and dk vanish
            assert np.max(np.abs(g)) <= 1e-6
            continue
        if dtype == "f32":
            np.testing.assert_allclose(g, r, rtol=0, atol=1e-4 * scale)
        else:
            cos = np.sum(g * r) / (np.linalg.norm(g) * np.linalg.norm(r) + 1e-300)
            assert cos > 0.9995, cos
            assert np.max(np.abs(g - r)) <= 3e-2 * scale


def test_expired_wait_reaches_the_host(nc):
    # a wait that nothing completes runs out after 20 ms and is reported, not hung
    import torch
    st = torch.cuda.current_stream().cuda_stream
    assert nc.nc_ops_status(st, 60000) == nc.NC_OK
    assert nc.nc_check_wait_expiry(20000, st) == nc.NC_OK
    assert nc.nc_ops_status(st, 60000) == nc.NC_ETIMEOUT
    assert nc.nc_ops_status(st, 60000) == nc.NC_OK  # read once, then cleared
    # the context is still usable afterwards
    x = torch.ones(1024, device="cuda")
    assert float(x.sum().item()) == 1024.0


def test_misaligned_bf16_operands_are_rejected(nc):
    import torch
    st = torch.cuda.current_stream().cuda_stream
    buf = torch.zeros(1 << 16, dtype=torch.bfloat16, device="cuda")
    p = buf.data_ptr()
    H, B, T = 2, 1, 64
    ld = 128 * (H + 2)
    assert nc.nc_attention_fwd(p + 2, ld, p, p, B, T, H, nc.NC_BF16, 0, st) == nc.NC_EALIGN
    assert nc.nc_gemm(p, 100, 0, p, 128, 0, p, 128, 64, 64, 100, nc.NC_BF16, nc.NC_EPI_STORE, 0,
                      st) == nc.NC_EALIGN
    # the CUDA-core test engine takes any stride
    assert nc.nc_gemm(p, 100, 0, p, 128, 0, p + 4096, 128, 64, 64, 100, nc.NC_BF16, nc.NC_EPI_STORE, 1,
                      st) == nc.NC_OK
    assert nc.nc_ops_status(st, 60000) == nc.NC_OK


WINDOW_CASES = [(1, 515, 3, 1), (1, 515, 3, 64), (2, 256, 2, 129), (1, 300, 10, 200), (1, 1030, 2, 384),
                (2, 130, 1, 128)]


@pytest.mark.parametrize("B,T,H,window", WINDOW_CASES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("engine", [0, 1, 2, 3])
def test_windowed_attention_fwd_bwd(nc, B, T, H, window, dtype, engine):
    # sliding window (query i sees keys j with 0 <= i - j < window) against the
    # full-block oracle's windowed attention
    import torch

    from oracle import full_block as fb
    code = nc.NC_BF16 if dtype == "bf16" else nc.NC_F32
    qkv, ld, q, k, v = _attn_inputs(B, T, H, 300 + T + H + window, dtype)
    st = torch.cuda.current_stream().cuda_stream
    qkv_d = _dev(qkv, dtype)
    O = torch.zeros(B * T, H * 128, dtype=qkv_d.dtype, device="cuda")
    lse = torch.zeros(B, H, T, dtype=torch.float32, device="cuda")
    assert nc.nc_attention_fwd(qkv_d.data_ptr(), ld, O.data_ptr(), lse.data_ptr(), B, T, H, code, engine, st,
                               window=window) == 0
    O_ref = np.empty((B, T, H, 128))
    for b in range(B):
        O_ref[b], _ = fb.attention(q[b], k[b], v[b], window)
    got_O = O.float().cpu().numpy().reshape(B, T, H, 128)
    tolO = 1e-5 if dtype == "f32" else 1.5e-2
    np.testing.assert_allclose(got_O, O_ref, rtol=0, atol=tolO * np.abs(O_ref).max())
    if window == 1:
        # one key: O = v of the query's own position, lse = q.k / sqrt(d)
        np.testing.assert_allclose(got_O, np.broadcast_to(v[:, :, None, :], got_O.shape), rtol=0,
                                   atol=tolO * np.abs(v).max())
    dO = synth.normal(9 + T, 4, B * T * H * 128).reshape(B * T, H * 128)
    dO = _bf16(dO) if dtype == "bf16" else dO.astype(np.float32).astype(np.float64)
    dO_d = _dev(dO, dtype)
    Drow = torch.zeros(B, H, T, dtype=torch.float32, device="cuda")
    dqkv = torch.zeros(B * T, ld, dtype=qkv_d.dtype, device="cuda")
    assert nc.nc_attention_bwd(qkv_d.data_ptr(), ld, O.data_ptr(), dO_d.data_ptr(), lse.data_ptr(),
                               Drow.data_ptr(), dqkv.data_ptr(), B, T, H, code, engine % 2, st,
                               window=window) == 0
    assert nc.nc_ops_status(st, 60000) == nc.NC_OK
    got = dqkv.float().cpu().numpy().astype(np.float64)
    refs = [np.empty((B, T, H, 128)), np.empty((B, T, 128)), np.empty((B, T, 128))]
    for b in range(B):
        refs[0][b], refs[1][b], refs[2][b] = fb.attention_bwd(dO.reshape(B, T, H, 128)[b], q[b], k[b], v[b], window)
    parts = [(got[:, :H * 128], refs[0].reshape(B * T, -1)), (got[:, H * 128:H * 128 + 128], refs[1].reshape(B * T, -1)),
             (got[:, H * 128 + 128:], refs[2].reshape(B * T, -1))]
    for i, (g, r) in enumerate(parts):
        scale = np.abs(r).max()
        if window == 1 and i < 2:
            # one key per query: the softmax is constant, dq = dk = 0 up to the
            # rounding of dP - D (a few ulps of dv's size)
            assert np.max(np.abs(g)) <= 1e-5 * np.abs(parts[2][1]).max()
            continue
        if dtype == "f32":
            np.testing.assert_allclose(g, r, rtol=0, atol=1e-4 * scale)
        else:
            cos = np.sum(g * r) / (np.linalg.norm(g) * np.linalg.norm(r) + 1e-300)
            assert cos > 0.9995, cos
            assert np.max(np.abs(g - r)) <= 3e-2 * scale


def test_window_covering_the_context_is_the_causal_kernel(nc):
    # window >= T is the plain causal mask: bit-identical to window 0
    import torch
    B, T, H = 1, 300, 2
    qkv, ld, q, k, v = _attn_inputs(B, T, H, 77, "bf16")
    st = torch.cuda.current_stream().cuda_stream
    qkv_d = _dev(qkv, "bf16")
    outs = []
    for window in (0, T, T + 5):
        O = torch.zeros(B * T, H * 128, dtype=torch.bfloat16, device="cuda")
        lse = torch.zeros(B, H, T, dtype=torch.float32, device="cuda")
        assert nc.nc_attention_fwd(qkv_d.data_ptr(), ld, O.data_ptr(), lse.data_ptr(), B, T, H, nc.NC_BF16, 0, st,
                                   window=window) == 0
        outs.append((O.view(torch.int16).cpu(), lse.cpu()))
    for O, lse in outs[1:]:
        assert torch.equal(O, outs[0][0]) and torch.equal(lse, outs[0][1])


CUT_CASES = [(1, 130, 3, 0), (1, 515, 10, 0), (1, 515, 3, 64), (1, 1030, 2, 384), (1, 300, 10, 200),
             (3, 1024, 4, 0)]


@pytest.mark.parametrize("B,T,H,window", CUT_CASES)
def test_attention_bwd_with_cut_key_tiles(nc, B, T, H, window):
    # nc_attention_bwd_ex with its scratch cuts the dK/dV work of the larger key
    # tiles into pieces whose fp32 partial sums a second kernel adds in piece
    # order: against the oracle, against the uncut call (dq bit-identical: the
    # same dQ kernel), and bit-identical from one call to the next
    import torch

    from oracle import full_block as fb
    qkv, ld, q, k, v = _attn_inputs(B, T, H, 500 + T + H + window, "bf16")
    st = torch.cuda.current_stream().cuda_stream
    qkv_d = _dev(qkv, "bf16")
    O = torch.zeros(B * T, H * 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(B, H, T, dtype=torch.float32, device="cuda")
    assert nc.nc_attention_fwd(qkv_d.data_ptr(), ld, O.data_ptr(), lse.data_ptr(), B, T, H, nc.NC_BF16, 0, st,
                               window=window) == 0
    dO = _bf16(synth.normal(11 + T, 4, B * T * H * 128).reshape(B * T, H * 128))
    dO_d = _dev(dO, "bf16")
    rc, nbytes = nc.nc_attention_bwd_scratch_bytes(B, T, H, window)
    assert rc == nc.NC_OK and nbytes > 0, "these shapes are cut"
    scratch = torch.full((nbytes // 4,), float("nan"), dtype=torch.float32, device="cuda")
    Drow = torch.zeros(B, H, T, dtype=torch.float32, device="cuda")
    runs = []
    for _ in range(2):
        dqkv = torch.zeros(B * T, ld, dtype=torch.bfloat16, device="cuda")
        assert nc.nc_attention_bwd_ex(qkv_d.data_ptr(), ld, O.data_ptr(), dO_d.data_ptr(), lse.data_ptr(),
                                      Drow.data_ptr(), scratch.data_ptr(), nbytes, dqkv.data_ptr(), B, T, H,
                                      nc.NC_BF16, 0, st, window=window) == 0
        runs.append(dqkv)
    whole = torch.zeros(B * T, ld, dtype=torch.bfloat16, device="cuda")
    assert nc.nc_attention_bwd(qkv_d.data_ptr(), ld, O.data_ptr(), dO_d.data_ptr(), lse.data_ptr(),
                               Drow.data_ptr(), whole.data_ptr(), B, T, H, nc.NC_BF16, 0, st, window=window) == 0
    assert nc.nc_ops_status(st, 60000) == nc.NC_OK
    assert torch.equal(runs[0].view(torch.int16), runs[1].view(torch.int16)), "cut schedule is deterministic"
    assert torch.equal(runs[0][:, :H * 128].view(torch.int16), whole[:, :H * 128].view(torch.int16))
    got = runs[0].float().cpu().numpy().astype(np.float64)
    uncut = whole.float().cpu().numpy().astype(np.float64)
    # the cut changes only the order of fp32 sums before one bf16 rounding
    kv = slice(H * 128, ld)
    assert np.max(np.abs(got[:, kv] - uncut[:, kv])) <= 2.0 ** -7 * np.abs(uncut[:, kv]).max()
    refs = [np.empty((B, T, 128)), np.empty((B, T, 128))]
    for b in range(B):
        # (window None: the full-block oracle's plain causal mask)
        _, refs[0][b], refs[1][b] = fb.attention_bwd(dO.reshape(B, T, H, 128)[b], q[b], k[b], v[b], window or None)
    for g, r in ((got[:, H * 128:H * 128 + 128], refs[0].reshape(B * T, -1)),
                 (got[:, H * 128 + 128:], refs[1].reshape(B * T, -1))):
        cos = np.sum(g * r) / (np.linalg.norm(g) * np.linalg.norm(r) + 1e-300)
        assert cos > 0.9995, cos
        assert np.max(np.abs(g - r)) <= 3e-2 * np.abs(r).max()


PERSIST_CASES = [(1, 515, 3, 0), (2, 300, 2, 0), (1, 515, 3, 64), (1, 1030, 2, 384), (2, 512, 2, 1)]


@pytest.mark.parametrize("B,T,H,window", PERSIST_CASES)
def test_persistent_attention_with_few_ctas(nc, B, T, H, window):
    # the persistent forward and dQ kernels with their CTA count capped at 3,
    # so every CTA walks several query tiles (one-key-tile tiles among them):
    # bit-identical to one CTA per SM (each tile's arithmetic is the same),
    # and against the oracle through the earlier tests' tolerances
    import torch

    from oracle import full_block as fb
    qkv, ld, q, k, v = _attn_inputs(B, T, H, 700 + T + H + window, "bf16")
    st = torch.cuda.current_stream().cuda_stream
    qkv_d = _dev(qkv, "bf16")
    dO = _bf16(synth.normal(13 + T, 4, B * T * H * 128).reshape(B * T, H * 128))
    dO_d = _dev(dO, "bf16")
    outs = []
    try:
        for cap in (0, 3, 0):
            assert nc.nc_set_attention_ctas(cap) == nc.NC_OK
            O = torch.zeros(B * T, H * 128, dtype=torch.bfloat16, device="cuda")
            lse = torch.zeros(B, H, T, dtype=torch.float32, device="cuda")
            assert nc.nc_attention_fwd(qkv_d.data_ptr(), ld, O.data_ptr(), lse.data_ptr(), B, T, H, nc.NC_BF16, 0,
                                       st, window=window) == 0
            Drow = torch.zeros(B, H, T, dtype=torch.float32, device="cuda")
            dqkv = torch.zeros(B * T, ld, dtype=torch.bfloat16, device="cuda")
            assert nc.nc_attention_bwd(qkv_d.data_ptr(), ld, O.data_ptr(), dO_d.data_ptr(), lse.data_ptr(),
                                       Drow.data_ptr(), dqkv.data_ptr(), B, T, H, nc.NC_BF16, 0, st,
                                       window=window) == 0
            assert nc.nc_ops_status(st, 60000) == nc.NC_OK
            outs.append((O.view(torch.int16).cpu(), lse.cpu(), dqkv.view(torch.int16).cpu(), Drow.cpu()))
    finally:
        nc.nc_set_attention_ctas(0)
    for a, b in zip(outs[0], outs[1]):
        assert torch.equal(a, b), "capped CTAs change no bit"
    got = outs[1][2].view(torch.bfloat16).float().numpy().astype(np.float64)
    dq_ref = np.empty((B, T, H, 128))
    for bb in range(B):
        dq_ref[bb], _, _ = fb.attention_bwd(dO.reshape(B, T, H, 128)[bb], q[bb], k[bb], v[bb], window or None)
    g, r = got[:, :H * 128], dq_ref.reshape(B * T, -1)
    if window == 1:
        assert np.max(np.abs(g)) <= 1e-5 * np.abs(v).max()
    else:
        cos = np.sum(g * r) / (np.linalg.norm(g) * np.linalg.norm(r) + 1e-300)
        assert cos > 0.9995, cos
