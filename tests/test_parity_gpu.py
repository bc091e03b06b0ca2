"""CUDA step vs the fp64 oracle on the same seeded inputs, through the C ABI.

Small cases span several GEMM / attention tiles and ragged tails (T not a
multiple of the tile, vocab not a multiple of the tile, one query head);
the d4 workload runs at its full size.  Tolerances: fp32 -- loss relative
error <= 1e-5 and per-tensor max-abs gradient error <= 1e-4 max|grad|;
bf16 -- |dloss| <= 1e-2 and per-tensor gradient cosine >= 0.999.
"""
import numpy as np
import pytest

import oracle
import synth
from tests._gpu_helpers import compare, cosine, gpu_step, make_case, split_grads, to_device, token_loss_bound

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from decoder_only_transformer_nanochat_b200 import build
    build.build()
    return torch


def _model(depth, V, seq, dtype):
    from decoder_only_transformer_nanochat_b200 import Model
    return Model(depth, vocab=V, seq=seq, dtype=dtype)


def _check_layout(model, lay):
    assert [(n, r, c) for n, _, r, c in model.layout] == lay
    off = 0
    for (n, o, r, c) in model.layout:
        assert o == off
        off += r * c


CASES = [
    # depth, V, B, T, dtype, seed, dist, head std
    (2, 96, 2, 9, "f32", 11, "uniform", 0.5),        # H=1, vocab tail, T < one tile
    (4, 1000, 3, 77, "f32", 12, "uniform", 0.3),     # H=2, ragged T and V
    (4, 65536, 2, 256, "f32", 0, "uniform", None),   # the d4 workload at full size
    (4, 65536, 2, 256, "bf16", 13, "zipf", None),
    (6, 5000, 2, 200, "bf16", 14, "zipf", 0.05),     # H=3, ragged V and T
    (2, 65536, 3, 130, "bf16", 15, "zipf", 0.02),    # H=1, T just above a tile
]


@pytest.mark.parametrize("depth,V,B,T,dtype,seed,dist,hstd", CASES)
def test_step_matches_oracle(torch_cuda, depth, V, B, T, dtype, seed, dist, hstd):
    std = {"lm_head": hstd} if hstd is not None else None
    lay, flat, W, tok, tgt = make_case(depth, V, B, T, dtype, seed, dist, std)
    model = _model(depth, V, max(T, 16), dtype)
    _check_layout(model, lay)
    rc, loss, tl, g = gpu_step(model, flat, tok, tgt, dtype)
    assert rc == 0
    loss_ref, tl_ref, g_ref = oracle.loss_and_grads(W, tok, tgt, depth)
    compare(dtype, lay, loss, g, loss_ref, g_ref, tl, tl_ref, tag=f"d{depth}-V{V}-B{B}-T{T}-{dtype}",
            tl_bound=token_loss_bound(W["lm_head"]))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_forward_logits_match_oracle(torch_cuda, dtype):
    torch = torch_cuda
    depth, V, B, T = 4, 3000, 2, 70
    lay, flat, W, tok, tgt = make_case(depth, V, B, T, dtype, 21, "uniform", {"lm_head": 0.5})
    model = _model(depth, V, 128, dtype)
    logits = model.fwd(to_device(flat, dtype), torch.from_numpy(tok).cuda())
    assert model.sync_status(60000) == 0
    got = logits.float().cpu().numpy().astype(np.float64)
    ref = oracle.forward_logits(W, tok, depth)
    assert np.max(np.abs(got)) <= 15.0
    if dtype == "f32":
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-4 * np.abs(ref).max())
    else:
        # bf16 activations and logits: a few bf16 roundings of values up to 15
        assert np.max(np.abs(got - ref)) <= 0.03 * np.abs(ref).max()
        assert np.mean(np.abs(got - ref)) <= 0.01 * np.mean(np.abs(ref))
        c = np.sum(got * ref) / np.linalg.norm(got) / np.linalg.norm(ref)
        assert c > 0.9995


def test_zero_unembedding_gives_ln_vocab(torch_cuda):
    # W_out = 0: every logit is 0, loss = ln V, and only the unembedding has a gradient
    depth, V, B, T = 4, 65536, 2, 64
    lay, flat, W, tok, tgt = make_case(depth, V, B, T, "bf16", 3, "zipf", {"lm_head": 0.0})
    model = _model(depth, V, 64, "bf16")
    rc, loss, tl, g = gpu_step(model, flat, tok, tgt, "bf16")
    assert rc == 0
    assert abs(loss - np.log(V)) < 1e-3
    n_head = V * 256
    assert np.all(g[:-n_head] == 0.0)
    assert np.any(g[-n_head:] != 0.0)


def test_error_paths(torch_cuda):
    torch = torch_cuda
    import decoder_only_transformer_nanochat_b200 as nc
    depth, V, B, T = 2, 512, 1, 32
    lay, flat, W, tok, tgt = make_case(depth, V, B, T, "f32", 5, "uniform")
    model = _model(depth, V, 32, "f32")
    w = to_device(flat, "f32")
    t = torch.from_numpy(tok).cuda()
    g = torch.from_numpy(tgt).cuda()
    loss = torch.empty(1, device="cuda")
    grads = torch.empty(model.n_params, device="cuda")
    rc, need = nc.nc_workspace_bytes(model.handle, B, T)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    args = lambda Bb, Tt, wsb: (model.handle, w.data_ptr(), t.data_ptr(), g.data_ptr(), Bb, Tt,
                                ws.data_ptr(), wsb, loss.data_ptr(), None, grads.data_ptr(), st)
    assert nc.nc_fwd_bwd(*args(B, 33, need)) == nc.NC_ESHAPE      # T > seq
    assert nc.nc_fwd_bwd(*args(0, T, need)) == nc.NC_ESHAPE
    assert nc.nc_fwd_bwd(*args(B, T, need - 1)) == nc.NC_ENOMEM
    assert nc.nc_workspace_bytes(model.handle, B, 33)[0] == nc.NC_ESHAPE
    assert nc.nc_param_layout(model.handle, 2 + 6 * depth)[0] == nc.NC_EINVAL
    assert nc.nc_fwd_bwd(*args(B, T, need)) == nc.NC_OK
    assert nc.nc_sync_status(model.handle, st, 60000) == nc.NC_OK
    # an out-of-range token is flagged on the device and read back once
    t[0, 3] = V + 7
    assert nc.nc_fwd_bwd(*args(B, T, need)) == nc.NC_OK
    assert nc.nc_sync_status(model.handle, st, 60000) == nc.NC_ERANGE
    assert nc.nc_sync_status(model.handle, st, 60000) == nc.NC_OK
    t[0, 3] = 1
    g[0, 5] = -1
    assert nc.nc_fwd_bwd(*args(B, T, need)) == nc.NC_OK
    assert nc.nc_sync_status(model.handle, st, 60000) == nc.NC_ERANGE
    # NaN weights give a non-finite loss
    g[0, 5] = 1
    w2 = w.clone()
    w2[-5] = float("nan")
    rc = nc.nc_fwd_bwd(model.handle, w2.data_ptr(), t.data_ptr(), g.data_ptr(), B, T, ws.data_ptr(),
                       need, loss.data_ptr(), None, grads.data_ptr(), st)
    assert rc == nc.NC_OK
    assert nc.nc_sync_status(model.handle, st, 60000) == nc.NC_ENONFINITE
    # a zero timeout on a busy stream reports a timeout instead of blocking
    big = torch.empty(1 << 28, device="cuda")
    for _ in range(20):
        big.mul_(1.0001)
    assert nc.nc_sync_status(model.handle, st, 0) in (nc.NC_ETIMEOUT, nc.NC_OK)
    torch.cuda.synchronize()


def _token_patterns(V, B, T):
    """Token rows that put segment boundaries where the summation's chunks
    (16 sorted positions each) make them delicate."""
    M = B * T
    same = np.full(M, 5)                                   # one segment over every chunk
    distinct = np.arange(M) % V                            # runs of one (V >= M) or a few
    runs16 = (np.arange(M) // 16) % V                      # every run ends on a chunk boundary
    runs17 = (np.arange(M) // 17) % V                      # runs cross boundaries by one
    mixed = np.where(np.arange(M) % 3 == 0, 0, (np.arange(M) * 7919) % V)  # one hot token among scattered ones
    return {"same": same, "distinct": distinct, "runs16": runs16, "runs17": runs17, "mixed": mixed}


@pytest.mark.parametrize("pattern", ["same", "distinct", "runs16", "runs17", "mixed"])
def test_embedding_gradient_segments(torch_cuda, pattern):
    # fp32 model: the embedding gradient row by row against the oracle, with
    # the tokens in shuffled order so that positions of a token are far apart
    depth, V, B, T = 2, 700, 2, 150
    lay, flat, W, _, tgt = make_case(depth, V, B, T, "f32", 17, "uniform", {"lm_head": 0.5})
    toks = _token_patterns(V, B, T)[pattern]
    perm = np.argsort(synth.uniform01(23, 1, B * T))
    tok = np.ascontiguousarray(toks[perm].reshape(B, T).astype(np.int32))
    model = _model(depth, V, T, "f32")
    rc, loss, tl, g = gpu_step(model, flat, tok, tgt, "f32")
    assert rc == 0
    loss_ref, tl_ref, g_ref = oracle.loss_and_grads(W, tok, tgt, depth)
    compare("f32", lay, loss, g, loss_ref, g_ref, tl, tl_ref, tag=f"segments-{pattern}")
    dwte = g[:V * 128].reshape(V, 128)
    ref = g_ref["wte"]
    absent = np.setdiff1d(np.arange(V), tok)
    assert np.all(dwte[absent] == 0.0)
    np.testing.assert_allclose(dwte, ref, rtol=0, atol=1e-4 * np.abs(ref).max())


def test_deterministic_step(torch_cuda):
    # Loss, token losses and the embedding and unembedding gradients are
    # bit-identical run to run (fixed summation orders, no floating-point
    # atomics).  The weight gradients of the blocks split their reductions
    # over K across CTAs that add into fp32 in arrival order, so those may
    # differ in the last bits; they are compared to the gradient tolerance.
    depth, V, B, T = 4, 65536, 2, 128
    lay, flat, W, tok, tgt = make_case(depth, V, B, T, "bf16", 6, "zipf")
    model = _model(depth, V, 128, "bf16")
    r1 = gpu_step(model, flat, tok, tgt, "bf16")
    r2 = gpu_step(model, flat, tok, tgt, "bf16")
    assert r1[1] == r2[1]
    np.testing.assert_array_equal(r1[2], r2[2])
    g1, g2 = split_grads(r1[3], lay), split_grads(r2[3], lay)
    np.testing.assert_array_equal(g1["wte"], g2["wte"])
    np.testing.assert_array_equal(g1["lm_head"], g2["lm_head"])
    for name, _, _ in lay:
        assert cosine(g1[name], g2[name]) >= 1 - 1e-6, name
