"""The four bf16 workloads at the sizes bench.py runs (d12: B=8 x T=1024;
d20: 16 x 2048; d24: 8 x 2048; d32: 4 x 2048), checked against the fp64
oracle where it can follow:

  * full-size step: the per-token losses of one sampled row against the
    oracle's forward pass over that row alone (rows are independent in the
    forward pass), the loss as the mean of the token losses, and gradient
    properties that hold at any size -- the scale invariances the
    parameterless norms create (<dWq_h, Wq_h> = <dWk, Wk> = 0,
    <dwte_v, wte_v> = 0), zero rows for tokens that never occur, finiteness;
  * oracle-sized step: loss and every gradient against the oracle on the
    full d12 workload and on one-row slices (B=1 at the workload's T=2048)
    of d20, d24 and d32, with the bf16 tolerances |dloss| <= 1e-2 and
    per-tensor cosine >= 0.999.
"""
import numpy as np
import pytest

import oracle
import synth
from tests._gpu_helpers import compare, cosine, gpu_step, split_grads, token_loss_bound

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from decoder_only_transformer_nanochat_b200 import build
    build.build()
    return torch


def _model(wl):
    from decoder_only_transformer_nanochat_b200 import Model
    return Model(wl.depth, vocab=wl.vocab, seq=wl.seq, dtype=wl.dtype)


@pytest.mark.parametrize("name", ["d12", "d20", "d24", "d32"])
def test_full_size_step(torch_cuda, name):
    wl = synth.WORKLOADS[name]
    lay = oracle.param_layout(wl.depth, wl.vocab)
    flat, W = synth.make_weights(lay, wl.seed, wl.dtype)
    tok, tgt = synth.token_rows(wl.seed, wl.B, wl.T, wl.vocab, wl.tokens)
    model = _model(wl)
    rc, loss, tl, g = gpu_step(model, flat, tok, tgt, wl.dtype)
    del model
    assert rc == 0
    assert np.isfinite(loss) and np.all(np.isfinite(g))
    assert abs(loss - tl.mean()) <= 1e-4 * abs(loss)

    # sampled row vs the oracle's forward over that row alone
    b = wl.B - 1
    _, tl_ref = oracle.forward_loss(W, tok[b:b + 1], tgt[b:b + 1], wl.depth)
    d = np.abs(tl[b] - tl_ref[0])
    from tests._gpu_helpers import record
    record("full_size_row", tag=name, tl_max=float(d.max()), tl_mean=float(d.mean()))
    bound = token_loss_bound(W["lm_head"])
    assert d.max() <= bound and d.mean() <= bound / 4, (d.mean(), d.max(), bound)

    G = split_grads(g, lay)
    for name_, _, _ in lay:
        assert np.any(G[name_] != 0.0), name_
    # scale invariances of the parameterless norms
    for l in range(wl.depth):
        wq, dwq = W[f"h{l}.wq"], G[f"h{l}.wq"]
        for h in range(wq.shape[0] // 128):
            rows = slice(128 * h, 128 * (h + 1))
            assert abs(cosine(dwq[rows], wq[rows])) <= 1e-2, (l, h)
        assert abs(cosine(G[f"h{l}.wk"], W[f"h{l}.wk"])) <= 1e-2, l
    used = np.unique(tok)
    dots = np.sum(G["wte"][used] * W["wte"][used], axis=1)
    norms = np.linalg.norm(G["wte"][used], axis=1) * np.linalg.norm(W["wte"][used], axis=1)
    assert np.max(np.abs(dots) / norms) <= 2e-2
    unused = np.setdiff1d(np.arange(wl.vocab), used)
    assert unused.size > 0 and np.all(G["wte"][unused] == 0.0)


SLICES = [("d12", 8, 1024), ("d20", 1, 2048), ("d24", 1, 2048), ("d32", 1, 2048)]


@pytest.mark.parametrize("name,B,T", SLICES)
def test_oracle_sized_step(torch_cuda, name, B, T):
    wl = synth.WORKLOADS[name]
    lay = oracle.param_layout(wl.depth, wl.vocab)
    flat, W = synth.make_weights(lay, wl.seed, wl.dtype)
    tok, tgt = synth.token_rows(wl.seed, wl.B, wl.T, wl.vocab, wl.tokens)
    tok, tgt = np.ascontiguousarray(tok[:B, :T]), np.ascontiguousarray(tgt[:B, :T])
    model = _model(wl)
    rc, loss, tl, g = gpu_step(model, flat, tok, tgt, wl.dtype)
    del model
    assert rc == 0
    loss_ref, tl_ref, g_ref = oracle.loss_and_grads(W, tok, tgt, wl.depth)
    compare(wl.dtype, lay, loss, g, loss_ref, g_ref, tl, tl_ref, tag=f"{name}-B{B}-T{T}",
            tl_bound=token_loss_bound(W["lm_head"]))
