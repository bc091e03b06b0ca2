"""The full reference block on the GPU -- sliding-window "SSSL" attention,
gated value embeddings, residual scalars -- against the fp64 full-block
oracle (oracle/full_block.py) on the same seeded inputs, through the C ABI.

Cases span the pages' window schedule at windows 1, 64, 129 and 1,024 (the
pages' short window), ragged T and vocabularies, one and several query
heads, fp32 (loss relative error <= 1e-5, per-tensor max-abs gradient error
<= 1e-4 max|grad|) and bf16 (|dloss| <= 1e-2, per-tensor cosine >= 0.999),
each feature alone and all together.  Features that are off are neutral in
the oracle: resid_lambdas 1, x0_lambdas 0, gates 0, no window.

The value-embedding gate is one scalar per layer: the pages name the gate
without its form, so this part is checked for consistency with the oracle's
reading, not against nanochat itself.
"""
import numpy as np
import pytest

import oracle
import synth
from oracle import full_block as fb
from tests._gpu_helpers import compare, gpu_step, split_grads, token_loss_bound

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from decoder_only_transformer_nanochat_b200 import build
    build.build()
    return torch


def _case(depth, V, B, T, dtype, seed, window, ve, scalars, dist="zipf", head_std=None):
    from decoder_only_transformer_nanochat_b200 import Model
    model = Model(depth, vocab=V, seq=T, dtype=dtype, window=window, value_embeds=ve, resid_scalars=scalars)
    lay = [(n, r, c) for n, _, r, c in model.layout]
    n_ve = len(fb.ve_layers(depth))
    # scalars away from special values, so every term of their gradients acts
    values = {"resid_lambdas": np.array([[0.9 + 0.05 * l for l in range(depth)]]),
              "x0_lambdas": np.array([[0.15 - 0.01 * l for l in range(depth)]]),
              "ve_gates": np.array([[0.7 + 0.1 * i for i in range(n_ve)]])}
    std = {"lm_head": head_std} if head_std is not None else None
    flat, W = synth.make_weights(lay, seed, dtype, std_override=std, values=values)
    W = dict(W)
    # the oracle's neutral extras for the features that are off
    full = fb.full_param_layout(depth, V)
    if not ve:
        for name, r, c in full:
            if name.startswith("ve") and name[2:].isdigit():
                W[name] = np.zeros((r, c))
        W["ve_gates"] = np.zeros((1, n_ve))
    if not scalars:
        W["resid_lambdas"] = np.ones((1, depth))
        W["x0_lambdas"] = np.zeros((1, depth))
    windows = fb.window_schedule(depth, short=window) if window else [None] * depth
    assert model.windows == [w or 0 for w in windows]
    tok, tgt = synth.token_rows(seed, B, T, V, dist)
    return model, lay, flat, W, tok, tgt, windows


CASES = [
    # depth, V, B, T, dtype, seed, window, value embeds, residual scalars, head std
    (2, 96, 2, 9, "f32", 11, 4, True, True, 0.5),         # H=1, vocab tail, window inside one tile
    (4, 1000, 2, 150, "f32", 12, 64, True, True, 0.3),    # ragged T and V, SSS then L
    (5, 700, 1, 300, "f32", 13, 1, True, True, 0.3),      # window 1: each S layer sees only itself
    (4, 65536, 2, 256, "bf16", 14, 129, True, True, None),
    (6, 5000, 2, 200, "bf16", 15, 64, True, True, 0.05),  # H=3
    (4, 4096, 1, 515, "bf16", 16, 129, False, False, 0.05),   # windows alone
    (4, 4096, 1, 300, "bf16", 17, 0, True, False, 0.05),      # value embeddings alone
    (4, 4096, 1, 300, "bf16", 18, 0, False, True, 0.05),      # residual scalars alone
    (12, 65536, 1, 1536, "bf16", 19, 1024, True, True, None),  # d12 width, the pages' 1,024 window
]


@pytest.mark.parametrize("depth,V,B,T,dtype,seed,window,ve,scalars,hstd", CASES)
def test_full_block_step_matches_oracle(torch_cuda, depth, V, B, T, dtype, seed, window, ve, scalars, hstd):
    model, lay, flat, W, tok, tgt, windows = _case(depth, V, B, T, dtype, seed, window, ve, scalars,
                                                   dist="uniform" if dtype == "f32" else "zipf", head_std=hstd)
    rc, loss, tl, g = gpu_step(model, flat, tok, tgt, dtype)
    assert rc == 0
    loss_ref, tl_ref, g_ref = fb.loss_and_grads(W, tok, tgt, depth, windows=windows)
    compare(dtype, lay, loss, g, loss_ref, g_ref, tl, tl_ref,
            tag=f"full-d{depth}-V{V}-B{B}-T{T}-{dtype}-w{window}-ve{int(ve)}-s{int(scalars)}",
            tl_bound=token_loss_bound(W["lm_head"]))
    G = split_grads(g, lay)
    if ve:
        # rows of tokens that never occur get no value-embedding gradient
        unused = np.setdiff1d(np.arange(V), tok)
        for l in fb.ve_layers(depth):
            assert np.all(G[f"ve{l}"][unused] == 0.0)


def test_neutral_full_block_is_the_baseline(torch_cuda):
    # all features on but neutral (no window reaching below T, gates 0,
    # resid 1, x0 0) gives the baseline model's loss and gradients
    torch = torch_cuda
    from decoder_only_transformer_nanochat_b200 import Model
    depth, V, B, T = 4, 1000, 2, 100
    base = Model(depth, vocab=V, seq=T, dtype="f32")
    full = Model(depth, vocab=V, seq=T, dtype="f32", window=T, value_embeds=True, resid_scalars=True)
    lay_b = [(n, r, c) for n, _, r, c in base.layout]
    lay_f = [(n, r, c) for n, _, r, c in full.layout]
    n_ve = len(fb.ve_layers(depth))
    flat_f, _ = synth.make_weights(lay_f, 5, "f32", values=synth.full_block_values(depth, n_ve, 1.0, 0.0, 0.0))
    nb = sum(r * c for _, r, c in lay_b)
    tok, tgt = synth.token_rows(5, B, T, V, "uniform")
    rb = gpu_step(base, flat_f[:nb].copy(), tok, tgt, "f32")
    rf = gpu_step(full, flat_f, tok, tgt, "f32")
    assert rb[0] == 0 and rf[0] == 0
    assert abs(rb[1] - rf[1]) <= 1e-6 * abs(rb[1])
    gb, gf = rb[3], rf[3][:nb]
    assert np.max(np.abs(gb - gf)) <= 1e-5 * np.abs(gb).max()
