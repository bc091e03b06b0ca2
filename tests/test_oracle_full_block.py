"""Pins of the full-block oracle (oracle.full_block): SSSL sliding-window
attention, value embeddings and per-layer residual scalars.

Each pin checks the oracle against something other than itself: the schedule
the pages spell out, a brute-force evaluation with Python loops, a closed form
(a one-token window returns v), the baseline model that the block reduces to
when its extra parameters are neutral, a window that covers the whole context,
and central finite differences on every tensor.  Citations: p1 = "Nanochat:
full-stack LLM training in 8,000 lines for $72", section "A Llama-class
transformer with ten modern departures"; p4 = "nanochat - full-stack ChatGPT
in ~8k lines", section "0. The model".
"""
import math

import numpy as np
import pytest

import oracle
import synth
from oracle import full_block as fb


def _tiny(depth=2, V=48, B=2, T=9, seed=11):
    lay = fb.full_param_layout(depth, V)
    _, W = synth.make_weights(lay, seed, "f32", std_override={"lm_head": 0.5})
    W = dict(W)
    # scalars away from special values, so every term of their gradients acts
    W["resid_lambdas"] = np.array([[0.9 + 0.1 * l for l in range(depth)]])
    W["x0_lambdas"] = np.array([[0.15 - 0.04 * l for l in range(depth)]])
    W["ve_gates"] = np.array([[0.7 + 0.2 * i for i in range(len(fb.ve_layers(depth)))]])
    tok, tgt = synth.token_rows(seed, B, T, V, "uniform")
    return lay, W, tok, tgt


# ---------------------------------------------------------------------------
# the schedule (p1: three short-window layers of 1,024 tokens, then one with
# the full 2,048 context, the final layer always full; p4: window_pattern "SSSL")

def test_sssl_schedule_as_the_pages_state_it():
    w = fb.window_schedule(20)
    assert len(w) == 20
    for l in range(20):
        expect_long = (l % 4 == 3) or l == 19
        assert (w[l] is None) == expect_long, l
        if not expect_long:
            assert w[l] == 1024
    assert fb.window_schedule(6) == [1024, 1024, 1024, None, 1024, None]
    assert fb.window_schedule(1) == [None]
    # three short layers for every long one: depth 16 has long layers 3, 7, 11, 15
    assert sum(x is not None for x in fb.window_schedule(16)) == 12


def test_init_values_of_the_residual_scalars():
    W = fb.init_scalars({}, 5)
    assert np.all(W["resid_lambdas"] == 1.0) and np.all(W["x0_lambdas"] == 0.1)
    assert W["ve_gates"].shape == (1, 3)  # layers 0, 2, 4


# ---------------------------------------------------------------------------
# windowed attention

def _brute_force(q, k, v, window):
    T, H, d = q.shape
    O = np.zeros_like(q)
    for h in range(H):
        for i in range(T):
            keys = [j for j in range(T) if j <= i and (window is None or i - j < window)]
            s = [sum(q[i, h, t] * k[j, t] for t in range(d)) / math.sqrt(d) for j in keys]
            m = max(s)
            e = [math.exp(x - m) for x in s]
            z = sum(e)
            for t in range(d):
                O[i, h, t] = sum(e[n] * v[keys[n], t] for n in range(len(keys))) / z
    return O


@pytest.mark.parametrize("window", [1, 3, None])
def test_windowed_attention_against_loops(window):
    rng = np.random.default_rng(3)
    T, H, d = 7, 2, 128
    q, k, v = rng.standard_normal((T, H, d)), rng.standard_normal((T, d)), rng.standard_normal((T, d))
    O, _ = fb.attention(q, k, v, window)
    np.testing.assert_allclose(O, _brute_force(q, k, v, window), rtol=1e-11, atol=1e-11)


def test_one_token_window_returns_v():
    rng = np.random.default_rng(4)
    T, H, d = 11, 3, 128
    q, k, v = rng.standard_normal((T, H, d)), rng.standard_normal((T, d)), rng.standard_normal((T, d))
    O, lse = fb.attention(q, k, v, 1)
    for h in range(H):
        assert np.array_equal(O[:, h, :], v)
        np.testing.assert_allclose(lse[h], np.sum(q[:, h, :] * k, axis=1) / math.sqrt(d), rtol=1e-13)


def test_window_covering_the_context_is_plain_causal():
    lay, W, tok, tgt = _tiny(depth=3)
    T = tok.shape[1]
    l1, _, g1 = fb.loss_and_grads(W, tok, tgt, 3, windows=[T, T + 5, None])
    l2, _, g2 = fb.loss_and_grads(W, tok, tgt, 3, windows=[None, None, None])
    assert l1 == l2
    for name in g2:
        assert np.array_equal(g1[name], g2[name]), name


def test_short_window_changes_only_layers_that_have_one():
    # with T <= window nothing changes; with a small window the loss moves
    lay, W, tok, tgt = _tiny(depth=2, T=9)
    base, _ = fb.forward_loss(W, tok, tgt, 2, windows=[None, None])
    assert fb.forward_loss(W, tok, tgt, 2, windows=[9, None])[0] == base
    assert fb.forward_loss(W, tok, tgt, 2, windows=[3, None])[0] != base


# ---------------------------------------------------------------------------
# neutral extra parameters give back the baseline model exactly

def test_neutral_block_is_the_baseline():
    depth, V = 3, 48
    lay, W, tok, tgt = _tiny(depth=depth, V=V)
    W["resid_lambdas"][:] = 1.0
    W["x0_lambdas"][:] = 0.0
    W["ve_gates"][:] = 0.0
    loss, tl, g = fb.loss_and_grads(W, tok, tgt, depth, windows=[None] * depth)
    loss0, tl0, g0 = oracle.loss_and_grads(W, tok, tgt, depth)
    np.testing.assert_allclose(tl, tl0, rtol=1e-13, atol=0)
    for name, _, _ in oracle.param_layout(depth, V):
        np.testing.assert_allclose(g[name], g0[name], rtol=1e-11, atol=1e-14 * np.abs(g0[name]).max(),
                                   err_msg=name)
    # the tables get no gradient through a zero gate, the gate itself does
    for l in fb.ve_layers(depth):
        assert np.all(g[f"ve{l}"] == 0.0)
    assert np.all(np.abs(g["ve_gates"]) > 0)


def test_value_embedding_rows_of_absent_tokens_get_no_gradient():
    lay, W, tok, tgt = _tiny(depth=2, V=48)
    _, _, g = fb.loss_and_grads(W, tok, tgt, 2, windows=[4, None])
    unused = np.setdiff1d(np.arange(48), tok.reshape(-1))
    assert unused.size > 0
    assert np.all(g["ve0"][unused] == 0.0)


# ---------------------------------------------------------------------------
# whole backward of the full block: central finite differences on every tensor

def test_finite_differences_every_tensor_full_block():
    depth = 2
    lay, W, tok, tgt = _tiny(depth=depth)
    windows = fb.window_schedule(depth, short=4)  # [4, None]: the short window is active at T = 9
    assert windows == [4, None]
    loss, _, g = fb.loss_and_grads(W, tok, tgt, depth, windows=windows)
    rng = np.random.default_rng(5)
    flat_tok = tok.reshape(-1)
    for name, rows, cols in lay:
        w = W[name]
        gmax = np.abs(g[name]).max()
        assert gmax > 0, name
        for _ in range(3):
            if name == "wte" or (name.startswith("ve") and name[2:].isdigit()):  # rows the tokens select
                i = int(flat_tok[rng.integers(flat_tok.size)])
            else:
                i = int(rng.integers(rows))
            j = int(rng.integers(cols))
            h = 1e-5 * max(1.0, abs(w[i, j]))
            old = w[i, j]
            w[i, j] = old + h
            lp, _ = fb.forward_loss(W, tok, tgt, depth, windows=windows)
            w[i, j] = old - h
            lm, _ = fb.forward_loss(W, tok, tgt, depth, windows=windows)
            w[i, j] = old
            fd = (lp - lm) / (2 * h)
            assert abs(fd - g[name][i, j]) <= 1e-6 * gmax, (name, i, j, fd, g[name][i, j])


def test_forward_logits_agree_with_the_loss():
    # the logits function and the loss function share the forward: the loss
    # recomputed from the logits (log-sum-exp minus the target's logit) agrees
    depth = 2
    lay, W, tok, tgt = _tiny(depth=depth)
    windows = fb.window_schedule(depth, short=4)
    s = fb.forward_logits(W, tok, depth, windows=windows)
    m = s.max(axis=2, keepdims=True)
    lse = (m + np.log(np.exp(s - m).sum(axis=2, keepdims=True)))[..., 0]
    tl = lse - np.take_along_axis(s, tgt[..., None], axis=2)[..., 0]
    loss, tl_ref = fb.forward_loss(W, tok, tgt, depth, windows=windows)
    np.testing.assert_allclose(tl, tl_ref, rtol=0, atol=1e-12)
    # causality: logits at position t do not change when later tokens change
    tok2 = tok.copy()
    tok2[:, -1] = (tok2[:, -1] + 1) % W["wte"].shape[0]
    s2 = fb.forward_logits(W, tok2, depth, windows=windows)
    np.testing.assert_array_equal(s[:, :-1], s2[:, :-1])
