"""Pins of the fp64 oracle against what the nanochat pages and mathematics fix.

None of these compares the oracle with itself: each checks a closed form, an
invariant, a brute-force evaluation or a library routine that the method
reduces to in a special case.  Citations name the page and section:
p1 = "Nanochat: full-stack LLM training in 8,000 lines for $72",
p4 = "nanochat - full-stack ChatGPT in ~8k lines", p5 = energyai.berlin walk-through.
"""
import math

import numpy as np
import pytest

import oracle
import synth


def _tiny(depth=4, V=96, B=2, T=9, seed=7, head_std=0.5, dist="uniform"):
    lay = oracle.param_layout(depth, V)
    _, W = synth.make_weights(lay, seed, "f32", std_override={"lm_head": head_std})
    tok, tgt = synth.token_rows(seed, B, T, V, dist)
    return lay, W, tok, tgt


# ---------------------------------------------------------------------------
# one dial (p1 "One dial controls everything"; p4 "How it works": depth 20 ->
# 1280 channels, 10 heads of dim 128)

def test_one_dial_dims():
    assert oracle.dims(20, 65536) == dict(L=20, C=1280, H=10, F=5120, V=65536, d=128)
    for depth, C in [(4, 256), (12, 768), (24, 1536), (32, 2048), (3, 256)]:
        D = oracle.dims(depth, 65536)
        assert D["C"] == C and D["H"] == C // 128 and D["F"] == 4 * C


def test_param_count_mqa():
    # MQA count: L*(2C^2 + 2*128*C + 8C^2) + 2*V*C  (one shared KV head)
    counts = {4: 36_438_016, 20: 502_005_760, 32: 1_627_389_952}
    for depth, n in counts.items():
        lay = oracle.param_layout(depth, 65536)
        assert sum(r * c for _, r, c in lay) == n


# ---------------------------------------------------------------------------
# whole backward: central finite differences in fp64 (H=2 so MQA is exercised)

def test_finite_differences_every_tensor():
    depth = 4
    lay, W, tok, tgt = _tiny(depth=depth)
    loss, _, g = oracle.loss_and_grads(W, tok, tgt, depth)
    rng = np.random.default_rng(0)
    flat_tok = tok.reshape(-1)
    for name, rows, cols in lay:
        w = W[name]
        gmax = np.abs(g[name]).max()
        assert gmax > 0
        for _ in range(3):
            i = int(flat_tok[rng.integers(flat_tok.size)]) if name == "wte" else int(rng.integers(rows))
            j = int(rng.integers(cols))
            h = 1e-5 * max(1.0, abs(w[i, j]))
            old = w[i, j]
            w[i, j] = old + h
            lp, _ = oracle.forward_loss(W, tok, tgt, depth)
            w[i, j] = old - h
            lm, _ = oracle.forward_loss(W, tok, tgt, depth)
            w[i, j] = old
            fd = (lp - lm) / (2 * h)
            assert abs(fd - g[name][i, j]) <= 1e-6 * gmax, (name, i, j, fd, g[name][i, j])


def test_unused_embedding_rows_have_zero_grad():
    lay, W, tok, tgt = _tiny()
    _, _, g = oracle.loss_and_grads(W, tok, tgt, 4)
    unused = np.setdiff1d(np.arange(96), tok.reshape(-1))
    assert unused.size > 0
    assert np.all(g["wte"][unused] == 0.0)


# ---------------------------------------------------------------------------
# parameterless RMSNorm (p1 "ten modern departures": bare F.rms_norm)

def test_rmsnorm_rms_is_one():
    x = synth.normal(3, 1, 64 * 300).reshape(64, 300) * np.linspace(0.01, 100, 64)[:, None]
    y, r = oracle.rmsnorm(x)
    ms = np.mean(x * x, axis=1)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=1)), np.sqrt(ms / (ms + oracle.EPS)), rtol=1e-14)
    big = ms >= 1.0
    assert big.sum() > 30
    np.testing.assert_allclose(np.sqrt(np.mean(y[big] * y[big], axis=1)), 1.0, atol=1e-7)


def test_rmsnorm_bwd_orthogonal_to_input():
    # y is invariant to scaling x, so the gradient is orthogonal to x (up to eps)
    x = synth.normal(4, 1, 16 * 128).reshape(16, 128)
    dy = synth.normal(4, 2, 16 * 128).reshape(16, 128)
    y, r = oracle.rmsnorm(x)
    dx = oracle.rmsnorm_bwd(dy, y, r)
    assert np.max(np.abs(np.sum(dx * x, axis=1))) < 1e-6 * np.max(np.abs(dx))


# ---------------------------------------------------------------------------
# RoPE (p5 "Rotary Position Embeddings": dot products depend on relative
# distance; rotation preserves norms)

def test_rope_preserves_norm_per_pair():
    T = 50
    cos, sin = oracle.rope_tables(T)
    x = synth.normal(5, 1, T * 128).reshape(T, 128)
    y = oracle.rope(x, cos, sin)
    pair = lambda z: z[:, :64] ** 2 + z[:, 64:] ** 2
    np.testing.assert_allclose(pair(y), pair(x), rtol=1e-12)


def test_rope_relative_offset():
    T = 64
    cos, sin = oracle.rope_tables(T)
    q = synth.normal(6, 1, 128)
    k = synth.normal(6, 2, 128)
    Q = oracle.rope(np.tile(q, (T, 1)), cos, sin)
    K = oracle.rope(np.tile(k, (T, 1)), cos, sin)
    for m, n, p in [(10, 3, 20), (5, 5, 40), (0, 7, 30)]:
        assert abs(Q[m] @ K[n] - Q[m + p] @ K[n + p]) < 1e-10
    # position 0 is the identity; angle of pair 0 at position t is t radians
    np.testing.assert_allclose(Q[0], q, atol=0)
    assert abs(cos[3, 0] - math.cos(3.0)) < 1e-15 and abs(sin[1, 63] - math.sin(10000 ** (-63 / 64))) < 1e-15


def test_rope_bwd_is_transpose():
    T = 7
    cos, sin = oracle.rope_tables(T)
    x = synth.normal(8, 1, T * 128).reshape(T, 128)
    dy = synth.normal(8, 2, T * 128).reshape(T, 128)
    assert abs(np.sum(oracle.rope(x, cos, sin) * dy) - np.sum(x * oracle.rope_bwd(dy, cos, sin))) < 1e-10


# ---------------------------------------------------------------------------
# attention (p5 "Multi-Query Attention"; causal)

def _brute_attention(q, k, v):
    """Pure-Python causal softmax attention, one query at a time."""
    T, H, d = q.shape
    O = np.zeros_like(q)
    for h in range(H):
        for i in range(T):
            w = [math.exp(sum(q[i, h, c] * k[j, c] for c in range(d)) / math.sqrt(d)) for j in range(i + 1)]
            Z = sum(w)
            for c in range(d):
                O[i, h, c] = sum(w[j] * v[j, c] for j in range(i + 1)) / Z
    return O


def test_attention_brute_force_mqa():
    T, H = 6, 3
    q = synth.normal(9, 1, T * H * 128).reshape(T, H, 128) * 0.3
    k = synth.normal(9, 2, T * 128).reshape(T, 128) * 0.3
    v = synth.normal(9, 3, T * 128).reshape(T, 128)
    O, lse = oracle.attention(q, k, v)
    np.testing.assert_allclose(O, _brute_attention(q, k, v), rtol=1e-12, atol=1e-13)
    # row 0 attends only to itself: O = v_0, lse = score
    np.testing.assert_allclose(O[0], np.tile(v[0], (H, 1)), rtol=1e-14)
    np.testing.assert_allclose(lse[:, 0], q[0] @ k[0] / math.sqrt(128), rtol=1e-13)


def test_attention_matches_sdpa_fp64():
    torch = pytest.importorskip("torch")
    T, H = 33, 4
    q = synth.normal(10, 1, T * H * 128).reshape(T, H, 128)
    k = synth.normal(10, 2, T * 128).reshape(T, 128)
    v = synth.normal(10, 3, T * 128).reshape(T, 128)
    O, _ = oracle.attention(q, k, v)
    tq = torch.tensor(q).permute(1, 0, 2)[None]
    tk = torch.tensor(k)[None, None].expand(1, H, T, 128)
    tv = torch.tensor(v)[None, None].expand(1, H, T, 128)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
    np.testing.assert_allclose(O, ref[0].permute(1, 0, 2).numpy(), rtol=1e-11, atol=1e-12)


def test_attention_bwd_matches_autograd_fp64():
    torch = pytest.importorskip("torch")
    T, H = 17, 2
    q = synth.normal(11, 1, T * H * 128).reshape(T, H, 128)
    k = synth.normal(11, 2, T * 128).reshape(T, 128)
    v = synth.normal(11, 3, T * 128).reshape(T, 128)
    dO = synth.normal(11, 4, T * H * 128).reshape(T, H, 128)
    dq, dk, dv = oracle.attention_bwd(dO, q, k, v)
    tq = torch.tensor(q, requires_grad=True)
    tk = torch.tensor(k, requires_grad=True)
    tv = torch.tensor(v, requires_grad=True)
    o = torch.nn.functional.scaled_dot_product_attention(
        tq.permute(1, 0, 2)[None], tk[None, None].expand(1, H, T, 128),
        tv[None, None].expand(1, H, T, 128), is_causal=True)
    o.backward(torch.tensor(dO).permute(1, 0, 2)[None])
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_attention_T1_returns_v():
    q = synth.normal(12, 1, 5 * 128).reshape(1, 5, 128)
    k = synth.normal(12, 2, 128).reshape(1, 128)
    v = synth.normal(12, 3, 128).reshape(1, 128)
    O, _ = oracle.attention(q, k, v)
    np.testing.assert_array_equal(O[0], np.tile(v[0], (5, 1)))


def test_causality_future_tokens_do_not_change_past_losses():
    lay, W, tok, tgt = _tiny(T=12)
    _, tl = oracle.forward_loss(W, tok, tgt, 4)
    tok2 = tok.copy()
    tok2[:, 8:] = (tok2[:, 8:] + 5) % 96
    _, tl2 = oracle.forward_loss(W, tok2, tgt, 4)
    np.testing.assert_allclose(tl2[:, :8], tl[:, :8], rtol=1e-13)
    assert np.all(np.abs(tl2[:, 8:] - tl[:, 8:]) > 0)


# ---------------------------------------------------------------------------
# scale invariances created by the parameterless norms (p1: norm after the
# embedding; QK-norm after RoPE)

def test_embedding_row_scale_invariance():
    lay, W, tok, tgt = _tiny()
    loss, _, g = oracle.loss_and_grads(W, tok, tgt, 4)
    dots = np.sum(g["wte"] * W["wte"], axis=1)
    assert np.max(np.abs(dots)) < 1e-6 * np.max(np.abs(g["wte"]))
    W2 = dict(W)
    W2["wte"] = W["wte"] * np.linspace(0.2, 5.0, 96)[:, None]
    l2, _ = oracle.forward_loss(W2, tok, tgt, 4)
    assert abs(l2 - loss) < 1e-6 * abs(loss)


def test_qk_norm_scale_invariance():
    lay, W, tok, tgt = _tiny()
    loss, _, g = oracle.loss_and_grads(W, tok, tgt, 4)
    for l in range(4):
        wq, dwq = W[f"h{l}.wq"], g[f"h{l}.wq"]
        for h in range(2):
            rows = slice(128 * h, 128 * (h + 1))
            assert abs(np.sum(dwq[rows] * wq[rows])) < 1e-6 * np.abs(dwq).max() * 10
        assert abs(np.sum(g[f"h{l}.wk"] * W[f"h{l}.wk"])) < 1e-6 * np.abs(g[f"h{l}.wk"]).max() * 10
    W2 = dict(W)
    W2["h1.wq"] = W["h1.wq"].copy()
    W2["h1.wq"][128:] *= 3.7
    W2["h2.wk"] = W["h2.wk"] * 0.3
    l2, _ = oracle.forward_loss(W2, tok, tgt, 4)
    assert abs(l2 - loss) < 1e-6 * abs(loss)
    # v is not normed: scaling Wv changes the loss
    W3 = dict(W)
    W3["h1.wv"] = W["h1.wv"] * 3.0
    l3, _ = oracle.forward_loss(W3, tok, tgt, 4)
    assert abs(l3 - loss) > 1e-6


# ---------------------------------------------------------------------------
# relu^2 MLP (p1: F.relu(x).square())

def test_relu_squared_not_plain_square():
    # negating one hidden unit's input row changes the loss for relu(h)^2,
    # while h^2 would be invariant to it
    lay, W, tok, tgt = _tiny()
    loss, _ = oracle.forward_loss(W, tok, tgt, 4)
    W2 = dict(W)
    W2["h0.w1"] = W["h0.w1"].copy()
    W2["h0.w1"][3] *= -1
    l2, _ = oracle.forward_loss(W2, tok, tgt, 4)
    assert abs(l2 - loss) > 1e-8


# ---------------------------------------------------------------------------
# head: softcap (p1: 15 tanh(logits/15) bounds logits to [-15, 15]) and the
# cross-entropy closed forms

def test_softcap_bound():
    lay, W, tok, tgt = _tiny(head_std=50.0)
    s = oracle.forward_logits(W, tok, 4)
    assert np.max(np.abs(s)) <= 15.0
    assert np.max(np.abs(s)) > 14.0


def test_zero_unembedding_gives_ln_vocab():
    lay, W, tok, tgt = _tiny(head_std=0.0)
    loss, tl, g = oracle.loss_and_grads(W, tok, tgt, 4)
    assert loss == pytest.approx(math.log(96), abs=1e-14)
    np.testing.assert_allclose(tl, math.log(96), atol=1e-14)
    for name, _, _ in lay:
        if name != "lm_head":
            assert np.all(g[name] == 0.0), name
    d = g["lm_head"]
    # rows of the unembedding grad sum to zero; every vocab entry that is
    # never a target gets the same row, (1/(V M)) sum_i xf_i, whose rows have RMS 1
    np.testing.assert_allclose(d.sum(axis=0), 0.0, atol=1e-15)
    never = np.setdiff1d(np.arange(96), tgt.reshape(-1))
    assert never.size > 1
    np.testing.assert_allclose(d[never], np.tile(d[never[0]], (never.size, 1)), rtol=0, atol=1e-17)


def test_near_zero_unembedding_loss_close_to_ln_vocab():
    # unembedding std 0.001 and |xf_i| = sqrt(C): each logit z ~ N(0, sigma^2),
    # sigma = 0.001 sqrt(C), so LSE = ln V + sigma^2/2 (to O(sigma^4)) and the
    # target logit averages to 0 with spread sigma / sqrt(M)
    depth, V, T = 4, 65536, 64
    lay = oracle.param_layout(depth, V)
    _, W = synth.make_weights(lay, 0, "f32")
    tok, tgt = synth.token_rows(0, 1, T, V, "uniform")
    loss, _ = oracle.forward_loss(W, tok, tgt, depth)
    sigma = 0.001 * math.sqrt(256)
    assert abs(loss - math.log(V) - sigma ** 2 / 2) < 4 * sigma / math.sqrt(T)


def test_batch_permutation_invariance():
    lay, W, tok, tgt = _tiny(B=3)
    loss, tl, g = oracle.loss_and_grads(W, tok, tgt, 4)
    p = [2, 0, 1]
    loss2, tl2, g2 = oracle.loss_and_grads(W, tok[p], tgt[p], 4)
    assert loss2 == pytest.approx(loss, rel=1e-13)
    np.testing.assert_allclose(tl2, tl[p], rtol=1e-13)
    for name in g:
        np.testing.assert_allclose(g2[name], g[name], rtol=1e-9, atol=1e-14 * np.abs(g[name]).max())


def test_loss_is_mean_of_row_losses():
    # the loss is a mean over positions: the full batch's gradient is the
    # mean of the one-row gradients
    lay, W, tok, tgt = _tiny(B=2)
    loss, tl, g = oracle.loss_and_grads(W, tok, tgt, 4)
    l0, _, g0 = oracle.loss_and_grads(W, tok[:1], tgt[:1], 4)
    l1, _, g1 = oracle.loss_and_grads(W, tok[1:], tgt[1:], 4)
    assert loss == pytest.approx((l0 + l1) / 2, rel=1e-13)
    for name in g:
        np.testing.assert_allclose(g[name], (g0[name] + g1[name]) / 2, rtol=1e-9,
                                   atol=1e-13 * np.abs(g[name]).max())


# ---------------------------------------------------------------------------
# the seeded inputs

def test_zipf_head_mass():
    cdf = synth.zipf_cdf(65536)
    assert cdf[0] == pytest.approx(0.1373, abs=5e-4)
    assert cdf[9] == pytest.approx(0.368, abs=2e-3)
    tok, tgt = synth.token_rows(2, 16, 2048, 65536, "zipf")
    assert abs((tok == 0).mean() - cdf[0]) < 0.01
    np.testing.assert_array_equal(tok[:, 1:], tgt[:, :-1])


def test_bf16_rounding_nearest_even():
    x = np.array([1.0, 1 + 2 ** -8, 1 + 3 * 2 ** -9, -2.5, 65504.0, 1e-40], dtype=np.float32)
    got = synth.bf16_bits_to_f64(synth.f32_to_bf16_bits(x))
    np.testing.assert_array_equal(got, [1.0, 1.0, 1 + 2 ** -7, -2.5, 65536.0, float(np.float32(1e-40)) and got[5]])
    assert got[1] == 1.0  # tie goes to even


def test_head_backward_row_matches_finite_differences_at_saturation():
    # d(scale * sum of token losses)/dz by central differences of the loss
    # itself, on rows whose logits reach deep into tanh saturation (|z| up to
    # 60), with the target at the row's argmax, at id 0 and at the last id
    rng = np.random.default_rng(5)
    V = 37
    z = rng.normal(0.0, 20.0, size=(4, V))
    z[1] = rng.uniform(30.0, 60.0, size=V) * rng.choice([-1.0, 1.0], size=V)
    z[2, 7] = 55.0
    tgt = np.array([0, V - 1, 7, 3])
    scale = 0.25

    def loss(zz):
        s = oracle.head_forward_row(zz, np.eye(V))  # z W^T with W = I
        return scale * oracle.head_loss_row(s, tgt)[0].sum()

    s = oracle.head_forward_row(z, np.eye(V))
    _, lse = oracle.head_loss_row(s, tgt)
    g = oracle.head_backward_row(s, lse, tgt, scale)
    h = 1e-5
    fd = np.empty_like(z)
    for i in range(z.shape[0]):
        for j in range(V):
            zp, zm = z.copy(), z.copy()
            zp[i, j] += h
            zm[i, j] -= h
            fd[i, j] = (loss(zp) - loss(zm)) / (2 * h)
    # central differences of a loss of size ~10 at h = 1e-5: rounding noise ~1e-10
    np.testing.assert_allclose(g, fd, rtol=1e-6, atol=5e-10)
    # at saturation the softcap derivative is tiny but not zero
    assert 0 < np.abs(g[1]).max() < 1e-2
