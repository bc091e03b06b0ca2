"""Third opinion on the fp64 oracle: the whole model restated with PyTorch
fp64 CPU ops and differentiated by autograd, written from the model's
definition (not from the oracle's code), compared tensor by tensor with the
oracle's hand-derived backward.  Finite differences check sampled entries;
this checks every entry of every gradient.

Definitions followed (p1 = "Nanochat: full-stack LLM training in 8,000 lines
for $72", "A Llama-class transformer with ten modern departures"; p4 =
"nanochat - full-stack ChatGPT in ~8k lines", "0. The model"; readings as in
the design notes): x = norm(wte[tok]); per block xn = norm(x), q, k, v
projections with one shared KV head, q, k = norm(rope(q)), norm(rope(k)) with
half-split pairs and theta 10,000, causal softmax attention scaled by
1/sqrt(128), x += O Wo^T, x += relu(norm(x) W1^T)^2 W2^T; head 15 tanh(z/15)
and the mean token cross-entropy.  The full block adds the sliding window,
the value embedding on even layers and the x0 / residual mixing.
"""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import synth  # noqa: E402
from oracle import full_block as fb  # noqa: E402

D_HEAD = 128
EPS = 2.0 ** -23


def _norm(x):
    return x / torch.sqrt((x * x).mean(dim=-1, keepdim=True) + EPS)


def _rope(x, T):
    # x [..., T, ..., 128] with the position on axis 1 of a [B, T, (H,) 128] tensor
    half = D_HEAD // 2
    inv = 10000.0 ** (-torch.arange(half, dtype=torch.float64) / half)
    ang = torch.arange(T, dtype=torch.float64)[:, None] * inv[None, :]  # [T, 64]
    shape = [1, T] + [1] * (x.dim() - 3) + [half]
    c, s = torch.cos(ang).reshape(shape), torch.sin(ang).reshape(shape)
    x1, x2 = x[..., :half], x[..., half:]
    return torch.cat([x1 * c - x2 * s, x1 * s + x2 * c], dim=-1)


def _attention(q, k, v, window=None):
    # q [B, T, H, d], k, v [B, T, d]
    T = q.shape[1]
    S = torch.einsum("bihd,bjd->bhij", q, k) / math.sqrt(D_HEAD)
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    keep = j <= i
    if window is not None:
        keep = keep & ((i - j) < window)
    S = S.masked_fill(~keep, float("-inf"))
    P = torch.softmax(S, dim=-1)
    return torch.einsum("bhij,bjd->bihd", P, v)


def _model_loss(Wt, tok, tgt, depth, full=False, windows=None):
    B, T = tok.shape
    tok_t = torch.from_numpy(tok).long()
    x0 = _norm(Wt["wte"][tok_t])  # [B, T, C]
    x = x0
    C = x.shape[-1]
    H = C // D_HEAD
    ve_layers = fb.ve_layers(depth) if full else []
    for l in range(depth):
        if full:
            x = Wt["resid_lambdas"][0, l] * x + Wt["x0_lambdas"][0, l] * x0
        xn = _norm(x)
        q = (xn @ Wt[f"h{l}.wq"].T).reshape(B, T, H, D_HEAD)
        k = xn @ Wt[f"h{l}.wk"].T
        v = xn @ Wt[f"h{l}.wv"].T
        if l in ve_layers:
            v = v + Wt["ve_gates"][0, ve_layers.index(l)] * Wt[f"ve{l}"][tok_t]
        q = _norm(_rope(q, T))
        k = _norm(_rope(k, T))
        O = _attention(q, k, v, windows[l] if windows is not None else None).reshape(B, T, C)
        x = x + O @ Wt[f"h{l}.wo"].T
        h = _norm(x) @ Wt[f"h{l}.w1"].T
        x = x + torch.relu(h) ** 2 @ Wt[f"h{l}.w2"].T
    s = 15.0 * torch.tanh((_norm(x) @ Wt["lm_head"].T) / 15.0)
    return torch.nn.functional.cross_entropy(s.reshape(B * T, -1), torch.from_numpy(tgt).long().reshape(-1))


def _compare(W, g_oracle, loss_oracle, loss_t, Wt):
    loss_t.backward()
    assert float(loss_t.detach()) == pytest.approx(loss_oracle, rel=1e-12)
    for name, w in Wt.items():
        g = w.grad.numpy()
        ref = g_oracle[name]
        np.testing.assert_allclose(ref, g, rtol=0, atol=1e-10 * max(np.abs(g).max(), 1e-30), err_msg=name)


def test_baseline_model_matches_autograd():
    depth, V = 2, 96
    lay = oracle.param_layout(depth, V)
    _, W = synth.make_weights(lay, 21, "f32", std_override={"lm_head": 0.5})
    tok, tgt = synth.token_rows(21, 2, 9, V, "uniform")
    loss, _, g = oracle.loss_and_grads(W, tok, tgt, depth)
    Wt = {n: torch.tensor(W[n], dtype=torch.float64, requires_grad=True) for n, _, _ in lay}
    _compare(W, g, loss, _model_loss(Wt, tok, tgt, depth), Wt)


def test_full_block_matches_autograd():
    depth, V = 3, 64
    lay = fb.full_param_layout(depth, V)
    _, W = synth.make_weights(lay, 22, "f32", std_override={"lm_head": 0.5})
    W = dict(W)
    W["resid_lambdas"] = np.array([[0.9, 1.05, 1.2]])
    W["x0_lambdas"] = np.array([[0.1, 0.2, -0.05]])
    W["ve_gates"] = np.array([[0.8, -0.6]])
    tok, tgt = synth.token_rows(22, 2, 11, V, "uniform")
    windows = [3, 5, None]
    loss, _, g = fb.loss_and_grads(W, tok, tgt, depth, windows=windows)
    Wt = {n: torch.tensor(W[n], dtype=torch.float64, requires_grad=True) for n, _, _ in lay}
    _compare(W, g, loss, _model_loss(Wt, tok, tgt, depth, full=True, windows=windows), Wt)
