"""fp64 CPU oracle of the full reference block: the baseline decoder plus
sliding-window "SSSL" attention, value embeddings and per-layer residual
scalars.

TEST INFRASTRUCTURE ONLY, like oracle.model (whose primitives it reuses):
nothing on the product path imports it.  No CUDA kernel implements these
features yet; this module and its pins come first.

What the pages fix (p1 = "Nanochat: full-stack LLM training in 8,000 lines
for $72", section "A Llama-class transformer with ten modern departures";
p4 = "nanochat - full-stack ChatGPT in ~8k lines", section "0. The model"):
  * sliding windows follow the pattern "SSSL": three layers with a short
    window of 1,024 tokens, then one layer with the full 2,048 context, and
    the final layer always full;
  * at alternating layers a gated embedding lookup is added to v (value
    embeddings, gate "ve_gate");
  * per-layer scalars resid_lambdas (init 1.0) and x0_lambdas (init 0.1) mix
    each layer's residual stream with the normalised embedding.

Readings taken where the pages stop (listed in the design notes too):
  * a window of w tokens lets query i see keys j with 0 <= i - j < w
    (the query itself and the w - 1 before it); "L" is the plain causal mask;
  * the pattern repeats from layer 0: layer l is "SSSL"[l % 4], except the
    last layer, which is "L";
  * the mixing happens at the entry of every block:
    x <- resid_lambdas[l] * x + x0_lambdas[l] * x0, with x0 = norm(wte[tok]),
    and the block's two residual adds then apply to the mixed stream;
  * value embeddings sit on the even layers 0, 2, 4, ...; each has its own
    table [vocab, 128] (the width of the one shared v head) and adds
    g_l * ve_l[tok] to v before attention (v is neither roped nor normed);
  * the gate g_l is one learnable scalar per value-embedding layer.  The
    pages name ve_gate without saying what it is computed from, so this part
    is "parity unpinned" against nanochat itself: it is only checked for
    internal consistency (finite differences, reduction to the baseline).
"""
from __future__ import annotations

import math

import numpy as np

from .model import (HEAD_DIM, _softmax_rows, dims, head_backward_row, head_forward_row, head_loss_row,
                    param_layout, rmsnorm, rmsnorm_bwd, rope, rope_bwd, rope_tables)

SHORT_WINDOW = 1024        # p1: short-window layers see 1,024 tokens
WINDOW_PATTERN = "SSSL"    # p1, p4: three short-window layers, then one long
RESID_LAMBDA_INIT = 1.0    # p1: resid_lambdas initialised to 1.0
X0_LAMBDA_INIT = 0.1       # p1: x0_lambdas initialised to 0.1


def window_schedule(depth: int, pattern: str = WINDOW_PATTERN, short: int = SHORT_WINDOW):
    """Window of every layer: `short` for an "S" layer, None (plain causal)
    for an "L" layer; the last layer is always "L"."""
    out = []
    for l in range(depth):
        kind = "L" if l == depth - 1 else pattern[l % len(pattern)]
        out.append(short if kind == "S" else None)
    return out


def ve_layers(depth: int) -> list[int]:
    """Layers that carry a value embedding (reading: the even ones)."""
    return [l for l in range(0, depth, 2)]


def full_param_layout(depth: int, vocab: int) -> list[tuple[str, int, int]]:
    """The baseline layout, then one value-embedding table per VE layer, then
    the scalars: resid_lambdas [1, L], x0_lambdas [1, L], ve_gates [1, n_ve]."""
    out = list(param_layout(depth, vocab))
    ve = ve_layers(depth)
    out += [(f"ve{l}", vocab, HEAD_DIM) for l in ve]
    out += [("resid_lambdas", 1, depth), ("x0_lambdas", 1, depth), ("ve_gates", 1, len(ve))]
    return out


def init_scalars(W: dict, depth: int, gate: float = 1.0) -> dict:
    """The pages' initial values of the residual scalars; the gate value is a
    free choice (the pages give none)."""
    W = dict(W)
    W["resid_lambdas"] = np.full((1, depth), RESID_LAMBDA_INIT)
    W["x0_lambdas"] = np.full((1, depth), X0_LAMBDA_INIT)
    W["ve_gates"] = np.full((1, len(ve_layers(depth))), gate)
    return W


# ---------------------------------------------------------------------------
# causal attention with an optional sliding window, one shared KV head
# (per batch row: q [T,H,d], k, v [T,d]); window None = plain causal.

def _scores(qh, k, window):
    T = qh.shape[0]
    S = (qh @ k.T) / math.sqrt(HEAD_DIM)
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    keep = j <= i
    if window is not None:
        keep &= (i - j) < window
    return np.where(keep, S, -np.inf)


def attention(q, k, v, window=None):
    T, H, _ = q.shape
    O = np.empty_like(q)
    lse = np.empty((H, T))
    for h in range(H):
        P, lse[h] = _softmax_rows(_scores(q[:, h, :], k, window))
        O[:, h, :] = P @ v
    return O, lse


def attention_bwd(dO, q, k, v, window=None):
    T, H, _ = q.shape
    dq = np.empty_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for h in range(H):
        P, _ = _softmax_rows(_scores(q[:, h, :], k, window))
        dP = dO[:, h, :] @ v.T
        dv += P.T @ dO[:, h, :]
        dS = P * (dP - np.sum(dP * P, axis=1, keepdims=True))
        dq[:, h, :] = (dS @ k) / math.sqrt(HEAD_DIM)
        dk += (dS.T @ q[:, h, :]) / math.sqrt(HEAD_DIM)
    return dq, dk, dv


# ---------------------------------------------------------------------------
# one block: mixing with x0, then the baseline block with the layer's window
# and (on VE layers) the value embedding added to v.

def block_forward(x, x0, W, l, B, T, cos, sin, tokens, windows):
    d = HEAD_DIM
    M, C = x.shape
    H = C // d
    lam_r, lam_0 = W["resid_lambdas"][0, l], W["x0_lambdas"][0, l]
    xin = lam_r * x + lam_0 * x0
    xn, r1 = rmsnorm(xin)
    q = (xn @ W[f"h{l}.wq"].T).reshape(B, T, H, d)
    k = (xn @ W[f"h{l}.wk"].T).reshape(B, T, d)
    v = (xn @ W[f"h{l}.wv"].T).reshape(B, T, d)
    ve = None
    if l in ve_layers(len(windows)):
        gi = ve_layers(len(windows)).index(l)
        ve = W[f"ve{l}"][tokens.reshape(-1)].reshape(B, T, d)
        v = v + W["ve_gates"][0, gi] * ve
    qn, rq = rmsnorm(rope(q, cos[None, :, None, :], sin[None, :, None, :]))
    kn, rk = rmsnorm(rope(k, cos[None], sin[None]))
    O = np.empty((B, T, H, d))
    for b in range(B):
        O[b], _ = attention(qn[b], kn[b], v[b], windows[l])
    O = O.reshape(M, C)
    x1 = xin + O @ W[f"h{l}.wo"].T
    xn2, r2 = rmsnorm(x1)
    h = xn2 @ W[f"h{l}.w1"].T
    a = np.maximum(h, 0.0) ** 2
    x2 = x1 + a @ W[f"h{l}.w2"].T
    cache = dict(x=x, x0=x0, xn=xn, r1=r1, qn=qn, rq=rq, kn=kn, rk=rk, v=v, ve=ve, O=O,
                 xn2=xn2, r2=r2, h=h, a=a)
    return x2, cache


def block_backward(dx2, cache, W, l, B, T, cos, sin, tokens, windows, grads):
    """Returns (d x, d x0) of this block's inputs and fills `grads`."""
    d = HEAD_DIM
    M, C = dx2.shape
    H = C // d
    c = cache
    grads[f"h{l}.w2"] = dx2.T @ c["a"]
    da = dx2 @ W[f"h{l}.w2"]
    dh = da * 2.0 * np.maximum(c["h"], 0.0)
    grads[f"h{l}.w1"] = dh.T @ c["xn2"]
    dxn2 = dh @ W[f"h{l}.w1"]
    dx1 = dx2 + rmsnorm_bwd(dxn2, c["xn2"], c["r2"])
    grads[f"h{l}.wo"] = dx1.T @ c["O"]
    dO = (dx1 @ W[f"h{l}.wo"]).reshape(B, T, H, d)
    dqn = np.empty((B, T, H, d))
    dkn = np.empty((B, T, d))
    dv = np.empty((B, T, d))
    for b in range(B):
        dqn[b], dkn[b], dv[b] = attention_bwd(dO[b], c["qn"][b], c["kn"][b], c["v"][b], windows[l])
    if c["ve"] is not None:
        gi = ve_layers(len(windows)).index(l)
        grads["ve_gates"][0, gi] = np.sum(dv * c["ve"])
        dtab = np.zeros_like(W[f"ve{l}"])
        np.add.at(dtab, tokens.reshape(-1), W["ve_gates"][0, gi] * dv.reshape(M, d))
        grads[f"ve{l}"] = dtab
    dq = rope_bwd(rmsnorm_bwd(dqn, c["qn"], c["rq"]), cos[None, :, None, :], sin[None, :, None, :])
    dk = rope_bwd(rmsnorm_bwd(dkn, c["kn"], c["rk"]), cos[None], sin[None])
    dq, dk, dv = dq.reshape(M, C), dk.reshape(M, d), dv.reshape(M, d)
    xn = c["xn"]
    grads[f"h{l}.wq"] = dq.T @ xn
    grads[f"h{l}.wk"] = dk.T @ xn
    grads[f"h{l}.wv"] = dv.T @ xn
    dxn = dq @ W[f"h{l}.wq"] + dk @ W[f"h{l}.wk"] + dv @ W[f"h{l}.wv"]
    dxin = dx1 + rmsnorm_bwd(dxn, xn, c["r1"])
    # xin = lam_r x + lam_0 x0
    grads["resid_lambdas"][0, l] = np.sum(dxin * c["x"])
    grads["x0_lambdas"][0, l] = np.sum(dxin * c["x0"])
    return W["resid_lambdas"][0, l] * dxin, W["x0_lambdas"][0, l] * dxin


def _stream(W, tokens, depth, windows):
    B, T = tokens.shape
    cos, sin = rope_tables(T)
    x0, r0 = rmsnorm(W["wte"][tokens.reshape(-1)])
    xs = [x0]
    x = x0
    for l in range(depth):
        x, _ = block_forward(x, x0, W, l, B, T, cos, sin, tokens, windows)
        xs.append(x)
    return xs, x0, r0, cos, sin


def forward_loss(W, tokens, targets, depth, windows=None):
    """Mean loss and per-token losses [B,T]; windows defaults to SSSL."""
    windows = window_schedule(depth) if windows is None else windows
    B, T = tokens.shape
    xs, _, _, _, _ = _stream(W, tokens, depth, windows)
    xf, _ = rmsnorm(xs[-1])
    tl = np.empty((B, T))
    for b in range(B):
        tl[b], _ = head_loss_row(head_forward_row(xf[b * T:(b + 1) * T], W["lm_head"]), targets[b])
    return tl.mean(), tl


def forward_logits(W, tokens, depth, windows=None):
    """Softcapped logits s [B,T,V] of every position; windows defaults to SSSL."""
    windows = window_schedule(depth) if windows is None else windows
    B, T = tokens.shape
    xs, _, _, _, _ = _stream(W, tokens, depth, windows)
    xf, _ = rmsnorm(xs[-1])
    V = W["lm_head"].shape[0]
    s = np.empty((B, T, V))
    for b in range(B):
        s[b] = head_forward_row(xf[b * T:(b + 1) * T], W["lm_head"])
    return s


def loss_and_grads(W, tokens, targets, depth, windows=None):
    """Loss, per-token losses and the gradient of every weight of
    full_param_layout (float64); windows defaults to the SSSL schedule."""
    windows = window_schedule(depth) if windows is None else windows
    B, T = tokens.shape
    M = B * T
    xs, x0, r0, cos, sin = _stream(W, tokens, depth, windows)
    xf, rf = rmsnorm(xs[-1])
    Wout = W["lm_head"]
    grads = {"resid_lambdas": np.zeros((1, depth)), "x0_lambdas": np.zeros((1, depth)),
             "ve_gates": np.zeros((1, len(ve_layers(depth))))}
    dWout = np.zeros_like(Wout)
    dxf = np.empty_like(xf)
    tl = np.empty((B, T))
    for b in range(B):
        rows = slice(b * T, (b + 1) * T)
        s = head_forward_row(xf[rows], Wout)
        tl[b], lse = head_loss_row(s, targets[b])
        dz = head_backward_row(s, lse, targets[b], 1.0 / M)
        dWout += dz.T @ xf[rows]
        dxf[rows] = dz @ Wout
    grads["lm_head"] = dWout
    dx = rmsnorm_bwd(dxf, xf, rf)
    dx0 = np.zeros_like(x0)
    for l in reversed(range(depth)):
        _, cache = block_forward(xs[l], x0, W, l, B, T, cos, sin, tokens, windows)
        dx, dx0_l = block_backward(dx, cache, W, l, B, T, cos, sin, tokens, windows, grads)
        dx0 += dx0_l
    # x0 is both the stream entering block 0 and the mixing input of every block
    demb = rmsnorm_bwd(dx + dx0, x0, r0)
    dwte = np.zeros_like(W["wte"])
    np.add.at(dwte, tokens.reshape(-1), demb)
    grads["wte"] = dwte
    return tl.mean(), tl, grads


__all__ = ["SHORT_WINDOW", "WINDOW_PATTERN", "RESID_LAMBDA_INIT", "X0_LAMBDA_INIT", "window_schedule",
           "ve_layers", "full_param_layout", "init_scalars", "attention", "attention_bwd",
           "forward_loss", "forward_logits", "loss_and_grads", "dims"]
