"""fp64 CPU oracle of one nanochat decoder training step (forward + backward).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, links or runs
this file; only tests/, the smoke check and the bench's CPU-baseline leg do.
It shares no code with the CUDA library.

Every function follows the nanochat pages directly, in float64, with numpy's
matmul as the only library step and no blocking or fusion beyond what the
definitions state.  Where the pages are silent the reading taken is written
beside the function.  Citations name the page and its section:

  p1 = "Nanochat: full-stack LLM training in 8,000 lines for $72" (aethryn.com)
  p4 = "nanochat - full-stack ChatGPT in ~8k lines" (atlas.blal.pro)
  p5 = the energyai.berlin nanochat walk-through

Model (p1 "A Llama-class transformer with ten modern departures";
p4 "0. The model (nanochat/gpt.py)"; p5 "Architectural decisions"):
  x = norm(wte[tok])
  per block: xn = norm(x); q,k,v = xn Wq^T, xn Wk^T, xn Wv^T (one shared KV head);
             q,k = norm(rope(q)), norm(rope(k)); O = causal softmax attention;
             x += O Wo^T; x += relu(norm(x) W1^T)^2 W2^T
  head: s = 15 tanh((norm(x) Wout^T) / 15); loss = mean over tokens of CE.
"""
from __future__ import annotations

import math

import numpy as np

HEAD_DIM = 128          # p1 "One dial controls everything": heads = width / 128
ROPE_THETA = 10000.0    # p1 "ten modern departures": base theta 10,000
SOFTCAP = 15.0          # p1 "ten modern departures": 15 * tanh(logits / 15)
EPS = 2.0 ** -23        # reading: F.rms_norm's default eps for float32 inputs


# ---------------------------------------------------------------------------
# one dial (p1 "One dial controls everything"; p4 "2. Pretrain": width snaps
# to a multiple of head_dim)

def dims(depth: int, vocab: int) -> dict:
    C = HEAD_DIM * math.ceil(64 * depth / HEAD_DIM)
    return dict(L=depth, C=C, H=C // HEAD_DIM, F=4 * C, V=vocab, d=HEAD_DIM)


def param_layout(depth: int, vocab: int) -> list[tuple[str, int, int]]:
    """(name, rows, cols) of every weight in storage order, each [out, in]."""
    D = dims(depth, vocab)
    C, F, V, d = D["C"], D["F"], D["V"], D["d"]
    out = [("wte", V, C)]
    for l in range(depth):
        out += [(f"h{l}.wq", C, C), (f"h{l}.wk", d, C), (f"h{l}.wv", d, C),
                (f"h{l}.wo", C, C), (f"h{l}.w1", F, C), (f"h{l}.w2", C, F)]
    out.append(("lm_head", V, C))
    return out


# ---------------------------------------------------------------------------
# parameterless RMSNorm over the last axis (p1 "ten modern departures": bare
# F.rms_norm, no gain, no bias).  Reading: y = x / sqrt(mean(x^2) + eps).

def rmsnorm(x):
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + EPS)
    return x * r, r


def rmsnorm_bwd(dy, y, r):
    """d/dx of y = x r(x):  dx = r (dy - y mean(dy * y))."""
    return r * (dy - y * np.mean(dy * y, axis=-1, keepdims=True))


# ---------------------------------------------------------------------------
# RoPE (p1 "ten modern departures": theta 10,000; p4: apply_rotary_emb(q, cos,
# sin)).  Reading: half-split pairs (i, i+64), omega_i = theta^(-i/64),
# angle = position * omega_i, positions 0..T-1 within each row.

def rope_tables(T: int):
    half = HEAD_DIM // 2
    omega = ROPE_THETA ** (-np.arange(half, dtype=np.float64) / half)
    ang = np.arange(T, dtype=np.float64)[:, None] * omega[None, :]
    return np.cos(ang), np.sin(ang)


def rope(x, cos, sin):
    """Rotate each pair (x_i, x_{i+64}) by the angle; cos/sin broadcast to x[..., :64]."""
    half = HEAD_DIM // 2
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x1 * sin + x2 * cos], axis=-1)


def rope_bwd(dy, cos, sin):
    """The transpose of a rotation is the rotation by the opposite angle."""
    half = HEAD_DIM // 2
    d1, d2 = dy[..., :half], dy[..., half:]
    return np.concatenate([d1 * cos + d2 * sin, -d1 * sin + d2 * cos], axis=-1)


# ---------------------------------------------------------------------------
# causal softmax attention with one shared KV head (p5 "Multi-Query
# Attention"; p1: causal FA3 / SDPA).  Per batch row: q [T,H,d], k,v [T,d].
# Reading: scale 1/sqrt(d), mask j <= i.

def _scores(qh, k):
    """S[i, j] = q_i . k_j / sqrt(d) for j <= i, -inf above the diagonal."""
    T = qh.shape[0]
    S = (qh @ k.T) / math.sqrt(HEAD_DIM)
    return np.where(np.tril(np.ones((T, T), dtype=bool)), S, -np.inf)


def _softmax_rows(S):
    m = S.max(axis=1, keepdims=True)
    lse = m + np.log(np.exp(S - m).sum(axis=1, keepdims=True))
    return np.exp(S - lse), lse[:, 0]


def attention(q, k, v):
    """O [T,H,d] and the log-sum-exp of each score row [H,T]."""
    T, H, _ = q.shape
    O = np.empty_like(q)
    lse = np.empty((H, T))
    for h in range(H):
        P, lse[h] = _softmax_rows(_scores(q[:, h, :], k))
        O[:, h, :] = P @ v
    return O, lse


def attention_bwd(dO, q, k, v):
    T, H, _ = q.shape
    dq = np.empty_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for h in range(H):
        P, _ = _softmax_rows(_scores(q[:, h, :], k))
        dP = dO[:, h, :] @ v.T
        dv += P.T @ dO[:, h, :]
        dS = P * (dP - np.sum(dP * P, axis=1, keepdims=True))
        dq[:, h, :] = (dS @ k) / math.sqrt(HEAD_DIM)
        dk += (dS.T @ q[:, h, :]) / math.sqrt(HEAD_DIM)
    return dq, dk, dv


# ---------------------------------------------------------------------------
# one transformer block, pre-norm, residual adds (p4 "0. The model": pre-norm
# RMSNorm before attention and MLP, bias=False; p1: relu^2 MLP at 4x).

def block_forward(x, W, l, B, T, cos, sin):
    """x: [B*T, C] residual stream entering block l.  Returns (x_out, cache)."""
    d = HEAD_DIM
    M, C = x.shape
    H = C // d
    xn, r1 = rmsnorm(x)
    q = (xn @ W[f"h{l}.wq"].T).reshape(B, T, H, d)
    k = (xn @ W[f"h{l}.wk"].T).reshape(B, T, d)
    v = (xn @ W[f"h{l}.wv"].T).reshape(B, T, d)
    qn, rq = rmsnorm(rope(q, cos[None, :, None, :], sin[None, :, None, :]))
    kn, rk = rmsnorm(rope(k, cos[None], sin[None]))
    O = np.empty((B, T, H, d))
    lse = np.empty((B, H, T))
    for b in range(B):
        O[b], lse[b] = attention(qn[b], kn[b], v[b])
    O = O.reshape(M, C)
    x1 = x + O @ W[f"h{l}.wo"].T
    xn2, r2 = rmsnorm(x1)
    h = xn2 @ W[f"h{l}.w1"].T
    a = np.maximum(h, 0.0) ** 2
    x2 = x1 + a @ W[f"h{l}.w2"].T
    cache = dict(xn=xn, r1=r1, qn=qn, rq=rq, kn=kn, rk=rk, v=v, O=O, lse=lse,
                 xn2=xn2, r2=r2, h=h, a=a)
    return x2, cache


def block_backward(dx2, cache, W, l, B, T, cos, sin, grads):
    d = HEAD_DIM
    M, C = dx2.shape
    H = C // d
    c = cache
    # x2 = x1 + a W2^T,  a = relu(h)^2,  h = xn2 W1^T
    grads[f"h{l}.w2"] = dx2.T @ c["a"]
    da = dx2 @ W[f"h{l}.w2"]
    dh = da * 2.0 * np.maximum(c["h"], 0.0)
    grads[f"h{l}.w1"] = dh.T @ c["xn2"]
    dxn2 = dh @ W[f"h{l}.w1"]
    dx1 = dx2 + rmsnorm_bwd(dxn2, c["xn2"], c["r2"])
    # x1 = x + O Wo^T
    grads[f"h{l}.wo"] = dx1.T @ c["O"]
    dO = (dx1 @ W[f"h{l}.wo"]).reshape(B, T, H, d)
    dqn = np.empty((B, T, H, d))
    dkn = np.empty((B, T, d))
    dv = np.empty((B, T, d))
    for b in range(B):
        dqn[b], dkn[b], dv[b] = attention_bwd(dO[b], c["qn"][b], c["kn"][b], c["v"][b])
    dq = rope_bwd(rmsnorm_bwd(dqn, c["qn"], c["rq"]), cos[None, :, None, :], sin[None, :, None, :])
    dk = rope_bwd(rmsnorm_bwd(dkn, c["kn"], c["rk"]), cos[None], sin[None])
    dq = dq.reshape(M, C)
    dk = dk.reshape(M, d)
    dv = dv.reshape(M, d)
    xn = c["xn"]
    grads[f"h{l}.wq"] = dq.T @ xn
    grads[f"h{l}.wk"] = dk.T @ xn
    grads[f"h{l}.wv"] = dv.T @ xn
    dxn = dq @ W[f"h{l}.wq"] + dk @ W[f"h{l}.wk"] + dv @ W[f"h{l}.wv"]
    return dx1 + rmsnorm_bwd(dxn, xn, c["r1"])


# ---------------------------------------------------------------------------
# head: final norm, untied unembedding, softcap in fp32 (here fp64), token-level
# cross-entropy averaged over all B*T positions (p1 "ten modern departures";
# p4: untied wte / lm_head, logits = softcap * tanh(logits / softcap)).

def head_forward_row(xf_row, Wout):
    z = xf_row @ Wout.T
    return SOFTCAP * np.tanh(z / SOFTCAP)


def head_loss_row(s, tgt):
    m = s.max(axis=1, keepdims=True)
    lse = (m + np.log(np.exp(s - m).sum(axis=1, keepdims=True)))[:, 0]
    return lse - s[np.arange(s.shape[0]), tgt], lse


def head_backward_row(s, lse, tgt, scale):
    """d (scale * sum of the rows' losses) / d z for softcapped logits s [T,V]:
    (softmax(s) - onehot(target)) * (1 - (s/15)^2) * scale, since
    s = 15 tanh(z/15) has ds/dz = 1 - tanh^2 = 1 - (s/15)^2."""
    ds = np.exp(s - lse[:, None])
    ds[np.arange(s.shape[0]), tgt] -= 1.0
    return ds * (1.0 - (s / SOFTCAP) ** 2) * scale


def _embed(W, tokens):
    B, T = tokens.shape
    return W["wte"][tokens.reshape(-1)]


def forward_logits(W, tokens, depth):
    """Softcapped logits s [B,T,V] of every position."""
    B, T = tokens.shape
    cos, sin = rope_tables(T)
    x, _ = rmsnorm(_embed(W, tokens))
    for l in range(depth):
        x, _ = block_forward(x, W, l, B, T, cos, sin)
    xf, _ = rmsnorm(x)
    V = W["lm_head"].shape[0]
    s = np.empty((B, T, V))
    for b in range(B):
        s[b] = head_forward_row(xf[b * T:(b + 1) * T], W["lm_head"])
    return s


def forward_loss(W, tokens, targets, depth):
    """Mean loss and per-token losses [B,T] (forward only)."""
    B, T = tokens.shape
    cos, sin = rope_tables(T)
    x, _ = rmsnorm(_embed(W, tokens))
    for l in range(depth):
        x, _ = block_forward(x, W, l, B, T, cos, sin)
    xf, _ = rmsnorm(x)
    tl = np.empty((B, T))
    for b in range(B):
        s = head_forward_row(xf[b * T:(b + 1) * T], W["lm_head"])
        tl[b], _ = head_loss_row(s, targets[b])
    return tl.mean(), tl


def loss_and_grads(W, tokens, targets, depth):
    """Loss, per-token losses [B,T] and the gradient of the loss w.r.t. every
    weight (dict name -> array of the weight's shape), all float64.

    Block caches are recomputed in the backward pass from each block's saved
    input, which yields the same values as keeping them.
    """
    B, T = tokens.shape
    M = B * T
    cos, sin = rope_tables(T)
    x_emb, r0 = rmsnorm(_embed(W, tokens))
    xs = [x_emb]
    x = x_emb
    for l in range(depth):
        x, _ = block_forward(x, W, l, B, T, cos, sin)
        xs.append(x)
    xf, rf = rmsnorm(x)
    Wout = W["lm_head"]
    grads = {}
    dWout = np.zeros_like(Wout)
    dxf = np.empty_like(xf)
    tl = np.empty((B, T))
    for b in range(B):
        rows = slice(b * T, (b + 1) * T)
        s = head_forward_row(xf[rows], Wout)
        tl[b], lse = head_loss_row(s, targets[b])
        # d loss / d s = (softmax(s) - onehot(target)) / M;  ds/dz = 1 - (s / 15)^2
        dz = head_backward_row(s, lse, targets[b], 1.0 / M)
        dWout += dz.T @ xf[rows]
        dxf[rows] = dz @ Wout
    grads["lm_head"] = dWout
    dx = rmsnorm_bwd(dxf, xf, rf)
    for l in reversed(range(depth)):
        _, cache = block_forward(xs[l], W, l, B, T, cos, sin)
        dx = block_backward(dx, cache, W, l, B, T, cos, sin, grads)
    dx0 = rmsnorm_bwd(dx, x_emb, r0)
    dwte = np.zeros_like(W["wte"])
    np.add.at(dwte, tokens.reshape(-1), dx0)
    grads["wte"] = dwte
    return tl.mean(), tl, grads
