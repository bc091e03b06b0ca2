"""fp64 CPU oracle of the optimizer step (Muon for the block matrices, AdamW
for the rest).

TEST INFRASTRUCTURE ONLY, like oracle.model: nothing on the product path
imports it, and it shares no code with the CUDA library.

What the pages fix ("Nanochat: full-stack LLM training in 8,000 lines for
$72", section "A Llama-class transformer with ten modern departures";
"nanochat - full-stack ChatGPT in ~8k lines", section "2. Pretrain"; the
energyai.berlin page, "Muon optimizer"):
  * a dual optimizer: Muon -- a momentum update orthogonalised before it is
    applied -- for the transformer's matrix weights, AdamW for the
    embeddings, the unembedding and the scalars, each group with its own
    learning rate;
  * Muon's momentum follows a schedule (0.85 -> 0.97 -> 0.90): here it is
    the caller's per-step input.

Readings taken where the pages stop (listed in the design notes too):
  * Muon: buf <- mu buf + g; the update is the orthogonal polar factor of
    buf (U V^T of its SVD U S V^T), approximated by k steps of the cubic
    Newton-Schulz iteration X <- 1.5 X - 0.5 X X^T X from X0 = buf / |buf|_F
    (a published method for the polar decomposition: Higham, "Functions of
    Matrices", 2008, section 8.9).  The pages name "Polar Express"
    orthogonalisation without its coefficients, so the orthogonalisation
    is "parity unpinned" against nanochat itself; it is pinned against the
    exact polar factor.  No extra shape-dependent scale.
  * AdamW: the textbook update with bias correction and decoupled weight
    decay (Loshchilov and Hutter):  m <- b1 m + (1-b1) g,
    v <- b2 v + (1-b2) g^2,  w <- w - lr (m/(1-b1^t)) / (sqrt(v/(1-b2^t)) + eps)
    - lr wd w.
  * weight decay is decoupled for both groups: w <- w - lr wd w.
  * groups: "matrix" = wq, wk, wv, wo, w1, w2 of every block (each its own
    matrix); "embed" = wte and the value-embedding tables; "head" = lm_head;
    "scalar" = resid_lambdas, x0_lambdas, ve_gates.
"""
from __future__ import annotations

import numpy as np


def param_group(name: str) -> str:
    """The optimizer group of a weight tensor, by name."""
    if name == "lm_head":
        return "head"
    if name == "wte" or (name.startswith("ve") and name[2:].isdigit()):
        return "embed"
    if name in ("resid_lambdas", "x0_lambdas", "ve_gates"):
        return "scalar"
    return "matrix"


def polar_factor(M):
    """U V^T of the SVD M = U S V^T: the orthogonal matrix nearest to M."""
    U, _, Vt = np.linalg.svd(M, full_matrices=False)
    return U @ Vt


def newton_schulz(M, steps: int):
    """Cubic Newton-Schulz iteration towards the polar factor of M, from
    M / |M|_F (every singular value then lies in (0, 1], inside the
    iteration's region of convergence (0, sqrt 3))."""
    X = M / np.linalg.norm(M)
    for _ in range(steps):
        X = 1.5 * X - 0.5 * X @ (X.T @ X)
    return X


def muon_update(w, g, buf, lr, mu, wd, steps):
    """One Muon step of one matrix: returns (w, buf)."""
    buf = mu * buf + g
    U = newton_schulz(buf, steps)
    return w - lr * U - lr * wd * w, buf


def adamw_update(w, g, m, v, t, lr, beta1, beta2, eps, wd):
    """One AdamW step (t >= 1): returns (w, m, v)."""
    m = beta1 * m + (1.0 - beta1) * g
    v = beta2 * v + (1.0 - beta2) * g * g
    mhat = m / (1.0 - beta1 ** t)
    vhat = v / (1.0 - beta2 ** t)
    return w - lr * mhat / (np.sqrt(vhat) + eps) - lr * wd * w, m, v


def optimizer_step(W, G, state, t, opts):
    """One step over every tensor.  W, G: name -> array; state: name ->
    (m, v) (Muon's momentum is m; v unused); opts: dict with lr_matrix,
    lr_embed, lr_head, lr_scalar, weight_decay, muon_momentum, ns_steps,
    beta1, beta2, eps.  Returns (W, state), new dicts."""
    lr = {"matrix": opts["lr_matrix"], "embed": opts["lr_embed"], "head": opts["lr_head"],
          "scalar": opts["lr_scalar"]}
    W2, S2 = {}, {}
    for name, w in W.items():
        m, v = state[name]
        grp = param_group(name)
        if grp == "matrix":
            w2, m2 = muon_update(w, G[name], m, lr[grp], opts["muon_momentum"], opts["weight_decay"],
                                 opts["ns_steps"])
            W2[name], S2[name] = w2, (m2, v)
        else:
            w2, m2, v2 = adamw_update(w, G[name], m, v, t, lr[grp], opts["beta1"], opts["beta2"], opts["eps"],
                                      opts["weight_decay"])
            W2[name], S2[name] = w2, (m2, v2)
    return W2, S2
