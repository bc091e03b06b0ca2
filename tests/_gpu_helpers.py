"""Shared pieces of the GPU parity tests: run the CUDA step through the C ABI
on seeded inputs and compare it with the fp64 oracle on the same inputs."""
from __future__ import annotations

import json
import os

import numpy as np

import oracle
import synth


def record(kind: str, **fields):
    """Append one line of measured errors to the file named by NC_PARITY_LOG
    (if set), for deriving and reviewing tolerances."""
    path = os.environ.get("NC_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"kind": kind, **fields}) + "\n")

# tolerances of the two precisions
F32_LOSS_REL = 1e-5          # |dloss| / |loss|
F32_GRAD_MAXABS = 1e-4       # per tensor: max|dg| <= 1e-4 * max|g|
BF16_LOSS_ABS = 1e-2         # |dloss|
BF16_GRAD_COS = 0.999        # per tensor cosine similarity


def token_loss_bound(w_out) -> float:
    """Bound on |per-token loss (bf16 model) - oracle|: a logit z_v = xf . w_v
    moves by at most u |xf| |w_v| when xf carries a relative error u (one
    bf16 rounding, u = 2^-8) in the 2-norm, |xf| = sqrt(C) after the final
    norm; the softcap's slope is at most 1, and a token's loss
    logsumexp(s) - s_target moves by at most twice the largest logit change."""
    C = w_out.shape[1]
    return 2.0 * 2.0 ** -8 * np.sqrt(C) * float(np.linalg.norm(w_out, axis=1).max())


def to_device(flat: np.ndarray, dtype: str):
    import torch
    if dtype == "f32":
        return torch.from_numpy(flat).cuda()
    return torch.from_numpy(flat.view(np.int16)).cuda().view(torch.bfloat16)


def make_case(depth, V, B, T, dtype, seed, dist, std_override=None):
    lay = oracle.param_layout(depth, V)
    flat, W = synth.make_weights(lay, seed, dtype, std_override=std_override)
    tok, tgt = synth.token_rows(seed, B, T, V, dist)
    return lay, flat, W, tok, tgt


def gpu_step(model, flat, tok, tgt, dtype):
    import torch
    w = to_device(flat, dtype)
    t = torch.from_numpy(tok).cuda()
    g = torch.from_numpy(tgt).cuda()
    tl = torch.empty(tok.shape, dtype=torch.float32, device="cuda")
    loss, grads = model.fwd_bwd(w, t, g, token_loss=tl)
    rc = model.sync_status(120000)
    torch.cuda.synchronize()
    return rc, float(loss.item()), tl.cpu().numpy().astype(np.float64), grads.cpu().numpy().astype(np.float64)


def split_grads(grads_flat, lay):
    out, off = {}, 0
    for name, r, c in lay:
        out[name] = grads_flat[off:off + r * c].reshape(r, c)
        off += r * c
    return out


def cosine(a, b):
    na, nb = np.linalg.norm(a), np.linalg.norm(b)
    if na == 0 and nb == 0:
        return 1.0
    return float(np.sum(a * b) / (na * nb))


def compare(dtype, lay, loss_gpu, g_gpu_flat, loss_ref, g_ref, tl_gpu=None, tl_ref=None, tag="", tl_bound=None):
    """Assert the precision's tolerances; return a per-tensor report."""
    g_gpu = split_grads(g_gpu_flat, lay)
    report = {}
    fields = {"tag": tag, "dtype": dtype, "dloss": float(loss_gpu - loss_ref)}
    if tl_gpu is not None:
        d = np.abs(tl_gpu - tl_ref)
        fields.update(tl_max=float(d.max()), tl_mean=float(d.mean()),
                      tl_ref_absmax=float(np.abs(tl_ref).max()))
    cos = {name: cosine(g_gpu[name], g_ref[name]) for name, _, _ in lay}
    worst = min(cos, key=cos.get)
    fields.update(min_cos=cos[worst], min_cos_tensor=worst)
    record("step", **fields)
    # A tensor whose exact gradient vanishes (a one-key window, or identical
    # value rows: attention then does not depend on its scores, so dq = dk = 0)
    # holds rounding noise of the quantities that cancel: it is bounded
    # against the largest gradient instead (fp32: 1e-6, about 16 units of
    # fp32 roundoff; bf16: 1e-3).
    gmax = max(float(np.max(np.abs(g_ref[name]))) for name, _, _ in lay)
    vanishing = {name for name, _, _ in lay if np.max(np.abs(g_ref[name])) <= 1e-6 * gmax}
    if dtype == "f32":
        assert abs(loss_gpu - loss_ref) <= F32_LOSS_REL * abs(loss_ref), (loss_gpu, loss_ref)
        for name, _, _ in lay:
            ref = g_ref[name]
            err = np.max(np.abs(g_gpu[name] - ref))
            if name in vanishing:
                assert np.max(np.abs(g_gpu[name])) <= 1e-6 * gmax, (name, err, gmax)
                continue
            scale = float(np.max(np.abs(ref)))
            report[name] = err / scale
            assert err <= F32_GRAD_MAXABS * scale, (name, err, scale)
        if tl_gpu is not None:
            np.testing.assert_allclose(tl_gpu, tl_ref, rtol=1e-5, atol=1e-5)
    else:
        assert abs(loss_gpu - loss_ref) <= BF16_LOSS_ABS, (loss_gpu, loss_ref)
        for name, _, _ in lay:
            if name in vanishing:
                assert np.max(np.abs(g_gpu[name])) <= 1e-3 * gmax, name
                continue
            c = cosine(g_gpu[name], g_ref[name])
            report[name] = c
            assert c >= BF16_GRAD_COS, (name, c)
        if tl_gpu is not None:
            # tl_bound: token_loss_bound(lm_head); the mean error is far below the worst case
            d = np.abs(tl_gpu - tl_ref)
            assert tl_bound is not None
            assert d.max() <= tl_bound and d.mean() <= tl_bound / 4, (d.max(), d.mean(), tl_bound)
    return report
