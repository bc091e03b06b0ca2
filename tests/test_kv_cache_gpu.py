"""Inference with a KV cache (nc_prefill / nc_decode) against the fp64 oracle.

A causal model's logits at position t depend only on tokens 0..t, so one
oracle forward over the whole sequence gives the reference for every step:
prefill a prompt, then decode token by token, and compare each step's
logits with the oracle's logits at that position.  Cases: the baseline
model in fp32 and bf16, and the full reference block (short windows that
bite inside the sequence, value embeddings, residual scalars).  Tolerances:
fp32 1e-4 of the largest logit; bf16 the forward-logits test's bounds (a few
bf16 roundings of values up to 15).
"""
import numpy as np
import pytest

import oracle
import synth
from oracle import full_block as fb
from tests._gpu_helpers import to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from decoder_only_transformer_nanochat_b200 import build
    build.build()
    return torch


def _close(got, ref, dtype):
    got = got.astype(np.float64)
    assert np.all(np.isfinite(got)) and np.max(np.abs(got)) <= 15.0
    if dtype == "f32":
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-4 * np.abs(ref).max())
    else:
        assert np.max(np.abs(got - ref)) <= 0.03 * np.abs(ref).max()
        assert np.mean(np.abs(got - ref)) <= 0.01 * np.mean(np.abs(ref))
        c = np.sum(got * ref) / np.linalg.norm(got) / np.linalg.norm(ref)
        assert c > 0.9995


CASES = [
    # depth, V, B, prompt, decode steps, T_max, dtype, window, value embeds, scalars
    (2, 1000, 2, 17, 12, 40, "f32", 0, False, False),
    (4, 4096, 3, 37, 20, 64, "bf16", 0, False, False),
    (4, 4096, 2, 30, 25, 64, "bf16", 8, True, True),
    (4, 2000, 2, 5, 30, 48, "f32", 4, True, True),
]


@pytest.mark.parametrize("depth,V,B,T0,steps,T_max,dtype,window,ve,scalars", CASES)
def test_decode_matches_the_full_forward(torch_cuda, depth, V, B, T0, steps, T_max, dtype, window, ve, scalars):
    torch = torch_cuda
    from decoder_only_transformer_nanochat_b200 import Model
    model = Model(depth, vocab=V, seq=T_max, dtype=dtype, window=window, value_embeds=ve, resid_scalars=scalars)
    lay = [(n, r, c) for n, _, r, c in model.layout]
    n_ve = len(fb.ve_layers(depth))
    values = synth.full_block_values(depth, n_ve, 0.95, 0.12, 0.8) if (ve or scalars) else None
    flat, W = synth.make_weights(lay, 31 + depth, dtype, std_override={"lm_head": 0.5}, values=values)
    W = dict(W)
    full = window or ve or scalars
    if full:
        if not ve:
            for name, r, c in fb.full_param_layout(depth, V):
                if name.startswith("ve") and name[2:].isdigit():
                    W[name] = np.zeros((r, c))
            W["ve_gates"] = np.zeros((1, n_ve))
        if not scalars:
            W["resid_lambdas"], W["x0_lambdas"] = np.ones((1, depth)), np.zeros((1, depth))
    T = T0 + steps
    tok, _ = synth.token_rows(40 + depth, B, T, V, "uniform")
    if full:
        windows = fb.window_schedule(depth, short=window) if window else [None] * depth
        ref = fb.forward_logits(W, tok, depth, windows=windows)
    else:
        ref = oracle.forward_logits(W, tok, depth)
    w = to_device(flat, dtype)
    t = torch.from_numpy(tok).cuda()
    cache = model.kv_cache(B, T_max)
    logits = model.prefill(w, t[:, :T0].contiguous(), cache, T_max)
    assert model.sync_status(60000) == 0
    _close(logits.float().cpu().numpy(), ref[:, T0 - 1], dtype)
    assert cache[1].cpu().tolist() == [T0] * B
    for k in range(steps):
        pos = T0 + k
        logits = model.decode(w, t[:, pos].contiguous(), cache, T_max)
        assert model.sync_status(60000) == 0
        _close(logits.float().cpu().numpy(), ref[:, pos], dtype)
    assert cache[1].cpu().tolist() == [T] * B


def test_decode_past_the_cache_is_flagged(torch_cuda):
    torch = torch_cuda
    from decoder_only_transformer_nanochat_b200 import Model
    depth, V, B, T_max = 2, 512, 2, 16
    model = Model(depth, vocab=V, seq=T_max, dtype="bf16")
    lay = [(n, r, c) for n, _, r, c in model.layout]
    flat, _ = synth.make_weights(lay, 3, "bf16")
    w = to_device(flat, "bf16")
    kv, seqlens = model.kv_cache(B, T_max)
    seqlens.fill_(T_max)  # the cache is full: the next position does not exist
    model.decode(w, torch.zeros(B, dtype=torch.int32, device="cuda"), (kv, seqlens), T_max)
    import decoder_only_transformer_nanochat_b200 as nc
    assert model.sync_status(60000) == nc.NC_ERANGE
    assert model.sync_status(60000) == 0
