"""The optimizer step (nc_optim_step: Muon for the block matrices, AdamW for
the rest) against the fp64 optimizer oracle (oracle/optim.py), through the C
ABI, on seeded weights and seeded synthetic gradients (the step is a function
of weights, gradients and state; no input comes from the CUDA path).

Two steps in a row, so the moments carry over.  Matrices cover both shapes
of the Newton-Schulz product (rows >= cols and rows < cols).  Tolerances:
  * AdamW (fp32 arithmetic on the fp32 master copy, both dtypes): relative
    Frobenius error of each tensor's update <= 1e-5, moments likewise;
  * Muon, fp32 model (CUDA-core GEMMs in fp32): <= 1e-4 per matrix update;
  * Muon, bf16 model (tensor-core GEMMs on bf16 operands): each
    Newton-Schulz step rounds X and its coefficient matrix to bf16 (unit
    roundoff u = 2^-8); the step removes the symmetric part of an error and
    keeps its skew part, so the skew parts of k steps' roundings add up like
    a random walk: <= 4 u sqrt(k) per matrix update.
The bf16 weights must be the master copy rounded to nearest.
"""
import numpy as np
import pytest

import synth
from oracle import full_block as fb
from oracle import optim
from tests._gpu_helpers import to_device

pytestmark = pytest.mark.gpu

OPTS = dict(lr_matrix=0.02, lr_embed=0.3, lr_head=0.004, lr_scalar=0.5, weight_decay=0.01,
            muon_momentum=0.9, ns_steps=10, beta1=0.8, beta2=0.95, eps=1e-10)


@pytest.fixture(scope="module")
def torch_cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from decoder_only_transformer_nanochat_b200 import build
    build.build()
    return torch


def _split(flat, lay):
    out, off = {}, 0
    for name, r, c in lay:
        out[name] = flat[off:off + r * c].reshape(r, c)
        off += r * c
    return out


def _rel(a, b):
    return float(np.linalg.norm(a - b) / (np.linalg.norm(b) + 1e-300))


@pytest.mark.parametrize("dtype,full", [("f32", False), ("bf16", False), ("bf16", True)])
def test_two_optimizer_steps_match_the_oracle(torch_cuda, dtype, full):
    torch = torch_cuda
    from decoder_only_transformer_nanochat_b200 import Model
    depth, V = 2, 300
    kw = dict(window=16, value_embeds=True, resid_scalars=True) if full else {}
    model = Model(depth, vocab=V, seq=64, dtype=dtype, **kw)
    lay = [(n, r, c) for n, _, r, c in model.layout]
    n_ve = len(fb.ve_layers(depth))
    flat, W = synth.make_weights(lay, 50, dtype, values=synth.full_block_values(depth, n_ve) if full else None)
    N = model.n_params
    w = to_device(flat, dtype)
    state = model.optimizer_state(w)
    S = {name: (np.zeros((r, c)), np.zeros((r, c))) for name, r, c in lay}
    Wref = dict(W)
    for t in (1, 2):
        g = (synth.normal(60 + t, 1, N) * 0.01).astype(np.float32)
        G = _split(g.astype(np.float64), lay)
        model.optimizer_step(w, torch.from_numpy(g).cuda(), state, t, OPTS)
        assert model.sync_status(60000) == 0
        Wprev = Wref
        Wref, S = optim.optimizer_step(Wref, G, S, t, OPTS)
        st = state.cpu().numpy().astype(np.float64)
        master, mom, vel = _split(st[:N], lay), _split(st[N:2 * N], lay), _split(st[2 * N:], lay)
        for name, r, c in lay:
            upd, upd_ref = master[name] - Wprev[name], Wref[name] - Wprev[name]
            if optim.param_group(name) == "matrix":
                bound = 1e-4 if dtype == "f32" else 4 * 2.0 ** -8 * np.sqrt(OPTS["ns_steps"])
            else:
                bound = 1e-5
                assert _rel(vel[name], S[name][1]) <= 1e-5, name
            assert _rel(upd, upd_ref) <= bound, (name, t, _rel(upd, upd_ref))
            assert _rel(mom[name], S[name][0]) <= 1e-5, name
        # the next step starts from the GPU's own master copy
        Wref = {name: master[name].copy() for name in master}
    got = w.float().cpu().numpy().astype(np.float64) if dtype == "bf16" else w.cpu().numpy().astype(np.float64)
    st = state.cpu().numpy()
    if dtype == "bf16":
        rounded = synth.bf16_bits_to_f64(synth.f32_to_bf16_bits(st[:N]))
        np.testing.assert_array_equal(got, rounded)
    else:
        np.testing.assert_array_equal(got, st[:N].astype(np.float64))


def test_optimizer_rejects_bad_options(torch_cuda):
    torch = torch_cuda
    import decoder_only_transformer_nanochat_b200 as nc
    from decoder_only_transformer_nanochat_b200 import Model
    model = Model(2, vocab=300, seq=64, dtype="bf16")
    lay = [(n, r, c) for n, _, r, c in model.layout]
    flat, _ = synth.make_weights(lay, 51, "bf16")
    w = to_device(flat, "bf16")
    state = model.optimizer_state(w)
    g = torch.zeros(model.n_params, dtype=torch.float32, device="cuda")
    for bad in (dict(OPTS, beta1=1.0), dict(OPTS, ns_steps=-1), dict(OPTS, eps=-1.0)):
        with pytest.raises(nc.NcError):
            model.optimizer_step(w, g, state, 1, bad)
    with pytest.raises(nc.NcError):
        model.optimizer_step(w, g, state, 0, OPTS)
