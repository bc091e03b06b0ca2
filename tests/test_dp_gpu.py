"""Gradient accumulation, gradient buckets and the data-parallel step on the
GPU, through the C ABI.

  * NC_ACCUMULATE adds a step's gradients to the buffer: two accumulated
    calls equal the sum of the two calls made separately, and, on the fp32
    model, half of it equals the full batch's gradient (each call's loss is
    the mean over its own rows, the halves are the same size);
  * the buckets the library reports are the plan dp.bucket_plan derives from
    the layout (a partition of the gradient, in backward order), and every
    bucket's event has fired once the step is done;
  * DataParallel over a one-rank NCCL group (all-reduce is the identity)
    returns the plain step's loss and gradients bit for bit, with the
    per-bucket event waits and collectives on their own stream.
"""
import os
import socket

import numpy as np
import pytest

import synth
from decoder_only_transformer_nanochat_b200 import dp
from tests._gpu_helpers import make_case, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from decoder_only_transformer_nanochat_b200 import build
    build.build()
    return torch


def _model(depth, V, seq, dtype, **kw):
    from decoder_only_transformer_nanochat_b200 import Model
    return Model(depth, vocab=V, seq=seq, dtype=dtype, **kw)


@pytest.mark.parametrize("dtype,full", [("f32", False), ("bf16", False), ("bf16", True)])
def test_accumulate_adds_the_gradients(torch_cuda, dtype, full):
    torch = torch_cuda
    depth, V, B, T = 3, 2000, 4, 96
    kw = dict(window=32, value_embeds=True, resid_scalars=True) if full else {}
    model = _model(depth, V, T, dtype, **kw)
    lay = [(n, r, c) for n, _, r, c in model.layout]
    flat, _ = synth.make_weights(lay, 8, dtype, std_override={"lm_head": 0.3},
                                 values=synth.full_block_values(depth, 2, 0.9, 0.2, 0.7) if full else None)
    w = to_device(flat, dtype)
    tok, tgt = synth.token_rows(8, B, T, V, "zipf")
    t = torch.from_numpy(tok).cuda()
    g = torch.from_numpy(tgt).cuda()
    half = B // 2
    ga = model.fwd_bwd(w, t[:half].contiguous(), g[:half].contiguous())[1].clone()
    gb = model.fwd_bwd(w, t[half:].contiguous(), g[half:].contiguous())[1].clone()
    acc = torch.zeros(model.n_params, dtype=torch.float32, device="cuda")
    model.fwd_bwd(w, t[:half].contiguous(), g[:half].contiguous(), grads=acc, accumulate=True)
    model.fwd_bwd(w, t[half:].contiguous(), g[half:].contiguous(), grads=acc, accumulate=True)
    assert model.sync_status(60000) == 0
    s = (ga + gb).cpu().numpy().astype(np.float64)
    a = acc.cpu().numpy().astype(np.float64)
    # same terms, one fp32 addition each (two for split-K reductions)
    assert np.max(np.abs(a - s)) <= 1e-6 * np.abs(s).max()
    if dtype == "f32":
        full_g = model.fwd_bwd(w, t, g)[1].cpu().numpy().astype(np.float64)
        assert np.max(np.abs(0.5 * a - full_g)) <= 1e-5 * np.abs(full_g).max()


@pytest.mark.parametrize("full", [False, True])
def test_buckets_follow_the_plan_and_their_events_fire(torch_cuda, full):
    torch = torch_cuda
    depth, V, B, T = 4, 1000, 2, 64
    kw = dict(window=16, value_embeds=True, resid_scalars=True) if full else {}
    model = _model(depth, V, T, "bf16", **kw)
    buckets = model.grad_buckets()
    assert buckets == dp.bucket_plan(model.layout, depth)
    lay = [(n, r, c) for n, _, r, c in model.layout]
    flat, _ = synth.make_weights(lay, 9, "bf16")
    events = [torch.cuda.Event() for _ in buckets]
    for e in events:
        e.record()
    torch.cuda.synchronize()
    model.set_grad_events([e.cuda_event for e in events])
    tok, tgt = synth.token_rows(9, B, T, V, "zipf")
    model.fwd_bwd(to_device(flat, "bf16"), torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda())
    # the last bucket's event is recorded at the end of the step: waiting on it waits for the step
    events[-1].synchronize()
    assert all(e.query() for e in events)
    model.set_grad_events([])
    torch.cuda.synchronize()


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_data_parallel_step_on_one_rank(torch_cuda):
    torch = torch_cuda
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        depth, V, B, T = 3, 3000, 2, 128
        lay, flat, W, tok, tgt = make_case(depth, V, B, T, "bf16", 10, "zipf")
        model = _model(depth, V, T, "bf16")
        w = to_device(flat, "bf16")
        t, g = torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda()
        loss0, g0 = model.fwd_bwd(w, t, g)
        loss0, g0 = loss0.clone(), g0.clone()
        step = dp.DataParallel(model)
        grads = torch.empty(model.n_params, dtype=torch.float32, device="cuda")
        loss = torch.empty(1, dtype=torch.float32, device="cuda")
        step.step(w, t, g, grads, loss)
        torch.cuda.synchronize()
        assert model.sync_status(60000) == 0
        assert torch.equal(loss, loss0)
        assert torch.equal(grads, g0)
        step.close()
    finally:
        torch.cuda.synchronize()
        dist.destroy_process_group()
