"""The data-parallel gradient exchange (dp.py) on CPU with two `gloo` ranks.

bucket_plan must partition the gradient buffer (every element in exactly one
bucket) in the order the backward finishes it; reduce_buckets must turn the
ranks' gradients into their mean bucket by bucket.  With the fp64 oracle's
gradients of each rank's own rows, that mean is the oracle gradient of the
concatenated batch: the data-parallel step computes the single-GPU step.
"""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

import oracle  # noqa: E402
from decoder_only_transformer_nanochat_b200 import dp  # noqa: E402
from oracle import full_block as fb  # noqa: E402

WORLD = 2


def _with_offsets(lay):
    out, off = [], 0
    for name, r, c in lay:
        out.append((name, off, r, c))
        off += r * c
    return out, off


@pytest.mark.parametrize("full", [False, True])
def test_bucket_plan_partitions_the_gradient(full):
    depth, V = 5, 100
    lay = fb.full_param_layout(depth, V) if full else oracle.param_layout(depth, V)
    layout, total = _with_offsets(lay)
    plan = dp.bucket_plan(layout, depth)
    assert len(plan) == depth + 2 + (1 if full else 0)
    cover = np.zeros(total, dtype=np.int64)
    for off, n in plan:
        assert n > 0
        cover[off:off + n] += 1
    assert np.all(cover == 1)
    by = {name: off for name, off, _, _ in layout}
    # completion order: the head first, then the blocks from the last, then the embedding
    assert plan[0][0] == by["lm_head"]
    assert [p[0] for p in plan[1:depth + 1]] == [by[f"h{l}.wq"] for l in reversed(range(depth))]
    assert plan[depth + 1] == (0, by["h0.wq"])  # wte: rows [0, V*C)


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, port: int, out_dir: str):
    import datetime

    import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=60))
    try:
        depth, V, B, T = 2, 64, 2, 8
        lay = oracle.param_layout(depth, V)
        layout, total = _with_offsets(lay)
        plan = dp.bucket_plan(layout, depth)
        _, W = synth.make_weights(lay, 3, "f32")
        tok, tgt = synth.token_rows(100 + rank, B, T, V, "uniform")
        loss, _, g = oracle.loss_and_grads(W, tok, tgt, depth)
        flat = torch.from_numpy(np.concatenate([g[n].ravel() for n, _, _ in lay]))
        seen = []
        works, finish = dp.reduce_buckets(flat, plan, before=lambda k: seen.append(k))
        for w in works:
            w.wait()
        finish()
        np.save(os.path.join(out_dir, f"rank{rank}.npy"), flat.numpy())
        np.save(os.path.join(out_dir, f"order{rank}.npy"), np.array(seen))
        np.save(os.path.join(out_dir, f"tok{rank}.npy"), np.stack([tok, tgt]))
    finally:
        dist.destroy_process_group()


def test_bucketed_mean_is_the_full_batch_gradient(tmp_path):
    import synth
    port = _free_port()
    mp.start_processes(_worker, args=(port, str(tmp_path)), nprocs=WORLD, join=True, start_method="spawn")
    r0 = np.load(tmp_path / "rank0.npy")
    r1 = np.load(tmp_path / "rank1.npy")
    np.testing.assert_array_equal(r0, r1)  # every rank holds the same mean
    depth, V = 2, 64
    assert list(np.load(tmp_path / "order0.npy")) == list(range(depth + 2))
    t0, t1 = np.load(tmp_path / "tok0.npy"), np.load(tmp_path / "tok1.npy")
    tok = np.concatenate([t0[0], t1[0]])
    tgt = np.concatenate([t0[1], t1[1]])
    lay = oracle.param_layout(depth, V)
    _, W = synth.make_weights(lay, 3, "f32")
    _, _, g = oracle.loss_and_grads(W, tok, tgt, depth)
    ref = np.concatenate([g[n].ravel() for n, _, _ in lay])
    np.testing.assert_allclose(r0, ref, rtol=0, atol=1e-12 * np.abs(ref).max())
