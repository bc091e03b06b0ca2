"""The multi-rank host path of bench.py, on CPU with two `gloo` ranks.

bench.py runs one process per GPU; each rank draws its own rows (its shard),
runs the step with no collective on the data path, and the job's time is the
maximum over ranks.  These tests run that host logic with world size 2 on the
gloo backend: the shard seeds give disjoint token rows, the max-over-ranks
reduction and the whole-job rate are right, and averaging the ranks' fp64
oracle gradients reproduces the oracle gradient of the concatenated batch (the
quantity a data-parallel all-reduce of the gradients would deliver).
"""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

WORLD = 2


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, port: int, out_dir: str):
    import datetime

    import bench
    import oracle
    import synth

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=60))
    try:
        res = {}
        # max over ranks, as the bench takes the slowest rank's time
        res["max"] = bench.reduce_max(10.0 + 5.0 * rank, WORLD, device="cpu")
        res["rate"] = bench.job_rate(1000, res["max"], WORLD)
        bench.barrier(WORLD)

        # shards: each rank's rows come from its own seed
        depth, V, B, T = 2, 64, 2, 8
        tok, tgt = synth.token_rows(bench.shard_seed(7, rank), B, T, V, "uniform")
        shards = [None] * WORLD
        dist.all_gather_object(shards, (tok, tgt))
        res["shards"] = shards

        # the ranks' gradients, averaged over ranks with a gloo all-reduce
        lay = oracle.param_layout(depth, V)
        _, W = synth.make_weights(lay, 3, "f32")
        loss, _, grads = oracle.loss_and_grads(W, tok, tgt, depth)
        names = sorted(grads)
        flat = torch.from_numpy(np.concatenate([grads[n].ravel() for n in names]))
        dist.all_reduce(flat, op=dist.ReduceOp.SUM)
        flat /= WORLD
        lt = torch.tensor([loss], dtype=torch.float64)
        dist.all_reduce(lt, op=dist.ReduceOp.SUM)
        res["mean_loss"] = float(lt.item()) / WORLD
        res["avg_grad"] = flat.numpy()
        res["names"] = names
        np.save(os.path.join(out_dir, f"rank{rank}.npy"), np.array([res], dtype=object), allow_pickle=True)
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def results(tmp_path_factory):
    out = tmp_path_factory.mktemp("dist")
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, str(out))) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    for p in procs:
        if p.is_alive():
            p.kill()
            p.join()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    return [np.load(os.path.join(out, f"rank{r}.npy"), allow_pickle=True)[0] for r in range(WORLD)]


def test_max_over_ranks_and_job_rate(results):
    for r in results:
        assert r["max"] == 15.0
        # both ranks' tokens over the slowest rank's 15 ms
        assert r["rate"] == pytest.approx(2 * 1000 / 0.015)


def test_shards_are_distinct_and_agree_on_every_rank(results):
    s0, s1 = results[0]["shards"], results[1]["shards"]
    for a, b in zip(s0, s1):
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    (tok0, tgt0), (tok1, tgt1) = s0
    assert not np.array_equal(tok0, tok1)
    # targets are the tokens shifted by one within each rank's rows
    assert np.array_equal(tok0[:, 1:], tgt0[:, :-1]) and np.array_equal(tok1[:, 1:], tgt1[:, :-1])


def test_averaged_rank_gradients_equal_the_full_batch_gradient(results):
    import oracle
    import synth

    depth, V = 2, 64
    (tok0, tgt0), (tok1, tgt1) = results[0]["shards"]
    lay = oracle.param_layout(depth, V)
    _, W = synth.make_weights(lay, 3, "f32")
    loss, _, grads = oracle.loss_and_grads(W, np.concatenate([tok0, tok1]), np.concatenate([tgt0, tgt1]), depth)
    names = results[0]["names"]
    full = np.concatenate([grads[n].ravel() for n in names])
    for r in results:
        assert r["mean_loss"] == pytest.approx(loss, rel=1e-12)
        # equal row counts per rank: the batch mean is the mean of the rank means
        np.testing.assert_allclose(r["avg_grad"], full, rtol=0, atol=1e-12 * np.abs(full).max())
