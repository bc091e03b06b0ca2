"""Data-parallel training step over torch.distributed ranks, one GPU per rank.

The pages train on 8 GPUs with a distributed optimizer that shards state
(ZeRO-2) and syncs gradients asynchronously ("Nanochat: full-stack LLM
training in 8,000 lines for $72", section "A Llama-class transformer with ten
modern departures"; energyai.berlin page, "Scaling across GPUs": torchrun /
DDP).  Here each rank runs the library's forward + backward on its own rows,
and the gradient of the global mean loss is the mean over ranks of the
ranks' gradients: the one exchange the step needs.

The backward finishes the gradient in buckets (nc_grad_bucket: lm_head, then
each block from the last to the first, then the embedding and the full
block's extras) and records one CUDA event per bucket.  A communication
stream waits on bucket k's event and hands that slice of the gradient to an
NCCL all-reduce, so the exchange of block l's gradient overlaps the backward
of the blocks below it.  PyTorch is plumbing here: the process group, the
streams and the events; the collective is NCCL's.
"""
from __future__ import annotations


def bucket_plan(layout, depth: int):
    """The buckets the library reports, from its parameter layout
    [(name, offset, rows, cols)]: lm_head; blocks depth-1 .. 0 (wq .. w2 of
    a block are contiguous); wte; then everything after lm_head, if any."""
    by = {name: (off, r * c) for name, off, r, c in layout}
    out = [by["lm_head"]]
    for l in reversed(range(depth)):
        a = by[f"h{l}.wq"][0]
        z_off, z_n = by[f"h{l}.w2"]
        out.append((a, z_off + z_n - a))
    out.append(by["wte"])
    names = [n for n, _, _, _ in layout]
    extras = names[names.index("lm_head") + 1:]
    if extras:
        first = by[extras[0]][0]
        last_off, last_n = by[extras[-1]]
        out.append((first, last_off + last_n - first))
    return out


def reduce_buckets(grads, buckets, group=None, before=None, average=True):
    """All-reduce grads[off:off+n] of every bucket, in order, asynchronously.
    before(k), if given, runs just before bucket k is handed to the collective
    (a stream wait on its event).  average: divide by the world size -- NCCL's
    AVG reduction; backends without it (gloo) sum and scale after the wait.
    Returns (works, finish): wait on the works, then call finish()."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    nccl = dist.get_backend(group) == "nccl"
    op = dist.ReduceOp.AVG if (average and nccl) else dist.ReduceOp.SUM
    works = []
    for k, (off, n) in enumerate(buckets):
        if before is not None:
            before(k)
        works.append(dist.all_reduce(grads[off:off + n], op=op, group=group, async_op=True))

    def finish():
        if average and not nccl and world > 1:
            for off, n in buckets:
                grads[off:off + n].div_(world)

    return works, finish


class DataParallel:
    """Runs Model.fwd_bwd on this rank's rows and averages loss and gradients
    over the ranks of `group`, overlapping the gradient all-reduce with the
    backward.  Every rank must call step() the same number of times."""

    def __init__(self, model, group=None):
        import torch
        import torch.distributed as dist
        self.model = model
        self.group = group
        self.world = dist.get_world_size(group)
        self.buckets = model.grad_buckets()
        self.stream = torch.cuda.Stream()
        self.events = [torch.cuda.Event() for _ in self.buckets]
        cur = torch.cuda.current_stream()
        for e in self.events:
            e.record(cur)  # creates the CUDA events the library will record
        model.set_grad_events([e.cuda_event for e in self.events])

    def step(self, weights, tokens, targets, grads, loss, accumulate: bool = False, reduce: bool = True):
        """reduce=False: micro-batch of a gradient accumulation, no exchange yet."""
        import torch
        import torch.distributed as dist
        self.model.fwd_bwd(weights, tokens, targets, grads=grads, loss=loss, accumulate=accumulate)
        if not reduce:
            return loss, grads
        with torch.cuda.stream(self.stream):
            works, finish = reduce_buckets(grads, self.buckets, self.group,
                                           before=lambda k: self.stream.wait_event(self.events[k]))
            # the loss is final before bucket 0's event (the head's gradient follows it)
            works.append(dist.all_reduce(loss, op=dist.ReduceOp.AVG, group=self.group, async_op=True))
        for w in works:
            w.wait()  # the current stream waits for the collectives
        finish()
        return loss, grads

    def close(self) -> None:
        self.model.set_grad_events([])
