"""Data-parallel gradient exchange overlapped with the backward pass.

The data-parallel step [LECTURE: DDP, gradients averaged over the ranks
before the optimizer step, no exchange until the last micro-batch; CH28 §28.3:
rank r reads the windows at offsets (i * N + r) * B * T]: every rank runs
forward and backward on its own windows, the gradient arenas are averaged,
and every rank applies the same clip + AdamW.

The library cuts the gradient arena into buckets in the order its backward
finishes them (gpt2_grad_buckets: one per layer's weight matrices, last
layer first, then the embeddings and every vector).  Two ways to average them:

* inside the library (init_library_exchange -> gpt2_dp_init): the backward
  itself enqueues an NCCL all-reduce of each bucket on its communication
  stream as soon as the bucket is final; this is stream-ordered, so it is also
  recorded into the graph of gpt2_stream_begin (what bench.py uses);
* by the caller, through gpt2_set_bucket_callback: GradExchange averages a
  bucket as soon as it is reported with any collective (NCCL all-reduce with
  ReduceOp.AVG on a side stream in nccl_exchange, gloo in the CPU tests).

Either way all but the last bucket cross NVLink while the earlier layers'
backward still runs.
"""
from __future__ import annotations


class GradExchange:
    """Averages the buckets of a gradient arena as they are reported.

    grad: 1-D float tensor (the arena); plan: [(bucket, offset, count)] as
    returned by grad_buckets(); average(view) must leave in `view` the
    element-wise mean of that view over the ranks.  ready(b) must be called
    for b = 0, 1, ... in order, once each per step; finish() checks that every
    bucket was seen and re-arms the exchange for the next step.
    """

    def __init__(self, grad, plan, average):
        self.grad = grad
        self.average = average
        self.ranges = {}
        for b, off, cnt in plan:
            self.ranges.setdefault(b, []).append((off, cnt))
        self.n_buckets = len(self.ranges)
        if sorted(self.ranges) != list(range(self.n_buckets)):
            raise ValueError("bucket indices must be 0 .. n-1")
        self.next = 0

    def ready(self, b):
        if b != self.next:
            raise RuntimeError(f"bucket {b} reported, {self.next} expected")
        self.next += 1
        for off, cnt in self.ranges[b]:
            self.average(self.grad[off:off + cnt])

    def finish(self):
        if self.next != self.n_buckets:
            raise RuntimeError(f"{self.next} of {self.n_buckets} buckets were reported")
        self.next = 0


class CudaGradExchange(GradExchange):
    """GradExchange for a model on a GPU: each bucket's averaging is enqueued
    on a side stream behind an event recorded on the model's stream when the
    bucket is reported, so it overlaps the rest of the backward; finish()
    makes the model's stream wait for the side stream (the clip + AdamW that
    follows then reads the averaged gradients)."""

    def __init__(self, model, average, comm_stream=None):
        import torch
        from decoder_only_lm_b200 import GRAD, grad_buckets
        self.torch = torch
        self.model = model
        self.comm = comm_stream or torch.cuda.Stream()
        super().__init__(model.arena(GRAD), grad_buckets(model.cfg), average)

    def arm(self):
        """Report buckets during the next backward (the last micro-batch's)."""
        self.model.set_bucket_callback(self.ready)

    def ready(self, b):
        ev = self.torch.cuda.Event()
        ev.record(self.model.stream)
        self.comm.wait_event(ev)
        with self.torch.cuda.stream(self.comm):
            super().ready(b)

    def finish(self):
        self.model.set_bucket_callback(None)
        super().finish()
        self.model.stream.wait_stream(self.comm)


def nccl_exchange(model, group=None):
    """CudaGradExchange whose averaging is an NCCL all-reduce (ReduceOp.AVG)
    of each bucket range over `group` (torch.distributed, backend nccl)."""
    import torch.distributed as dist

    def average(view):
        dist.all_reduce(view, op=dist.ReduceOp.AVG, group=group)

    return CudaGradExchange(model, average)


def init_library_exchange(model, group=None):
    """gpt2_dp_init over the ranks of `group` (torch.distributed, initialised):
    rank 0 makes the NCCL id and broadcasts it; every rank joins."""
    import torch.distributed as dist
    from decoder_only_lm_b200 import dp_unique_id
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    box = [dp_unique_id() if rank == 0 else None]
    dist.broadcast_object_list(box, src=0, group=group)
    model.dp_init(box[0], rank, world)
