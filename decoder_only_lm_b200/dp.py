"""Data-parallel gradient exchange overlapped with the backward pass.

The data-parallel step [LECTURE: DDP, gradients averaged over the ranks
before the optimizer step, no exchange until the last micro-batch; CH28 §28.3:
rank r reads the windows at offsets (i * N + r) * B * T]: every rank runs
forward and backward on its own windows, the gradient arenas are averaged,
and every rank applies the same clip + AdamW.

The library cuts the gradient arena into buckets in the order its backward
finishes them (gpt2_grad_buckets: one per layer's weight matrices, last
layer first, then the embeddings and every vector) and calls back as each one
becomes final (gpt2_set_bucket_callback).  GradExchange averages a bucket as
soon as it is reported, so all but the last bucket cross NVLink while the
earlier layers' backward still runs.  Averaging a range of elements in place
is the caller's collective: NCCL all-reduce with ReduceOp.AVG on a side
stream for GPUs (nccl_exchange), any callable for tests.
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
