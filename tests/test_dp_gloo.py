"""The data-parallel path on CPU with two gloo ranks.

The benchmark's N > 1 step is: rank r takes the windows at offsets
(i * N + r) * B * T of the token stream (CH28 §28.3: rank r starts at B*T*r and
advances B*T*N), runs forward + backward on its shard, averages the gradient
arena with one all-reduce, then every rank applies the same clip + AdamW.
Here the per-rank gradients come from the oracle (float64) and the exchange
runs over gloo; the averaged gradient must equal the gradient of the combined
batch, and every rank must end with the same parameters.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, B, T, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import synth
        m = oracle.Model(2, 64, 4, 512, 512, 64)
        flat = m.pack(synth.init_params(0, m.shapes()))
        stream = synth.uniform_stream(1, 4 * B * T * world + 1, 512)
        mm, vv = np.zeros_like(flat), np.zeros_like(flat)
        for i in range(2):  # two steps: offsets advance by B*T*world
            off = (i * world + rank) * B * T
            x, y = oracle.batch_from_stream(stream, off, B, T)
            _, _, g, _ = m.fwd_bwd(flat, x, y)
            gt = torch.from_numpy(g)
            dist.all_reduce(gt, op=dist.ReduceOp.SUM)
            g = gt.numpy() / world
            m.clip_adamw(flat, g, mm, vv, i + 1)
            if i == 0:
                first_grad = g.copy()
        pt = torch.from_numpy(flat.copy())
        gathered = [torch.zeros_like(pt) for _ in range(world)]
        dist.all_gather(gathered, pt)
        if rank == 0:
            q.put((first_grad, [t.numpy() for t in gathered]))
    finally:
        dist.destroy_process_group()


def test_two_rank_gradient_average_equals_full_batch():
    import oracle
    import synth
    world, B, T = 2, 2, 16
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, B, T, q)) for r in range(world)]
    for p in procs:
        p.start()
    first_grad, params = q.get(timeout=300)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # the same step on one process with the combined batch (rank 0 rows, then rank 1 rows)
    m = oracle.Model(2, 64, 4, 512, 512, 64)
    flat = m.pack(synth.init_params(0, m.shapes()))
    stream = synth.uniform_stream(1, 4 * B * T * world + 1, 512)
    x, y = oracle.batch_from_stream(stream, 0, B * world, T)
    _, _, g_full, _ = m.fwd_bwd(flat, x, y)
    assert np.linalg.norm(first_grad - g_full) <= 1e-12 * np.linalg.norm(g_full)
    # every rank holds the same parameters after the updates
    assert np.array_equal(params[0], params[1])


def test_rank_offsets_follow_the_worked_example(golden_dir):
    import json
    g = json.load(open(os.path.join(golden_dir, "slicing_ch28.json")))["ranks"]
    B, T, R = g["B"], g["T"], g["R"]
    for r in range(R):
        assert (0 * R + r) * B * T == g["first_inputs"][str(r)][0]
        assert (1 * R + r) * B * T == g["next_start"][str(r)]
