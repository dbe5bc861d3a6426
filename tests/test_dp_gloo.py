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


# ------------------------------------------------------------- bucketed exchange
TINY_CFG = dict(n_layer=2, n_embd=64, n_head=4, vocab_size=512, padded_vocab=512, max_T=64)


def _to_arena(named, layout, n_arena):
    a = np.zeros(n_arena)
    for name, off, cnt in layout:
        a[off:off + cnt] = np.asarray(named[name], np.float64).reshape(-1)
    return a


def _bucket_rank_main(rank, world, port, B, T, q):
    """One rank of the bucketed exchange: its oracle gradient, laid out as the
    library's gradient arena, averaged bucket by bucket in the order the
    library's backward reports them."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import decoder_only_lm_b200 as g
        from decoder_only_lm_b200.dp import GradExchange
        import oracle
        import synth
        cfg = g.make_config(**TINY_CFG)
        layout = g.arena_layout(cfg)
        plan = g.grad_buckets(cfg)
        m = oracle.Model(2, 64, 4, 512, 512, 64)
        flat = m.pack(synth.init_params(0, m.shapes()))
        stream = synth.uniform_stream(1, 4 * B * T * world + 1, 512)
        x, y = oracle.batch_from_stream(stream, rank * B * T, B, T)
        _, _, gr, _ = m.fwd_bwd(flat, x, y)
        n_arena = max(off + cnt for _, off, cnt in plan)
        arena = torch.from_numpy(_to_arena(m.unpack(gr), layout, n_arena))

        def average(view):
            dist.all_reduce(view, op=dist.ReduceOp.SUM)
            view.div_(world)

        ex = GradExchange(arena, plan, average)
        for b in range(ex.n_buckets):  # the order gpt2_backward reports them in
            ex.ready(b)
        ex.finish()
        if rank == 0:
            q.put(arena.numpy().copy())
    finally:
        dist.destroy_process_group()


def test_bucket_plan_partitions_the_arena_in_backward_order():
    """The plan covers every element of the gradient arena exactly once; bucket
    b < L is exactly layer L-1-b's four weight matrices, bucket L the
    embeddings and every vector."""
    import decoder_only_lm_b200 as g
    for kw in (TINY_CFG, dict(n_layer=12, n_embd=768, n_head=12, vocab_size=50257,
                              padded_vocab=50304, max_T=1024)):
        cfg = g.make_config(**kw)
        layout = g.arena_layout(cfg)
        plan = g.grad_buckets(cfg)
        n_arena = max(off + cnt for _, off, cnt in plan)
        cover = np.zeros(n_arena, np.int32)
        for _, off, cnt in plan:
            cover[off:off + cnt] += 1
        assert (cover == 1).all()
        L = kw["n_layer"]
        assert sorted({b for b, _, _ in plan}) == list(range(L + 1))
        for name, off, cnt in layout:
            owners = {b for b, o, c in plan if o <= off and off + cnt <= o + c}
            assert len(owners) == 1, name
            (b,) = owners
            if name.startswith("h.") and name.endswith(".w") and ("attn" in name or "mlp" in name):
                assert b == L - 1 - int(name.split(".")[1]), name
            else:
                assert b == L, name


def test_bucketed_exchange_equals_full_batch_gradient():
    """Two gloo ranks average their shards' gradients bucket by bucket through
    the exchange the GPU path uses; the result is the gradient of the combined
    batch (equal shards: the mean of the shard means), and the arena's padding
    stays zero."""
    import decoder_only_lm_b200 as g
    import oracle
    import synth
    world, B, T = 2, 2, 16
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bucket_rank_main, args=(r, world, port, B, T, q))
             for r in range(world)]
    for p in procs:
        p.start()
    avg = q.get(timeout=300)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    m = oracle.Model(2, 64, 4, 512, 512, 64)
    flat = m.pack(synth.init_params(0, m.shapes()))
    stream = synth.uniform_stream(1, 4 * B * T * world + 1, 512)
    x, y = oracle.batch_from_stream(stream, 0, B * world, T)
    _, _, g_full, _ = m.fwd_bwd(flat, x, y)
    cfg = g.make_config(**TINY_CFG)
    layout = g.arena_layout(cfg)
    full = _to_arena(m.unpack(g_full), layout, avg.size)
    assert np.linalg.norm(avg - full) <= 1e-12 * np.linalg.norm(full)
    used = np.zeros(avg.size, bool)
    for _, off, cnt in layout:
        used[off:off + cnt] = True
    assert (avg[~used] == 0).all()


def test_exchange_refuses_buckets_out_of_order():
    from decoder_only_lm_b200.dp import GradExchange
    ex = GradExchange(torch.zeros(8), [(0, 0, 4), (1, 4, 4)], lambda v: None)
    with pytest.raises(RuntimeError):
        ex.ready(1)
    ex.ready(0)
    with pytest.raises(RuntimeError):
        ex.finish()
    ex.ready(1)
    ex.finish()
    ex.ready(0)  # re-armed for the next step
