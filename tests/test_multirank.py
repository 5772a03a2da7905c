"""The multi-GPU path on CPU: world-size-2 gloo ranks.

bench.py shards a job across ranks with no collective on the data path,
either as independent sequences (rank r runs batch element r, drawn from the
stream of that batch index) or as the heads of one call (rank r runs a
contiguous run of heads), then reduces timings as max-over-ranks and work as
a sum.  These tests run that logic with gloo on CPU: the sharded results
equal a single-process run of the whole batch or call, and the reduction is
right.
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


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from block_sparse_video_sol_b200 import synth
        from oracle import sol_ref
        w = synth.Workload("mr", B=1, H=2, N=200, D=16, grid=(2, 10, 10), n_topics=4, seed=77, tau=0.5)
        q, k, v = (synth.bf16_bits_to_f64(x) for x in synth.generate(w, b_offset=bench.shard_b_offset(rank, w)))
        o = sol_ref.sol_forward(q, k, v, tau=w.tau, bq=16, bk=16)["O"]
        ot = torch.from_numpy(o)
        gathered = [torch.empty_like(ot) for _ in range(world)]
        dist.all_gather(gathered, ot)
        t_ms, e2e_ms, work = bench.job_reduce((10.0 + rank, 20.0 - rank, 100.0 * (rank + 1)), "cpu", world)
        if rank == 0:
            np.save(os.path.join(out_dir, "gathered.npy"), torch.cat(gathered, dim=0).numpy())
            np.save(os.path.join(out_dir, "reduced.npy"), np.array([t_ms, e2e_ms, work]))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def _head_worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from block_sparse_video_sol_b200 import synth
        from oracle import sol_ref
        w = synth.Workload("mrh", B=1, H=5, N=200, D=16, grid=(2, 10, 10), n_topics=4, seed=78, tau=0.5)
        heads = bench.shard_heads(rank, world, w.H)
        q, k, v = (synth.bf16_bits_to_f64(x) for x in synth.generate(w, heads=heads))
        r = sol_ref.sol_forward(q, k, v, tau=w.tau, bq=16, bk=16, log_mass_bias_on=True)
        parts = [torch.from_numpy(r["O"]).contiguous(), torch.from_numpy(r["sel"]).to(torch.int64).contiguous()]
        sizes = [len(bench.shard_heads(i, world, w.H)) for i in range(world)]
        out = []
        for t, axis in zip(parts, (2, 1)):
            gathered = []
            for i in range(world):   # uneven shards: every rank sends its part to every other in turn
                shape = list(t.shape)
                shape[axis] = sizes[i]
                buf = t.clone() if i == rank else torch.empty(shape, dtype=t.dtype)
                dist.broadcast(buf, src=i)
                gathered.append(buf)
            out.append(torch.cat(gathered, dim=axis).numpy())
        if rank == 0:
            np.save(os.path.join(out_dir, "o.npy"), out[0])
            np.save(os.path.join(out_dir, "sel.npy"), out[1])
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_rank_head_split_matches_the_whole_call(tmp_path):
    """One B=1 call with 5 heads split 2 / 3 over two ranks: gathered along the head axis,
    outputs and routing masks equal the single-process call."""
    world, port = 2, _free_port()
    mp.start_processes(_head_worker, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn",
                       join=True)
    from block_sparse_video_sol_b200 import synth
    from oracle import sol_ref
    w = synth.Workload("mrh", B=1, H=5, N=200, D=16, grid=(2, 10, 10), n_topics=4, seed=78, tau=0.5)
    q, k, v = (synth.bf16_bits_to_f64(x) for x in synth.generate(w))
    ref = sol_ref.sol_forward(q, k, v, tau=w.tau, bq=16, bk=16, log_mass_bias_on=True)
    assert np.array_equal(np.load(tmp_path / "sel.npy"), ref["sel"].astype(np.int64))
    np.testing.assert_allclose(np.load(tmp_path / "o.npy"), ref["O"], rtol=1e-12, atol=1e-13)


def test_head_shards_cover_every_head_once():
    import bench
    for H in (1, 5, 7, 56):
        for world in (1, 2, 3, 8):
            got = [h for r in range(world) for h in bench.shard_heads(r, world, H)]
            assert got == list(range(H))
            sizes = [len(bench.shard_heads(r, world, H)) for r in range(world)]
            assert max(sizes) - min(sizes) <= 1


def test_two_rank_sharding_matches_batched_oracle(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn", join=True)
    gathered = np.load(tmp_path / "gathered.npy")
    from block_sparse_video_sol_b200 import synth
    from oracle import sol_ref
    w = synth.Workload("mr", B=2, H=2, N=200, D=16, grid=(2, 10, 10), n_topics=4, seed=77, tau=0.5)
    q, k, v = (synth.bf16_bits_to_f64(x) for x in synth.generate(w))
    ref = sol_ref.sol_forward(q, k, v, tau=w.tau, bq=16, bk=16)["O"]
    np.testing.assert_allclose(gathered, ref, rtol=1e-12, atol=1e-13)
    t_ms, e2e_ms, work = np.load(tmp_path / "reduced.npy")
    assert (t_ms, e2e_ms, work) == (11.0, 20.0, 300.0)


def test_single_rank_reduce_is_identity():
    import bench
    assert bench.job_reduce((1.5, 2.5, 7.0), "cpu", 1) == (1.5, 2.5, 7.0)
