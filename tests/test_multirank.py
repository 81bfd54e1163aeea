"""The N > 1 path of bench.py on CPU: two ranks over gloo (127.0.0.1).

Each rank packs its own users (weak scaling, no data-path collective); the reported time is the
max over ranks and the work the sum; the reference arm runs on rank 0 only.  The ranks run as
spawned processes; the collectives are the same calls bench.py makes with NCCL on GPUs.
"""
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench
    import mtfm_synth as syn

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # rank r: time r + 1 ms, work [10 (r + 1), r + 1]
        ms, work = bench.reduce_over_ranks(rank + 1.0, [10.0 * (rank + 1), rank + 1.0], "cpu")
        b = syn.pair_batch(4, seed=bench.rank_batch_seed(rank))

        class Args:
            users, steps, warmup = 4, 1, 3

        ref = bench.run_reference(Args, rank, world) if rank != 0 else "rank0"
        out[rank] = (ms, work, b.L_H.tolist(), b.total_tokens, ref)
    finally:
        dist.destroy_process_group()


def test_two_ranks_reduce_and_shard():
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    assert sorted(out.keys()) == [0, 1]
    for r in range(world):
        ms, work, _, _, _ = out[r]
        assert ms == 2.0                      # max of 1 and 2
        assert work == [30.0, 3.0]            # sums over both ranks
    # the two ranks hold different users
    assert out[0][2] != out[1][2] or out[0][3] != out[1][3]
    # the reference arm does no work off rank 0
    assert out[1][4] is None


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    ms, work = bench.reduce_over_ranks(3.5, [1.0, 2.0], "cpu")
    assert ms == 3.5 and work == [1.0, 2.0]
    seeds = {bench.rank_batch_seed(r) for r in range(8)}
    assert len(seeds) == 8
