"""The N > 1 host logic of bench.py on CPU ranks (gloo, world size 2): the
replicas share nothing on the data path; only the whole-job aggregation (max of
the ranks' device times, sum of their committed tokens) and a barrier cross
ranks, and every replica decodes its own prompts."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        import synth
        ms, tokens = 10.0 + 3.5 * rank, 100.0 * (rank + 1)
        dist.barrier()
        got = bench.combine_ranks(dist, ms, tokens, "cpu")
        cfg = dict(synth.CONFIGS["qwen3_8b_b16"])
        first = [int(p[0]) for p in bench.rank_prompts(cfg, rank)[:4]]
        lens = [len(p) for p in bench.rank_prompts(cfg, rank)]
        out[rank] = (got, first, lens, [len(p) for p in bench.rank_prompts(cfg, rank)])
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_and_own_prompts():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert sorted(res) == [0, 1]
    for r in range(world):
        (ms_max, tok_sum), first, lens, lens_again = res[r]
        assert ms_max == 13.5 and tok_sum == 300.0  # max of 10.0 and 13.5; 100 + 200
        assert lens == lens_again  # a replica's prompts are deterministic
        assert all(128 <= n <= 1024 for n in lens)
    assert res[0][1] != res[1][1] or res[0][2] != res[1][2]  # the replicas decode different prompts
