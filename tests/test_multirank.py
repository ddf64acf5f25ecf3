"""The multi-GPU path on CPU: two gloo ranks run bench.py's rank logic --
one independent batch per rank, device time taken as the max over ranks,
whole-job throughput = all ranks' units over that time.  No GPU needed."""

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
import workloads as W


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        # each rank's own batch: a small decode case seeded by the rank
        q, k, v, lens, meta = W.gqa_case("decode_gqa", bench.rank_seed(rank), b_override=2, n_override=64)
        fingerprint = float(np.abs(k).sum() + np.abs(q).sum())
        # pretend device times: the slower rank sets the job time
        ms, e2e = 10.0 + 5.0 * rank, 20.0 - 3.0 * rank
        got = bench.max_over_ranks([ms, e2e, fingerprint], world)
        dist.barrier()
        np.save(os.path.join(out_dir, f"rank{rank}.npy"), np.array([ms, e2e, fingerprint] + got))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    r0 = np.load(tmp_path / "rank0.npy")
    r1 = np.load(tmp_path / "rank1.npy")
    # every rank sees the same reduced values: the max over ranks
    assert np.array_equal(r0[3:], r1[3:])
    assert r0[3] == max(r0[0], r1[0]) == 15.0
    assert r0[4] == max(r0[1], r1[1]) == 20.0
    # the ranks attended different batches (independent shards)
    assert r0[2] != r1[2]
    assert r0[5] == max(r0[2], r1[2])


def test_whole_job_rate_uses_all_ranks_and_slowest_time():
    # 2 ranks x 100 MB each in 15 ms (slowest rank) -> 200 MB / 15 ms
    assert bench.whole_job_rate(100e6, 2, 15.0) == pytest.approx(200e6 / 15e-3)
    assert bench.whole_job_rate(100e6, 1, 10.0) == pytest.approx(1e10)


def test_rank_batches_are_deterministic():
    a = W.gqa_case("decode_gqa", bench.rank_seed(1), b_override=2, n_override=64)
    b = W.gqa_case("decode_gqa", bench.rank_seed(1), b_override=2, n_override=64)
    for x, y in zip(a[:4], b[:4]):
        assert np.array_equal(x, y)
