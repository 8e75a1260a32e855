"""Host logic of the multi-rank bench path on CPU: two gloo ranks (no GPU).

The weight-sync path shards without exchange (every rank quantizes and checks its own tensors);
the only collectives are the timing barrier, the max over ranks of the step time and the sum of
the mismatch counts. These run here over gloo exactly as over NCCL on the GPUs.
"""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        ms = bench.max_over_ranks(dist, 1.0 + rank * 0.5, device="cpu")
        mism = bench.sum_over_ranks(dist, 3 * rank + 1, device="cpu")
        e2e = bench.aggregate_e2e(dist, {"ms_per_step": 100.0 + 10 * rank, "grid_equal": rank == 0,
                                         "h2d_bytes_per_step": 7, "d2h_bytes_per_step": 3, "steps": 3},
                                  world, 10 ** 9, device="cpu")
        res = {"ms": ms, "mismatches": mism, "e2e": e2e,
               "value": bench.job_throughput_gbs(world, 10 ** 9, ms),
               "seeds": [bench.rank_seed(layer, idx, rank) for layer in range(36) for idx in range(4)]}
        # The reference arm under torchrun: ranks other than 0 exit at once with status 0.
        if rank != 0:
            os.environ["RANK"] = str(rank)

            class A:
                steps, warmup, gpus = 1, 3, world
            res["reference_rc"] = bench.run_reference(A)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_like_the_bench(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    r = [json.load(open(tmp_path / f"rank{i}.json")) for i in range(world)]
    for x in r:
        assert x["ms"] == pytest.approx(1.5)               # the slowest rank's time
        assert x["mismatches"] == 1 + 4                     # summed over ranks
        assert x["value"] == pytest.approx(2 * 1e9 / 1.5e-3 / 1e9)
    assert r[1]["reference_rc"] == 0
    for x in r:
        e = x["e2e"]
        assert e["ms_per_step"] == 110.0 and e["grid_equal"] is False     # rank 1 reported a mismatch
        assert e["value"] == pytest.approx(2 * 1e9 / 0.110 / 1e9, rel=1e-3)
        assert e["h2d_bytes_per_step"] == 14 and e["d2h_bytes_per_step"] == 6
    # Every rank synchronizes its own tensors: no seed is shared between ranks.
    assert len(set(r[0]["seeds"]) | set(r[1]["seeds"])) == 2 * 144
