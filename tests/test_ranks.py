"""The multi-rank path of bench.py on CPU: two gloo ranks, as
torch.distributed.run would launch them, take the barrier and the maximum of
their step times, and the job value counts one call per rank."""

import hashlib
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import torch
    import bench
    ranks = bench.Ranks("gloo", torch.device("cpu"))
    ranks.barrier()
    t = ranks.max(10.0 + 5.0 * rank)       # rank r "took" 10 + 5 r ms
    ranks.barrier()
    out[rank] = (ranks.world, ranks.rank, t, bench.whole_job_ms_per_call(t, ranks.world))
    ranks.close()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_slowest_time():
    world = 2
    with mp.Manager() as man:
        out = man.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert sorted(res) == [0, 1]
    for r in range(world):
        w, rk, t, v = res[r]
        assert (w, rk) == (world, r)
        assert t == 15.0                      # the slowest rank's time on every rank
        assert v == 7.5                       # two calls finished in 15 ms


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import torch
    import bench
    for k in ("RANK", "WORLD_SIZE"):
        os.environ.pop(k, None)
    ranks = bench.Ranks("gloo", torch.device("cpu"))
    assert (ranks.world, ranks.rank) == (1, 0)
    assert ranks.max(3.0) == 3.0
    ranks.barrier()
    ranks.close()
    assert bench.whole_job_ms_per_call(12.0, 1) == 12.0


def test_profiled_traffic_only_for_the_captured_kernel_and_workload():
    """The bench reports the ncu DRAM traffic only while the attention source
    is the one captured, and only for the captured workload, scaled by heads."""
    import bench
    from synthetic import get_workload
    w = get_workload("wide")
    t = bench.profiled_traffic(w)
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "attention_tc_wide_h4.json")))
    src = open(os.path.join(bench.ROOT, rec["source"]), "rb").read()
    if hashlib.sha256(src).hexdigest() == rec["source_sha256"]:
        assert t == (rec["dram_bytes_read"] + rec["dram_bytes_write"]) * 40 / rec["heads"]
        assert bench.profiled_traffic(w.replace(name="wide_h4", H=4)) == rec["dram_bytes_read"] + rec["dram_bytes_write"]
    else:
        assert t is None
    assert bench.profiled_traffic(get_workload("large")) is None
