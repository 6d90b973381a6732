"""The replica (N > 1) path of bench.py on CPU: two gloo ranks run the same host logic the
torchrun launch runs on GPUs (rank-distinct inputs, work summed and times maxed over ranks)."""
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime

    import torch.distributed as dist

    import bench
    import synth
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = bench.replica_workload(synth.WORKLOADS["mha4-L2048-B64"].with_lens([300, 77]), rank)
        x = synth.make_inputs(w)
        # per-rank "measurements": rank r did (r + 1) units in (10 + r) ms, etc.
        work, times = bench.reduce_over_ranks([float(rank + 1)], [10.0 + rank, 5.0 - rank], dist)
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), work=np.array(work), times=np.array(times),
                 q=x["q"][:64], seeds=np.array(w.seeds))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_sum_work_and_max_times(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    mp.spawn(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    r0, r1 = (np.load(tmp_path / f"r{r}.npz") for r in range(2))
    for r in (r0, r1):  # every rank sees the same whole-job totals
        assert r["work"].tolist() == [3.0]
        assert r["times"].tolist() == [11.0, 5.0]
    # replicas are independent problems: distinct seeds, distinct bytes
    assert r0["seeds"].tolist() != r1["seeds"].tolist()
    assert not np.array_equal(r0["q"], r1["q"])


def test_single_process_passes_values_through():
    import bench
    assert bench.reduce_over_ranks([2.0], [1.5, 0.5]) == ([2.0], [1.5, 0.5])
    import synth
    w = synth.WORKLOADS["mha4-L2048-B64"]
    assert bench.replica_workload(w, 0) is w
