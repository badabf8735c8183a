"""The N > 1 host path of bench.py on CPU: two gloo ranks, each drawing its own
replica of the workload (weak scaling), timings reduced to the slowest rank."""
import os
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from long_context_sparse_rtp_b200 import synth
        w = synth.WORKLOADS["prefill_2k"]
        w = w.with_(seed=bench.rank_seed(w.seed, rank))
        inp = synth.make_inputs(w, "cpu", L=64)
        # every rank takes the same collective steps in the same order
        slowest = bench.max_over_ranks(1.0 + rank, world)
        q0 = inp["q"].float().flatten()[:8].clone()
        gathered = [torch.zeros_like(q0) for _ in range(world)]
        dist.all_gather(gathered, q0)
        out[rank] = (slowest, [g.tolist() for g in gathered])
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling(tmp_path):
    world = 2
    port = 29500 + (os.getpid() % 1000)
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    assert sorted(out.keys()) == [0, 1]
    for r in range(world):
        slowest, gathered = out[r]
        assert slowest == 2.0                 # max over ranks
        assert gathered[0] != gathered[1]     # distinct replicas per rank
    assert out[0][1] == out[1][1]             # both ranks saw the same exchange
