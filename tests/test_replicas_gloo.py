"""The multi-GPU form of this path is replicas (one batch per rank, no
collective on the data path): its host logic, run as two gloo ranks on CPU.

Each rank builds its replica's inputs with bench.replica_inputs, the ranks
agree on the step time through bench.max_over_ranks, and each rank's layer
output, computed by the oracle on a few tokens, depends only on its own
inputs."""
import os
import socket

import numpy as np


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    import oracle
    import synth
    dist, r, ws, _ = bench._dist("gloo")
    assert (r, ws) == (rank, world)
    wl = synth.workload("tiny")
    inp = bench.replica_inputs(wl, rank)
    # step times differ per rank; every rank must see the largest
    t = bench.max_over_ranks(1.5 + rank, dist, "cpu")
    y, _, _ = oracle.moe_forward(**inp, tokens=np.arange(4, dtype=np.int32))
    np.savez(os.path.join(out_dir, f"rank{rank}.npz"), t=t, x=inp["x"], w1=inp["w1"],
             idx=inp["topk_idx"], y=y)
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_replicas(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    r0 = np.load(tmp_path / "rank0.npz")
    r1 = np.load(tmp_path / "rank1.npz")
    assert float(r0["t"]) == float(r1["t"]) == 2.5          # max over ranks
    assert np.array_equal(r0["w1"], r1["w1"])                # shared weights
    assert not np.array_equal(r0["x"], r1["x"])              # own activations
    assert not np.array_equal(r0["idx"], r1["idx"])          # own routing
    # rank 1's output is the single-process oracle on rank 1's inputs
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import oracle
    import synth
    inp1 = bench.replica_inputs(synth.workload("tiny"), 1)
    y1, _, _ = oracle.moe_forward(**inp1, tokens=np.arange(4, dtype=np.int32))
    assert np.array_equal(r1["y"], y1)


def test_reference_arm_other_ranks_do_no_work(capsys):
    """Under torchrun the reference arm runs on rank 0 only: rank 1 returns at
    once and prints nothing."""
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import synth

    class A:
        steps, warmup = 1, 0
    bench.run_reference(A(), synth.workload("tiny"), rank=1)
    assert capsys.readouterr().out == ""
