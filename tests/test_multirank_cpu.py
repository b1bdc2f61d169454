"""The benchmark's multi-rank host logic with two gloo ranks on the CPU:
barriers, the max over ranks of the timed region, the whole-job throughput,
and the reference arm running on rank 0 only."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist

    import bench
    r, w, local = bench.init_distributed(backend="gloo")
    try:
        bench.barrier(w, local)
        cpu = torch.device("cpu")
        maxes = bench.max_over_ranks([float(r + 1), 10.0 - r], w, cpu)
        # each rank "ran" 100 TFLOP; rank r took (r + 1) seconds
        value, slowest = bench.aggregate(100e12, 1000.0 * (r + 1), w, cpu)
        args = bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "3",
                                 "--workload", "single_head_f32_64"])
        ref = bench.run_reference(args, bench.synth.workload("single_head_f32_64"), r, w)
        q.put((r, maxes, value, slowest, ref is None, None if ref is None else ref["impl"]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, maxes, value, slowest, ref_none, impl in results:
        assert maxes == [2.0, 10.0]
        assert slowest == pytest.approx(2000.0)
        assert value == pytest.approx(100.0)     # 2 x 100 TFLOP over the slowest 2 s
        assert ref_none == (r != 0)
        assert impl == ("reference" if r == 0 else None)
