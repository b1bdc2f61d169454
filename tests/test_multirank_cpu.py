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


def _split_worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist

    import bench
    r, w_, local = bench.init_distributed(backend="gloo")
    try:
        wl = bench.synth.make_small(3, 5, 70, 70, 16, 16, "bf16", True, seed=9,
                                    lengths=(70, 33, 1))
        full = bench.synth.make_inputs(wl)
        parts = bench.make_parts(wl, "heads", r, w_)
        problems, same = [], True
        for sub, ts, kl, flops in parts:
            b0 = int(sub.name.split("[b")[1].split(":")[0])
            h0 = int(sub.name.split(",h")[1].split(":")[0])
            problems += [(b0 + b, h0 + h) for b in range(sub.B) for h in range(sub.H)]
            for t, f in zip(ts, full):
                same = same and torch.equal(t, f[b0:b0 + sub.B, h0:h0 + sub.H])
            same = same and (kl == wl.key_len()[b0:b0 + sub.B])
        local_flops = sum(p[3] for p in parts)
        job = bench.sum_over_ranks(local_flops, w_, torch.device("cpu"))
        gathered = [None] * w_
        dist.all_gather_object(gathered, problems)
        q.put((r, same, job, wl.bwd_flops(), gathered))
    finally:
        dist.destroy_process_group()


def test_heads_split_over_two_gloo_ranks():
    """--split heads: the two ranks' slices cover every (batch, head) problem
    exactly once, carry the 1-GPU run's inputs and key lengths, and their
    FLOPs add up to the workload's."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, same, job, want, gathered in results:
        assert same
        assert job == pytest.approx(want)
        flat = [x for g in gathered for x in g]
        assert sorted(flat) == [(b, h) for b in range(3) for h in range(5)]
        assert len(flat) == len(set(flat))


@pytest.mark.parametrize("B,H", [(1, 1), (2, 32), (3, 5), (8, 16), (1, 32)])
def test_rank_slices_tile_the_problems(B, H):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    for world in range(1, 10):
        seen = []
        for r in range(world):
            for b0, nb, h0, nh in bench.slice_runs(B, H, *bench.rank_slice(B * H, r, world)):
                assert nb == 1 or (h0 == 0 and nh == H)
                seen += [(b0 + b) * H + h0 + h for b in range(nb) for h in range(nh)]
        assert seen == list(range(B * H))
