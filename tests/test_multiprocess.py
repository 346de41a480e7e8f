"""Multi-process host logic of the benchmark on CPU (gloo, world size 2).

The rasterizer partitions by image, so ranks exchange nothing on the data path; the
only collectives are the measurement's: the maximum of the device times and the sums
of samples and pixels.  Each rank renders its own seeded batch (weak scaling).
"""
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    from differentiable_mesh_rasterization_b200 import synthetic as syn
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b = syn.make_batch(2, seed=bench.rank_seed(2, rank), n_meshes=2)
        samples = bench.count_samples(b)
        dev_ms = 10.0 + 5.0 * rank
        out = bench.combine_ranks(dev_ms, float(samples), float(b.N * 137 * 137))
        q.put((rank, samples, out, float(b.verts.sum())))
    finally:
        dist.destroy_process_group()


def test_two_ranks_weak_scaling_reduction():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, s0, out0, v0), (r1, s1, out1, v1) = res
    assert out0 == out1                          # every rank sees the same totals
    assert out0[0] == 15.0                       # max over ranks of the device time
    assert out0[1] == s0 + s1                    # samples summed over ranks
    assert out0[2] == 2 * 2 * 137 * 137
    assert v0 != v1                              # ranks render different batches


def test_single_process_reduction_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.combine_ranks(3.0, 5.0, 7.0) == (3.0, 5.0, 7.0)
    assert bench.rank_seed(5, 0) == 1005 and bench.rank_seed(5, 3) == 4005
