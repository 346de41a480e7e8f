"""Per-image sharding of a packed batch (host logic, CPU only).

The split is checked against brute force on small cost lists; the cut-out shards against
the whole batch: every rank renders its meshes with the float64 oracle (standing in for
the GPU, which these CPU tests do not have) and the ranks' images and vertex gradients,
summed over two gloo processes, equal the oracle run on the whole batch.
"""
import itertools
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from differentiable_mesh_rasterization_b200 import sharding
from differentiable_mesh_rasterization_b200 import synthetic as syn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def best_makespan(costs, world):
    best = float("inf")
    for assign in itertools.product(range(world), repeat=len(costs)):
        load = [0.0] * world
        for c, r in zip(costs, assign):
            load[r] += c
        best = min(best, max(load))
    return best


@pytest.mark.parametrize("seed", range(6))
def test_partition_is_a_balanced_split(seed):
    rng = np.random.default_rng(seed)
    n, world = int(rng.integers(1, 9)), int(rng.integers(1, 4))
    costs = rng.integers(0, 100, n).astype(float)
    parts = sharding.partition_meshes(costs, world)
    assert len(parts) == world
    assert sorted(np.concatenate(parts).tolist()) == list(range(n))     # each mesh exactly once
    assert all(np.all(np.diff(p) > 0) for p in parts)
    span = max(costs[p].sum() for p in parts)
    assert span <= 4 / 3 * best_makespan(costs, world) + 1e-9           # LPT bound
    assert all(np.array_equal(a, b) for a, b in zip(parts, sharding.partition_meshes(costs, world)))


def test_partition_edge_cases():
    assert [p.tolist() for p in sharding.partition_meshes([], 3)] == [[], [], []]
    assert [p.tolist() for p in sharding.partition_meshes([5.0, 5.0], 4)] == [[0], [1], [], []]
    assert [p.tolist() for p in sharding.partition_meshes([1.0, 7.0, 3.0], 1)] == [[0, 1, 2]]
    assert [p.tolist() for p in sharding.partition_meshes([0.0] * 5, 2)] == [[0, 2, 4], [1, 3]]
    with pytest.raises(ValueError):
        sharding.partition_meshes([1.0], 0)


def test_shard_index_maps():
    b = syn.make_batch(2, n_meshes=4)
    sh = sharding.Shard(b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, [3, 1])
    assert np.array_equal(sh.num, b.num_faces_per_mesh[[3, 1]])
    assert sh.first.tolist() == [0, int(b.num_faces_per_mesh[3])]
    # the cut-out faces, mapped back, are the batch's faces of meshes 3 and 1
    assert np.array_equal(sh.vert_ids[sh.faces], b.faces[sh.face_ids])
    f3 = b.mesh_to_face_first_idx[3]
    assert sh.face_ids[0] == f3 and sh.global_faces(np.array([[0, -1]])).tolist() == [[f3, -1]]
    empty = sharding.Shard(b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, [])
    assert empty.faces.shape == (0, 3) and empty.first.size == 0
    counts = sharding.mesh_sample_counts(b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh,
                                         b.workload.H, b.workload.W, b.workload.blur_radius)
    assert counts.shape == (4,) and np.all(counts > 0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _render(oracle, verts, faces, first, num, w, ga):
    """Oracle forward (silhouette) and fused backward of one packed batch."""
    p2f, _, _, dists, _ = oracle.rasterize_fwd(verts, faces, first, num, w.H, w.W, np.float32(w.blur_radius), w.K,
                                               w.perspective_correct, exempt=False)
    alpha = oracle.silhouette_fwd(p2f, dists, np.float32(w.sigma))
    gd = oracle.silhouette_bwd(ga, p2f, dists, np.float32(w.sigma))
    gv = oracle.rasterize_bwd(verts, faces, p2f, w.perspective_correct, grad_dists=gd)
    return p2f, alpha, gv


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b = syn.make_batch(2, n_meshes=5)
        w = b.workload
        ga = syn.grad_alpha(b)
        costs = sharding.mesh_sample_counts(b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh,
                                            w.H, w.W, w.blur_radius)
        mine = sharding.partition_meshes(costs, world)[rank]
        sh = sharding.Shard(b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, mine)
        p2f, alpha, gv = _render(oracle, b.verts[sh.vert_ids], sh.faces, sh.first, sh.num, w, ga[mine])
        # only to compare on one rank: the data path itself exchanges nothing
        P = torch.from_numpy(sh.scatter_images(sh.global_faces(p2f) + 1, b.N))
        A = torch.from_numpy(sh.scatter_images(alpha, b.N))
        G = torch.from_numpy(sh.scatter_vertex_rows(gv, b.verts.shape[0]))
        for t in (P, A, G):
            dist.all_reduce(t)
        q.put((rank, len(mine), P.numpy() - 1, A.numpy(), G.numpy()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_reproduce_the_whole_batch(oracle_mod):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    b = syn.make_batch(2, n_meshes=5)
    w = b.workload
    p2f, alpha, gv = _render(oracle_mod, b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, w,
                             syn.grad_alpha(b))
    assert res[0][1] > 0 and res[1][1] > 0 and res[0][1] + res[1][1] == b.N
    for _, _, P, A, G in res:
        assert np.array_equal(P, p2f)
        assert np.array_equal(A, alpha)
        assert np.allclose(G, gv, rtol=1e-10, atol=1e-12 * np.abs(gv).max())


@pytest.mark.parametrize("cfg", [2, 5])
def test_shard_costs_add_up_to_the_benchmark_sample_count(cfg):
    """The cost model of the split and the benchmark's sample count are written separately;
    summed over meshes they must agree, so a split run reports the same total work."""
    sys.path.insert(0, ROOT)
    import bench
    b = syn.make_batch(cfg)
    w = b.workload
    costs = sharding.mesh_sample_counts(b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, w.H, w.W,
                                        w.blur_radius)
    assert int(costs.sum()) == bench.count_samples(b)
