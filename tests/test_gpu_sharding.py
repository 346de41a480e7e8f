"""The per-image split of a batch over ranks, rendered through the CUDA library.

Each rank's shard (its meshes cut out of the packed batch by ``sharding.Shard``) is
rendered here one after the other on the one GPU, exactly as that rank would render it on
its own GPU, and the results are put back in the batch's numbering.  Face ids keep their
order inside a shard, so depth ties break the same way: pix_to_face and the silhouette
equal the whole-batch run bit for bit; the vertex gradients come from float atomics, whose
order of addition differs, so they agree to rounding.
"""
import numpy as np
import pytest
import torch

import differentiable_mesh_rasterization_b200 as mr
from differentiable_mesh_rasterization_b200 import sharding
from differentiable_mesh_rasterization_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from differentiable_mesh_rasterization_b200 import build
    build.build()


def _render(verts, faces, first, num, w, ga):
    v = torch.from_numpy(np.ascontiguousarray(verts)).cuda()
    f = torch.from_numpy(np.ascontiguousarray(faces)).cuda()
    p2f, _, _, dists, alpha = mr.rasterize_fwd(v, f, first, num, w.H, w.W, w.blur_radius, w.K,
                                               w.perspective_correct, sigma=w.sigma)
    gv = mr.silhouette_rasterize_bwd(v, f, p2f, dists, w.sigma, torch.from_numpy(np.ascontiguousarray(ga)).cuda())
    return p2f.cpu().numpy(), alpha.cpu().numpy(), gv.cpu().numpy()


@pytest.mark.parametrize("cfg", [2, 5])
@pytest.mark.parametrize("world", [2, 4])
def test_shards_reproduce_the_whole_batch(cfg, world):
    b = syn.make_batch(cfg)
    w = b.workload
    ga = syn.grad_alpha(b)[:b.N]
    p2f, alpha, gv = _render(b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, w, ga)
    costs = sharding.mesh_sample_counts(b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, w.H, w.W,
                                        w.blur_radius)
    parts = sharding.partition_meshes(costs, world)
    assert sorted(np.concatenate(parts).tolist()) == list(range(b.N))
    P = np.full_like(p2f, -1)
    A = np.zeros_like(alpha)
    G = np.zeros_like(gv)
    loads = []
    for mine in parts:
        if len(mine) == 0:
            continue
        sh = sharding.Shard(b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, mine)
        sp, sa, sg = _render(b.verts[sh.vert_ids], sh.faces, sh.first, sh.num, w, ga[mine])
        P[mine] = sh.global_faces(sp)
        A[mine] = sa
        G += sh.scatter_vertex_rows(sg, b.verts.shape[0])
        loads.append(int(costs[mine].sum()))
    assert np.array_equal(P, p2f)
    assert np.array_equal(A, alpha)
    scale = np.abs(gv).max()
    assert np.allclose(G, gv, rtol=1e-5, atol=1e-6 * scale)
    # the split balances the fine pass's work: no rank above 4/3 of the mean plus one mesh
    assert max(loads) <= sum(loads) / world * 4 / 3 + costs.max()
