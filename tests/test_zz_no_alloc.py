"""The scratch-free forward entry point (mr_rasterize_fwd_noalloc), checked on the GPU.

Some callers of this library cannot allocate device memory while they render (their
host owns all device memory in its own pool, or an allocation could stall or fail
inside a latency-critical loop).  mr_rasterize_fwd_noalloc serves them: it takes all
of its scratch from one fixed device array inside the library.  These tests call it
through the C ABI and compare it with the allocating mr_rasterize_fwd, on two calls in
a row (the shared array keeps the previous call's contents, so the second call checks
that everything that must start at zero is cleared).

This file is named to be collected last, so a run that stops at the first failure has
already run every other test; it also passes when run alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import differentiable_mesh_rasterization_b200 as mr
from differentiable_mesh_rasterization_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

ABS = 1e-5
ULP = 2.0 ** -23


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from differentiable_mesh_rasterization_b200 import build
    build.build()


def _same(a, b, label):
    p_a, z_a, b_a, d_a = a
    p_b, z_b, b_b, d_b = b
    assert torch.equal(p_a, p_b), f"{label}: pix_to_face differs"
    for name, x, y in (("zbuf", z_a, z_b), ("bary", b_a, b_b), ("dists", d_a, d_b)):
        tol = ABS + ULP * y.abs()
        assert bool(((x - y).abs() <= tol).all()), f"{label}: {name} differs beyond tolerance"


def _inputs(cfg, n_meshes, H=None, W=None):
    b = syn.make_batch(cfg, n_meshes=n_meshes)
    w = b.workload
    v = torch.from_numpy(b.verts).cuda()
    f = torch.from_numpy(b.faces).cuda()
    return (v, f, b.mesh_to_face_first_idx, b.num_faces_per_mesh, H or w.H, W or w.W, w.blur_radius, w.K,
            w.perspective_correct)


def test_noalloc_matches_allocating_forward_on_two_calls():
    big = _inputs(2, None)                 # 8 images 137x137, K=8: fits the fixed scratch
    small = _inputs(3, 1, 96, 80)          # a different, smaller batch next
    for label, args in (("first call", big), ("second call", small), ("third call", big)):
        want = mr.rasterize_fwd(*args)
        got = mr.rasterize_fwd_noalloc(*args)
        torch.cuda.synchronize()
        _same(got, want, label)
        assert int((got[0] >= 0).sum()) > 1000


def test_noalloc_rejects_batches_beyond_its_scratch():
    """The first limit: the 64 meshes of the 512x512 batch hold 2.35 M faces, whose records
    (160 bytes each) alone exceed the fixed array; rejected before anything is launched
    (a small image keeps the outputs small)."""
    b = syn.make_batch(5)
    v = torch.from_numpy(b.verts).cuda()
    f = torch.from_numpy(b.faces).cuda()
    with pytest.raises(mr.MeshRastError) as e:
        mr.rasterize_fwd_noalloc(v, f, b.mesh_to_face_first_idx, b.num_faces_per_mesh, 32, 32, 1e-5, 4, False)
    assert e.value.code == -1 and "scratch" in str(e.value)



def test_noalloc_rejects_bin_lists_beyond_its_scratch_and_recovers():
    """The second limit: the fixed part of the scratch fits (one 2048x2048 image, K=1), but
    the per-bin face lists found by the count pass do not (a blur radius of 1.4 in NDC puts
    each of the 1280 faces into all 16384 bins).  The call has already run kernels on the
    shared array when it refuses; the next call must still match mr_rasterize_fwd."""
    verts, faces = syn.icosphere(3)
    v = torch.from_numpy(syn.project(verts * 0.5).astype(np.float32)).cuda()
    f = torch.from_numpy(faces.astype(np.int64)).cuda()
    with pytest.raises(mr.MeshRastError) as e:
        mr.rasterize_fwd_noalloc(v, f, [0], [faces.shape[0]], 2048, 2048, 2.0, 1, False)
    assert e.value.code == -1 and "bin lists" in str(e.value)
    args = _inputs(2, None)
    want = mr.rasterize_fwd(*args)
    got = mr.rasterize_fwd_noalloc(*args)
    torch.cuda.synchronize()
    _same(got, want, "after the refused call")


def test_noalloc_takes_device_resident_mesh_arrays():
    v, f, first, num, H, W, blur, K, persp = _inputs(2, None)
    want = mr.rasterize_fwd(v, f, first, num, H, W, blur, K, persp)
    got = mr.rasterize_fwd_noalloc(v, f, torch.as_tensor(first).cuda(), torch.as_tensor(num).cuda(), H, W, blur, K,
                                   persp)
    torch.cuda.synchronize()
    _same(got, want, "device-resident per-mesh arrays")

