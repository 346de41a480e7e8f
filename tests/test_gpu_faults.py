"""Error paths under injected host-side failures (no GPU fault is ever caused).

mr_inject_fault makes the library's n-th scratch allocation fail with MR_ERR_OOM or
MR_ERR_CUDA before it allocates.  Each case checks that the entry point returns that code
with its message, that the scratch it had already taken is released (the default pool's
used bytes return to their level before the call), and that the next call succeeds and
matches a clean run.
"""
import pytest
import torch

import differentiable_mesh_rasterization_b200 as mr
from differentiable_mesh_rasterization_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from differentiable_mesh_rasterization_b200 import build
    build.build()
    yield
    mr.inject_fault("off")


@pytest.fixture(scope="module")
def batch():
    b = syn.make_batch(2)
    w = b.workload
    v = torch.from_numpy(b.verts).cuda()
    f = torch.from_numpy(b.faces).cuda()
    args = (v, f, b.mesh_to_face_first_idx, b.num_faces_per_mesh, w.H, w.W, w.blur_radius, w.K)
    ref = mr.rasterize_fwd(*args, sigma=w.sigma)
    torch.cuda.synchronize()
    return b, args, ref


def _expect_failure(kind, skip, call):
    code = {"oom": -2, "cuda": -3}[kind]
    torch.cuda.synchronize()
    before = mr.scratch_in_use()
    mr.inject_fault(kind, skip)
    with pytest.raises(mr.MeshRastError) as e:
        call()
    assert e.value.code == code and "injected" in str(e.value)
    torch.cuda.synchronize()
    assert mr.scratch_in_use() == before, "scratch taken before the failure was not released"


@pytest.mark.parametrize("kind", ["oom", "cuda"])
@pytest.mark.parametrize("skip", [0, 1])
def test_forward_fails_cleanly_and_recovers(batch, kind, skip):
    """skip 0: the first allocation (face records, counts) fails; skip 1: the bin lists'
    allocation fails after the face setup and count kernels have run on the first."""
    b, args, ref = batch
    w = b.workload
    _expect_failure(kind, skip, lambda: mr.rasterize_fwd(*args, sigma=w.sigma))
    got = mr.rasterize_fwd(*args, sigma=w.sigma)
    for x, y in zip(got, ref):
        assert torch.equal(x, y)


@pytest.mark.parametrize("kind", ["oom", "cuda"])
def test_backward_fails_cleanly_and_recovers(batch, kind):
    b, args, ref = batch
    w = b.workload
    v, f = args[0], args[1]
    ga = torch.from_numpy(syn.grad_alpha(b)).cuda()
    want = mr.silhouette_rasterize_bwd(v, f, ref[0], ref[3], w.sigma, ga)
    _expect_failure(kind, 0, lambda: mr.silhouette_rasterize_bwd(v, f, ref[0], ref[3], w.sigma, ga))
    got = mr.silhouette_rasterize_bwd(v, f, ref[0], ref[3], w.sigma, ga)
    # float atomics: the order of the additions, and so the last bits, vary from run to run
    assert torch.allclose(got, want, rtol=1e-5, atol=1e-5 * float(want.abs().max()))


def test_point_and_knn_paths_fail_cleanly_and_recover():
    pb = syn.make_point_batch(2)
    w = pb.workload
    P = torch.from_numpy(pb.points).cuda()
    call = lambda: mr.rasterize_points_fwd(P, pb.cloud_first_idx, pb.num_points_per_cloud, w.H, w.W, w.radius, w.K)
    want = call()
    _expect_failure("oom", 0, call)
    for x, y in zip(call(), want):
        assert torch.equal(x, y)
    kb = syn.make_knn_batch(2)
    A, B = torch.from_numpy(kb.p1).cuda(), torch.from_numpy(kb.p2).cuda()
    call = lambda: mr.knn_fwd(A, kb.first1, kb.num1, B, kb.first2, kb.num2, 8)
    want = call()
    _expect_failure("cuda", 0, call)
    for x, y in zip(call(), want):
        assert torch.equal(x, y)


def test_scratch_free_forward_is_not_affected_by_the_hook(batch):
    """The scratch-free forward allocates nothing, so an armed hook never fires there."""
    b, args, ref = batch
    mr.inject_fault("oom", 0)
    try:
        got = mr.rasterize_fwd_noalloc(*args)
    finally:
        mr.inject_fault("off")
    for x, y in zip(got, ref[:4]):
        assert torch.equal(x, y)


def test_scratch_peak_reports_the_forward_scratch(batch):
    """The pool's high-water mark covers the forward's scratch (160 bytes of records per
    face, bin counts and lists), all of which is released when the call's stream is done."""
    b, args, ref = batch
    torch.cuda.synchronize()
    base = mr.scratch_in_use()
    mr.scratch_peak(reset=True)
    mr.rasterize_fwd(*args)
    torch.cuda.synchronize()
    peak = mr.scratch_peak(reset=True)
    assert peak - base >= b.faces.shape[0] * 160
    assert mr.scratch_in_use() == base
