"""Parity of the CUDA point-cloud renderer (rasterization, compositing, their gradients)
and of the batched KNN with the float64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import differentiable_mesh_rasterization_b200 as mr
from differentiable_mesh_rasterization_b200 import synthetic as syn

from _parity import EXEMPT_MAX, compare_grad, np_

pytestmark = pytest.mark.gpu

ABS = 1e-5
ULP = 2.0 ** -23


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from differentiable_mesh_rasterization_b200 import build
    build.build()


def cuda(a, dtype=None):
    return torch.from_numpy(np.ascontiguousarray(a if dtype is None else a.astype(dtype))).cuda()


def _compare_slots(got, want, flags, label):
    """idx exact outside flagged pixels; zbuf, dists within 1e-5 + 1 ulp there."""
    gi, gz, gd = (np_(x) for x in got)
    wi, wz, wd, = want
    ok = ~flags
    assert flags.mean() <= EXEMPT_MAX, f"{label}: {flags.mean():.3%} flagged"
    assert np.array_equal(gi[ok], wi[ok]), f"{label}: idx differs at {np.argwhere((gi != wi).any(-1) & ok)[:5]}"
    for name, x, y in (("zbuf", gz, wz), ("dists", gd, wd)):
        err = (np.abs(x - y) - (ABS + ULP * np.abs(y)))[ok]
        assert err.size == 0 or err.max() <= 0, f"{label}: {name} off by {err.max():.3g}"


@pytest.fixture(scope="module")
def pts2(oracle_mod):
    pb = syn.make_point_batch(2)
    w = pb.workload
    o = oracle_mod.rasterize_points(pb.points, pb.cloud_first_idx, pb.num_points_per_cloud, w.H, w.W, w.radius, w.K)
    return pb, o


def test_point_rasterizer_matches_oracle(pts2):
    pb, (wi, wz, wd, flags) = pts2
    w = pb.workload
    got = mr.rasterize_points_fwd(cuda(pb.points), pb.cloud_first_idx, pb.num_points_per_cloud, w.H, w.W,
                                  np.float32(w.radius), w.K)
    assert (wi >= 0).mean() > 0.05
    _compare_slots(got, (wi, wz, wd), flags[..., None].repeat(w.K, -1), "points batch 2")
    mr.device_status()


@pytest.mark.parametrize("K,H,W,radius", [(1, 33, 47, 0.03), (3, 64, 40, 0.01), (16, 50, 50, 0.05)])
def test_point_rasterizer_shapes_and_ragged_tiles(oracle_mod, K, H, W, radius):
    pb = syn.make_point_batch(2, n_clouds=3)
    got = mr.rasterize_points_fwd(cuda(pb.points), pb.cloud_first_idx, pb.num_points_per_cloud, H, W,
                                  np.float32(radius), K)
    wi, wz, wd, flags = oracle_mod.rasterize_points(pb.points, pb.cloud_first_idx, pb.num_points_per_cloud, H, W,
                                                    np.float32(radius), K)
    _compare_slots(got, (wi, wz, wd), flags[..., None].repeat(K, -1), f"K={K} {H}x{W}")


def test_point_rasterizer_edge_cases(oracle_mod):
    """Empty clouds, points behind the camera, points off screen, a cloud of one point."""
    rng = np.random.default_rng(5)
    pts = np.concatenate([rng.uniform(-1.2, 1.2, size=(300, 2)), rng.uniform(-0.5, 3, size=(300, 1))], 1)
    pts = pts.astype(np.float32)
    first = np.array([0, 100, 100, 299], np.int64)
    num = np.array([100, 0, 199, 1], np.int64)
    got = mr.rasterize_points_fwd(cuda(pts), first, num, 24, 20, np.float32(0.2), 5)
    wi, wz, wd, flags = oracle_mod.rasterize_points(pts, first, num, 24, 20, np.float32(0.2), 5)
    assert np.all(np_(got[0])[1] == -1)
    _compare_slots(got, (wi, wz, wd), flags[..., None].repeat(5, -1), "edge cases")
    empty = mr.rasterize_points_fwd(cuda(pts), first, num, 8, 8, np.float32(0.0), 2)
    assert int((np_(empty[0]) >= 0).sum()) <= 4            # radius 0: only exact centre hits



@pytest.mark.parametrize("H,W,K", [(64, 64, 8), (40, 72, 4), (37, 53, 3)])
def test_point_outputs_are_fully_written(H, W, K):
    """Outputs pre-filled with a sentinel: a few points leave most 16 x 16 bins empty (those
    write their padding before any pixel arithmetic); every element is written and equals
    a call into fresh buffers."""
    rng = np.random.default_rng(5)
    pts = np.concatenate([rng.uniform(-0.15, 0.15, (40, 2)), rng.uniform(1.0, 3.0, (40, 1))], 1).astype(np.float32)
    p = torch.from_numpy(pts).cuda()
    ref = mr.rasterize_points_fwd(p, [0], [40], H, W, 0.05, K)
    idx = torch.full((1, H, W, K), 987654, dtype=torch.int64, device="cuda")
    zbuf, dists = (torch.full((1, H, W, K), 7.5, device="cuda") for _ in range(2))
    first, num = np.array([0], np.int64), np.array([40], np.int64)
    rc = mr.load_library().mr_rasterize_points_fwd(p.data_ptr(), 40, first.ctypes.data, num.ctypes.data, 1, H, W,
                                                   0.05, K, idx.data_ptr(), zbuf.data_ptr(), dists.data_ptr(),
                                                   torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == 0
    for got, want in zip((idx, zbuf, dists), ref):
        assert torch.equal(got, want)
    assert (ref[0] >= 0).any() and (ref[0][..., 0] == -1).float().mean() > 0.5


def test_point_at_exactly_the_radius_is_kept(oracle_mod):
    """Dyadic point and radius (two pixel pitches): the squared distance ties r^2 exactly in
    float32 too, and the threshold is inclusive on both sides."""
    H = W = 32
    x0, y0 = -1 + 21 / W, 1 - 21 / H                # pixel (10, 10)
    r = 4.0 / W
    pts = np.array([[x0, y0, 1.0]], np.float32)
    gi = np_(mr.rasterize_points_fwd(cuda(pts), np.array([0]), np.array([1]), H, W, np.float32(r), 1)[0])
    wi, *_ = oracle_mod.rasterize_points(pts, [0], [1], H, W, r, 1)
    assert np.array_equal(gi, wi)
    for i, j in ((10, 12), (10, 8), (12, 10), (8, 10)):
        assert gi[0, i, j, 0] == 0

def test_point_rasterizer_full_size_sampled(oracle_mod):
    """The benchmark batch (64 clouds, 1.18 M points, 512x512, K=8) in the benchmark's launch,
    checked at sampled pixels against the oracle and everywhere by properties."""
    pb = syn.make_point_batch(5)
    w = pb.workload
    P = cuda(pb.points)
    idx, zbuf, dists = (np_(x) for x in mr.rasterize_points_fwd(P, pb.cloud_first_idx, pb.num_points_per_cloud,
                                                                 w.H, w.W, np.float32(w.radius), w.K))
    mr.device_status()
    # properties at every slot: the reported point is within the radius, in front, of the
    # pixel's own cloud; slots are in (z, id) order; zbuf / dists recompute from the point
    valid = idx >= 0
    assert valid.mean() > 0.05
    n_of = np.repeat(np.arange(pb.N), pb.num_points_per_cloud)
    n_img = np.broadcast_to(np.arange(pb.N)[:, None, None, None], idx.shape)
    assert np.all(n_of[idx[valid]] == n_img[valid])
    pv = pb.points.astype(np.float64)[idx[valid]]
    assert np.all(pv[:, 2] >= 0) and np.array_equal(zbuf[valid], pb.points[idx[valid], 2])
    jj = np.broadcast_to(np.arange(w.W)[None, None, :, None], idx.shape)[valid]
    ii = np.broadcast_to(np.arange(w.H)[None, :, None, None], idx.shape)[valid]
    d2 = (-1 + (2 * jj + 1) / w.W - pv[:, 0]) ** 2 + (1 - (2 * ii + 1) / w.H - pv[:, 1]) ** 2
    assert np.all(np.abs(dists[valid] - d2) <= ABS + ULP * d2)
    assert np.all(d2 <= np.float64(np.float32(w.radius)) ** 2 * (1 + 1e-5))
    z = np.where(valid, zbuf, np.inf)
    zi = np.where(valid, idx, np.iinfo(np.int64).max)
    order_ok = (z[..., :-1] < z[..., 1:]) | ((z[..., :-1] == z[..., 1:]) & (zi[..., :-1] < zi[..., 1:]))
    assert np.all(order_ok | ~valid[..., 1:])
    assert np.all(valid[..., :-1] | ~valid[..., 1:])        # padding only at the end
    # sampled pixels against the oracle
    rng = np.random.default_rng(11)
    pix = np.concatenate([rng.choice(np.flatnonzero(valid[..., 0].reshape(-1)), 3000, replace=False),
                          rng.integers(0, pb.N * w.H * w.W, 500)])
    wi, wz, wd, flags = oracle_mod.rasterize_points(pb.points, pb.cloud_first_idx, pb.num_points_per_cloud, w.H,
                                                    w.W, np.float32(w.radius), w.K, pixels=pix)
    got = tuple(x.reshape(-1, w.K)[pix] for x in (idx, zbuf, dists))
    _compare_slots(got, (wi, wz, wd), flags[:, None].repeat(w.K, -1), "batch 5 sampled")


@pytest.mark.parametrize("mode", ["alpha", "norm_weighted"])
def test_compositing_matches_oracle(oracle_mod, pts2, mode):
    pb, (wi, wz, wd, flags) = pts2
    w = pb.workload
    d32 = wd.astype(np.float32)
    feats = pb.features
    got = np_(mr.composite_points_fwd(cuda(wi), cuda(d32), cuda(feats), np.float32(w.radius), mode))
    want = oracle_mod.composite_points(wi, d32, feats, np.float32(w.radius), mode)
    err = np.abs(got - want) - (1e-4 * np.abs(want) + 1e-6)
    assert err.max() <= 0, f"{mode}: off by {err.max():.3g}"
    g = syn.random_grads(want.shape, 21)
    gf, gd = mr.composite_points_bwd(cuda(wi), cuda(d32), cuda(feats), np.float32(w.radius), cuda(g), mode)
    wf, wdd = oracle_mod.composite_points_bwd(wi, d32, feats, np.float32(w.radius), g, mode)
    compare_grad(gf, wf, label=f"{mode} grad_features")
    compare_grad(gd, wdd, label=f"{mode} grad_dists")


def test_point_rasterizer_backward_matches_oracle(oracle_mod, pts2):
    pb, (wi, wz, wd, flags) = pts2
    gz = syn.random_grads(wi.shape, 22)
    gd = syn.random_grads(wi.shape, 23)
    got = mr.rasterize_points_bwd(cuda(pb.points), cuda(wi), cuda(gz), cuda(gd))
    want = oracle_mod.rasterize_points_bwd(pb.points, wi, gz, gd)
    compare_grad(got, want, label="point raster bwd")
    only_z = mr.rasterize_points_bwd(cuda(pb.points), cuda(wi), grad_zbuf=cuda(gz))
    compare_grad(only_z, oracle_mod.rasterize_points_bwd(pb.points, wi, gz, None), label="only zbuf")


def test_point_render_end_to_end(oracle_mod):
    """points, features -> K nearest -> alpha compositing -> loss, and back to the points'
    screen positions and features, against the oracle's chain (flagged pixels left out)."""
    pb = syn.make_point_batch(2)
    w = pb.workload
    P, F = cuda(pb.points), cuda(pb.features)
    r = np.float32(w.radius)
    idx, zbuf, dists = mr.rasterize_points_fwd(P, pb.cloud_first_idx, pb.num_points_per_cloud, w.H, w.W, r, w.K)
    img = mr.composite_points_fwd(idx, dists, F, r)
    g = syn.random_grads(tuple(img.shape), 24)
    gf, gd = mr.composite_points_bwd(idx, dists, F, r, cuda(g))
    gp = mr.rasterize_points_bwd(P, idx, grad_dists=gd)
    mr.device_status()
    wi, wz, wd, flags = oracle_mod.rasterize_points(pb.points, pb.cloud_first_idx, pb.num_points_per_cloud, w.H, w.W,
                                                    r, w.K)
    wimg = oracle_mod.composite_points(wi, wd, pb.features, r)
    ok = ~flags
    err = (np.abs(np_(img) - wimg) - (1e-4 * np.abs(wimg) + 1e-5))[ok]
    assert err.max() <= 0
    wf, wdd = oracle_mod.composite_points_bwd(wi, wd, pb.features, r, g)
    wp = oracle_mod.rasterize_points_bwd(pb.points, wi, None, wdd)
    touched = np.zeros(pb.points.shape[0], bool)
    for a in (wi[flags], np_(idx)[flags]):
        touched[a[a >= 0]] = True
    keep = ~touched
    assert keep.mean() > 0.9
    compare_grad(np_(gf)[keep], wf[keep], label="grad features")
    compare_grad(np_(gp)[keep], wp[keep], label="grad points")


def _compare_knn(gi, gd, wi, wd, flags, label):
    ok = ~flags
    assert flags.mean() < 0.02, f"{label}: {flags.mean():.3%} flagged"
    assert np.array_equal(gi[ok], wi[ok]), f"{label}: idx differs at {np.argwhere((gi != wi).any(-1) & ok)[:5]}"
    # float32 distances from float32 differences: a few ulps of the value
    tol = 1e-9 + 8 * ULP * np.abs(wd)
    assert np.all(np.abs(gd - wd) <= tol), f"{label}: dists off by {np.max(np.abs(gd - wd) - tol):.3g}"
    # flagged queries: the same K distances (the order of near-ties is rounding's)
    assert np.array_equal(gi[flags] >= 0, wi[flags] >= 0)


@pytest.mark.parametrize("K", [1, 8, 20])
def test_knn_matches_oracle(oracle_mod, K):
    kb = syn.make_knn_batch(2)
    gi, gd = mr.knn_fwd(cuda(kb.p1), kb.first1, kb.num1, cuda(kb.p2), kb.first2, kb.num2, K)
    wi, wd, flags = oracle_mod.knn(kb.p1, kb.first1, kb.num1, kb.p2, kb.first2, kb.num2, K)
    _compare_knn(np_(gi), np_(gd), wi, wd, flags, f"knn batch 2 K={K}")


def test_knn_edge_cases(oracle_mod):
    """Fewer references than K, an empty reference cloud, queries outside every cloud, D=2."""
    rng = np.random.default_rng(6)
    p1 = rng.normal(size=(50, 2)).astype(np.float32)
    p2 = rng.normal(size=(30, 2)).astype(np.float32)
    f1, n1 = np.array([0, 20, 35]), np.array([20, 10, 10])      # queries 30..34 and 45..49 in no cloud
    f2, n2 = np.array([0, 5, 5]), np.array([5, 0, 25])
    gi, gd = mr.knn_fwd(cuda(p1), f1, n1, cuda(p2), f2, n2, 8)
    wi, wd, flags = oracle_mod.knn(p1, f1, n1, p2, f2, n2, 8)
    gi, gd = np_(gi), np_(gd)
    outside = np.r_[30:35, 45:50]
    assert np.all(gi[outside] == -1) and np.all(gd[outside] == -1)
    inside = np.setdiff1d(np.arange(50), outside)
    _compare_knn(gi[inside], gd[inside], wi[inside], wd[inside], flags[inside], "edge cases")
    assert np.all(gi[:20, 5:] == -1) and np.all(gi[20:30] == -1)


def test_knn_full_size_sampled(oracle_mod):
    """The benchmark batch (64 clouds, 1.18 M points, D=3, K=8) in the benchmark's launch,
    checked on sampled queries of every cloud against the oracle."""
    kb = syn.make_knn_batch(5)
    K = kb.workload.K
    gi, gd = (np_(x) for x in mr.knn_fwd(cuda(kb.p1), kb.first1, kb.num1, cuda(kb.p2), kb.first2, kb.num2, K))
    rng = np.random.default_rng(12)
    sel, n1 = [], []
    for n in range(kb.N):
        q = np.sort(rng.choice(kb.num1[n], min(40, kb.num1[n]), replace=False)) + kb.first1[n]
        n1.append(len(q))
        sel.append(q)
    sel = np.concatenate(sel)
    f1 = np.cumsum([0] + n1[:-1])
    wi, wd, flags = oracle_mod.knn(kb.p1[sel], f1, n1, kb.p2, kb.first2, kb.num2, K)
    _compare_knn(gi[sel], gd[sel], wi, wd, flags, "knn batch 5 sampled")


def test_knn_backward_matches_oracle(oracle_mod):
    kb = syn.make_knn_batch(2)
    K = 8
    wi, wd, flags = oracle_mod.knn(kb.p1, kb.first1, kb.num1, kb.p2, kb.first2, kb.num2, K)
    g = syn.random_grads(wi.shape, 25)
    g1, g2 = mr.knn_bwd(cuda(kb.p1), cuda(kb.p2), cuda(wi), cuda(g))
    w1, w2 = oracle_mod.knn_bwd(kb.p1, kb.p2, wi, g)
    compare_grad(g1, w1, label="knn grad p1")
    compare_grad(g2, w2, label="knn grad p2")


@pytest.mark.parametrize("D,K", [(1, 5), (4, 32)])
def test_knn_other_dimensions(oracle_mod, D, K):
    """D = 1 and D = 4 (the widest supported), K up to 32, heterogeneous clouds."""
    rng = np.random.default_rng(20 + D)
    sizes = [700, 37, 1500, 5]
    p2 = rng.normal(size=(sum(sizes), D)).astype(np.float32)
    p1 = (p2 + 0.05 * rng.normal(size=p2.shape)).astype(np.float32)
    f = np.cumsum([0] + sizes[:-1]).astype(np.int64)
    n = np.array(sizes, np.int64)
    gi, gd = mr.knn_fwd(cuda(p1), f, n, cuda(p2), f, n, K)
    wi, wd, flags = oracle_mod.knn(p1, f, n, p2, f, n, K)
    _compare_knn(np_(gi), np_(gd), wi, wd, flags, f"knn D={D} K={K}")
    g = syn.random_grads(wi.shape, 30 + D)
    g1, g2 = mr.knn_bwd(cuda(p1), cuda(p2), cuda(wi), cuda(g))
    w1, w2 = oracle_mod.knn_bwd(p1, p2, wi, g)
    compare_grad(g1, w1, label=f"knn D={D} grad p1")
    compare_grad(g2, w2, label=f"knn D={D} grad p2")


def test_point_rasterizer_many_slots_and_dense_bins(oracle_mod):
    """K = 32 and a radius that puts thousands of points in a bin (several 256-point chunks)."""
    pb = syn.make_point_batch(2, n_clouds=3)             # the third cloud has 2562 points
    H, W, K, r = 45, 38, 32, np.float32(0.15)
    got = mr.rasterize_points_fwd(cuda(pb.points), pb.cloud_first_idx, pb.num_points_per_cloud, H, W, r, K)
    wi, wz, wd, flags = oracle_mod.rasterize_points(pb.points, pb.cloud_first_idx, pb.num_points_per_cloud, H, W,
                                                    r, K)
    assert (wi[..., -1] >= 0).mean() > 0.05              # some pixels fill all 32 slots
    _compare_slots(got, (wi, wz, wd), flags[..., None].repeat(K, -1), "K=32 dense")


def test_device_resident_cloud_arrays_match_host_ones():
    """Per-cloud index arrays given as CUDA tensors: the point rasterizer and KNN read them
    with one device-to-host copy and give identical outputs."""
    pb = syn.make_point_batch(2)
    w = pb.workload
    dev = lambda a: torch.as_tensor(np.asarray(a, np.int64)).cuda()
    P = cuda(pb.points)
    want = mr.rasterize_points_fwd(P, pb.cloud_first_idx, pb.num_points_per_cloud, w.H, w.W, w.radius, w.K)
    got = mr.rasterize_points_fwd(P, dev(pb.cloud_first_idx), dev(pb.num_points_per_cloud), w.H, w.W, w.radius, w.K)
    for x, y in zip(got, want):
        assert torch.equal(x, y)
    kb = syn.make_knn_batch(2)
    a, b = cuda(kb.p1), cuda(kb.p2)
    want = mr.knn_fwd(a, kb.first1, kb.num1, b, kb.first2, kb.num2, 8)
    got = mr.knn_fwd(a, dev(kb.first1), kb.num1, b, dev(kb.first2), dev(kb.num2), 8)
    for x, y in zip(got, want):
        assert torch.equal(x, y)


def test_knn_pair_count_is_the_work_of_the_search():
    """mr_knn_count_pairs returns the same neighbours as mr_knn_fwd and the pairs the search
    evaluated: exactly num1 x num2 when every cloud holds at most 32 references (one group,
    nothing to prune: the first group is always staged), and below the exhaustive count on
    the full-size batch, where whole groups are bounded away."""
    rng = np.random.default_rng(70)
    num1, num2 = np.array([50, 7, 0, 33]), np.array([20, 32, 5, 1])
    f1 = np.concatenate([[0], np.cumsum(num1)[:-1]])
    f2 = np.concatenate([[0], np.cumsum(num2)[:-1]])
    a = cuda(rng.normal(size=(num1.sum(), 3)).astype(np.float32))
    b = cuda(rng.normal(size=(num2.sum(), 3)).astype(np.float32))
    count, ci, cd = mr.knn_count_pairs(a, f1, num1, b, f2, num2, 4)
    gi, gd = mr.knn_fwd(a, f1, num1, b, f2, num2, 4)
    assert torch.equal(ci, gi) and torch.equal(cd, gd)
    assert count == int(np.sum(num1 * num2))
    kb = syn.make_knn_batch(5, n_clouds=8)
    A, B = cuda(kb.p1), cuda(kb.p2)
    count, ci, cd = mr.knn_count_pairs(A, kb.first1, kb.num1, B, kb.first2, kb.num2, 8)
    gi, gd = mr.knn_fwd(A, kb.first1, kb.num1, B, kb.first2, kb.num2, 8)
    assert torch.equal(ci, gi) and torch.equal(cd, gd)
    exhaustive = int(np.sum(kb.num1.astype(np.int64) * kb.num2))
    assert int(kb.p1.shape[0]) * 8 <= count < exhaustive
