"""Pins of the oracle's point-cloud renderer and batched KNN (steps 22-28), CPU only.

Checked against facts fixed outside the oracle: the pixels a single point covers are
the integer lattice points of a disc, with squared distances that are integers times
the squared pixel pitch; depth order, depth ties and points behind the camera on a
hand-built stack; packing clouds into one batch changes nothing; whole-pixel
translation shifts the image; closed forms of alpha and norm-weighted compositing for
one and two points; scipy's KD-tree for the K nearest neighbours of heterogeneous
clouds; a hand-solved 1-D neighbour list; and central differences for every gradient.
"""
import numpy as np
import pytest
from scipy.spatial import cKDTree

from differentiable_mesh_rasterization_b200 import synthetic as syn

H = W = 32
PITCH = 2.0 / 32


def centre(i, j):
    return -1 + (2 * j + 1) / W, 1 - (2 * i + 1) / H



def test_radius_is_inclusive(oracle_mod):
    """Step 22 keeps a point at distance exactly r (squared distance <= r^2): with r two
    pixel pitches every quantity is a dyadic rational, so the tie is exact."""
    x0, y0 = centre(10, 10)
    r = 2 * PITCH
    pts = np.array([[x0, y0, 1.0]], np.float32)
    idx, _, dists, flags = oracle_mod.rasterize_points(pts, [0], [1], H, W, r, 1)
    for i, j in ((10, 12), (10, 8), (12, 10), (8, 10)):
        assert idx[0, i, j, 0] == 0 and dists[0, i, j, 0] == r * r and flags[0, i, j]
    assert idx[0, 10, 13, 0] == -1 and idx[0, 11, 12, 0] == -1

def test_single_point_covers_a_lattice_disc(oracle_mod):
    x0, y0 = centre(13, 17)
    r = 2.5 * PITCH
    pts = np.array([[x0, y0, 1.0]], np.float32)
    idx, zbuf, dists, flags = oracle_mod.rasterize_points(pts, [0], [1], H, W, r, 2)
    covered = set()
    for a in range(-3, 4):
        for b in range(-3, 4):
            if 4 * (a * a + b * b) <= 25:          # a^2 + b^2 <= 2.5^2 in integers
                covered.add((13 + a, 17 + b))
    got = {tuple(ij) for ij in np.argwhere(idx[0, :, :, 0] == 0)}
    assert got == covered and len(covered) == 21
    for (i, j) in covered:
        a, b = i - 13, j - 17
        assert abs(dists[0, i, j, 0] - (a * a + b * b) * PITCH ** 2) < 1e-12
        assert zbuf[0, i, j, 0] == 1.0 and idx[0, i, j, 1] == -1
    assert np.all(idx[0, :, :, 1] == -1) and np.all(dists[idx < 0] == -1)
    assert not flags.any()


def test_depth_order_ties_and_points_behind(oracle_mod):
    x0, y0 = centre(5, 6)
    z = [5.0, 3.0, 4.0, 1.0, -0.5, 3.0, 2.0]
    pts = np.array([[x0, y0, zz] for zz in z], np.float32)
    idx, zbuf, _, _ = oracle_mod.rasterize_points(pts, [0], [len(z)], H, W, 0.5 * PITCH, 4)
    # nearest first; the two points at depth 3 by id; the one behind the camera never
    assert list(idx[0, 5, 6]) == [3, 6, 1, 5]
    assert list(zbuf[0, 5, 6]) == [1.0, 2.0, 3.0, 3.0]
    assert np.all(idx[0, 5, 5] == -1)


def test_packing_and_whole_pixel_translation(oracle_mod):
    pb = syn.make_point_batch(2, n_clouds=3)
    w = pb.workload
    args = (36, 40, w.radius, 4)
    idx, zbuf, dists, _ = oracle_mod.rasterize_points(pb.points, pb.cloud_first_idx, pb.num_points_per_cloud, *args)
    for n in range(3):
        f, c = pb.cloud_first_idx[n], pb.num_points_per_cloud[n]
        i1, z1, d1, _ = oracle_mod.rasterize_points(pb.points[f:f + c], [0], [c], *args)
        assert np.array_equal(np.where(i1[0] >= 0, i1[0] + f, -1), idx[n])
        assert np.array_equal(z1[0], zbuf[n]) and np.allclose(d1[0], dists[n], rtol=0, atol=1e-15)
        assert (idx[n] >= 0).sum() > 100
    # shift cloud 0 by 3 pixels right and 2 down (dyadic pitches keep it exact)
    Hs, Ws = 32, 64
    f, c = pb.cloud_first_idx[0], pb.num_points_per_cloud[0]
    p = pb.points[f:f + c].astype(np.float64) * 0.5
    a, _, da, _ = oracle_mod.rasterize_points(p.astype(np.float32), [0], [c], Hs, Ws, 0.02, 3)
    q = p + np.array([3 * 2.0 / Ws, -2 * 2.0 / Hs, 0.0])
    b, _, db, _ = oracle_mod.rasterize_points(q.astype(np.float32), [0], [c], Hs, Ws, 0.02, 3)
    assert np.array_equal(a[0, 4:-4, 4:-8], b[0, 6:-2, 7:-5])
    assert np.allclose(da[0, 4:-4, 4:-8], db[0, 6:-2, 7:-5], atol=1e-9)


def test_margin_flag(oracle_mod):
    x0, y0 = centre(10, 10)
    r = 2 * PITCH
    pts = np.array([[x0, y0 + r, 1.0]], np.float32)     # exactly r from pixel (10, 10)
    _, _, _, flags = oracle_mod.rasterize_points(pts, [0], [1], H, W, r, 2)
    assert flags[0, 10, 10]


def test_compositing_closed_forms(oracle_mod):
    r = 0.1
    f = np.array([[0.2, 0.5, 0.9], [0.7, 0.1, 0.3]])
    idx = np.array([[[[0, -1]], [[0, 1]]]], np.int64)         # (1, 2, 1, 2): two pixels
    d = np.array([[[[0.003, -1]], [[0.002, 0.006]]]])
    a0, a1 = 1 - 0.003 / r ** 2, 1 - 0.002 / r ** 2
    a2 = 1 - 0.006 / r ** 2
    out = oracle_mod.composite_points(idx, d, f, r, "alpha")
    assert np.allclose(out[0, 0, 0], a0 * f[0], atol=1e-15)
    assert np.allclose(out[0, 1, 0], a1 * f[0] + (1 - a1) * a2 * f[1], atol=1e-15)
    out = oracle_mod.composite_points(idx, d, f, r, "norm_weighted")
    assert np.allclose(out[0, 0, 0], f[0], atol=1e-15)
    assert np.allclose(out[0, 1, 0], (a1 * f[0] + a2 * f[1]) / (a1 + a2), atol=1e-15)
    same = np.stack([f[0], f[0]])
    assert np.allclose(oracle_mod.composite_points(idx, d, same, r, "norm_weighted")[0, 1, 0], f[0], atol=1e-15)
    # below the floor the weights are not normalised
    dd = np.array([[[[0.99995 * r ** 2, -1]], [[0.02, 0.02]]]])
    out = oracle_mod.composite_points(idx, dd, f, r, "norm_weighted")
    assert np.allclose(out[0, 0, 0], (1 - 0.99995) * f[0] / 1e-4, atol=1e-12)


def _fd(fun, x, i, h):
    xp, xm = x.copy(), x.copy()
    xp[i] += h
    xm[i] -= h
    return (fun(xp) - fun(xm)) / (2 * h)


@pytest.mark.parametrize("mode", ["alpha", "norm_weighted"])
def test_compositing_backward_finite_differences(oracle_mod, mode):
    pb = syn.make_point_batch(2, n_clouds=2)
    w = pb.workload
    idx, _, dists, _ = oracle_mod.rasterize_points(pb.points, pb.cloud_first_idx, pb.num_points_per_cloud, 30, 30,
                                                   w.radius, 4)
    feats = pb.features.astype(np.float64)
    rng = np.random.default_rng(0)
    g = rng.normal(size=idx.shape[:-1] + (3,))
    gf, gd = oracle_mod.composite_points_bwd(idx, dists, feats, w.radius, g, mode)
    loss_f = lambda F: float(np.sum(oracle_mod.composite_points(idx, dists, F, w.radius, mode) * g))
    loss_d = lambda D: float(np.sum(oracle_mod.composite_points(idx, D, feats, w.radius, mode) * g))
    used = np.unique(idx[idx >= 0])
    for m in used[:: max(1, len(used) // 10)]:
        for c in range(3):
            assert abs(_fd(loss_f, feats, (m, c), 1e-6) - gf[m, c]) < 1e-7
    slots = np.argwhere(idx >= 0)
    assert len(slots) > 50
    for s in slots[:: max(1, len(slots) // 20)]:
        s = tuple(s)
        assert abs(_fd(loss_d, dists, s, 1e-9) - gd[s]) < 1e-5 * (1 + abs(gd[s])), (s, gd[s])
    assert np.all(gd[idx < 0] == 0)


def test_point_rasterizer_backward_finite_differences(oracle_mod):
    pb = syn.make_point_batch(2, n_clouds=2)
    w = pb.workload
    idx, zbuf, dists, _ = oracle_mod.rasterize_points(pb.points, pb.cloud_first_idx, pb.num_points_per_cloud, 30, 30,
                                                      w.radius, 4)
    rng = np.random.default_rng(1)
    gz = rng.normal(size=idx.shape)
    gd = rng.normal(size=idx.shape)
    gp = oracle_mod.rasterize_points_bwd(pb.points, idx, gz, gd)
    # with the slot assignment held, zbuf and dists are explicit functions of the points
    jj, ii = np.meshgrid(np.arange(30), np.arange(30))
    px = (-1 + (2 * jj + 1) / 30)[None, :, :, None]
    py = (1 - (2 * ii + 1) / 30)[None, :, :, None]
    valid = idx >= 0
    safe = np.where(valid, idx, 0)

    def loss(P):
        z = P[safe, 2]
        d = (px - P[safe, 0]) ** 2 + (py - P[safe, 1]) ** 2
        return float(np.sum(np.where(valid, z * gz + d * gd, 0.0)))

    P = pb.points.astype(np.float64)
    assert np.allclose(np.where(valid, P[safe, 2], -1), zbuf)
    assert np.allclose(np.where(valid, (px - P[safe, 0]) ** 2 + (py - P[safe, 1]) ** 2, -1), dists, atol=1e-12)
    for m in np.unique(idx[valid])[::37]:
        for e in range(3):
            assert abs(_fd(loss, P, (m, e), 1e-6) - gp[m, e]) < 1e-6 * (1 + abs(gp[m, e]))


def test_knn_matches_kdtree_on_heterogeneous_clouds(oracle_mod):
    kb = syn.make_knn_batch(2, n_clouds=4)
    K = kb.workload.K
    idx, dists, flags = oracle_mod.knn(kb.p1, kb.first1, kb.num1, kb.p2, kb.first2, kb.num2, K)
    for n in range(kb.N):
        a = slice(kb.first1[n], kb.first1[n] + kb.num1[n])
        b0 = kb.first2[n]
        tree = cKDTree(kb.p2[b0:b0 + kb.num2[n]].astype(np.float64))
        d, j = tree.query(kb.p1[a].astype(np.float64), k=K)
        assert np.allclose(dists[a], d ** 2, rtol=1e-12, atol=1e-15)
        ok = ~flags[a]
        assert ok.mean() > 0.99
        assert np.array_equal(idx[a][ok], (j + b0)[ok])



@pytest.mark.parametrize("D", [1, 2, 4])
def test_knn_matches_kdtree_in_other_dimensions(oracle_mod, D):
    """Heterogeneous clouds (one query cloud empty) against scipy's KD-tree.  The tie flag is
    pinned too: a query is flagged exactly when two of its K+1 nearest KD-tree distances
    (squared) lie within 1e-6 of each other, relative to the larger."""
    rng = np.random.default_rng(40 + D)
    num1, num2 = np.array([37, 0, 64]), np.array([50, 9, 130])
    first1 = np.concatenate([[0], np.cumsum(num1)[:-1]])
    first2 = np.concatenate([[0], np.cumsum(num2)[:-1]])
    p1 = rng.normal(size=(num1.sum(), D)).astype(np.float32)
    p2 = rng.normal(size=(num2.sum(), D)).astype(np.float32)
    K = 6
    idx, dists, flags = oracle_mod.knn(p1, first1, num1, p2, first2, num2, K)
    for n in range(3):
        a = slice(first1[n], first1[n] + num1[n])
        if num1[n] == 0:
            continue
        tree = cKDTree(p2[first2[n]:first2[n] + num2[n]].astype(np.float64))
        d, j = tree.query(p1[a].astype(np.float64), k=K + 1)
        d2 = d ** 2
        assert np.allclose(dists[a], d2[:, :K], rtol=1e-12, atol=1e-15)
        # (a cloud smaller than K + 1 pads the KD-tree's answer with inf: no tie there)
        tied = (np.isfinite(d2[:, 1:]) & ((d2[:, 1:] - d2[:, :-1]) <= 1e-6 * d2[:, 1:])).any(1)
        assert np.array_equal(flags[a].astype(bool), tied)
        ok = ~flags[a]
        assert np.array_equal(idx[a][ok], (j[:, :K] + first2[n])[ok])


def test_knn_hand_solved_and_padding(oracle_mod):
    ref = np.array([[0, 0, 0], [1, 0, 0], [3, 0, 0], [6, 0, 0], [10, 0, 0]], np.float32)
    q = np.array([[2.2, 0, 0], [6, 0, 0], [0, 0, 0]], np.float32)
    idx, dists, _ = oracle_mod.knn(q, [0, 2], [2, 1], ref, [0, 3], [3, 2], 3)
    # cloud 0: queries 2.2 and 6 against 0, 1, 3; cloud 1: query 0 against 6, 10 (+ padding)
    assert idx[0].tolist() == [2, 1, 0] and np.allclose(dists[0], [0.8 ** 2, 1.2 ** 2, 2.2 ** 2], atol=1e-6)
    assert idx[1].tolist() == [2, 1, 0] and np.allclose(dists[1], [9, 25, 36])
    assert idx[2].tolist() == [3, 4, -1] and np.allclose(dists[2], [36, 100, -1])


def test_knn_invariant_under_rigid_motion(oracle_mod):
    kb = syn.make_knn_batch(2, n_clouds=2)
    rng = np.random.default_rng(2)
    R = syn.random_rotation(rng)
    t = rng.normal(size=3)
    i1, d1, f1 = oracle_mod.knn(kb.p1, kb.first1, kb.num1, kb.p2, kb.first2, kb.num2, 8)
    mv = lambda p: (p.astype(np.float64) @ R.T + t).astype(np.float32)
    i2, d2, f2 = oracle_mod.knn(mv(kb.p1), kb.first1, kb.num1, mv(kb.p2), kb.first2, kb.num2, 8)
    assert np.allclose(d1, d2, rtol=1e-4, atol=1e-8)       # float32 rounding of the moved points
    ok = ~(f1 | f2)
    assert np.mean(np.all(i1 == i2, axis=1)[ok]) > 0.99


def test_knn_backward_finite_differences(oracle_mod):
    kb = syn.make_knn_batch(2, n_clouds=1)
    idx, dists, _ = oracle_mod.knn(kb.p1, kb.first1, kb.num1, kb.p2, kb.first2, kb.num2, 4)
    rng = np.random.default_rng(3)
    g = rng.normal(size=dists.shape)
    g1, g2 = oracle_mod.knn_bwd(kb.p1, kb.p2, idx, g)
    A, B = kb.p1.astype(np.float64), kb.p2.astype(np.float64)

    def loss(A_, B_):
        return float(np.sum(((A_[:, None, :] - B_[idx]) ** 2).sum(-1) * g))

    assert np.allclose(((A[:, None, :] - B[idx]) ** 2).sum(-1), dists, rtol=1e-9, atol=1e-14)
    for i in range(0, A.shape[0], 97):
        for e in range(3):
            assert abs(_fd(lambda t: loss(t, B), A, (i, e), 1e-6) - g1[i, e]) < 1e-6
    for j in np.unique(idx)[::53]:
        for e in range(3):
            assert abs(_fd(lambda t: loss(A, t), B, (j, e), 1e-6) - g2[j, e]) < 1e-6


def test_knn_flags_a_tie_at_the_kth_neighbour(oracle_mod):
    ref = np.array([[1, 0, 0], [0, 2, 0], [0, 0, 3], [0, -3, 0], [5, 0, 0]], np.float32)
    q = np.zeros((1, 3), np.float32)
    _, d, flags = oracle_mod.knn(q, [0], [1], ref, [0], [5], 3)
    assert flags[0] and np.allclose(d[0], [1, 4, 9])
    _, _, flags = oracle_mod.knn(q, [0], [1], ref, [0], [5], 2)
    assert not flags[0]
