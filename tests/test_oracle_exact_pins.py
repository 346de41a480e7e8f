"""Exact-rational pins of the float64 oracle (CPU only).

Inputs are dyadic rationals, exact in float32, so every quantity the rasterizer defines
has an exact rational value.  These tests compute those values with ``fractions.Fraction``
by routes other than the oracle's (barycentrics by solving the 3x3 affine system,
point-segment distance by the perpendicular cross product), and compare.  They also pin
the soft silhouette of an axis-aligned square and its gradient against torch float64
autograd, and the perspective depth of a face whose depth varies along x only.

Source: "Accelerating 3D Deep Learning with PyTorch3D" (method: the per-pixel K nearest
faces with barycentric coordinates, signed squared distance, blur radius and the
perspective_correct switch; the soft silhouette of the second stage).
"""
from fractions import Fraction as Fr
import math

import numpy as np
import pytest


def centre(i, j, H, W):
    return Fr(-1) + Fr(2 * j + 1, W), Fr(1) - Fr(2 * i + 1, H)


def solve3(M, r):
    """Gaussian elimination over the rationals."""
    A = [list(row) + [rv] for row, rv in zip(M, r)]
    for c in range(3):
        piv = next(k for k in range(c, 3) if A[k][c] != 0)
        A[c], A[piv] = A[piv], A[c]
        for k in range(3):
            if k != c and A[k][c] != 0:
                f = A[k][c] / A[c][c]
                A[k] = [x - f * y for x, y in zip(A[k], A[c])]
    return [A[k][3] / A[k][k] for k in range(3)]


def seg_d2(p, u, v):
    ex, ey = v[0] - u[0], v[1] - u[1]
    qx, qy = p[0] - u[0], p[1] - u[1]
    L = ex * ex + ey * ey
    s = qx * ex + qy * ey
    if s <= 0:
        return qx * qx + qy * qy
    if s >= L:
        rx, ry = p[0] - v[0], p[1] - v[1]
        return rx * rx + ry * ry
    cr = ex * qy - ey * qx
    return cr * cr / L


def exact_eval(p, tri, persp):
    """(inside, d2, bary, z) of pixel centre p against a face, all as Fractions."""
    M = [[tri[0][0], tri[1][0], tri[2][0]], [tri[0][1], tri[1][1], tri[2][1]], [1, 1, 1]]
    lam = solve3(M, [p[0], p[1], Fr(1)])
    inside = all(l >= 0 for l in lam)
    d2 = min(seg_d2(p, tri[a], tri[b]) for a, b in ((0, 1), (1, 2), (2, 0)))
    if persp:
        mu = [lam[k] / tri[k][2] for k in range(3)]
        s = sum(mu)
        bary = [m / s for m in mu]
        z = 1 / s
    else:
        bary = lam
        z = sum(lam[k] * tri[k][2] for k in range(3))
    return inside, d2, bary, z


def dyadic_triangle(rng, den=128):
    while True:
        xy = rng.integers(-den + 8, den - 8, size=(3, 2))
        z = rng.integers(den, 4 * den, size=3)
        area = (xy[1, 0] - xy[0, 0]) * (xy[2, 1] - xy[0, 1]) - (xy[2, 0] - xy[0, 0]) * (xy[1, 1] - xy[0, 1])
        if abs(area) > den * den // 16:
            return [[Fr(int(xy[k, 0]), den), Fr(int(xy[k, 1]), den), Fr(int(z[k]), den)] for k in range(3)]


def one_face(tri):
    verts = np.array([[float(c) for c in v] for v in tri], np.float32)
    assert all(Fr(float(verts[k, e])) == tri[k][e] for k in range(3) for e in range(3))
    return verts, np.array([[0, 1, 2]], np.int64), np.array([0], np.int64), np.array([1], np.int64)


@pytest.mark.parametrize("persp", [False, True])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_single_triangle_against_exact_rationals(oracle_mod, seed, persp):
    rng = np.random.default_rng(100 + seed)
    tri = dyadic_triangle(rng)
    H = W = 32
    blur = Fr(3, 1024)                        # reach of about 0.87 pixel pitches
    p2f, zbuf, bary, dists, _ = oracle_mod.rasterize_fwd(*one_face(tri), H, W, float(blur), 1, persp)
    n_in = n_ring = 0
    for i in range(H):
        for j in range(W):
            p = centre(i, j, H, W)
            inside, d2, eb, ez = exact_eval(p, tri, persp)
            if not inside and abs(d2 - blur) <= blur * Fr(1, 10 ** 9):
                continue                        # candidacy on its threshold: rounding decides
            cand = inside or d2 <= blur
            assert (p2f[0, i, j, 0] == 0) == cand, (i, j)
            if not cand:
                assert zbuf[0, i, j, 0] == -1 and dists[0, i, j, 0] == -1
                continue
            n_in += inside
            n_ring += not inside
            sd = -d2 if inside else d2
            assert abs(dists[0, i, j, 0] - float(sd)) <= 1e-15 + 1e-13 * float(d2)
            assert abs(zbuf[0, i, j, 0] - float(ez)) <= 1e-13 * float(ez)
            scale = max(1.0, max(abs(float(b)) for b in eb))
            for k in range(3):
                assert abs(bary[0, i, j, 0, k] - float(eb[k])) <= 1e-13 * scale
            assert abs(bary[0, i, j, 0].sum() - 1.0) <= 1e-12
            assert (bary[0, i, j, 0].min() >= 0) == inside
    assert n_in > 20 and n_ring > 10


def test_perspective_depth_varying_along_x_only(oracle_mod):
    """Vertex depths 1/z = alpha + beta x make 1/z affine in x alone, so z(p) = 1/(alpha + beta px)."""
    alpha, beta = Fr(1, 2), Fr(1, 4)
    xy = [(Fr(-3, 4), Fr(-5, 8)), (Fr(3, 4), Fr(-1, 2)), (Fr(-1, 8), Fr(3, 4))]
    z = [1 / (alpha + beta * x) for x, _ in xy]          # not dyadic: float32 rounds them
    verts = np.array([[float(x), float(y), float(zk)] for (x, y), zk in zip(xy, z)], np.float64)
    H = W = 32
    p2f, zbuf, _, _, _ = oracle_mod.rasterize_fwd(
        verts.astype(np.float32), np.array([[0, 1, 2]]), np.array([0]), np.array([1]), H, W, 0.0, 1, True)
    zf = verts[:, 2].astype(np.float32).astype(np.float64)      # the depths the oracle sees
    # with the float32-rounded depths 1/z is still affine in screen space; take it exactly
    xyf = [(Fr(float(x)), Fr(float(y))) for x, y in xy]
    inv = [1 / Fr(float(v)) for v in zf]
    M = [[x for x, _ in xyf], [y for _, y in xyf], [1, 1, 1]]
    n = 0
    for i in range(H):
        for j in range(W):
            if p2f[0, i, j, 0] < 0:
                continue
            px, py = centre(i, j, H, W)
            lam = solve3(M, [px, py, Fr(1)])
            zz = 1 / sum(l * q for l, q in zip(lam, inv))
            assert abs(zbuf[0, i, j, 0] - float(zz)) <= 1e-13 * float(zz)
            # and the closed form of the unrounded mesh, to float32 depth rounding
            assert abs(zbuf[0, i, j, 0] - 1.0 / float(alpha + beta * px)) <= 1e-6
            n += 1
    assert n > 100


# ------------------------------------------------------------- axis-aligned square
def square_mesh(lo, hi, z=2.0):
    v = np.array([[lo, lo, z], [hi, lo, z], [hi, hi, z], [lo, hi, z]], np.float32)
    f = np.array([[0, 1, 2], [0, 2, 3]], np.int64)
    return v, f, np.array([0], np.int64), np.array([2], np.int64)


def test_square_hard_coverage_count(oracle_mod):
    H = W = 64
    lo, hi = -0.5, 0.25                     # both edges between pixel centres (centres are odd/64)
    p2f, _, _, dists, _ = oracle_mod.rasterize_fwd(*square_mesh(lo, hi), H, W, 0.0, 2)
    xs = [-1 + (2 * j + 1) / W for j in range(W)]
    n_cols = sum(lo <= x <= hi for x in xs)
    n_rows = sum(lo <= y <= hi for y in xs)
    cov = (p2f[0, :, :, 0] >= 0)
    assert cov.sum() == n_cols * n_rows == 24 * 24
    a = oracle_mod.silhouette_fwd(p2f, dists, 1e-4)[0]
    assert np.all(a[~cov] == 0) and np.all(a[cov] > 0.5)


def test_square_soft_silhouette_exact(oracle_mod):
    H = W = 64
    lo, hi = Fr(-1, 2), Fr(1, 4)
    sigma = 1e-4
    blur = Fr(1, 256)                        # sqrt(blur) = 1/16 = two pixel pitches
    p2f, zbuf, bary, dists, _ = oracle_mod.rasterize_fwd(*square_mesh(float(lo), float(hi)), H, W, float(blur), 2)
    alpha = oracle_mod.silhouette_fwd(p2f, dists, sigma)[0]
    V = [(lo, lo), (hi, lo), (hi, hi), (lo, hi)]
    tris = [[V[0], V[1], V[2]], [V[0], V[2], V[3]]]
    counts = {"out": 0, "ring": 0, "in": 0}
    for i in range(H):
        for j in range(W):
            p = centre(i, j, H, W)
            terms = []
            for t in tris:
                tz = [(x, y, Fr(2)) for x, y in t]
                inside, d2, _, _ = exact_eval(p, tz, False)
                if inside or d2 <= blur:
                    terms.append(float(-d2 if inside else d2))
            if not terms:
                counts["out"] += 1
                assert alpha[i, j] == 0 and p2f[0, i, j, 0] == -1
                continue
            counts["in" if min(terms) <= 0 else "ring"] += 1
            expect = 1.0 - math.prod(1.0 - 1.0 / (1.0 + math.exp(d / sigma)) for d in terms)
            assert abs(alpha[i, j] - expect) <= 1e-12, (i, j, alpha[i, j], expect)
            assert sorted(dists[0, i, j][p2f[0, i, j] >= 0]) == pytest.approx(sorted(terms), abs=1e-15)
    assert counts["ring"] > 50 and counts["in"] > 400 and counts["out"] > 2000


def test_silhouette_bwd_matches_torch_autograd(oracle_mod):
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(4)
    sigma = 2e-4
    P, K = 200, 6
    p2f = rng.integers(-1, 5, size=(P, K))
    d = rng.normal(0, 5e-4, size=(P, K))
    ga = rng.normal(size=P)
    dt = torch.tensor(d, dtype=torch.float64, requires_grad=True)
    valid = torch.tensor(p2f >= 0)
    p = torch.sigmoid(-dt / sigma)
    alpha = 1 - torch.where(valid, 1 - p, torch.ones_like(p)).prod(-1)
    (alpha * torch.tensor(ga)).sum().backward()
    g = oracle_mod.silhouette_bwd(ga, p2f, d, sigma)
    assert np.allclose(oracle_mod.silhouette_fwd(p2f, d, sigma), alpha.detach().numpy(), rtol=0, atol=1e-14)
    ref = dt.grad.numpy()
    assert np.allclose(g, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    assert np.all(g[p2f < 0] == 0)


def test_closed_triangle_counts_its_boundary_as_inside(oracle_mod):
    """Step 4 takes the closed triangle: vertices and edge points are inside."""
    tri = np.array([[-0.5, -0.5, 2.0], [0.5, -0.5, 2.0], [0.0, 0.5, 2.0]], np.float64)
    for px, py in ((-0.5, -0.5), (0.0, -0.5), (0.25, 0.0), (-0.25, 0.0), (0.0, 0.0)):
        r = oracle_mod.probe(px, py, tri, False)
        assert r["inside"], (px, py)
    for px, py in ((0.0, -0.5 - 2.0 ** -20), (0.5, 0.0)):
        assert not oracle_mod.probe(px, py, tri, False)["inside"]


@pytest.mark.parametrize("persp", [False, True])
def test_equal_depth_ties_go_to_the_lower_face_id(oracle_mod, persp):
    """Step 10 orders by (z, face id): copies of one face tie exactly in depth."""
    H = W = 16
    tri = [[-0.7, -0.6, 2.0], [0.6, -0.5, 2.5], [0.0, 0.7, 3.0]]
    far = [[-0.7, -0.6, 4.0], [0.6, -0.5, 4.0], [0.0, 0.7, 4.0]]
    verts = np.array(far + tri + tri + tri, np.float32)           # faces 0 (behind), 1, 2, 3 (copies)
    faces = np.arange(12, dtype=np.int64).reshape(4, 3)
    p2f, zbuf, _, _, ex = oracle_mod.rasterize_fwd(verts, faces, np.array([0]), np.array([4]), H, W, 0.0, 4,
                                                   persp, exempt=False)
    cov = p2f[0, :, :, 0] >= 0
    assert cov.sum() > 50
    assert np.all(p2f[0][cov] == [1, 2, 3, 0])
    assert np.all(zbuf[0][cov][:, 0] == zbuf[0][cov][:, 2])
    one, *_ = oracle_mod.rasterize_fwd(verts, faces[::-1].copy(), np.array([0]), np.array([4]), H, W, 0.0, 2,
                                       persp, exempt=False)
    # reversed face order: the copies are now faces 0, 1, 2 and the far face is 3
    assert np.all(one[0][cov] == [0, 1])
