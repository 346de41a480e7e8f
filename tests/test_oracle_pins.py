"""Pins of the float64 oracle against facts fixed outside of it (CPU only).

Every check below compares the oracle with something it does not compute itself:
closed-form barycentrics of lattice points, the Voronoi-region distance to a right
triangle, ray-plane intersection depths in 3-D, exact translation / permutation /
batching invariants, finite differences of its own forward (for the backward), and
the sigmoid closed forms of the blur radius used by the benchmark batches.
"""

import numpy as np
import pytest

from differentiable_mesh_rasterization_b200 import synthetic as syn


def centre(i, j, H, W):
    return -1.0 + (2 * j + 1) / W, 1.0 - (2 * i + 1) / H


def mesh(tris, z=None):
    """tris: list of 3x2 or 3x3 vertex lists -> (verts f32, faces, first, num) for one mesh."""
    v = []
    for t in tris:
        for p in t:
            v.append([p[0], p[1], p[2] if len(p) > 2 else (2.0 if z is None else z)])
    verts = np.array(v, np.float32)
    faces = np.arange(len(tris) * 3, dtype=np.int64).reshape(-1, 3)
    return verts, faces, np.array([0], np.int64), np.array([len(tris)], np.int64)


def idx_tri(pts, H, W, z=2.0):
    """Triangle whose vertices sit on pixel centres given as (row, col)."""
    return [[*centre(i, j, H, W), z] for i, j in pts]


# ---------------------------------------------------------------- step 1: pixel centres
@pytest.mark.parametrize("H,W,i,j", [(8, 8, 2, 5), (6, 10, 4, 1), (10, 6, 0, 5)])
def test_pixel_centre_convention(oracle_mod, H, W, i, j):
    x, y = centre(i, j, H, W)
    h = 0.3 * min(2.0 / W, 2.0 / H)
    tri = [[x - h, y - h], [x + h, y - h], [x, y + h]]
    p2f, zbuf, bary, dists, _ = oracle_mod.rasterize_fwd(*mesh([tri]), H, W, 0.0, 1)
    cov = p2f[0, :, :, 0] >= 0
    assert cov.sum() == 1 and cov[i, j]
    # row 0 is the top (y = +1 side): a pixel above has larger y
    assert centre(0, 0, H, W)[1] > centre(H - 1, 0, H, W)[1]


# ------------------------------------------------- steps 3, 4, 7: lattice barycentrics
def right_triangle_expect(H, W, L=12, o=2):
    u = np.arange(H)[:, None] - o + np.zeros((1, W))
    v = np.arange(W)[None, :] - o + np.zeros((H, 1))
    inside = (u >= 0) & (v >= 0) & (u + v <= L)
    bary = np.stack([1 - u / L - v / L, v / L, u / L], -1)
    return u, v, inside, bary


def test_right_triangle_barycentrics_closed_form(oracle_mod):
    H = W = 16
    tri = idx_tri([(2, 2), (2, 14), (14, 2)], H, W)
    p2f, zbuf, bary, dists, _ = oracle_mod.rasterize_fwd(*mesh([tri]), H, W, 0.0, 1)
    u, v, inside, eb = right_triangle_expect(H, W)
    cov = p2f[0, :, :, 0] == 0
    assert np.array_equal(cov, inside)
    assert inside.sum() == 13 * 14 // 2          # lattice points of the closed triangle
    assert np.allclose(bary[0, :, :, 0][inside], eb[inside], atol=1e-14)
    assert np.allclose(zbuf[0, :, :, 0][inside], 2.0, atol=1e-14)
    # vertices, edge midpoints and centroid
    assert np.allclose(bary[0, 2, 2, 0], [1, 0, 0]) and np.allclose(bary[0, 2, 8, 0], [0.5, 0.5, 0])
    assert np.allclose(bary[0, 8, 8, 0], [0, 0.5, 0.5]) and np.allclose(bary[0, 6, 6, 0], [1 / 3] * 3)
    # inside: dist = -(distance to the nearest side)^2
    s = 2.0 / W
    d2 = np.minimum(np.minimum(u ** 2, v ** 2), (12 - u - v) ** 2 / 2.0) * s * s
    assert np.allclose(dists[0, :, :, 0][inside], -d2[inside], atol=1e-14)
    assert np.all(p2f[0, :, :, 0][~inside] == -1)
    assert np.all(zbuf[0, :, :, 0][~inside] == -1) and np.all(dists[0, :, :, 0][~inside] == -1)
    assert np.all(bary[0, :, :, 0][~inside] == -1)


# ------------------------------------------------------ steps 5, 6, 9: blur distances
def voronoi_d2(u, v, L):
    """Squared distance from (u, v) to the triangle {u>=0, v>=0, u+v<=L} by Voronoi region."""
    if u >= 0 and v >= 0 and u + v <= L:
        return None
    if u < 0 and v < 0:
        return u * u + v * v
    if u < 0 and 0 <= v <= L:
        return u * u
    if v < 0 and 0 <= u <= L:
        return v * v
    if u >= L and u - v >= L:
        return (u - L) ** 2 + v * v
    if v >= L and v - u >= L:
        return u * u + (v - L) ** 2
    return (u + v - L) ** 2 / 2.0


@pytest.mark.parametrize("reach_px", [1.0, 2.5, 3.0])
def test_blur_distances_voronoi(oracle_mod, reach_px):
    H = W = 32
    s = 2.0 / W
    tri = idx_tri([(4, 4), (4, 16), (16, 4)], H, W)
    blur = (reach_px * s) ** 2
    p2f, zbuf, bary, dists, _ = oracle_mod.rasterize_fwd(*mesh([tri]), H, W, blur, 1)
    for i in range(H):
        for j in range(W):
            d = voronoi_d2(i - 4, j - 4, 12)
            if d is None:
                assert p2f[0, i, j, 0] == 0 and dists[0, i, j, 0] <= 0
            elif d * s * s <= blur * (1 + 1e-12):
                assert p2f[0, i, j, 0] == 0
                assert abs(dists[0, i, j, 0] - d * s * s) < 1e-14
                assert abs(bary[0, i, j, 0].sum() - 1) < 1e-13
            else:
                assert p2f[0, i, j, 0] == -1


# ---------------------------------------------------------------- step 10: depth order
def test_two_overlapping_triangles(oracle_mod):
    H = W = 16
    far = idx_tri([(2, 2), (2, 12), (12, 2)], H, W, z=2.0)
    near = idx_tri([(5, 5), (5, 15), (15, 5)], H, W, z=1.0)
    u0, v0, in0, _ = right_triangle_expect(H, W, L=10, o=2)
    u1, v1, in1, _ = right_triangle_expect(H, W, L=10, o=5)
    for order in ([far, near], [near, far]):
        fid_far, fid_near = (0, 1) if order[0] is far else (1, 0)
        for persp in (False, True):
            p2f, zbuf, _, _, ex = oracle_mod.rasterize_fwd(*mesh(order), H, W, 0.0, 2, persp)
            e0 = np.where(in1, fid_near, np.where(in0, fid_far, -1))
            e1 = np.where(in1 & in0, fid_far, -1)
            assert np.array_equal(p2f[0, :, :, 0], e0) and np.array_equal(p2f[0, :, :, 1], e1)
            assert np.allclose(zbuf[0, :, :, 0], np.where(in1, 1.0, np.where(in0, 2.0, -1.0)))
            assert not (ex & 1).any()          # no depth near-ties; edge lattice points are E2
            p1, *_ = oracle_mod.rasterize_fwd(*mesh(order), H, W, 0.0, 1, persp)
            assert np.array_equal(p1[..., 0], p2f[..., 0])


def test_stack_keeps_k_nearest(oracle_mod):
    H = W = 8
    rng = np.random.default_rng(3)
    zs = rng.permutation(np.arange(1, 8)).astype(float)
    tris = [[[-0.9, -0.9, z], [0.9, -0.9, z], [0.0, 0.9, z]] for z in zs]
    p2f, zbuf, _, _, _ = oracle_mod.rasterize_fwd(*mesh(tris), H, W, 0.0, 4)
    i, j = 4, 4
    assert np.array_equal(zbuf[0, i, j], [1, 2, 3, 4])
    assert np.array_equal(p2f[0, i, j], np.argsort(zs)[:4])


def test_degenerate_and_behind_camera_never_appear(oracle_mod):
    H = W = 16
    good = [[-0.5, -0.5, 2.0], [0.5, -0.5, 2.0], [0.0, 0.5, 2.0]]
    line = [[-0.8, -0.8, 1.0], [0.8, 0.8, 1.0], [0.0, 0.0, 1.0]]          # zero area
    behind = [[-0.9, -0.9, -1.0], [0.9, -0.9, -1.0], [0.0, 0.9, -1.0]]   # z < 0
    p2f, *_ = oracle_mod.rasterize_fwd(*mesh([line, good, behind]), H, W, 1e-3, 3)
    assert set(np.unique(p2f)) == {-1, 1}


# ----------------------------------------------------- steps 7, 8: perspective depth
def test_perspective_matches_ray_plane_intersection(oracle_mod):
    H = W = 32
    scr = np.array([[-0.45, -0.40, 2.0], [0.55, -0.25, 3.5], [0.05, 0.6, 2.6]], np.float32)
    verts, faces, first, num = scr, np.array([[0, 1, 2]], np.int64), np.array([0]), np.array([1])
    p2f, zbuf, bary, _, _ = oracle_mod.rasterize_fwd(verts, faces, first, num, H, W, 0.0, 1, True)
    s = scr.astype(np.float64)
    P = np.stack([s[:, 0] * s[:, 2], s[:, 1] * s[:, 2], s[:, 2]], 1)   # 3-D points (tan(fov/2) = 1)
    n = np.cross(P[1] - P[0], P[2] - P[0])
    M = np.vstack([P.T, np.ones(3)])
    cov = 0
    for i in range(H):
        for j in range(W):
            if p2f[0, i, j, 0] < 0:
                continue
            cov += 1
            x, y = centre(i, j, H, W)
            d = np.array([x, y, 1.0])
            t = n @ P[0] / (n @ d)
            X = t * d
            lam = np.linalg.lstsq(M, np.append(X, 1.0), rcond=None)[0]
            assert abs(zbuf[0, i, j, 0] - t) < 1e-12
            assert np.allclose(bary[0, i, j, 0], lam, atol=1e-10)
    assert cov > 50
    # the screen-affine (perspective off) depth differs visibly on this slanted face
    _, z2, _, _, _ = oracle_mod.rasterize_fwd(verts, faces, first, num, H, W, 0.0, 1, False)
    m = p2f[0, :, :, 0] >= 0
    assert np.abs(z2[0, :, :, 0][m] - zbuf[0, :, :, 0][m]).max() > 1e-2


def test_perspective_equal_depth_reduces_to_affine(oracle_mod):
    """A face of constant depth has screen-affine attributes, so both modes agree."""
    b = syn.make_batch(2, n_meshes=1)
    soup = b.verts[b.faces.reshape(-1)].copy()                 # unshared vertices
    nf = b.faces.shape[0]
    rng = np.random.default_rng(2)
    soup[:, 2] = np.repeat(rng.uniform(1.5, 3.5, nf), 3).astype(np.float32)
    faces = np.arange(3 * nf, dtype=np.int64).reshape(nf, 3)
    args = (soup, faces, np.array([0]), np.array([nf]), 40, 40, 5e-4, 3)
    a = oracle_mod.rasterize_fwd(*args, False)
    p = oracle_mod.rasterize_fwd(*args, True)
    ok = (a[4] == 0) & (p[4] == 0)
    assert ok.mean() > 0.95
    assert np.array_equal(a[0][ok], p[0][ok])
    assert np.allclose(a[2][ok], p[2][ok], atol=1e-12) and np.allclose(a[1][ok], p[1][ok], atol=1e-12)


# ---------------------------------------------------------- steps 11, 12: silhouette
def test_silhouette_closed_forms(oracle_mod):
    sigma = 1e-4
    br = syn.blur_for_sigma(sigma)
    p2f = np.array([[0, -1], [0, -1], [0, 1], [-1, -1]], np.int64)
    d = np.array([[br, -1], [-br, -1], [0.0, 0.0], [-1, -1]])
    a = oracle_mod.silhouette_fwd(p2f, d, sigma)
    assert abs(a[0] - 1e-4) < 1e-15          # weight at the blur radius is eps = 1e-4
    assert abs(a[1] - (1 - 1e-4)) < 1e-12
    assert abs(a[2] - 0.75) < 1e-15          # two faces on their edge: 1 - (1/2)^2
    assert a[3] == 0.0
    g = oracle_mod.silhouette_bwd(np.array([1.0, 2.0, 1.0, 5.0]), p2f, d, sigma)
    assert abs(g[2, 0] - (-0.5 * 0.25 / sigma)) < 1e-9     # -(1-p_other) p (1-p) / sigma
    assert abs(g[0, 0] - (-1e-4 * (1 - 1e-4) / sigma)) < 1e-12
    assert np.all(g[3] == 0) and g[0, 1] == 0


def test_silhouette_bwd_finite_difference(oracle_mod):
    rng = np.random.default_rng(0)
    sigma = 1e-4
    K = 5
    p2f = rng.integers(-1, 3, size=(64, K))
    d = rng.normal(0, 3e-4, size=(64, K))
    ga = rng.normal(size=64)
    g = oracle_mod.silhouette_bwd(ga, p2f, d, sigma)
    h = 1e-10
    for k in range(K):
        dp, dm = d.copy(), d.copy()
        dp[:, k] += h
        dm[:, k] -= h
        fd = ga * (oracle_mod.silhouette_fwd(p2f, dp, sigma) - oracle_mod.silhouette_fwd(p2f, dm, sigma)) / (2 * h)
        assert np.allclose(g[:, k], fd, rtol=1e-5, atol=1e-6 * np.abs(fd).max())


# ------------------------------------------------------------ step 13: raster backward
def _probe_loss(oracle_mod, px, py, abc, persp, gz, gb, gd):
    r = oracle_mod.probe(px, py, abc, persp)
    return gz * r["z"] + gb @ r["bary"] + gd * r["dist"], r


@pytest.mark.parametrize("persp", [False, True])
def test_raster_bwd_matches_finite_differences(oracle_mod, persp):
    """One pixel per image, one face per mesh: the per-slot gradient against central FD."""
    rng = np.random.default_rng(11 + persp)
    N = 40
    tris = []
    for _ in range(N):
        c = rng.uniform(-0.1, 0.1, 2)
        p = c + rng.uniform(-0.5, 0.5, (3, 2))
        z = rng.uniform(1.5, 3.5, 3)
        tris.append(np.concatenate([p, z[:, None]], 1))
    verts = np.concatenate(tris).astype(np.float32)
    faces = np.arange(3 * N, dtype=np.int64).reshape(N, 3)
    first = np.arange(N, dtype=np.int64)
    num = np.ones(N, np.int64)
    blur = 0.05
    p2f, zbuf, bary, dists, _ = oracle_mod.rasterize_fwd(verts, faces, first, num, 1, 1, blur, 1, persp)
    gz = rng.normal(size=(N, 1, 1, 1))
    gb = rng.normal(size=(N, 1, 1, 1, 3))
    gd = rng.normal(size=(N, 1, 1, 1))
    gv = oracle_mod.rasterize_bwd(verts, faces, p2f, persp, gz, gb, gd)
    checked = 0
    for n in range(N):
        if p2f[n, 0, 0, 0] < 0:
            assert np.all(gv[3 * n:3 * n + 3] == 0)
            continue
        abc = verts[3 * n:3 * n + 3].astype(np.float64)
        base = oracle_mod.probe(0.0, 0.0, abc, persp)
        g = (gz[n, 0, 0, 0], gb[n, 0, 0, 0], gd[n, 0, 0, 0])
        for q in range(3):
            for e in range(3):
                est, same = [], True
                for h in (2e-6, 1e-6):          # central differences + Richardson step
                    ap, am = abc.copy(), abc.copy()
                    ap[q, e] += h
                    am[q, e] -= h
                    lp, rp = _probe_loss(oracle_mod, 0, 0, ap, persp, *g)
                    lm, rm = _probe_loss(oracle_mod, 0, 0, am, persp, *g)
                    same &= all(r["inside"] == base["inside"] and r["edge"] == base["edge"] for r in (rp, rm))
                    est.append((lp - lm) / (2 * h))
                if not same:
                    continue
                fd = (4 * est[1] - est[0]) / 3
                assert abs(gv[3 * n + q, e] - fd) <= 1e-6 * max(1.0, abs(fd)), (n, q, e, gv[3 * n + q, e], fd)
                checked += 1
    assert checked > 200


def test_raster_bwd_sums_slots_over_image(oracle_mod):
    """Image-level gradient = sum over its slots of the per-slot gradients (probe FD)."""
    rng = np.random.default_rng(5)
    H = W = 12
    K = 3
    tris = [np.concatenate([rng.uniform(-0.7, 0.7, (3, 2)), rng.uniform(1.5, 3, (3, 1))], 1) for _ in range(4)]
    verts = np.concatenate(tris).astype(np.float32)
    faces = np.array([[0, 1, 2], [3, 4, 5], [6, 7, 8], [9, 10, 2]], np.int64)   # a shared vertex
    first, num = np.array([0]), np.array([4])
    p2f, *_ = oracle_mod.rasterize_fwd(verts, faces, first, num, H, W, 0.02, K)
    gd = rng.normal(size=p2f.shape)
    gb = rng.normal(size=p2f.shape + (3,))
    gv = oracle_mod.rasterize_bwd(verts, faces, p2f, False, None, gb, gd)
    expect = np.zeros((verts.shape[0], 3))
    h = 1e-6
    for i in range(H):
        for j in range(W):
            x, y = centre(i, j, H, W)
            for k in range(K):
                f = p2f[0, i, j, k]
                if f < 0:
                    continue
                abc = verts[faces[f]].astype(np.float64)
                for q in range(3):
                    for e in range(3):
                        ap, am = abc.copy(), abc.copy()
                        ap[q, e] += h
                        am[q, e] -= h
                        lp, _ = _probe_loss(oracle_mod, x, y, ap, False, 0.0, gb[0, i, j, k], gd[0, i, j, k])
                        lm, _ = _probe_loss(oracle_mod, x, y, am, False, 0.0, gb[0, i, j, k], gd[0, i, j, k])
                        expect[faces[f, q], e] += (lp - lm) / (2 * h)
    assert np.allclose(gv, expect, rtol=1e-5, atol=1e-5 * np.abs(expect).max())


# ---------------------------------------------------------------------- invariants
@pytest.fixture(scope="module")
def small_batch():
    b = syn.make_batch(2, n_meshes=3)
    return b


@pytest.mark.parametrize("persp", [False, True])
def test_invariants_on_seeded_batch(oracle_mod, small_batch, persp):
    b = small_batch
    H = W = 48
    blur = 9e-4
    p2f, zbuf, bary, dists, ex = oracle_mod.rasterize_fwd(
        b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, H, W, blur, 5, persp)
    valid = p2f >= 0
    assert valid.sum() > 1000
    assert np.allclose(bary.sum(-1)[valid], 1.0, atol=1e-10)
    zb = np.where(valid, zbuf, 1e30)
    assert np.all(np.diff(zb, axis=-1) >= 0)
    # valid slots come first
    assert np.all(valid[..., 1:] <= valid[..., :-1])
    mn = bary.min(-1)
    assert np.all(dists[valid & (mn > 1e-9)] <= 0)
    assert np.all(dists[valid & (mn < -1e-9)] > 0)
    assert np.all(np.abs(dists[valid & (dists > 0)]) <= blur)
    # faces belong to the pixel's own mesh
    for n in range(b.N):
        f = p2f[n][valid[n]]
        f0, nf = b.mesh_to_face_first_idx[n], b.num_faces_per_mesh[n]
        assert f.min() >= f0 and f.max() < f0 + nf
    assert ex.mean() < 0.02


def test_translation_by_one_pixel(oracle_mod, small_batch):
    b = small_batch
    H = W = 32
    v = b.verts.astype(np.float64)
    v[:, :2] = np.round(v[:, :2] * 2 ** 16) / 2 ** 16       # dyadic: x + 2/W stays exact
    v = v.astype(np.float32)
    vs = v.copy()
    vs[:, 0] += np.float32(2.0 / W)
    args = (b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, H, W, 6e-4, 4)
    a = oracle_mod.rasterize_fwd(v, *args)
    s = oracle_mod.rasterize_fwd(vs, *args)
    assert np.array_equal(a[0][:, :, :-1], s[0][:, :, 1:])
    for q in (1, 2):            # differences to the pixel centre are exact, so these are too
        assert np.array_equal(a[q][:, :, :-1], s[q][:, :, 1:])
    # the nearest point q = u + t (v - u) is rounded at the shifted magnitude
    assert np.allclose(a[3][:, :, :-1], s[3][:, :, 1:], rtol=0, atol=1e-15)


def test_face_permutation_relabels(oracle_mod, small_batch):
    b = small_batch
    H = W = 32
    rng = np.random.default_rng(9)
    perm = np.concatenate([f0 + rng.permutation(nf) for f0, nf in zip(b.mesh_to_face_first_idx, b.num_faces_per_mesh)])
    args = (b.mesh_to_face_first_idx, b.num_faces_per_mesh, H, W, 6e-4, 4)
    a = oracle_mod.rasterize_fwd(b.verts, b.faces, *args)
    p = oracle_mod.rasterize_fwd(b.verts, b.faces[perm], *args)
    ok = a[4] == 0
    mapped = np.where(p[0] >= 0, perm[np.maximum(p[0], 0)], -1)
    assert np.array_equal(mapped[ok], a[0][ok])
    assert np.allclose(p[1][ok], a[1][ok])


def test_batch_equals_concatenated_singles(oracle_mod, small_batch):
    b = small_batch
    H = W = 24
    full = oracle_mod.rasterize_fwd(b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, H, W, 7e-4, 3)
    for n in range(b.N):
        one = oracle_mod.rasterize_fwd(b.verts, b.faces, b.mesh_to_face_first_idx[n:n + 1],
                                       b.num_faces_per_mesh[n:n + 1], H, W, 7e-4, 3)
        for q in range(5):
            assert np.array_equal(full[q][n], one[q][0])


def test_k_prefix(oracle_mod, small_batch):
    b = small_batch
    args = (b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, 24, 24, 7e-4)
    k8 = oracle_mod.rasterize_fwd(*args, 8)
    k3 = oracle_mod.rasterize_fwd(*args, 3)
    assert np.array_equal(k8[0][..., :3], k3[0])
    assert np.array_equal(k8[1][..., :3], k3[1])


def test_pixel_list_matches_full_image(oracle_mod, small_batch):
    b = small_batch
    H = W = 20
    args = (b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, H, W, 7e-4, 4)
    full = oracle_mod.rasterize_fwd(*args)
    rng = np.random.default_rng(1)
    pix = rng.choice(b.N * H * W, size=200, replace=False)
    part = oracle_mod.rasterize_fwd(*args, pixels=pix)
    for q in range(5):
        assert np.array_equal(full[q].reshape((b.N * H * W,) + full[q].shape[3:])[pix], part[q])


def test_exempt_flags(oracle_mod):
    H = W = 8
    t = [[-0.9, -0.9], [0.9, -0.9], [0.0, 0.9]]
    close = [[*p, 2.0] for p in t], [[*p, 2.0 + 2e-7] for p in t]
    apart = [[*p, 2.0] for p in t], [[*p, 2.1] for p in t]
    _, _, _, _, ex = oracle_mod.rasterize_fwd(*mesh(list(close)), H, W, 0.0, 1)
    assert ex[0, 4, 4] & 1
    _, _, _, _, ex = oracle_mod.rasterize_fwd(*mesh(list(apart)), H, W, 0.0, 1)
    assert not ex[0, 4, 4]
    # a pixel whose squared distance equals the blur radius is marked E2
    s = 2.0 / W
    tri = idx_tri([(2, 2), (2, 6), (6, 2)], H, W)
    _, _, _, _, ex = oracle_mod.rasterize_fwd(*mesh([tri]), H, W, (1 * s) ** 2, 1)
    assert ex[0, 1, 3] & 2          # one pixel above edge (a, b)
    assert not ex[0, 4, 3]
    # hard rasterization (blur 0): a pixel centre on an edge has min w = 0 exactly, so its
    # coverage is rounding's; one a pixel inside is not
    _, _, _, _, ex = oracle_mod.rasterize_fwd(*mesh([tri]), H, W, 0.0, 1)
    assert ex[0, 2, 4] & 2 and ex[0, 4, 2] & 2 and ex[0, 4, 4] & 2      # edges ab, ca, bc
    assert not ex[0, 3, 3] and not ex[0, 0, 0]


def test_rejects_bad_arguments(oracle_mod):
    v, f, first, num = mesh([[[-0.5, -0.5], [0.5, -0.5], [0, 0.5]]])
    with pytest.raises(ValueError):
        oracle_mod.rasterize_fwd(v, f, first, num + 1, 4, 4, 0.0, 1)
    with pytest.raises(ValueError):
        oracle_mod.rasterize_fwd(v, f + 5, first, num, 4, 4, 0.0, 1)
    with pytest.raises(ValueError):
        oracle_mod.rasterize_fwd(v, f, first, num, 4, 4, -1.0, 1)
