"""Pins of the oracle's stage-two shading (interpolation and soft RGB blend), CPU only.

Checked against facts fixed outside the oracle: linear precision of barycentric
interpolation (an attribute that is an affine function of the vertex position
interpolates to that function at the pixel centre), closed forms of the blend for one
face, for faces of equal colour and for an empty pixel, the silhouette channel equal
to the silhouette of step 11, and central differences for both backward passes.
"""
import numpy as np
import pytest

from differentiable_mesh_rasterization_b200 import synthetic as syn


@pytest.fixture(scope="module")
def frag(oracle_mod):
    b = syn.make_batch(2, n_meshes=3)
    H = W = 40
    out = oracle_mod.rasterize_fwd(b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, H, W,
                                   np.float32(9e-4), 4, False, exempt=False)
    return b, H, W, out


def test_interpolation_has_linear_precision(oracle_mod, frag):
    b, H, W, (p2f, zbuf, bary, dists, _) = frag
    v = b.verts.astype(np.float64)
    A = np.array([[0.3, -1.2], [2.0, 0.5], [-0.7, 0.1]])
    attr = np.stack([v[:, 0], v[:, 1], v[:, 0] * A[0, 0] + v[:, 1] * A[0, 1] + 0.25,
                     np.full(v.shape[0], 3.5)], 1)           # x, y, an affine map, a constant
    out = oracle_mod.interpolate_fwd(p2f, bary, b.faces, attr)
    jj, ii = np.meshgrid(np.arange(W), np.arange(H))
    px = -1 + (2 * jj + 1) / W
    py = 1 - (2 * ii + 1) / H
    valid = p2f >= 0
    for k in range(p2f.shape[-1]):
        m = valid[..., k]
        assert np.allclose(out[..., k, 0][m], np.broadcast_to(px, m.shape)[m], atol=1e-11)
        assert np.allclose(out[..., k, 1][m], np.broadcast_to(py, m.shape)[m], atol=1e-11)
        aff = A[0, 0] * px + A[0, 1] * py + 0.25
        assert np.allclose(out[..., k, 2][m], np.broadcast_to(aff, m.shape)[m], atol=1e-10)
        assert np.allclose(out[..., k, 3][m], 3.5, atol=1e-11)
    assert np.all(out[~valid] == 0)


def test_interpolation_backward_finite_differences(oracle_mod, frag):
    b, H, W, (p2f, zbuf, bary, dists, _) = frag
    rng = np.random.default_rng(0)
    attr = rng.normal(size=(b.verts.shape[0], 3))
    g = rng.normal(size=p2f.shape + (3,))
    ga, gb = oracle_mod.interpolate_bwd(p2f, bary, b.faces, attr, g)
    loss = lambda a, bb: np.sum(oracle_mod.interpolate_fwd(p2f, bb, b.faces, a) * g)
    h = 1e-6
    for v_, d_ in [(int(b.faces[p2f[0, 20, 20, 0], 0]), 1), (int(b.faces[p2f[1, 18, 21, 1], 2]), 0)]:
        ap, am = attr.copy(), attr.copy()
        ap[v_, d_] += h
        am[v_, d_] -= h
        assert abs((loss(ap, bary) - loss(am, bary)) / (2 * h) - ga[v_, d_]) < 1e-6
    for idx in [(0, 20, 20, 0, 1), (1, 18, 21, 1, 2)]:
        bp, bm = bary.copy(), bary.copy()
        bp[idx] += h
        bm[idx] -= h
        assert abs((loss(attr, bp) - loss(attr, bm)) / (2 * h) - gb[idx]) < 1e-6


BL = dict(sigma=1e-4, gamma=1e-4, znear=1.0, zfar=100.0)


def test_blend_closed_forms(oracle_mod):
    bg = np.array([0.1, 0.2, 0.3])
    # one face at the pixel: weight p exp((s - s)/gamma) = p against the background exp((eps - s)/gamma)
    p2f = np.array([[0, -1]])
    c = np.array([[[0.9, 0.5, 0.1], [0, 0, 0]]])
    d = np.array([[-2e-4, 0.0]])
    z = np.array([[3.0, 0.0]])
    out = oracle_mod.blend_fwd(p2f, c, d, z, bg, **BL)
    p = 1 / (1 + np.exp(-2))
    s = (100.0 - 3.0) / 99.0
    wb = np.exp((1e-10 - s) / 1e-4)
    assert np.allclose(out[0, :3], (p * c[0, 0] + wb * bg) / (p + wb), atol=1e-14)
    assert abs(out[0, 3] - p) < 1e-15
    # faces of one colour far in front of the background blend to that colour
    p2f = np.array([[0, 1, 2]])
    c = np.tile(np.array([0.4, 0.6, 0.8]), (1, 3, 1))
    out = oracle_mod.blend_fwd(p2f, c, np.array([[-1e-3, 1e-4, 3e-4]]), np.array([[2.0, 2.1, 2.05]]), bg, **BL)
    assert np.allclose(out[0, :3], [0.4, 0.6, 0.8], atol=1e-12)
    # nearer face dominates with a small gamma
    out = oracle_mod.blend_fwd(np.array([[0, 1]]), np.array([[[1., 0, 0], [0, 1., 0]]]),
                               np.array([[-1e-3, -1e-3]]), np.array([[2.0, 2.5]]), bg, **BL)
    assert out[0, 0] > 1 - 1e-9 and out[0, 1] < 1e-9
    # empty pixel: background, alpha 0
    out = oracle_mod.blend_fwd(np.array([[-1, -1]]), np.zeros((1, 2, 3)), np.zeros((1, 2)), np.zeros((1, 2)), bg,
                               **BL)
    assert np.allclose(out[0], [0.1, 0.2, 0.3, 0.0])


def test_blend_alpha_is_the_silhouette(oracle_mod, frag):
    b, H, W, (p2f, zbuf, bary, dists, _) = frag
    rng = np.random.default_rng(1)
    c = rng.uniform(size=p2f.shape + (3,))
    out = oracle_mod.blend_fwd(p2f, c, dists, zbuf, np.array([0.2, 0.2, 0.2]), sigma=1e-4, gamma=1e-2, znear=1.0,
                               zfar=10.0)
    assert np.allclose(out[..., 3], oracle_mod.silhouette_fwd(p2f, dists, 1e-4), atol=1e-15)


def test_blend_backward_finite_differences(oracle_mod):
    rng = np.random.default_rng(2)
    P, K, D = 30, 4, 3
    p2f = rng.integers(-1, 5, size=(P, K))
    c = rng.uniform(size=(P, K, D))
    d = rng.normal(0, 3e-4, size=(P, K))
    z = rng.uniform(1.5, 3.5, size=(P, K))
    bg = np.array([0.3, 0.5, 0.7])
    kw = dict(sigma=1e-4, gamma=5e-2, znear=1.0, zfar=10.0)
    g = rng.normal(size=(P, D + 1))
    gc, gd, gz = oracle_mod.blend_bwd(p2f, c, d, z, bg, grad_rgba=g, **kw)
    loss = lambda c_, d_, z_: np.sum(oracle_mod.blend_fwd(p2f, c_, d_, z_, bg, **kw) * g)
    for arr, grad, h in ((c, gc, 1e-6), (d, gd, 1e-10), (z, gz, 1e-6)):
        for _ in range(25):
            idx = tuple(rng.integers(0, s) for s in arr.shape)
            ap, am = arr.copy(), arr.copy()
            ap[idx] += h
            am[idx] -= h
            args_p = [ap if x is arr else x for x in (c, d, z)]
            args_m = [am if x is arr else x for x in (c, d, z)]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-5 * max(1.0, abs(fd)), (idx, fd, grad[idx])
    assert np.all(gc[p2f < 0] == 0) and np.all(gd[p2f < 0] == 0) and np.all(gz[p2f < 0] == 0)
