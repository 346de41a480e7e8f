"""Pins of the oracle's Phong lighting (steps 18-21), CPU only.

Checked against facts fixed outside the oracle: hand-computed values of the Phong
reflection model for a unit normal on +z with the light and the camera placed so that
the diffuse cosine and the mirror cosine are 1, 1/sqrt(2) or negative; invariance
under scaling the normal and under a rigid motion of the whole scene; linear precision
of the per-fragment interpolation (attributes affine in the screen position shade like
the affine values at the pixel centre); and central differences for both gradients.
"""
import math

import numpy as np
import pytest

from differentiable_mesh_rasterization_b200 import synthetic as syn

AMB = np.array([0.1, 0.2, 0.05])
DIF = np.array([0.7, 0.5, 0.9])
SPE = np.array([0.3, 0.25, 0.2])
SHINE = 8.0
ALB = np.array([0.5, 0.25, 1.0])


def params(oracle_mod, L, C, shininess=SHINE):
    return oracle_mod.phong_params(L, C, AMB, DIF, SPE, shininess)


def one(oracle_mod, P, N, c, prm):
    out, flags = oracle_mod.phong_fwd(np.array([P], float), np.array([N], float), np.array([c], float), prm)
    return out[0], bool(flags[0])


def test_phong_hand_values(oracle_mod):
    P, N = [0.0, 0.0, 0.0], [0.0, 0.0, 1.0]
    r2 = 1.0 / math.sqrt(2.0)
    cases = [
        # light and camera on the normal: cos = 1, mirror cosine 1
        (([0, 0, 2], [0, 0, 5]), (AMB + DIF) * ALB + SPE),
        # camera at the mirror image of the light: cos = 1/sqrt2, mirror cosine 1
        (([1, 0, 1], [-1, 0, 1]), (AMB + DIF * r2) * ALB + SPE),
        # camera on the normal: cos = 1/sqrt2, mirror cosine 1/sqrt2
        (([1, 0, 1], [0, 0, 3]), (AMB + DIF * r2) * ALB + SPE * r2 ** SHINE),
        # camera on the light's side near the surface: mirror cosine < 0, no highlight
        (([1, 0, 1], [1, 0, 1e-3]), (AMB + DIF * r2) * ALB),
        # light below the surface: ambient only
        (([0, 0, -1], [0, 0, 5]), AMB * ALB),
    ]
    for (L, C), want in cases:
        got, flag = one(oracle_mod, P, N, ALB, params(oracle_mod, L, C))
        assert np.allclose(got, want, rtol=0, atol=1e-14), (L, C, got, want)
        assert not flag


def test_phong_flags_grazing_light(oracle_mod):
    """The flag marks |cos| < 1e-6 only: the light at height h over a unit distance gives
    cos = h / sqrt(1 + h^2), flagged below h = 1e-6 and not above it."""
    for h, want in ((1e-8, True), (-5e-7, True), (5e-6, False), (1e-4, False), (-1e-3, False)):
        prm = params(oracle_mod, [1.0, 0.0, h], [0.0, 0.0, 3.0])
        _, flag = one(oracle_mod, [0, 0, 0], [0, 0, 1], ALB, prm)
        assert flag == want, h


def test_phong_invariances(oracle_mod):
    rng = np.random.default_rng(5)
    M = 200
    P = rng.uniform(-1, 1, size=(M, 3))
    N = rng.normal(size=(M, 3))
    c = rng.uniform(size=(M, 3))
    L, C = np.array([1.5, 2.0, 3.0]), np.array([0.0, 0.0, 2.7])
    base, _ = oracle_mod.phong_fwd(P, N, c, params(oracle_mod, L, C))
    scaled, _ = oracle_mod.phong_fwd(P, N * rng.uniform(0.1, 10.0, size=(M, 1)), c, params(oracle_mod, L, C))
    assert np.allclose(scaled, base, rtol=1e-12, atol=1e-13)
    R = syn.random_rotation(rng)
    t = rng.normal(size=3)
    moved, _ = oracle_mod.phong_fwd(P @ R.T + t, N @ R.T, c, params(oracle_mod, R @ L + t, R @ C + t))
    assert np.allclose(moved, base, rtol=1e-10, atol=1e-12)
    # some points must be lit, some shiny, some dark for the checks to mean anything
    amb_only = np.all(np.isclose(base, AMB * c, atol=1e-14), axis=1)
    assert 10 < amb_only.sum() < M - 10


def _fd(f, x, idx, h):
    xp, xm = x.copy(), x.copy()
    xp[idx] += h
    xm[idx] -= h
    # fourth-order central difference
    xpp, xmm = x.copy(), x.copy()
    xpp[idx] += 2 * h
    xmm[idx] -= 2 * h
    return (8 * (f(xp) - f(xm)) - (f(xpp) - f(xmm))) / (12 * h)


def test_phong_backward_finite_differences(oracle_mod):
    rng = np.random.default_rng(6)
    M = 64
    P = rng.uniform(-0.5, 0.5, size=(M, 3))
    N = rng.normal(size=(M, 3))
    c = rng.uniform(size=(M, 3))
    prm = params(oracle_mod, [1.5, 2.0, 3.0], [0.0, 0.0, 2.7])
    g = rng.normal(size=(M, 3))
    out, flags = oracle_mod.phong_fwd(P, N, c, prm)
    gP, gN, gc = oracle_mod.phong_bwd(P, N, c, prm, g)
    loss = lambda P_, N_, c_: float(np.sum(oracle_mod.phong_fwd(P_, N_, c_, prm)[0] * g))
    checked = 0
    for i in range(M):
        if flags[i]:
            continue
        for e in range(3):
            for x, gx, wrap in ((P, gP, lambda t: loss(t, N, c)), (N, gN, lambda t: loss(P, t, c)),
                                (c, gc, lambda t: loss(P, N, t))):
                fd = _fd(wrap, x, (i, e), 1e-5)
                assert abs(fd - gx[i, e]) <= 1e-6 * (1 + abs(gx[i, e])), (i, e, fd, gx[i, e])
                checked += 1
    assert checked > 500
    assert np.any(np.abs(gP) > 1e-3) and np.any(np.abs(gN) > 1e-3)


@pytest.fixture(scope="module")
def frag(oracle_mod):
    b = syn.make_batch(2, n_meshes=3)
    H = W = 40
    out = oracle_mod.rasterize_fwd(b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, H, W,
                                   np.float32(9e-4), 4, False, exempt=False)
    return b, H, W, out


def _affine_attributes(x, y):
    P = np.stack([0.8 * x + 0.1, 0.6 * y - 0.2, 0.3 * x - 0.2 * y + 0.5], -1)
    N = np.stack([0.4 * x - 0.1, -0.3 * y + 0.2, np.ones_like(x)], -1)
    c = np.stack([0.5 + 0.2 * x, 0.5 - 0.3 * y, 0.4 + 0.1 * x + 0.1 * y], -1)
    return P, N, c


def test_phong_shading_has_linear_precision(oracle_mod, frag):
    """Vertex attributes that are affine in the screen position interpolate to the affine
    values at the pixel centre, so Phong shading there equals step 18 at those values."""
    b, H, W, (p2f, zbuf, bary, dists, _) = frag
    v = b.verts.astype(np.float64)
    vP, vN, vc = _affine_attributes(v[:, 0], v[:, 1])
    prm = params(oracle_mod, [1.0, 1.5, 2.0], [0.0, 0.0, 2.7])
    got, flags = oracle_mod.phong_shade_fwd(p2f, bary, b.faces, vP, vN, vc, prm)
    jj, ii = np.meshgrid(np.arange(W), np.arange(H))
    px = -1 + (2 * jj + 1) / W
    py = 1 - (2 * ii + 1) / H
    P, N, c = _affine_attributes(px.reshape(-1), py.reshape(-1))
    want, _ = oracle_mod.phong_fwd(P, N, c, prm)
    want = want.reshape(H, W, 3)
    valid = p2f >= 0
    assert valid.sum() > 500
    for n in range(p2f.shape[0]):
        for k in range(p2f.shape[-1]):
            m = valid[n, :, :, k]
            assert np.allclose(got[n, :, :, k][m], want[m], rtol=0, atol=1e-10)
    assert np.all(got[~valid] == 0) and not np.any(flags[~valid])


def test_phong_shading_backward_finite_differences(oracle_mod, frag):
    b, H, W, (p2f, zbuf, bary, dists, _) = frag
    rng = np.random.default_rng(7)
    V = b.verts.shape[0]
    vP = b.verts.astype(np.float64) + rng.normal(scale=0.01, size=(V, 3))
    vN = rng.normal(size=(V, 3))
    vc = rng.uniform(size=(V, 3))
    prm = params(oracle_mod, [1.0, 1.5, 4.0], [0.0, 0.0, 5.0])
    g = rng.normal(size=p2f.shape + (3,))
    gP, gN, gc, gb = oracle_mod.phong_shade_bwd(p2f, bary, b.faces, vP, vN, vc, prm, g)

    def loss(P_=vP, N_=vN, c_=vc, b_=bary):
        return float(np.sum(oracle_mod.phong_shade_fwd(p2f, b_, b.faces, P_, N_, c_, prm)[0] * g))

    _, flags = oracle_mod.phong_shade_fwd(p2f, bary, b.faces, vP, vN, vc, prm)
    bad_faces = np.unique(p2f[flags])
    bad_verts = set(b.faces[bad_faces].reshape(-1).tolist()) if bad_faces.size else set()
    seen = [int(v) for v in np.unique(b.faces[np.unique(p2f[p2f >= 0])]) if int(v) not in bad_verts]
    for v_ in seen[:: max(1, len(seen) // 6)]:
        for e in range(3):
            for x, gx, kw in ((vP, gP, "P_"), (vN, gN, "N_"), (vc, gc, "c_")):
                fd = _fd(lambda t: loss(**{kw: t}), x, (v_, e), 1e-5)
                assert abs(fd - gx[v_, e]) <= 1e-6 * (1 + abs(gx[v_, e])), (kw, v_, e, fd, gx[v_, e])
    slots = np.argwhere((p2f >= 0) & ~flags)
    for idx in slots[:: max(1, len(slots) // 8)]:
        for m in range(3):
            j = tuple(idx) + (m,)
            fd = _fd(lambda t: loss(b_=t), bary, j, 1e-5)
            assert abs(fd - gb[j]) <= 1e-6 * (1 + abs(gb[j])), (j, fd, gb[j])
    assert np.all(gb[p2f < 0] == 0)
