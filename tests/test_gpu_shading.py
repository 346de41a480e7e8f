"""Parity of the CUDA stage-two shading (interpolation, soft RGB blend, their gradients)
with the float64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import differentiable_mesh_rasterization_b200 as mr
from differentiable_mesh_rasterization_b200 import synthetic as syn

from _parity import Scene, compare_forward, compare_grad, np_

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from differentiable_mesh_rasterization_b200 import build
    build.build()


def cuda(a, dtype=None):
    return torch.from_numpy(np.ascontiguousarray(a if dtype is None else a.astype(dtype))).cuda()


def reconciled(oracle_mod, b, frags, H, W, blur, K, pixels=None):
    """The GPU fragments checked against the oracle's, and the oracle's fragments reconciled
    to the GPU's choice of faces at depth-tie and candidacy-margin pixels (the GPU's ids, the
    oracle's float64 values): the oracle's chain then runs on the same faces everywhere."""
    sc = Scene(oracle_mod, b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, H, W, blur, K, False,
               pixels)
    g = frags if pixels is None else tuple(np_(x).reshape((-1,) + tuple(x.shape[3:]))[pixels] for x in frags)
    return compare_forward(g, sc.fwd(), "fragments", scene=sc)["rec"]


@pytest.fixture(scope="module")
def frags(oracle_mod):
    """The oracle's fragments of batch 2 (8 icospheres, 137x137, K=8), rounded to float32."""
    b = syn.make_batch(2)
    w = b.workload
    o = oracle_mod.rasterize_fwd(b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, w.H, w.W,
                                 np.float32(w.blur_radius), w.K, False)
    p2f, zbuf, bary, dists, ex = o
    return b, p2f, zbuf.astype(np.float32), bary.astype(np.float32), dists.astype(np.float32), ex


def test_interpolation_matches_oracle(oracle_mod, frags):
    b, p2f, zbuf, bary, dists, _ = frags
    rng = np.random.default_rng(0)
    for D in (1, 3, 4):
        attr = rng.uniform(-1, 1, size=(b.verts.shape[0], D)).astype(np.float32)
        got = np_(mr.interpolate_fwd(cuda(p2f), cuda(bary), cuda(b.faces), cuda(attr)))
        want = oracle_mod.interpolate_fwd(p2f, bary, b.faces, attr)
        scale = oracle_mod.interpolate_fwd(p2f, np.abs(bary), b.faces, np.abs(attr))
        assert np.all(np.abs(got - want) <= 1e-6 + 2.0 ** -22 * scale), D
        g = rng.normal(size=got.shape).astype(np.float32)
        ga, gb = mr.interpolate_bwd(cuda(p2f), cuda(bary), cuda(b.faces), cuda(attr), cuda(g))
        wa, wb = oracle_mod.interpolate_bwd(p2f, bary, b.faces, attr, g)
        compare_grad(ga, wa, label=f"grad_attr D={D}")
        compare_grad(gb, wb, label=f"grad_bary D={D}")


@pytest.mark.parametrize("gamma", [1e-4, 1e-2])
def test_blend_matches_oracle(oracle_mod, frags, gamma):
    b, p2f, zbuf, bary, dists, _ = frags
    rng = np.random.default_rng(1)
    kw = dict(sigma=1e-4, gamma=gamma, znear=1.0, zfar=100.0)
    bg = np.array([0.2, 0.4, 0.6], np.float32)
    colors = rng.uniform(size=p2f.shape + (3,)).astype(np.float32)
    got = np_(mr.blend_fwd(cuda(p2f), cuda(colors), cuda(dists), cuda(zbuf), bg, **kw))
    want = oracle_mod.blend_fwd(p2f, colors, dists, zbuf, bg, **kw)
    err = np.abs(got - want) - (1e-4 * np.abs(want) + 1e-6)
    assert err.max() <= 0, f"rgba off by {err.max():.3g} beyond tolerance"
    g = rng.normal(size=want.shape).astype(np.float32)
    gc, gd, gz = mr.blend_bwd(cuda(p2f), cuda(colors), cuda(dists), cuda(zbuf), bg, grad_rgba=cuda(g), **kw)
    wc, wd, wz = oracle_mod.blend_bwd(p2f, colors, dists, zbuf, bg, grad_rgba=g, **kw)
    compare_grad(gc, wc, label="grad_colors")
    compare_grad(gd, wd, label="grad_dists")
    compare_grad(gz, wz, label="grad_zbuf")


def test_gouraud_render_end_to_end(oracle_mod):
    """verts, vertex colours -> fragments -> interpolated colours -> soft RGB blend -> loss,
    and back to vertex colours and screen-space vertices, against the oracle's chain."""
    b = syn.make_batch(2)
    w = b.workload
    rng = np.random.default_rng(2)
    vcol = rng.uniform(size=(b.verts.shape[0], 3)).astype(np.float32)
    bg = np.array([1.0, 1.0, 1.0], np.float32)
    kw = dict(sigma=1e-4, gamma=1e-2, znear=1.0, zfar=10.0)
    v, f = cuda(b.verts), cuda(b.faces)
    p2f, zbuf, bary, dists = mr.rasterize_fwd(v, f, b.mesh_to_face_first_idx, b.num_faces_per_mesh, w.H, w.W,
                                              w.blur_radius, w.K)
    col = mr.interpolate_fwd(p2f, bary, f, cuda(vcol))
    rgba = mr.blend_fwd(p2f, col, dists, zbuf, bg, **kw)
    g = syn.random_grads(tuple(rgba.shape), 7)
    gcol, gd, gz = mr.blend_bwd(p2f, col, dists, zbuf, bg, grad_rgba=cuda(g), **kw)
    gvcol, gbary = mr.interpolate_bwd(p2f, bary, f, cuda(vcol), gcol)
    gv = mr.rasterize_bwd(v, f, p2f, False, grad_zbuf=gz, grad_bary=gbary, grad_dists=gd)
    mr.device_status()

    op2f, oz, ob, od = reconciled(oracle_mod, b, (p2f, zbuf, bary, dists), w.H, w.W, w.blur_radius, w.K)
    ocol = oracle_mod.interpolate_fwd(op2f, ob, b.faces, vcol)
    orgba = oracle_mod.blend_fwd(op2f, ocol, od, oz, bg, **kw)
    err = np.abs(np_(rgba) - orgba) - (1e-4 * np.abs(orgba) + 1e-5)
    assert err.max() <= 0, f"rgba off by {err.max():.3g}"
    oc, odd, ozz = oracle_mod.blend_bwd(op2f, ocol, od, oz, bg, grad_rgba=g, **kw)
    ovcol, obary = oracle_mod.interpolate_bwd(op2f, ob, b.faces, vcol, oc)
    ogv = oracle_mod.rasterize_bwd(b.verts, b.faces, op2f, False, grad_zbuf=ozz, grad_bary=obary, grad_dists=odd)
    compare_grad(gvcol, ovcol, label="grad vertex colours")
    compare_grad(gv, ogv, label="grad vertices")


LIGHT = dict(light_location=[1.0, 1.5, 3.0], camera_position=[0.0, 0.0, 2.7], ambient=[0.1, 0.1, 0.15],
             diffuse=[0.6, 0.55, 0.5], specular=[0.3, 0.3, 0.3])


def _params(shininess):
    return mr.phong_params(shininess=shininess, **LIGHT)


def _light_tol(shininess):
    """Float32 rounding allowance of the lighting of one point: the attributes (below 2 in
    magnitude) are rounded once after interpolation, and the lighting magnifies an
    attribute error by at most about 1 + shininess (the specular power's slope)."""
    return 4.0 * (1.0 + shininess) * 2.0 ** -23


def _rounding_allowance(oracle_mod, p2f, bary, faces, vP, vN, vc, prm64, g):
    """What rounding the interpolated position, normal and albedo to float32 changes in the
    oracle's own lighting and gradient, slot by slot; spread to the vertices like the
    gradient itself (sum over slots of |b_m| |change|) and to grad_bary (sum over the
    attributes of |attr_m| . |change|).

    The CUDA path interpolates exactly and rounds once to float32 there.  Where the
    lighting is ill-conditioned (a blur-ring point extrapolated with barycentrics of
    magnitude ~40 to within a few hundredths of the camera or the light), that rounding
    alone moves the result beyond the relative tolerance.  Returns (per-slot colour
    change, [per-vertex change of grad P, N, c], per-slot change of grad_bary)."""
    valid = p2f >= 0
    b32 = np.asarray(bary, np.float32)
    X = [oracle_mod.interpolate_fwd(p2f, bary, faces, a)[valid] for a in (vP, vN, vc)]
    R = [oracle_mod.interpolate_fwd(p2f, b32, faces, a)[valid].astype(np.float32) for a in (vP, vN, vc)]
    gv = np.asarray(g, np.float64)[valid]
    col = np.zeros(p2f.shape + (3,))
    col[valid] = np.abs(oracle_mod.phong_fwd(*X, prm64)[0] - oracle_mod.phong_fwd(*R, prm64)[0])
    zeros = np.zeros((np.asarray(vP).shape[0], 3))
    f = np.asarray(faces)[np.where(valid, p2f, 0)]
    per_vertex, gb = [], np.zeros(p2f.shape + (3,))
    for attr, a, r in zip((vP, vN, vc), oracle_mod.phong_bwd(*X, prm64, gv), oracle_mod.phong_bwd(*R, prm64, gv)):
        sp = np.zeros(p2f.shape + (3,))
        sp[valid] = np.abs(a - r)
        per_vertex.append(oracle_mod.interpolate_bwd(p2f, np.abs(bary), faces, zeros, sp)[0])
        gb += (np.abs(np.asarray(attr, np.float64)[f]) * sp[..., None, :]).sum(-1)
    gb[~valid] = 0.0
    return col, per_vertex, gb


@pytest.mark.parametrize("shininess", [8.0, 64.0])
def test_phong_lighting_matches_oracle(oracle_mod, shininess):
    rng = np.random.default_rng(3)
    M = 100_003
    P = rng.uniform(-1, 1, size=(M, 3)).astype(np.float32)
    N = rng.normal(size=(M, 3)).astype(np.float32)
    c = rng.uniform(size=(M, 3)).astype(np.float32)
    prm = _params(shininess)
    got = np_(mr.phong_fwd(cuda(P), cuda(N), cuda(c), prm))
    want, flags = oracle_mod.phong_fwd(P, N, c, prm.astype(np.float64))
    ok = ~flags
    err = np.abs(got[ok] - want[ok]) - (1e-4 * np.abs(want[ok]) + 1e-6)
    assert err.max() <= 0, f"colours off by {err.max():.3g} beyond tolerance"
    g = rng.normal(size=(M, 3)).astype(np.float32)
    gP, gN, gc = mr.phong_bwd(cuda(P), cuda(N), cuda(c), prm, cuda(g))
    wP, wN, wc = oracle_mod.phong_bwd(P, N, c, prm.astype(np.float64), g)
    compare_grad(np_(gP)[ok], wP[ok], label="grad_points")
    compare_grad(np_(gN)[ok], wN[ok], label="grad_normals")
    compare_grad(np_(gc)[ok], wc[ok], label="grad_albedo")


def test_phong_shading_matches_oracle(oracle_mod, frags):
    b, p2f, zbuf, bary, dists, _ = frags
    rng = np.random.default_rng(4)
    alb = rng.uniform(size=(b.verts.shape[0], 3)).astype(np.float32)
    prm = _params(16.0)
    args = (b.world, b.normals, alb)
    got = np_(mr.phong_shade_fwd(cuda(p2f), cuda(bary), cuda(b.faces), *(cuda(a) for a in args), prm))
    want, flags = oracle_mod.phong_shade_fwd(p2f, bary, b.faces, *args, prm.astype(np.float64))
    ok = ~flags
    assert ok.mean() > 0.99
    g = rng.normal(size=want.shape).astype(np.float32)
    g[flags] = 0.0          # a flagged slot's switch is decided by rounding: no gradient through it
    col_a, vert_a, gb_a = _rounding_allowance(oracle_mod, p2f, bary, b.faces, *args, prm.astype(np.float64), g)
    tol = 1e-4 * np.abs(want) + 1e-6 + _light_tol(16.0) + 4.0 * col_a
    err = (np.abs(got - want) - tol)[ok]
    assert err.max() <= 0, f"colours off by {err.max():.3g} beyond tolerance"
    assert np.all(got[p2f < 0] == 0)
    outs = mr.phong_shade_bwd(cuda(p2f), cuda(bary), cuda(b.faces), *(cuda(a) for a in args), prm, cuda(g))
    wants = oracle_mod.phong_shade_bwd(p2f, bary, b.faces, *args, prm.astype(np.float64), g)
    for name, x, y, a in zip(("grad_points", "grad_normals", "grad_albedo", "grad_bary"), outs, wants,
                             vert_a + [gb_a]):
        compare_grad(x, y, label=name, extra=4.0 * a)


def test_phong_render_end_to_end(oracle_mod):
    """verts -> fragments -> per-fragment Phong colours -> soft RGB blend -> loss and back to
    the world positions, normals and albedo, and to the screen-space vertices."""
    b = syn.make_batch(2)
    w = b.workload
    rng = np.random.default_rng(5)
    alb = rng.uniform(size=(b.verts.shape[0], 3)).astype(np.float32)
    prm = _params(32.0)
    bg = np.array([0.0, 0.0, 0.0], np.float32)
    kw = dict(sigma=1e-4, gamma=1e-2, znear=1.0, zfar=10.0)
    v, f = cuda(b.verts), cuda(b.faces)
    P, N, A = cuda(b.world), cuda(b.normals), cuda(alb)
    p2f, zbuf, bary, dists = mr.rasterize_fwd(v, f, b.mesh_to_face_first_idx, b.num_faces_per_mesh, w.H, w.W,
                                              w.blur_radius, w.K)
    col = mr.phong_shade_fwd(p2f, bary, f, P, N, A, prm)
    rgba = mr.blend_fwd(p2f, col, dists, zbuf, bg, **kw)
    g = syn.random_grads(tuple(rgba.shape), 8)
    gcol, gd, gz = mr.blend_bwd(p2f, col, dists, zbuf, bg, grad_rgba=cuda(g), **kw)
    gP, gN, gA, gbary = mr.phong_shade_bwd(p2f, bary, f, P, N, A, prm, gcol)
    gv = mr.rasterize_bwd(v, f, p2f, False, grad_zbuf=gz, grad_bary=gbary, grad_dists=gd)
    mr.device_status()

    op2f, oz, ob, od = reconciled(oracle_mod, b, (p2f, zbuf, bary, dists), w.H, w.W, w.blur_radius, w.K)
    prm64 = prm.astype(np.float64)
    ocol, oflags = oracle_mod.phong_shade_fwd(op2f, ob, b.faces, b.world, b.normals, alb, prm64)
    orgba = oracle_mod.blend_fwd(op2f, ocol, od, oz, bg, **kw)
    ok = ~oflags.any(-1)          # a grazing light (|n.l| < 1e-6): the specular switch is rounding's
    oc, odd, ozz = oracle_mod.blend_bwd(op2f, ocol, od, oz, bg, grad_rgba=g, **kw)
    col_a, vert_a, gb_a = _rounding_allowance(oracle_mod, op2f, ob, b.faces, b.world, b.normals, alb, prm64, oc)
    extra = 4.0 * col_a.max(axis=(-2, -1))[..., None]
    err = (np.abs(np_(rgba) - orgba) - (1e-4 * np.abs(orgba) + 1e-5 + _light_tol(32.0) + extra))[ok]
    assert err.max() <= 0, f"rgba off by {err.max():.3g}"
    oP, oN, oA, obary = oracle_mod.phong_shade_bwd(op2f, ob, b.faces, b.world, b.normals, alb, prm64, oc)
    ogv = oracle_mod.rasterize_bwd(b.verts, b.faces, op2f, False, grad_zbuf=ozz, grad_bary=obary, grad_dists=odd)
    fs = np.unique(op2f[~ok].reshape(-1))
    keep = np.ones(b.verts.shape[0], bool)
    fs = fs[fs >= 0]
    keep[b.faces[fs].reshape(-1)] = False
    assert keep.mean() > 0.97
    for name, x, y, a in (("grad points", gP, oP, vert_a[0]), ("grad normals", gN, oN, vert_a[1]),
                          ("grad albedo", gA, oA, vert_a[2])):
        compare_grad(np_(x)[keep], y[keep], label=name, extra=4.0 * a[keep])
    # grad_bary of the ill-conditioned slots (see _rounding_allowance) reaches the screen
    # vertices through 1/area factors: their faces' vertices are left out there
    ill = gb_a.max(-1) > 1e-4 * np.sqrt(np.mean(obary ** 2))
    keep_v = keep.copy()
    keep_v[b.faces[np.unique(op2f[ill])].reshape(-1)] = False
    assert keep_v.mean() > 0.75
    compare_grad(np_(gv)[keep_v], ogv[keep_v], label="grad vertices")


def test_gouraud_lighting_at_vertices_end_to_end(oracle_mod):
    """Gouraud shading with lighting: Phong at the vertices, then interpolation and blend."""
    b = syn.make_batch(2, n_meshes=4)
    w = b.workload
    rng = np.random.default_rng(6)
    alb = rng.uniform(size=(b.verts.shape[0], 3)).astype(np.float32)
    prm = _params(8.0)
    bg = np.array([1.0, 1.0, 1.0], np.float32)
    kw = dict(sigma=1e-4, gamma=1e-2, znear=1.0, zfar=10.0)
    P, N, A = cuda(b.world), cuda(b.normals), cuda(alb)
    vcol = mr.phong_fwd(P, N, A, prm)
    o = oracle_mod.rasterize_fwd(b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, w.H, w.W,
                                 np.float32(w.blur_radius), w.K, False)
    op2f, oz, ob, od, ex = o
    p2f, zb, bb, dd = cuda(op2f), cuda(oz, np.float32), cuda(ob, np.float32), cuda(od, np.float32)
    col = mr.interpolate_fwd(p2f, bb, cuda(b.faces), vcol)
    rgba = mr.blend_fwd(p2f, col, dd, zb, bg, **kw)
    g = syn.random_grads(tuple(rgba.shape), 9)
    gcol, _, _ = mr.blend_bwd(p2f, col, dd, zb, bg, grad_rgba=cuda(g), **kw)
    gvcol, _ = mr.interpolate_bwd(p2f, bb, cuda(b.faces), vcol, gcol)
    gP, gN, gA = mr.phong_bwd(P, N, A, prm, gvcol)

    prm64 = prm.astype(np.float64)
    ovcol, vflags = oracle_mod.phong_fwd(b.world, b.normals, alb, prm64)
    ocol = oracle_mod.interpolate_fwd(op2f, ob.astype(np.float32), b.faces, ovcol)
    orgba = oracle_mod.blend_fwd(op2f, ocol, od.astype(np.float32), oz.astype(np.float32), bg, **kw)
    err = np.abs(np_(rgba) - orgba) - (1e-4 * np.abs(orgba) + 1e-5)
    assert err.max() <= 0, f"rgba off by {err.max():.3g}"
    oc, _, _ = oracle_mod.blend_bwd(op2f, ocol, od.astype(np.float32), oz.astype(np.float32), bg, grad_rgba=g, **kw)
    ogv, _ = oracle_mod.interpolate_bwd(op2f, ob.astype(np.float32), b.faces, ovcol, oc)
    oP, oN, oA = oracle_mod.phong_bwd(b.world, b.normals, alb, prm64, ogv)
    keep = ~vflags
    for name, x, y in (("grad points", gP, oP), ("grad normals", gN, oN), ("grad albedo", gA, oA)):
        compare_grad(np_(x)[keep], y[keep], label=name)


def _blend_input_allowance(oracle_mod, p2f, colors, dists, zbuf, bg, kw):
    """First-order change of the oracle's rgba under float32 rounding of its fragment inputs:
    sum_k |d rgba / d dists_k| 8u|dists_k| + |d rgba / d zbuf_k| 8u|zbuf_k| + |d rgba / d colour_k|
    8u (u = 2^-23; 8 ulps bound the GPU's rounding of a fragment).  At sigma = 1e-4 the blend
    multiplies a distance's error by up to w (1 - p) / sigma, so a float32 ulp of dists alone
    can exceed the relative tolerance."""
    u8 = 8 * 2.0 ** -23
    D = colors.shape[-1]
    allow = np.zeros(p2f.shape[:-1] + (D + 1,))
    for c in range(D + 1):
        g = np.zeros(p2f.shape[:-1] + (D + 1,))
        g[..., c] = 1.0
        gc, gd, gz = oracle_mod.blend_bwd(p2f, colors, dists, zbuf, bg, grad_rgba=g, **kw)
        allow[..., c] = (np.abs(gd) * u8 * np.abs(dists) + np.abs(gz) * u8 * np.abs(zbuf)
                         + np.abs(gc).sum(-1) * u8).sum(-1)
    return allow


def test_shading_full_size_sampled(oracle_mod):
    """The benchmark batch (64 meshes, 512x512, K=4) through the benchmark's launches:
    rasterize -> Gouraud colours -> soft RGB blend, and per-fragment Phong shading; sampled
    pixels against the oracle's chain computed from its own fragments at those pixels."""
    b = syn.make_batch(5)
    w = b.workload
    rng = np.random.default_rng(40)
    vcol = rng.uniform(size=(b.verts.shape[0], 3)).astype(np.float32)
    bg = np.array([1.0, 1.0, 1.0], np.float32)
    kw = dict(sigma=w.sigma, gamma=1e-2, znear=1.0, zfar=10.0)
    prm = _params(32.0)
    v, f = cuda(b.verts), cuda(b.faces)
    p2f, zbuf, bary, dists = mr.rasterize_fwd(v, f, b.mesh_to_face_first_idx, b.num_faces_per_mesh, w.H, w.W,
                                              w.blur_radius, w.K)
    col = mr.interpolate_fwd(p2f, bary, f, cuda(vcol))
    rgba = np_(mr.blend_fwd(p2f, col, dists, zbuf, bg, **kw)).reshape(-1, 4)
    pcol = np_(mr.phong_shade_fwd(p2f, bary, f, cuda(b.world), cuda(b.normals), cuda(vcol), prm)).reshape(-1, w.K, 3)
    mr.device_status()
    covered = np.flatnonzero((np_(p2f)[..., 0] >= 0).reshape(-1))
    pix = np.concatenate([rng.choice(covered, 1500, replace=False), rng.integers(0, b.N * w.H * w.W, 300)])
    op2f, oz, ob, od = reconciled(oracle_mod, b, (p2f, zbuf, bary, dists), w.H, w.W, w.blur_radius, w.K, pix)
    ok = np.ones(len(pix), bool)
    ocol = oracle_mod.interpolate_fwd(op2f, ob, b.faces, vcol)
    orgba = oracle_mod.blend_fwd(op2f, ocol, od, oz, bg, **kw)
    extra = 4.0 * _blend_input_allowance(oracle_mod, op2f, ocol, od, oz, bg, kw)
    err = (np.abs(rgba[pix] - orgba) - (1e-4 * np.abs(orgba) + 1e-5 + extra))[ok]
    assert err.max() <= 0, f"rgba off by {err.max():.3g}"
    opc, pflags = oracle_mod.phong_shade_fwd(op2f, ob, b.faces, b.world, b.normals, vcol, prm.astype(np.float64))
    sel = ok[:, None] & ~pflags & (op2f >= 0)
    col_a, _, _ = _rounding_allowance(oracle_mod, op2f, ob, b.faces, b.world, b.normals, vcol,
                                      prm.astype(np.float64), np.zeros(op2f.shape + (3,)))
    tol = 1e-4 * np.abs(opc) + 1e-5 + _light_tol(32.0) + 4.0 * col_a
    perr = (np.abs(pcol[pix] - opc) - tol)[sel]
    assert perr.max() <= 0, f"Phong colours off by {perr.max():.3g}"


@pytest.mark.parametrize("D", [1, 4])
def test_blend_other_channel_counts(oracle_mod, frags, D):
    """The element-wise blend path (D != 3) and a 4-channel attribute, on the oracle's fragments."""
    b, p2f, zbuf, bary, dists, _ = frags
    rng = np.random.default_rng(50 + D)
    kw = dict(sigma=1e-4, gamma=1e-2, znear=1.0, zfar=100.0)
    bg = rng.uniform(size=D).astype(np.float32)
    colors = rng.uniform(size=p2f.shape + (D,)).astype(np.float32)
    got = np_(mr.blend_fwd(cuda(p2f), cuda(colors), cuda(dists), cuda(zbuf), bg, **kw))
    want = oracle_mod.blend_fwd(p2f, colors, dists, zbuf, bg, **kw)
    assert np.all(np.abs(got - want) <= 1e-4 * np.abs(want) + 1e-6)
    g = rng.normal(size=want.shape).astype(np.float32)
    outs = mr.blend_bwd(cuda(p2f), cuda(colors), cuda(dists), cuda(zbuf), bg, grad_rgba=cuda(g), **kw)
    wants = oracle_mod.blend_bwd(p2f, colors, dists, zbuf, bg, grad_rgba=g, **kw)
    for name, x, y in zip(("grad_colors", "grad_dists", "grad_zbuf"), outs, wants):
        compare_grad(x, y, label=f"D={D} {name}")


def test_shading_on_perspective_correct_fragments(oracle_mod):
    """Interpolation and Phong shading on perspective-correct fragments with K = 16 (the
    element-wise kernels' widest slot template), against the oracle's own fragments."""
    b = syn.make_batch(3, n_meshes=2)
    H = W = 48
    o = oracle_mod.rasterize_fwd(b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, H, W,
                                 np.float32(b.workload.blur_radius), 16, True)
    p2f, bary = o[0], o[2].astype(np.float32)
    assert (p2f[..., 1] >= 0).mean() > 0.05
    rng = np.random.default_rng(60)
    attr = rng.uniform(-1, 1, size=(b.verts.shape[0], 4)).astype(np.float32)
    got = np_(mr.interpolate_fwd(cuda(p2f), cuda(bary), cuda(b.faces), cuda(attr)))
    want = oracle_mod.interpolate_fwd(p2f, bary, b.faces, attr)
    scale = oracle_mod.interpolate_fwd(p2f, np.abs(bary), b.faces, np.abs(attr))
    assert np.all(np.abs(got - want) <= 1e-6 + 2.0 ** -22 * scale)
    prm = _params(8.0)
    alb = rng.uniform(size=(b.verts.shape[0], 3)).astype(np.float32)
    pc = np_(mr.phong_shade_fwd(cuda(p2f), cuda(bary), cuda(b.faces), cuda(b.world), cuda(b.normals), cuda(alb), prm))
    wc, flags = oracle_mod.phong_shade_fwd(p2f, bary, b.faces, b.world, b.normals, alb, prm.astype(np.float64))
    col_a, _, _ = _rounding_allowance(oracle_mod, p2f, bary, b.faces, b.world, b.normals, alb,
                                      prm.astype(np.float64), np.zeros(p2f.shape + (3,)))
    tol = 1e-4 * np.abs(wc) + 1e-6 + _light_tol(8.0) + 4.0 * col_a
    assert np.all((np.abs(pc - wc) - tol)[~flags] <= 0)
