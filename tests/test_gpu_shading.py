"""Parity of the CUDA stage-two shading (interpolation, soft RGB blend, their gradients)
with the float64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import differentiable_mesh_rasterization_b200 as mr
from differentiable_mesh_rasterization_b200 import synthetic as syn

from _parity import compare_grad, np_

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from differentiable_mesh_rasterization_b200 import build
    build.build()


def cuda(a, dtype=None):
    return torch.from_numpy(np.ascontiguousarray(a if dtype is None else a.astype(dtype))).cuda()


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

    o = oracle_mod.rasterize_fwd(b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, w.H, w.W,
                                 np.float32(w.blur_radius), w.K, False)
    op2f, oz, ob, od, ex = o
    ocol = oracle_mod.interpolate_fwd(op2f, ob, b.faces, vcol)
    orgba = oracle_mod.blend_fwd(op2f, ocol, od, oz, bg, **kw)
    ok = ex == 0
    err = np.abs(np_(rgba)[ok] - orgba[ok]) - (1e-4 * np.abs(orgba[ok]) + 1e-5)
    assert err.max() <= 0, f"rgba off by {err.max():.3g}"
    oc, odd, ozz = oracle_mod.blend_bwd(op2f, ocol, od, oz, bg, grad_rgba=g, **kw)
    ovcol, obary = oracle_mod.interpolate_bwd(op2f, ob, b.faces, vcol, oc)
    ogv = oracle_mod.rasterize_bwd(b.verts, b.faces, op2f, False, grad_zbuf=ozz, grad_bary=obary, grad_dists=odd)
    # vertices of faces seen in exempt pixels (either side) are left out of the comparison
    fs = np.unique(np.concatenate([op2f[~ok].reshape(-1), np_(p2f)[~ok].reshape(-1)]))
    keep = np.ones(b.verts.shape[0], bool)
    fs = fs[fs >= 0]
    keep[b.faces[fs].reshape(-1)] = False
    assert keep.mean() > 0.75
    compare_grad(np_(gvcol)[keep], ovcol[keep], label="grad vertex colours")
    compare_grad(np_(gv)[keep], ogv[keep], label="grad vertices")
