"""Parity of the CUDA backward passes (silhouette and rasterizer) with the float64 oracle."""
import numpy as np
import pytest
import torch

import differentiable_mesh_rasterization_b200 as mr
from differentiable_mesh_rasterization_b200 import synthetic as syn

from _parity import Scene, compare_alpha, compare_forward, compare_grad, np_

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from differentiable_mesh_rasterization_b200 import build
    build.build()


def cuda(a, dtype=None):
    return torch.from_numpy(np.ascontiguousarray(a if dtype is None else a.astype(dtype))).cuda()


def test_silhouette_kernels_on_seeded_slots(oracle_mod):
    rng = np.random.default_rng(21)
    sigma = np.float32(1e-4)
    for K in (1, 3, 4, 8, 16, 32):
        p2f = rng.integers(-1, 50, size=(3, 9, 11, K)).astype(np.int64)
        d = rng.normal(0, 4e-4, size=p2f.shape).astype(np.float32)
        d[..., 0] = rng.uniform(-5e-2, 1e-3, size=d.shape[:-1])      # deep interior to the blur ring
        ga = rng.normal(size=p2f.shape[:-1]).astype(np.float32)
        a = mr.silhouette_blend_fwd(cuda(p2f), cuda(d), float(sigma))
        compare_alpha(a, oracle_mod.silhouette_fwd(p2f, d, sigma), label=f"K={K}")
        gd = mr.silhouette_blend_bwd(cuda(ga), cuda(p2f), cuda(d), float(sigma))
        go = oracle_mod.silhouette_bwd(ga, p2f, d, sigma)
        compare_grad(gd, go, label=f"grad_dists K={K}")
        assert torch.all(gd[cuda(p2f) < 0] == 0)


def _oracle_chain(oracle_mod, b, p2f, dists, ga, sigma):
    gd = oracle_mod.silhouette_bwd(ga, p2f, dists, sigma)
    return oracle_mod.rasterize_bwd(b.verts, b.faces, p2f, False, grad_dists=gd)


@pytest.mark.parametrize("cfg,nm", [(2, None), (3, 2)])
def test_backward_given_the_oracle_forward(oracle_mod, cfg, nm):
    """Both sides differentiate the same slots: the oracle's pix_to_face and dists."""
    b = syn.make_batch(cfg, n_meshes=nm)
    w = b.workload
    sigma = np.float32(w.sigma)
    o = oracle_mod.rasterize_fwd(b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, w.H, w.W,
                                 np.float32(w.blur_radius), w.K, False, exempt=False)
    p2f, dists = o[0], o[3].astype(np.float32)
    ga = syn.grad_alpha(b)[:b.N]
    want = _oracle_chain(oracle_mod, b, p2f, dists.astype(np.float64), ga, sigma)
    v, f = cuda(b.verts), cuda(b.faces)
    got = mr.silhouette_rasterize_bwd(v, f, cuda(p2f), cuda(dists), float(sigma), cuda(ga))
    rel = compare_grad(got, want, label=f"fused bwd batch{cfg}")
    assert rel < 1e-4
    # unfused: silhouette bwd kernel -> general raster bwd kernel
    gd = mr.silhouette_blend_bwd(cuda(ga), cuda(p2f), cuda(dists), float(sigma))
    got2 = mr.rasterize_bwd(v, f, cuda(p2f), False, grad_dists=gd)
    compare_grad(got2, want, label=f"unfused bwd batch{cfg}")
    mr.device_status()


@pytest.mark.parametrize("persp", [False, True])
def test_general_backward_all_outputs(oracle_mod, persp):
    b = syn.make_batch(2, n_meshes=4)
    w = b.workload
    H = W = 61
    o = oracle_mod.rasterize_fwd(b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, H, W,
                                 np.float32(w.blur_radius), 5, persp, exempt=False)
    p2f = o[0]
    rng = np.random.default_rng(3 + persp)
    gz = rng.normal(size=p2f.shape).astype(np.float32)
    gb = rng.normal(size=p2f.shape + (3,)).astype(np.float32)
    gd = (rng.normal(size=p2f.shape) * 100).astype(np.float32)
    want = oracle_mod.rasterize_bwd(b.verts, b.faces, p2f, persp, gz, gb, gd)
    got = mr.rasterize_bwd(cuda(b.verts), cuda(b.faces), cuda(p2f), persp, cuda(gz), cuda(gb), cuda(gd))
    compare_grad(got, want, label=f"general bwd persp={persp}")
    for only in ("z", "b", "d"):
        args = dict(grad_zbuf=cuda(gz) if only == "z" else None, grad_bary=cuda(gb) if only == "b" else None,
                    grad_dists=cuda(gd) if only == "d" else None)
        w1 = oracle_mod.rasterize_bwd(b.verts, b.faces, p2f, persp, gz if only == "z" else None,
                                      gb if only == "b" else None, gd if only == "d" else None)
        g1 = mr.rasterize_bwd(cuda(b.verts), cuda(b.faces), cuda(p2f), persp, **args)
        compare_grad(g1, w1, label=f"general bwd only {only}")
    mr.device_status()


def test_end_to_end_batch2(oracle_mod):
    """verts -> alpha -> grad_verts on both sides from the same seeded inputs. The oracle's
    backward runs on its own fragments reconciled to the GPU's choice of faces at flagged
    pixels (the GPU's ids with the oracle's float64 values), so every vertex is compared."""
    b = syn.make_batch(2)
    w = b.workload
    sigma = np.float32(w.sigma)
    ga = syn.grad_alpha(b)
    v, f = cuda(b.verts), cuda(b.faces)
    p2f, zb, ba, dists, alpha = mr.rasterize_fwd(v, f, b.mesh_to_face_first_idx, b.num_faces_per_mesh, w.H, w.W,
                                                 w.blur_radius, w.K, sigma=float(sigma))
    got = mr.silhouette_rasterize_bwd(v, f, p2f, dists, float(sigma), cuda(ga))
    sc = Scene(oracle_mod, b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, w.H, w.W,
               w.blur_radius, w.K, False)
    info = compare_forward((p2f, zb, ba, dists), sc.fwd(), "batch2", scene=sc)
    rp2f, rd = info["rec"][0], info["rec"][3]
    want = _oracle_chain(oracle_mod, b, rp2f, rd, ga, sigma)
    rel = compare_grad(got, want, label="end-to-end batch2")
    assert rel < 1e-4
    compare_alpha(alpha, oracle_mod.silhouette_fwd(rp2f, rd, sigma), label="alpha batch2")


def test_end_to_end_full_batch5_whole_images(oracle_mod):
    """The 64-image 512x512 batch on the GPU; the oracle redoes three whole images (their
    meshes own disjoint vertex ranges, so those vertices' gradients are complete)."""
    b = syn.make_batch(5)
    w = b.workload
    sigma = np.float32(w.sigma)
    ga = syn.grad_alpha(b)
    v, f = cuda(b.verts), cuda(b.faces)
    p2f, zb, ba, dists, alpha = mr.rasterize_fwd(v, f, b.mesh_to_face_first_idx, b.num_faces_per_mesh, w.H, w.W,
                                                 w.blur_radius, w.K, sigma=float(sigma))
    got = np_(mr.silhouette_rasterize_bwd(v, f, p2f, dists, float(sigma), cuda(ga)))
    imgs = np.argsort(b.num_faces_per_mesh)[:3]
    pix = np.concatenate([np.arange(n * w.H * w.W, (n + 1) * w.H * w.W) for n in imgs])
    sc = Scene(oracle_mod, b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, w.H, w.W,
               w.blur_radius, w.K, False, pix)
    sel = lambda x: np_(x).reshape((-1,) + tuple(x.shape[3:]))[pix]
    info = compare_forward(tuple(sel(x) for x in (p2f, zb, ba, dists)), sc.fwd(), "batch5 images", scene=sc)
    P2F = np.full((b.N, w.H, w.W, w.K), -1, np.int64)
    D = np.full((b.N, w.H, w.W, w.K), -1.0)
    P2F.reshape(-1, w.K)[pix] = info["rec"][0]
    D.reshape(-1, w.K)[pix] = info["rec"][3]
    want = _oracle_chain(oracle_mod, b, P2F, D, ga, sigma)
    for n in imgs:
        v0, nv = b.mesh_to_vert_first_idx[n], b.num_verts_per_mesh[n]
        rel = compare_grad(got[v0:v0 + nv], want[v0:v0 + nv], label=f"batch5 image {n}")
        assert rel < 1e-4
    compare_alpha(np_(alpha).reshape(-1)[pix], oracle_mod.silhouette_fwd(info["rec"][0], info["rec"][3], sigma),
                  label="batch5 alpha")


@pytest.mark.parametrize("hw", [199, 256])
def test_fused_backward_vector_and_scalar_loads(oracle_mod, hw):
    """With K = 4 the fused backward reads each pixel's ids and distances in 16-byte loads
    when both arrays start on a 16-byte boundary, one by one otherwise. Both forms agree
    (up to the order of the atomics) and match the oracle's backward on the same fragments,
    with H, W a power of two (exact pixel centres) and not; at 199 x 199 the last warp
    holds 2 of its 32 pixels."""
    b = syn.make_batch(5, n_meshes=2)
    w = b.workload
    sigma = np.float32(w.sigma)
    v, f = cuda(b.verts), cuda(b.faces)
    p2f, _, _, dists, _ = mr.rasterize_fwd(v, f, b.mesh_to_face_first_idx, b.num_faces_per_mesh, hw, hw,
                                           w.blur_radius, 4, sigma=float(sigma))
    assert (p2f >= 0).sum().item() > 1000
    ga = np.random.default_rng(hw).normal(size=(b.N, hw, hw)).astype(np.float32)
    assert p2f.data_ptr() % 16 == 0 and dists.data_ptr() % 16 == 0
    got = mr.silhouette_rasterize_bwd(v, f, p2f, dists, float(sigma), cuda(ga))
    # the same contiguous arrays, 8 (ids) and 4 (distances) bytes past a 16-byte boundary
    p2f_u = torch.empty(p2f.numel() + 1, dtype=torch.int64, device="cuda")[1:].view(p2f.shape)
    d_u = torch.empty(dists.numel() + 1, dtype=torch.float32, device="cuda")[1:].view(dists.shape)
    p2f_u.copy_(p2f)
    d_u.copy_(dists)
    assert p2f_u.data_ptr() % 16 == 8 and d_u.data_ptr() % 16 == 4
    got_u = mr.silhouette_rasterize_bwd(v, f, p2f_u, d_u, float(sigma), cuda(ga))
    diff = ((got - got_u).norm() / got.norm()).item()
    assert diff < 1e-5, diff
    want = _oracle_chain(oracle_mod, b, np_(p2f), np_(dists).astype(np.float64), ga, sigma)
    assert compare_grad(got, want, label=f"fused bwd 16-byte loads {hw}px") < 1e-4
    assert compare_grad(got_u, want, label=f"fused bwd scalar loads {hw}px") < 1e-4


def test_backward_rejects_bad_slots():
    v = cuda(np.array([[-0.5, -0.5, 2.0], [0.5, -0.5, 2.0], [0.0, 0.5, 2.0]], np.float32))
    f = cuda(np.array([[0, 1, 2]], np.int64))
    p2f = torch.full((1, 4, 4, 2), -1, dtype=torch.int64, device="cuda")
    p2f[0, 1, 1, 0] = 5          # beyond F: skipped and reported
    g = torch.ones((1, 4, 4, 2), device="cuda")
    out = mr.rasterize_bwd(v, f, p2f, False, grad_dists=g)
    with pytest.raises(mr.MeshRastError) as e:
        mr.device_status()
    assert e.value.code == -4
    assert torch.all(out == 0)
    mr.device_status()           # the word was cleared
