"""Parity of the CUDA forward (stage one + fused silhouette) with the float64 oracle.

Every GPU call goes through the C ABI (via the ctypes binding).  Small cases are
compared on every pixel; the full benchmark batches on seeded pixel samples.
"""
import numpy as np
import pytest
import torch

import differentiable_mesh_rasterization_b200 as mr
from differentiable_mesh_rasterization_b200 import synthetic as syn

from _parity import Scene, compare_alpha, compare_forward, np_, sample_pixels

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from differentiable_mesh_rasterization_b200 import build
    build.build()


def to_dev(verts, faces):
    return torch.from_numpy(np.ascontiguousarray(verts, np.float32)).cuda(), \
        torch.from_numpy(np.ascontiguousarray(faces, np.int64)).cuda()


def run_both(oracle_mod, verts, faces, first, num, H, W, blur, K, persp, pixels=None, sigma=None):
    """The CUDA forward and the oracle on the same inputs; returns (gpu, oracle, scene)."""
    v, f = to_dev(verts, faces)
    g = mr.rasterize_fwd(v, f, first, num, H, W, blur, K, persp, sigma=sigma)
    torch.cuda.synchronize()
    scene = Scene(oracle_mod, verts, faces, first, num, H, W, blur, K, persp, pixels)
    o = scene.fwd()
    if pixels is not None:
        N = len(first)
        g = tuple(np_(x).reshape((N * H * W,) + tuple(x.shape[3:]))[pixels] for x in g)
    return g, o, scene


def alpha_of(oracle_mod, info, sigma):
    """The oracle's silhouette of the GPU's choice of faces (reconciled at flagged pixels)."""
    rec = info["rec"]
    return oracle_mod.silhouette_fwd(rec[0], rec[3], np.float32(sigma))


def centre(i, j, H, W):
    return -1.0 + (2 * j + 1) / W, 1.0 - (2 * i + 1) / H


def soup(tris):
    v = np.array([p for t in tris for p in t], np.float32)
    return v, np.arange(len(v), dtype=np.int64).reshape(-1, 3)


# ---------------------------------------------------------------- hand-made cases
def test_right_triangle_hard_and_blur(oracle_mod):
    H = W = 32
    tri = [[*centre(4, 4, H, W), 2.0], [*centre(4, 16, H, W), 2.5], [*centre(16, 4, H, W), 3.0]]
    v, f = soup([tri])
    for blur in (0.0, (2.5 * 2 / W) ** 2):
        for persp in (False, True):
            g, o, sc = run_both(oracle_mod, v, f, [0], [1], H, W, blur, 1, persp)
            # the vertices sit on pixel centres, so whole edges run through centres: the
            # candidacy of those pixels is rounding's by construction (E2)
            compare_forward(g, o, f"blur={blur} persp={persp}", scene=sc, e2_max=0.2)


def test_overlap_stack_and_k_beyond_candidates(oracle_mod):
    H = W = 24
    rng = np.random.default_rng(4)
    tris = []
    for z in rng.permutation(np.arange(1, 7)):
        c = rng.uniform(-0.3, 0.3, 2)
        tris.append([[c[0] - 0.6, c[1] - 0.5, z], [c[0] + 0.6, c[1] - 0.4, z + 0.3], [c[0], c[1] + 0.7, z - 0.2]])
    v, f = soup(tris)
    for K in (1, 3, 4, 8, 32):
        g, o, sc = run_both(oracle_mod, v, f, [0], [len(tris)], H, W, 4e-3, K, False)
        compare_forward(g, o, f"K={K}", scene=sc)


def test_degenerate_behind_camera_and_empty_meshes(oracle_mod):
    H, W = 20, 36          # non-square, ragged in both directions
    good = [[-0.5, -0.5, 2.0], [0.5, -0.5, 2.0], [0.0, 0.5, 2.0]]
    line = [[-0.8, -0.8, 1.0], [0.8, 0.8, 1.0], [0.0, 0.0, 1.0]]
    behind = [[-0.9, -0.9, -1.0], [0.9, -0.9, -1.0], [0.0, 0.9, -1.0]]
    offscreen = [[3.0, 3.0, 2.0], [4.0, 3.0, 2.0], [3.5, 4.0, 2.0]]
    v, f = soup([line, good, behind, offscreen])
    first, num = [0, 4, 1], [4, 0, 2]     # mesh 1 is empty, mesh 2 re-uses faces 1..2
    g, o, sc = run_both(oracle_mod, v, f, first, num, H, W, 1e-3, 3, False)
    compare_forward(g, o, "mixed", scene=sc)
    assert np.all(np_(g[0])[1] == -1)
    assert set(np.unique(np_(g[0]))) <= {-1, 1}



@pytest.mark.parametrize("persp", [False, True])
def test_exact_depth_ties_go_to_the_lower_face_id(oracle_mod, persp):
    """Copies of one face tie exactly in depth (identical constants on both sides): the
    order is by face id, as in the oracle, at every covered pixel."""
    H = W = 32
    tri = [[-0.7, -0.6, 2.0], [0.6, -0.5, 2.5], [0.0, 0.7, 3.0]]
    far = [[-0.7, -0.6, 4.0], [0.6, -0.5, 4.0], [0.0, 0.7, 4.0]]
    v, f = soup([far, tri, tri, tri])
    dv, df = to_dev(v, f)
    g = np_(mr.rasterize_fwd(dv, df, [0], [4], H, W, 0.0, 4, persp)[0])
    o, _, _, _, ex = oracle_mod.rasterize_fwd(v, f, [0], [4], H, W, 0.0, 4, persp)
    cov = o[0, :, :, 0] >= 0
    assert cov.sum() > 150
    assert np.all(o[0][cov] == [1, 2, 3, 0])
    # every covered pixel is a depth tie (E1) by construction; only pixels whose coverage
    # rounding decides (E2: a pixel centre within 1e-6 of an edge) are left out
    ok = (ex & 2) == 0
    assert ok.mean() > 0.99
    assert np.array_equal(g[ok], o[ok])


@pytest.mark.parametrize("H,W", [(1, 3000), (3000, 1), (7, 4099)])
def test_extreme_aspect_ratios(oracle_mod, H, W):
    """Single-row and single-column images and a ragged wide one: one bin row or column,
    partial warp tiles along the short side, non-power-of-two centres (float-pair path)."""
    b = syn.make_batch(2, n_meshes=2)
    g, o, sc = run_both(oracle_mod, b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, H, W,
                        2e-3, 4, False, sigma=1e-4)
    info = compare_forward(g[:4], o, f"{H}x{W}", scene=sc)
    assert info["valid_slots"] > 100
    compare_alpha(g[4], alpha_of(oracle_mod, info, 1e-4), label=f"{H}x{W} alpha")


def test_no_faces_at_all():
    v = torch.zeros((0, 3), device="cuda")
    f = torch.zeros((0, 3), dtype=torch.int64, device="cuda")
    p2f, zbuf, bary, dists, alpha = mr.rasterize_fwd(v, f, [0, 0], [0, 0], 17, 33, 1e-3, 2, sigma=1e-4)
    assert torch.all(p2f == -1) and torch.all(zbuf == -1) and torch.all(bary == -1) and torch.all(dists == -1)
    assert torch.all(alpha == 0)


@pytest.mark.parametrize("H,W,K", [(64, 64, 4), (48, 80, 4), (37, 53, 2), (64, 64, 3)])
def test_every_output_element_is_written(H, W, K):
    """Outputs pre-filled with a sentinel: a small triangle leaves most 16 x 16 bins empty
    (the fine pass skips those and the epilogue pads them) and the rest partly covered; the
    vector path (K = 4, H and W multiples of 16) and the general one both write every
    element, and the results equal a call into fresh buffers."""
    v, f = to_dev(*soup([[[-0.2, -0.1, 2.0], [0.15, -0.2, 2.1], [0.0, 0.25, 2.2]]]))
    lib = mr.load_library()
    ref = mr.rasterize_fwd(v, f, [0], [1], H, W, 2e-3, K, sigma=1e-4)
    p2f = torch.full((1, H, W, K), 123456, dtype=torch.int64, device="cuda")
    zbuf, dists = (torch.full((1, H, W, K), 7.5, device="cuda") for _ in range(2))
    bary = torch.full((1, H, W, K, 3), 7.5, device="cuda")
    alpha = torch.full((1, H, W), 7.5, device="cuda")
    first, num = np.array([0], np.int64), np.array([1], np.int64)
    rc = lib.mr_rasterize_silhouette_fwd(v.data_ptr(), v.shape[0], f.data_ptr(), f.shape[0], first.ctypes.data,
                                         num.ctypes.data, 1, H, W, 2e-3, K, 0, 1e-4, p2f.data_ptr(),
                                         zbuf.data_ptr(), bary.data_ptr(), dists.data_ptr(), alpha.data_ptr(),
                                         torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == 0
    for got, want in zip((p2f, zbuf, bary, dists, alpha), ref):
        assert torch.equal(got, want)
    assert (ref[0] >= 0).any() and (ref[0][..., 0] == -1).float().mean() > 0.5


def test_face_covering_the_whole_image_and_crowded_bin(oracle_mod):
    H = W = 64
    big = [[-3.0, -3.0, 2.5], [3.0, -3.0, 2.5], [0.0, 3.0, 2.6]]
    rng = np.random.default_rng(8)
    tiny = []
    for _ in range(600):                       # hundreds of faces inside one 16x16 bin
        c = rng.uniform(-0.45, -0.05, 2)
        z = rng.uniform(1.5, 3.0)
        tiny.append([[c[0], c[1], z], [c[0] + 0.02, c[1], z + 0.01], [c[0], c[1] + 0.02, z - 0.01]])
    v, f = soup([big] + tiny)
    g, o, sc = run_both(oracle_mod, v, f, [0], [len(tiny) + 1], H, W, 2e-4, 8, False)
    compare_forward(g, o, "big+crowded", scene=sc)


def test_invalid_vertex_index_is_reported():
    v, f = to_dev(*soup([[[-0.5, -0.5, 2.0], [0.5, -0.5, 2.0], [0.0, 0.5, 2.0]]]))
    f[0, 1] = 7    # outside [0, V): the kernel skips the face and reports it
    with pytest.raises(mr.MeshRastError) as e:
        mr.rasterize_fwd(v, f, [0], [1], 8, 8, 0.0, 1)
    assert e.value.code == -4


def test_deterministic_and_stream_aware(oracle_mod):
    b = syn.make_batch(2, n_meshes=3)
    w = b.workload
    v, f = to_dev(b.verts, b.faces)
    a = mr.rasterize_fwd(v, f, b.mesh_to_face_first_idx, b.num_faces_per_mesh, w.H, w.W, w.blur_radius, w.K)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        c = mr.rasterize_fwd(v, f, b.mesh_to_face_first_idx, b.num_faces_per_mesh, w.H, w.W, w.blur_radius, w.K)
    s.synchronize()
    for x, y in zip(a, c):
        assert torch.equal(x, y)


# ---------------------------------------------------------------- benchmark batches
def test_batch1_full(oracle_mod):
    b = syn.make_batch(1)
    w = b.workload
    g, o, sc = run_both(oracle_mod, b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, w.H, w.W,
                        w.blur_radius, w.K, w.perspective_correct)
    compare_forward(g, o, "batch1", scene=sc)


@pytest.mark.parametrize("persp", [False, True])
def test_batch2_full_with_silhouette(oracle_mod, persp):
    b = syn.make_batch(2)
    w = b.workload
    v, f = to_dev(b.verts, b.faces)
    g = mr.rasterize_fwd(v, f, b.mesh_to_face_first_idx, b.num_faces_per_mesh, w.H, w.W, w.blur_radius, w.K,
                         persp, sigma=w.sigma)
    sc = Scene(oracle_mod, b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, w.H, w.W,
               w.blur_radius, w.K, persp)
    info = compare_forward(g[:4], sc.fwd(), "batch2", scene=sc)
    assert info["valid_slots"] > 100000
    assert info["e1"] > 0          # the tie rule is exercised, not skipped
    compare_alpha(g[4], alpha_of(oracle_mod, info, w.sigma), label="batch2 alpha")
    # the stand-alone silhouette kernel reproduces the fused epilogue bit for bit
    a2 = mr.silhouette_blend_fwd(g[0], g[3], w.sigma)
    assert torch.equal(a2, g[4])


def test_batch3_two_meshes_full(oracle_mod):
    b = syn.make_batch(3, n_meshes=2)
    w = b.workload
    g, o, sc = run_both(oracle_mod, b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, w.H, w.W,
                        w.blur_radius, w.K, w.perspective_correct, sigma=w.sigma)
    info = compare_forward(g[:4], o, "batch3[:2]", scene=sc)
    compare_alpha(g[4], alpha_of(oracle_mod, info, w.sigma), label="batch3[:2] alpha")


@pytest.mark.parametrize("cfg,per_image", [(3, 150), (4, 2500), (5, 40)])
def test_full_batch_sampled(oracle_mod, cfg, per_image):
    """Full benchmark batch on the GPU in its benchmark launch (fused silhouette);
    seeded pixel samples recomputed one by one by the oracle."""
    b = syn.make_batch(cfg)
    w = b.workload
    v, f = to_dev(b.verts, b.faces)
    sig = w.sigma
    out = mr.rasterize_fwd(v, f, b.mesh_to_face_first_idx, b.num_faces_per_mesh, w.H, w.W, w.blur_radius, w.K,
                           w.perspective_correct, sigma=sig)
    pix = sample_pixels(b, per_image, seed=cfg)
    N = b.N
    g = tuple(np_(x).reshape((N * w.H * w.W,) + tuple(x.shape[3:]))[pix] for x in out[:4])
    sc = Scene(oracle_mod, b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, w.H, w.W,
               w.blur_radius, w.K, w.perspective_correct, pix)
    info = compare_forward(g, sc.fwd(), f"batch{cfg} sampled", scene=sc)
    assert info["valid_slots"] > 500
    if sig is not None:
        compare_alpha(np_(out[4]).reshape(-1)[pix], alpha_of(oracle_mod, info, sig), label=f"batch{cfg} alpha")


def test_device_resident_mesh_arrays_match_host_ones():
    """The per-mesh index arrays may be CUDA tensors (as a packed mesh batch keeps them); the
    library reads them with one device-to-host copy and the outputs are identical."""
    b = syn.make_batch(2)
    w = b.workload
    v, f = to_dev(b.verts, b.faces)
    first, num = b.mesh_to_face_first_idx, b.num_faces_per_mesh
    want = mr.rasterize_fwd(v, f, first, num, w.H, w.W, w.blur_radius, w.K, sigma=w.sigma)
    got = mr.rasterize_fwd(v, f, torch.as_tensor(first).cuda(), torch.as_tensor(num).cuda(), w.H, w.W, w.blur_radius,
                           w.K, sigma=w.sigma)
    for x, y in zip(got, want):
        assert torch.equal(x, y)
