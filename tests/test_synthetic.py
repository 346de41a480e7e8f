"""Input generators: topology counts, Euler characteristic, determinism (CPU only)."""
import numpy as np
import pytest

from differentiable_mesh_rasterization_b200 import synthetic as syn


def euler(v, f):
    e = np.unique(np.sort(np.concatenate([f[:, [0, 1]], f[:, [1, 2]], f[:, [2, 0]]]), axis=1), axis=0)
    return v.shape[0] - e.shape[0] + f.shape[0]


@pytest.mark.parametrize("level", [0, 1, 2, 3, 4])
def test_icosphere_counts_and_euler(level):
    v, f = syn.icosphere(level)
    assert v.shape == (10 * 4 ** level + 2, 3)
    assert f.shape == (20 * 4 ** level, 3)
    assert euler(v, f) == 2
    assert np.allclose(np.linalg.norm(v, axis=1), 1.0)
    # outward, consistently wound faces: normal . centroid > 0
    a, b, c = v[f[:, 0]], v[f[:, 1]], v[f[:, 2]]
    assert np.all(np.einsum("ij,ij->i", np.cross(b - a, c - a), a + b + c) > 0)


@pytest.mark.parametrize("R,S", [(16, 16), (17, 40), (256, 33)])
def test_torus_counts_and_euler(R, S):
    v, f = syn.torus(R, S)
    assert v.shape == (R * S, 3) and f.shape == (2 * R * S, 3)
    assert euler(v, f) == 0
    # every edge shared by exactly two faces (closed 2-manifold)
    e = np.sort(np.concatenate([f[:, [0, 1]], f[:, [1, 2]], f[:, [2, 0]]]), axis=1)
    _, cnt = np.unique(e, axis=0, return_counts=True)
    assert np.all(cnt == 2)


def test_rotation_is_orthonormal():
    rng = np.random.Generator(np.random.PCG64(7))
    for _ in range(10):
        R = syn.random_rotation(rng)
        assert np.allclose(R @ R.T, np.eye(3), atol=1e-12)
        assert np.isclose(np.linalg.det(R), 1.0)


def test_projection_camera():
    w = np.array([[0.0, 0.0, 0.0], [1.0, 0.5, -0.3]])
    p = syn.project(w)
    t = np.tan(np.radians(30.0))
    assert np.allclose(p[0], [0, 0, 2.7])
    assert np.allclose(p[1], [1.0 / (3.0 * t), 0.5 / (3.0 * t), 3.0])


@pytest.mark.parametrize("cfg", [1, 2, 3])
def test_batches_deterministic_and_packed(cfg):
    a = syn.make_batch(cfg)
    b = syn.make_batch(cfg)
    assert np.array_equal(a.verts, b.verts) and np.array_equal(a.faces, b.faces)
    w = syn.WORKLOADS[cfg]
    assert a.N == w.N
    assert a.verts.dtype == np.float32 and a.faces.dtype == np.int64
    assert np.array_equal(a.mesh_to_face_first_idx, np.concatenate([[0], np.cumsum(a.num_faces_per_mesh)[:-1]]))
    # faces of mesh n reference only mesh n's vertices
    for n in range(a.N):
        f0, nf = a.mesh_to_face_first_idx[n], a.num_faces_per_mesh[n]
        v0, nv = a.mesh_to_vert_first_idx[n], a.num_verts_per_mesh[n]
        fs = a.faces[f0:f0 + nf]
        assert fs.min() >= v0 and fs.max() < v0 + nv
    assert np.all(a.verts[:, 2] > 1.0)   # everything in front of the camera
    c = syn.make_batch(cfg, seed=12345)
    assert not np.array_equal(a.verts, c.verts)


def test_config_face_counts():
    b2 = syn.make_batch(2)
    assert set(b2.num_faces_per_mesh.tolist()) <= {320, 1280, 5120}
    b3 = syn.make_batch(3)
    assert np.all(b3.num_faces_per_mesh == 20480)
    b5 = syn.make_batch(5, n_meshes=40)
    full_kinds = syn.make_batch(5, n_meshes=40).kinds
    assert all(k[0] == "ico" and 3 <= k[1] <= 6 for k in full_kinds[:32])
    assert all(k[0] == "torus" and 16 <= k[1] <= 256 and 16 <= k[2] <= 256 for k in full_kinds[32:40])
    for n, k in enumerate(full_kinds):
        if k[0] == "ico":
            assert b5.num_faces_per_mesh[n] == 20 * 4 ** k[1]
        else:
            assert b5.num_faces_per_mesh[n] == 2 * k[1] * k[2]


def test_truncated_batch_is_prefix():
    full = syn.make_batch(2)
    part = syn.make_batch(2, n_meshes=3)
    nv = int(part.num_verts_per_mesh.sum())
    assert np.array_equal(full.verts[:nv], part.verts)


def test_blur_sigma_relation():
    s = 1e-4
    br = syn.blur_for_sigma(s)
    assert abs(1.0 / (1.0 + np.exp(br / s)) - 1e-4) < 1e-15
