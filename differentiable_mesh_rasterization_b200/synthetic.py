"""Seeded synthetic inputs: icospheres, tori, random poses and the screen projection.

This module builds the inputs of the rasterizer and nothing else.  It holds none of
the rasterizer's arithmetic (no coverage, distance, depth ordering or blending), so
both the CUDA path and the float64 CPU oracle may consume what it produces.

Workloads follow the five benchmark batches of the PyTorch3D rasterizer evaluation
(*Accelerating 3D Deep Learning with PyTorch3D*, "Experiments": 137x137 renders of
heterogeneous batches; tutorial summary, "Data Structures and I/O": icosphere and torus
primitives).  Every random draw comes from numpy ``PCG64``; batch ``c`` uses seed
``1000 + c`` and mesh ``n`` draws from ``SeedSequence(1000 + c).spawn(N + 1)[n]``;
the last spawned child draws the upstream silhouette gradient.

Camera: the eye sits at distance 2.7 on +Z looking at the origin with a 60 degree
vertical field of view.  A world point (X, Y, Z) maps to view depth z = 2.7 - Z and to
normalised device coordinates x = X / (z tan 30deg), y = Y / (z tan 30deg): +x right,
+y up.  The rasterizer receives (x, y, z) per vertex.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

CAMERA_DIST = 2.7
FOV_DEG = 60.0


# --------------------------------------------------------------------------- meshes
def icosahedron() -> tuple[np.ndarray, np.ndarray]:
    """Regular icosahedron on the unit sphere, outward counter-clockwise faces."""
    p = (1.0 + math.sqrt(5.0)) / 2.0
    v = np.array(
        [[-1, p, 0], [1, p, 0], [-1, -p, 0], [1, -p, 0],
         [0, -1, p], [0, 1, p], [0, -1, -p], [0, 1, -p],
         [p, 0, -1], [p, 0, 1], [-p, 0, -1], [-p, 0, 1]], dtype=np.float64)
    v /= np.linalg.norm(v, axis=1, keepdims=True)
    f = np.array(
        [[0, 11, 5], [0, 5, 1], [0, 1, 7], [0, 7, 10], [0, 10, 11],
         [1, 5, 9], [5, 11, 4], [11, 10, 2], [10, 7, 6], [7, 1, 8],
         [3, 9, 4], [3, 4, 2], [3, 2, 6], [3, 6, 8], [3, 8, 9],
         [4, 9, 5], [2, 4, 11], [6, 2, 10], [8, 6, 7], [9, 8, 1]], dtype=np.int64)
    return v, f


def icosphere(level: int) -> tuple[np.ndarray, np.ndarray]:
    """Icosahedron subdivided ``level`` times (shared edge midpoints, re-normalised).

    V = 10 * 4**level + 2 and F = 20 * 4**level.  The four children of face ``f`` are
    faces ``4f .. 4f+3``, so neighbouring face ids stay close on the surface.
    """
    v, f = icosahedron()
    for _ in range(level):
        nf = f.shape[0]
        e = np.stack([f[:, [0, 1]], f[:, [1, 2]], f[:, [2, 0]]], axis=1).reshape(-1, 2)
        key = np.sort(e, axis=1)
        uniq, inv = np.unique(key, axis=0, return_inverse=True)
        inv = inv.reshape(nf, 3)
        mid = v[uniq[:, 0]] + v[uniq[:, 1]]
        mid /= np.linalg.norm(mid, axis=1, keepdims=True)
        base = v.shape[0]
        v = np.concatenate([v, mid], axis=0)
        a, b, c = f[:, 0], f[:, 1], f[:, 2]
        ab, bc, ca = base + inv[:, 0], base + inv[:, 1], base + inv[:, 2]
        f = np.stack([np.stack([a, ab, ca], 1), np.stack([ab, b, bc], 1),
                      np.stack([ca, bc, c], 1), np.stack([ab, bc, ca], 1)], axis=1).reshape(-1, 3)
    return v, f


def torus(rings: int, segments: int, major: float = 1.0, minor: float = 0.3) -> tuple[np.ndarray, np.ndarray]:
    """Torus in the XY plane: V = rings * segments, F = 2 * rings * segments."""
    th = 2.0 * math.pi * np.arange(rings) / rings
    ph = 2.0 * math.pi * np.arange(segments) / segments
    T, P = np.meshgrid(th, ph, indexing="ij")
    r = major + minor * np.cos(P)
    v = np.stack([r * np.cos(T), r * np.sin(T), minor * np.sin(P)], axis=-1).reshape(-1, 3)
    i = np.arange(rings)[:, None]
    j = np.arange(segments)[None, :]
    i1, j1 = (i + 1) % rings, (j + 1) % segments
    v00, v10 = i * segments + j, i1 * segments + j
    v11, v01 = i1 * segments + j1, i * segments + j1
    f = np.stack([np.stack([v00, v10, v11], -1), np.stack([v00, v11, v01], -1)], axis=2)
    return v, f.reshape(-1, 3).astype(np.int64)


def random_rotation(rng: np.random.Generator) -> np.ndarray:
    """Uniform rotation from a normalised 4-D Gaussian quaternion."""
    q = rng.standard_normal(4)
    q /= np.linalg.norm(q)
    w, x, y, z = q
    return np.array([
        [1 - 2 * (y * y + z * z), 2 * (x * y - z * w), 2 * (x * z + y * w)],
        [2 * (x * y + z * w), 1 - 2 * (x * x + z * z), 2 * (y * z - x * w)],
        [2 * (x * z - y * w), 2 * (y * z + x * w), 1 - 2 * (x * x + y * y)]])


def project(world: np.ndarray, dist: float = CAMERA_DIST, fov_deg: float = FOV_DEG) -> np.ndarray:
    """World (X, Y, Z) -> (x_ndc, y_ndc, z_view) for the fixed look-at camera."""
    t = math.tan(math.radians(fov_deg) / 2.0)
    z = dist - world[:, 2]
    return np.stack([world[:, 0] / (z * t), world[:, 1] / (z * t), z], axis=1)


# --------------------------------------------------------------------------- batches
def blur_for_sigma(sigma: float, eps: float = 1e-4) -> float:
    """Blur radius at which a face's sigmoid weight falls to ``eps``: ln(1/eps - 1) * sigma."""
    return math.log(1.0 / eps - 1.0) * sigma


@dataclass
class Workload:
    name: str
    N: int
    H: int
    W: int
    K: int
    blur_radius: float
    sigma: float | None
    perspective_correct: bool
    backward: bool
    description: str


WORKLOADS: dict[int, Workload] = {
    1: Workload("ico2_b1_64px_K1_hard", 1, 64, 64, 1, 0.0, None, False, False,
                "1 x icosphere L2 (320 faces), radial noise 0.02, 64x64, K=1, blur 0, forward"),
    2: Workload("ico234_b8_137px_K8_soft", 8, 137, 137, 8, blur_for_sigma(1e-4), 1e-4, False, True,
                "8 x icosphere L2/L3/L4, noise 0.03, SO(3), 137x137, K=8, sigma 1e-4, fwd+bwd"),
    3: Workload("ico5_b16_256px_K16_soft", 16, 256, 256, 16, blur_for_sigma(1e-4), 1e-4, False, True,
                "16 x icosphere L5 (20,480 faces), noise 0.05, SO(3), scale U(0.6,1), 256x256, K=16, fwd+bwd"),
    4: Workload("ico7_b1_1024px_K8_persp", 1, 1024, 1024, 8, 1e-5, None, True, False,
                "1 x icosphere L7 (327,680 faces), noise 0.01, 1024x1024, K=8, blur 1e-5, perspective, fwd"),
    5: Workload("ico36_torus_b64_512px_K4_soft", 64, 512, 512, 4, blur_for_sigma(1e-4), 1e-4, False, True,
                "64 meshes: 32 icospheres L3-L6 + 32 tori (16..256 rings/segments), SO(3), "
                "translation +-0.2, 512x512, K=4, sigma 1e-4, fwd+bwd"),
}


@dataclass
class MeshBatch:
    """A packed heterogeneous batch in screen space, ready for the rasterizer."""
    verts: np.ndarray               # (sum V, 3) float32: x_ndc, y_ndc, z_view
    faces: np.ndarray               # (sum F, 3) int64: global (packed) vertex ids
    mesh_to_face_first_idx: np.ndarray  # (N,) int64
    num_faces_per_mesh: np.ndarray      # (N,) int64
    mesh_to_vert_first_idx: np.ndarray  # (N,) int64
    num_verts_per_mesh: np.ndarray      # (N,) int64
    workload: Workload
    seed: int
    kinds: list = field(default_factory=list)   # per mesh: ("ico", level) or ("torus", R, S)
    world: np.ndarray | None = None     # (sum V, 3) float32: world positions (camera at (0, 0, 2.7))
    normals: np.ndarray | None = None   # (sum V, 3) float32: unit normals of the unperturbed shape

    @property
    def N(self) -> int:
        return int(self.num_faces_per_mesh.shape[0])


def _pack(meshes: list[tuple[np.ndarray, np.ndarray]]):
    verts, faces, ff, nf, vf, nv = [], [], [], [], [], []
    vo = fo = 0
    for v, f, *_ in meshes:
        verts.append(v)
        faces.append(f + vo)
        ff.append(fo); nf.append(f.shape[0]); vf.append(vo); nv.append(v.shape[0])
        vo += v.shape[0]; fo += f.shape[0]
    return (np.concatenate(verts).astype(np.float32), np.concatenate(faces).astype(np.int64),
            np.array(ff, np.int64), np.array(nf, np.int64), np.array(vf, np.int64), np.array(nv, np.int64))


def _mesh_rngs(seed: int, n: int) -> list[np.random.Generator]:
    return [np.random.Generator(np.random.PCG64(s)) for s in np.random.SeedSequence(seed).spawn(n + 1)]


def make_batch(config: int, seed: int | None = None, n_meshes: int | None = None) -> MeshBatch:
    """Seeded packed batch for benchmark batch ``config`` (1..5).

    ``n_meshes`` truncates the batch to its first meshes (same draws as the full batch).
    """
    w = WORKLOADS[config]
    seed = 1000 + config if seed is None else seed
    N = w.N
    rngs = _mesh_rngs(seed, N)
    top = np.random.Generator(np.random.PCG64(seed))
    meshes, kinds = [], []
    if config == 1:
        levels = [2]
    elif config == 2:
        levels = list(top.integers(2, 5, size=N))
    elif config == 3:
        levels = [5] * N
    elif config == 4:
        levels = [7]
    else:
        levels = list(top.integers(3, 7, size=N // 2))
        rs = top.integers(16, 257, size=(N - N // 2, 2))
    noise = {1: 0.02, 2: 0.03, 3: 0.05, 4: 0.01, 5: 0.0}[config]
    count = N if n_meshes is None else min(N, n_meshes)
    for n in range(count):
        rng = rngs[n]
        if config == 5 and n >= N // 2:
            R, S = int(rs[n - N // 2, 0]), int(rs[n - N // 2, 1])
            v, f = torus(R, S)
            ring = v.copy()
            ring[:, 2] = 0.0
            ring /= np.linalg.norm(ring, axis=1, keepdims=True)
            nrm = (v - ring) / np.linalg.norm(v - ring, axis=1, keepdims=True)   # away from the tube's core
            kinds.append(("torus", R, S))
        else:
            v, f = icosphere(int(levels[n]))
            nrm = v.copy()                                                     # unit sphere: normal = position
            kinds.append(("ico", int(levels[n])))
        if noise > 0:
            v = v * (1.0 + noise * rng.standard_normal((v.shape[0], 1)))
        if config == 3:
            v = v * rng.uniform(0.6, 1.0)
        if config in (2, 3, 5):
            R3 = random_rotation(rng)
            v = v @ R3.T
            nrm = nrm @ R3.T
        if config == 5:
            v = v + rng.uniform(-0.2, 0.2, size=3)
        meshes.append((project(v), f, v, nrm))
    verts, faces, ff, nf, vf, nv = _pack(meshes)
    world = np.concatenate([m[2] for m in meshes]).astype(np.float32)
    normals = np.concatenate([m[3] for m in meshes]).astype(np.float32)
    return MeshBatch(verts, faces, ff, nf, vf, nv, w, seed, kinds, world, normals)


def grad_alpha(batch: MeshBatch) -> np.ndarray:
    """Upstream gradient dL/dsilhouette ~ N(0, 1), shape (N, H, W), float32."""
    w = batch.workload
    rng = _mesh_rngs(batch.seed, w.N)[w.N]
    return rng.standard_normal((batch.N, w.H, w.W)).astype(np.float32)


def random_grads(shape: tuple, seed: int) -> np.ndarray:
    """Generic seeded N(0, 1) float32 array (upstream gradients for tests)."""
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape).astype(np.float32)


# --------------------------------------------------------------------------- point clouds
@dataclass
class PointWorkload:
    name: str
    mesh_config: int        # the mesh batch whose vertices are the clouds
    H: int
    W: int
    K: int
    radius: float           # NDC units
    C: int                  # feature channels
    description: str


POINT_WORKLOADS: dict[int, PointWorkload] = {
    2: PointWorkload("pts_ico234_b8_137px_K8", 2, 137, 137, 8, 0.02, 3,
                     "vertices of mesh batch 2 (8 clouds, 642-2562 points), 137x137, K=8, radius 0.02, RGB"),
    5: PointWorkload("pts_ico36_torus_b64_512px_K8", 5, 512, 512, 8, 0.01, 3,
                     "vertices of mesh batch 5 (64 clouds, 642-55,418 points, 1.18 M in all), 512x512, K=8, "
                     "radius 0.01, RGB"),
}


@dataclass
class PointBatch:
    """A packed heterogeneous batch of screen-space point clouds with per-point features."""
    points: np.ndarray              # (P, 3) float32: x_ndc, y_ndc, z_view
    cloud_first_idx: np.ndarray     # (N,) int64
    num_points_per_cloud: np.ndarray  # (N,) int64
    features: np.ndarray            # (P, C) float32 in [0, 1)
    workload: PointWorkload

    @property
    def N(self) -> int:
        return int(self.num_points_per_cloud.shape[0])


def make_point_batch(config: int, n_clouds: int | None = None) -> PointBatch:
    """Point clouds made of the vertices of mesh batch ``config`` (same draws), with
    features ~ U[0, 1) from ``PCG64(2000 + config)``."""
    w = POINT_WORKLOADS[config]
    b = make_batch(w.mesh_config, n_meshes=n_clouds)
    rng = np.random.Generator(np.random.PCG64(2000 + config))
    feats = rng.uniform(size=(b.verts.shape[0], w.C)).astype(np.float32)
    return PointBatch(b.verts, b.mesh_to_vert_first_idx.copy(), b.num_verts_per_mesh.copy(), feats, w)


@dataclass
class KnnWorkload:
    name: str
    mesh_config: int
    K: int
    jitter: float
    description: str


KNN_WORKLOADS: dict[int, KnnWorkload] = {
    2: KnnWorkload("knn_ico234_b8_K8", 2, 8, 0.01,
                   "8 clouds (world vertices of mesh batch 2, 642-2562 points) against their jittered copies, D=3, K=8"),
    5: KnnWorkload("knn_ico36_torus_b64_K8", 5, 8, 0.01,
                   "64 clouds (world vertices of mesh batch 5, 642-55,418 points, 1.18 M in all) against their "
                   "jittered copies, D=3, K=8"),
}


@dataclass
class KnnBatch:
    """Two packed heterogeneous sets of 3-D clouds: queries p1 and references p2 (cloud n of
    p1 searches cloud n of p2)."""
    p1: np.ndarray
    first1: np.ndarray
    num1: np.ndarray
    p2: np.ndarray
    first2: np.ndarray
    num2: np.ndarray
    workload: KnnWorkload

    @property
    def N(self) -> int:
        return int(self.num1.shape[0])


def make_knn_batch(config: int, n_clouds: int | None = None) -> KnnBatch:
    """References: the world vertices of mesh batch ``config``; queries: the same points
    moved by N(0, jitter^2) per coordinate from ``PCG64(3000 + config)``."""
    w = KNN_WORKLOADS[config]
    b = make_batch(w.mesh_config, n_meshes=n_clouds)
    rng = np.random.Generator(np.random.PCG64(3000 + config))
    p2 = b.world.astype(np.float32)
    p1 = (p2 + w.jitter * rng.standard_normal(p2.shape)).astype(np.float32)
    f, n = b.mesh_to_vert_first_idx.copy(), b.num_verts_per_mesh.copy()
    return KnnBatch(p1, f, n, p2, f.copy(), n.copy(), w)
