"""Per-image sharding of a packed mesh batch across ranks (one process per GPU).

The rasterizer's images are independent ("Accelerating 3D Deep Learning with PyTorch3D",
heterogeneous batching: image n is drawn from mesh n alone), so a batch splits by whole
meshes.  Each rank renders its meshes with the single-GPU entry points and computes the
gradient of the vertices they use; nothing crosses ranks on the data path.  A vertex
used by meshes on several ranks (packed batches normally give each mesh its own) gets
its gradient as the sum of the ranks' parts.  The helpers here are host-side index
bookkeeping (numpy): the cost model that balances the split, the split itself, and the
index maps that cut one rank's meshes out of the packed arrays and put its results back.
"""
from __future__ import annotations

import math

import numpy as np


def face_pixel_boxes(verts, faces, H: int, W: int, blur_radius: float):
    """Inclusive pixel boxes (jl, jh, il, ih) of the given faces grown by sqrt(blur_radius),
    clipped to the image, in float64; degenerate (|2 area| <= 1e-12) and off-image faces are
    dropped.  verts (V, 3), faces (F, 3) int64, host arrays."""
    r = math.sqrt(blur_radius)
    tri = np.asarray(verts, np.float64)[np.asarray(faces, np.int64)]          # (F, 3, 3)
    a, b, c = tri[:, 0], tri[:, 1], tri[:, 2]
    area2 = (b[:, 0] - a[:, 0]) * (c[:, 1] - a[:, 1]) - (b[:, 1] - a[:, 1]) * (c[:, 0] - a[:, 0])
    xmin, xmax = tri[:, :, 0].min(1) - r, tri[:, :, 0].max(1) + r
    ymin, ymax = tri[:, :, 1].min(1) - r, tri[:, :, 1].max(1) + r
    jl = np.maximum(np.ceil((xmin + 1) * W / 2 - 0.5), 0)
    jh = np.minimum(np.floor((xmax + 1) * W / 2 - 0.5), W - 1)
    il = np.maximum(np.ceil((1 - ymax) * H / 2 - 0.5), 0)
    ih = np.minimum(np.floor((1 - ymin) * H / 2 - 0.5), H - 1)
    ok = (np.abs(area2) > 1e-12) & (jl <= jh) & (il <= ih)
    return jl[ok], jh[ok], il[ok], ih[ok]


def mesh_sample_counts(verts, faces, first, num, H: int, W: int, blur_radius: float) -> np.ndarray:
    """Per mesh, its pixel-face samples: the (pixel, face) pairs whose pixel centre lies in
    the face's box grown by sqrt(blur_radius) -- the work the fine pass has to test, and
    the cost by which :func:`partition_meshes` balances ranks."""
    faces = np.asarray(faces, np.int64)
    out = np.zeros(len(first), np.int64)
    for n, (f0, nf) in enumerate(zip(np.asarray(first, np.int64), np.asarray(num, np.int64))):
        jl, jh, il, ih = face_pixel_boxes(verts, faces[f0:f0 + nf], H, W, blur_radius)
        out[n] = int(np.sum((jh - jl + 1) * (ih - il + 1)))
    return out


def partition_meshes(costs, world: int) -> list[np.ndarray]:
    """Split mesh indices 0..N-1 over `world` ranks, balancing the summed cost: meshes in
    decreasing cost (ties: lower index first) each go to the rank with the least cost so
    far (ties: fewer meshes, then lower rank, so zero-cost meshes spread too) -- the
    longest-processing-time rule, within 4/3 of the best makespan.  Deterministic, so every rank computes the same split without exchanging
    anything.  Returns per rank its mesh indices in increasing order."""
    if world < 1:
        raise ValueError("world must be >= 1")
    costs = np.asarray(costs, np.float64)
    order = sorted(range(len(costs)), key=lambda n: (-costs[n], n))
    load = [0.0] * world
    parts: list[list[int]] = [[] for _ in range(world)]
    for n in order:
        r = min(range(world), key=lambda q: (load[q], len(parts[q]), q))
        parts[r].append(n)
        load[r] += costs[n]
    return [np.array(sorted(p), np.int64) for p in parts]


class Shard:
    """One rank's meshes cut out of a packed batch.

    face_ids: the global face rows, mesh after mesh in `meshes` order; vert_ids: the
    global vertices those faces use (sorted); faces: the same faces with vertex ids local
    to vert_ids; first / num: the per-mesh face ranges inside `faces`.  The rank's inputs
    are verts[vert_ids] and faces; its images are the batch's images `meshes`.
    """

    def __init__(self, faces, first, num, meshes):
        faces = np.asarray(faces, np.int64)
        first = np.asarray(first, np.int64)
        num = np.asarray(num, np.int64)
        self.meshes = np.asarray(meshes, np.int64)
        self.num = num[self.meshes].copy()
        self.first = (np.cumsum(self.num) - self.num).astype(np.int64)
        self.face_ids = (np.concatenate([np.arange(first[n], first[n] + num[n]) for n in self.meshes])
                         if len(self.meshes) else np.zeros(0, np.int64)).astype(np.int64)
        used = faces[self.face_ids]
        self.vert_ids = np.unique(used)
        self.faces = np.searchsorted(self.vert_ids, used).astype(np.int64).reshape(-1, 3)

    def global_faces(self, pix_to_face):
        """A pix_to_face of this shard (local face ids, -1 for empty slots) in the batch's
        face ids."""
        p = np.asarray(pix_to_face, np.int64)
        return np.where(p >= 0, self.face_ids[np.maximum(p, 0)] if self.face_ids.size else -1, -1)

    def scatter_vertex_rows(self, local_rows, V: int):
        """Rows of a per-vertex result (e.g. grad_verts) of this shard placed at their global
        vertex ids in a zero (V, ...) array; the sum of all ranks' arrays is the whole
        batch's result."""
        local_rows = np.asarray(local_rows)
        out = np.zeros((V,) + local_rows.shape[1:], local_rows.dtype)
        out[self.vert_ids] = local_rows
        return out

    def scatter_images(self, local_images, N: int):
        """Per-image results (first axis = this shard's images) placed at their global image
        indices in a zero (N, ...) array."""
        local_images = np.asarray(local_images)
        out = np.zeros((N,) + local_images.shape[1:], local_images.dtype)
        out[self.meshes] = local_images
        return out
