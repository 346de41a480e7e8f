"""Writes the stored oracle outputs under tests/golden/ (calls only oracle/ and the input generators).

    python tests/golden/make_golden.py

batch1_oracle.txt: the 64x64 hard-rasterized icosphere (benchmark batch 1: level-2
icosphere, radial noise 0.02, 64x64, K=1, blur 0).  One line per covered pixel:
``row col face zbuf bary0 bary1 bary2 dist exempt`` with 17 significant digits.

next_rows_oracle.txt: Phong lighting of 40 seeded points (step 18), the point rasterizer on
the first cloud of point batch 2 at 24x24 with K=3 and radius 0.05 (step 22) with its alpha
compositing (step 24), and the 4 nearest neighbours of the first 50 queries of KNN batch 2
(step 27); one tagged line per point, covered pixel or query.
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from differentiable_mesh_rasterization_b200 import synthetic as syn  # noqa: E402


def batch1_lines():
    b = syn.make_batch(1)
    w = b.workload
    p2f, zbuf, bary, dists, ex = oracle.rasterize_fwd(b.verts, b.faces, b.mesh_to_face_first_idx,
                                                      b.num_faces_per_mesh, w.H, w.W, w.blur_radius, w.K,
                                                      w.perspective_correct)
    lines = []
    for i in range(w.H):
        for j in range(w.W):
            f = p2f[0, i, j, 0]
            if f < 0:
                continue
            vals = [zbuf[0, i, j, 0], *bary[0, i, j, 0], dists[0, i, j, 0]]
            lines.append(f"{i} {j} {f} " + " ".join(f"{x:.17g}" for x in vals) + f" {ex[0, i, j]}")
    return lines


PHONG_PARAMS = ([1.0, 1.5, 3.0], [0.0, 0.0, 2.7], [0.1, 0.2, 0.05], [0.7, 0.5, 0.9], [0.3, 0.25, 0.2], 8.0)


def next_rows_lines():
    f17 = lambda xs: " ".join(f"{float(x):.17g}" for x in xs)
    lines = []
    rng = np.random.default_rng(7)
    P = rng.uniform(-1, 1, size=(40, 3))
    N = rng.normal(size=(40, 3))
    c = rng.uniform(size=(40, 3))
    col, flags = oracle.phong_fwd(P, N, c, oracle.phong_params(*PHONG_PARAMS))
    for i in range(40):
        lines.append(f"phong {i} {int(flags[i])} " + f17(col[i]))
    pb = syn.make_point_batch(2, n_clouds=1)
    idx, zbuf, dists, pflags = oracle.rasterize_points(pb.points, pb.cloud_first_idx, pb.num_points_per_cloud, 24,
                                                       24, 0.05, 3)
    img = oracle.composite_points(idx, dists, pb.features, 0.05, "alpha")
    for i in range(24):
        for j in range(24):
            if idx[0, i, j, 0] < 0:
                continue
            lines.append(f"points {i} {j} {int(pflags[0, i, j])} " + " ".join(str(int(x)) for x in idx[0, i, j]) +
                         " " + f17(zbuf[0, i, j]) + " " + f17(dists[0, i, j]) + " " + f17(img[0, i, j]))
    kb = syn.make_knn_batch(2, n_clouds=1)
    q = kb.p1[:50]
    kidx, kd, kflags = oracle.knn(q, [0], [50], kb.p2, kb.first2, kb.num2, 4)
    for i in range(50):
        lines.append(f"knn {i} {int(kflags[i])} " + " ".join(str(int(x)) for x in kidx[i]) + " " + f17(kd[i]))
    return lines


if __name__ == "__main__":
    with open(os.path.join(HERE, "next_rows_oracle.txt"), "w") as fh:
        fh.write("# tag key... flag values -- written by make_golden.py\n")
        fh.write("\n".join(next_rows_lines()) + "\n")
    with open(os.path.join(HERE, "batch1_oracle.txt"), "w") as fh:
        fh.write("# row col face zbuf bary0 bary1 bary2 dist exempt -- written by make_golden.py\n")
        fh.write("\n".join(batch1_lines()) + "\n")
