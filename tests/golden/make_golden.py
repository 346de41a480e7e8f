"""Writes the stored oracle outputs under tests/golden/ (calls only oracle/ and the input generators).

    python tests/golden/make_golden.py

batch1_oracle.txt: the 64x64 hard-rasterized icosphere (benchmark batch 1: level-2
icosphere, radial noise 0.02, 64x64, K=1, blur 0).  One line per covered pixel:
``row col face zbuf bary0 bary1 bary2 dist exempt`` with 17 significant digits.
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


if __name__ == "__main__":
    with open(os.path.join(HERE, "batch1_oracle.txt"), "w") as fh:
        fh.write("# row col face zbuf bary0 bary1 bary2 dist exempt -- written by make_golden.py\n")
        fh.write("\n".join(batch1_lines()) + "\n")
