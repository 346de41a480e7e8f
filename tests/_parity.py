"""Comparison rules between the CUDA path (float32) and the float64 oracle.

pix_to_face: exact on every pixel the oracle does not mark exempt (E1: two of the K+1
nearest candidates within 1e-6 in depth; E2: a face whose candidacy sits on its
threshold and would rank in the first K).
zbuf, bary, dists: |gpu - oracle| <= 1e-5 + 2^-23 |oracle| on the slots of those
pixels (1e-5 absolute, widened by one float32 ulp of the value because a float32
result cannot be nearer than half an ulp to a float64 value above ~168).
alpha: |gpu - oracle| <= 1e-4 |oracle| + 1e-7.
grad_verts: |gpu - oracle| <= 1e-4 |oracle| + 1e-4 rms(oracle).
"""
from __future__ import annotations

import numpy as np

ABS = 1e-5
ULP = 2.0 ** -23
EXEMPT_MAX = 0.03     # E1 near-ties reach ~1.2% of covered pixels on sub-pixel meshes


def np_(t):
    return t.detach().cpu().numpy() if hasattr(t, "detach") else np.asarray(t)


def compare_forward(gpu, ora, label="", exempt_max=EXEMPT_MAX):
    """gpu: (p2f, zbuf, bary, dists) tensors/arrays; ora: oracle tuple incl. exempt."""
    pg, zg, bg, dg = (np_(x) for x in gpu)
    po, zo, bo, do, ex = ora
    ok = ex == 0
    assert ok.mean() >= 1 - exempt_max, f"{label}: exempt fraction {1 - ok.mean():.4%}"
    bad = (pg != po).any(-1) & ok
    if bad.any():
        idx = np.argwhere(bad)[:5]
        det = [(tuple(i), pg[tuple(i)].tolist(), po[tuple(i)].tolist(), zo[tuple(i)].tolist()) for i in idx]
        raise AssertionError(f"{label}: pix_to_face differs at {int(bad.sum())} non-exempt pixels: {det}")
    valid = (po >= 0) & ok[..., None]
    empty = (po < 0) & ok[..., None]
    for name, g, o in (("zbuf", zg, zo), ("dists", dg, do)):
        err = np.abs(g[valid] - o[valid]) - (ABS + ULP * np.abs(o[valid]))
        assert err.size == 0 or err.max() <= 0, f"{label}: {name} off by {err.max() + ABS:.3g}"
        assert np.all(g[empty] == -1), f"{label}: {name} empty slots not -1"
    err = np.abs(bg[valid] - bo[valid]) - (ABS + ULP * np.abs(bo[valid]))
    assert err.size == 0 or err.max() <= 0, f"{label}: bary off by {err.max() + ABS:.3g}"
    assert np.all(bg[empty] == -1), f"{label}: bary empty slots not -1"
    return dict(exempt=float(1 - ok.mean()), valid_slots=int(valid.sum()))


def compare_alpha(ag, ao, mask=None, label=""):
    ag, ao = np_(ag), np.asarray(ao)
    if mask is not None:
        ag, ao = ag[mask], ao[mask]
    err = np.abs(ag - ao) - (1e-4 * np.abs(ao) + 1e-7)
    assert err.size == 0 or err.max() <= 0, f"{label}: alpha off by {err.max():.3g} beyond tolerance"


def compare_grad(gg, go, mask=None, label="", extra=None):
    """Element-wise |gpu - oracle| <= 1e-4 |oracle| + 1e-4 rms(oracle) (+ ``extra``, an
    element-wise allowance for float32 rounding of ill-conditioned inputs)."""
    gg, go = np_(gg).astype(np.float64), np.asarray(go)
    extra = 0.0 if extra is None else np.asarray(extra, np.float64)
    if mask is not None:
        gg, go = gg[mask], go[mask]
        if np.ndim(extra):
            extra = extra[mask]
    rms = np.sqrt(np.mean(go ** 2)) if go.size else 0.0
    err = np.abs(gg - go) - (1e-4 * np.abs(go) + 1e-4 * rms + extra)
    if err.size and err.max() > 0:
        i = int(np.argmax(err))
        raise AssertionError(f"{label}: grad off at {i}: gpu {gg.reshape(-1)[i]:.6g} oracle {go.reshape(-1)[i]:.6g} "
                             f"rms {rms:.3g}")
    rel = np.linalg.norm(gg - go) / max(np.linalg.norm(go), 1e-30)
    return float(rel)


def sample_pixels(batch, count_per_image, seed):
    """Seeded pixel ids inside each mesh's screen box (widened by the blur reach)."""
    w = batch.workload
    rng = np.random.default_rng(seed)
    r = np.sqrt(w.blur_radius)
    out = []
    for n in range(batch.N):
        f0, nf = batch.mesh_to_face_first_idx[n], batch.num_faces_per_mesh[n]
        v = batch.verts[np.unique(batch.faces[f0:f0 + nf])]
        x0, x1 = v[:, 0].min() - r, v[:, 0].max() + r
        y0, y1 = v[:, 1].min() - r, v[:, 1].max() + r
        j0 = int(np.clip(np.floor((x0 + 1) * w.W / 2), 0, w.W - 1))
        j1 = int(np.clip(np.ceil((x1 + 1) * w.W / 2), 0, w.W - 1))
        i0 = int(np.clip(np.floor((1 - y1) * w.H / 2), 0, w.H - 1))
        i1 = int(np.clip(np.ceil((1 - y0) * w.H / 2), 0, w.H - 1))
        ii = rng.integers(i0, i1 + 1, count_per_image)
        jj = rng.integers(j0, j1 + 1, count_per_image)
        out.append((n * w.H + ii) * w.W + jj)
    return np.unique(np.concatenate(out))
