"""Comparison rules between the CUDA path (float32) and the float64 oracle.

pix_to_face (target specification: exact, except where two candidate depths differ by
less than 1e-6):
- pixels the oracle does not flag: exact;
- E1 pixels (two of the K+1 nearest candidates within 1e-6 in depth): equal up to a
  permutation inside each group of candidates whose depths chain within 1e-6; the oracle is
  asked again for more than K candidates there, so a group that straddles slot K may hand
  slot K-1 to the (K+1)-th candidate;
- E2 pixels (a face whose candidacy lies within a rounding margin of its threshold and
  would rank in the first K): the choice of faces is the only thing left open, and only
  for those marginal faces -- the faces that are not marginal must be the oracle's, in
  order, up to depth ties; the E2 rate must stay below 0.1% of the compared pixels.
zbuf, bary, dists: |gpu - oracle| <= 1e-5 + 2^-23 |oracle| on every valid slot of every
pixel (1e-5 absolute, widened by one float32 ulp of the value, because a float32 result
cannot be nearer than half an ulp to a float64 value above ~168). At flagged pixels each
GPU slot is compared with the oracle's value for the same face (zbuf also slot by slot).
Empty slots hold -1 in all four outputs.
alpha: |gpu - oracle| <= 1e-4 |oracle| + 1e-7.
grad_verts: |gpu - oracle| <= 1e-4 |oracle| + 1e-4 rms(oracle).

``compare_forward`` returns, besides counts, the oracle's outputs *reconciled* to the GPU's
choice of faces at flagged pixels (the GPU's face ids with the oracle's float64 values for
them), so that alpha and gradients are compared on every pixel and every vertex with no
mask.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

ABS = 1e-5
ULP = 2.0 ** -23
TIE = 1e-6            # depth-tie width of the target specification (E1)
E2_MAX = 1e-3         # candidacy-margin pixels (E2) allowed per compared pixel
MARGIN_W = 1e-6       # E2 margins, as the oracle flags them
MARGIN_BLUR = 1e-5
EXEMPT_MAX = E2_MAX   # point-radius margins (the analogue of E2 for point clouds)


def np_(t):
    return t.detach().cpu().numpy() if hasattr(t, "detach") else np.asarray(t)


@dataclass
class Scene:
    """The arguments of one forward call, so the comparator can ask the oracle for more
    candidates at flagged pixels and evaluate single (pixel, face) pairs."""
    oracle: object
    verts: np.ndarray
    faces: np.ndarray
    first: object
    num: object
    H: int
    W: int
    blur: float
    K: int
    persp: bool
    pixels: np.ndarray | None = None     # flat ids (n*H + i)*W + j of the compared rows

    def fwd(self, K=None, pixels=None, exempt=True):
        return self.oracle.rasterize_fwd(self.verts, self.faces, self.first, self.num, self.H, self.W,
                                         np.float32(self.blur), K or self.K, self.persp,
                                         pixels=self.pixels if pixels is None else pixels, exempt=exempt)

    def row_ids(self, nrows):
        return np.arange(nrows) if self.pixels is None else np.asarray(self.pixels, np.int64)

    def probe(self, pid, f):
        """The oracle's steps 2-9 for pixel ``pid`` and face ``f``."""
        rem = int(pid) % (self.H * self.W)
        i, j = rem // self.W, rem % self.W
        px, py = -1.0 + (2 * j + 1) / self.W, 1.0 - (2 * i + 1) / self.H
        abc = np.asarray(self.verts, np.float32)[np.asarray(self.faces)[f]].astype(np.float64)
        return self.oracle.probe(px, py, abc, self.persp)

    def marginal(self, pid, f):
        """A face whose candidacy at this pixel rounding decides (the oracle's E2 margins)."""
        r = self.probe(pid, f)
        if r["degenerate"] or r["z"] < 0:
            return False
        blur = float(np.float32(self.blur))
        if blur > 0:
            return (not r["inside"]) and abs(r["d2"] - blur) < MARGIN_BLUR * blur
        return -MARGIN_W < min(r["w"]) < MARGIN_W

    def mesh_of(self, pid):
        n = int(pid) // (self.H * self.W)
        f0 = int(np.asarray(self.first)[n])
        return f0, f0 + int(np.asarray(self.num)[n])


def _tol(o):
    return ABS + ULP * np.abs(o)


def _close(g, o):
    return bool(np.all(np.abs(np.asarray(g, np.float64) - o) <= _tol(o)))


def _groups(z, valid):
    """Label of the depth-tie group of each entry of a sorted candidate list."""
    lab = np.zeros(len(z), np.int64)
    for k in range(1, len(z)):
        lab[k] = lab[k - 1] + (not (valid[k] and valid[k - 1] and z[k] - z[k - 1] < TIE))
    return lab


def _requery(scene, ids, K):
    """The oracle's sorted candidates at ``ids``, enough of them that the tie group holding
    slot K-1 ends inside the list."""
    K2 = K + 1
    while True:
        q = scene.fwd(K=K2, pixels=ids, exempt=False)
        open_end = False
        for r in range(len(ids)):
            p, z = q[0][r], q[1][r]
            if p[-1] >= 0:
                lab = _groups(z, p >= 0)
                open_end |= lab[-1] == lab[K - 1]
        if not open_end:
            return q
        assert K2 < 512, "a depth-tie group longer than 512 candidates"
        K2 *= 2


def _check_e1_row(label, row, pid, k_gpu, q, rec):
    """pix_to_face up to permutation inside depth-tie groups; values by face id."""
    pg, zg, bg, dg = k_gpu
    qp, qz, qb, qd = q
    K = pg.shape[0]
    lab = _groups(qz, qp >= 0)
    seen = set()
    for k in range(K):
        gid = int(pg[k])
        if qp[k] < 0:
            if gid != -1 or zg[k] != -1 or dg[k] != -1 or np.any(bg[k] != -1):
                raise AssertionError(f"{label}: pixel {pid} slot {k} should be empty, gpu {gid}")
            continue
        members = qp[lab == lab[k]]
        if gid not in members or gid in seen:
            raise AssertionError(f"{label}: pix_to_face at tie pixel {pid} slot {k}: gpu {pg.tolist()}, "
                                 f"oracle {qp.tolist()} z {qz.tolist()}")
        seen.add(gid)
        m = int(np.flatnonzero(qp == gid)[0])
        for name, g, o in (("zbuf", zg[k], qz[m]), ("zbuf (slot)", zg[k], qz[k]), ("dists", dg[k], qd[m]),
                           ("bary", bg[k], qb[m])):
            if not _close(g, o):
                raise AssertionError(f"{label}: {name} at tie pixel {pid} slot {k} face {gid}: gpu {g} oracle {o}")
        rec[0][row, k], rec[1][row, k], rec[2][row, k], rec[3][row, k] = gid, qz[m], qb[m], qd[m]


def _check_e2_row(label, row, pid, k_gpu, scene, rec):
    """Faces that are not marginal: the oracle's, in order up to depth ties, as many as the
    slots the marginal ones leave. Every GPU slot's values: the oracle's for that face. Valid
    slots first, sorted by depth, faces of the pixel's own mesh."""
    pg, zg, bg, dg = k_gpu
    K = pg.shape[0]
    valid = pg >= 0
    if np.any(valid[1:] & ~valid[:-1]):
        raise AssertionError(f"{label}: empty slot before a valid one at pixel {pid}: {pg.tolist()}")
    f0, f1 = scene.mesh_of(pid)
    ids = [int(x) for x in pg[valid]]
    if len(set(ids)) != len(ids) or any(not (f0 <= x < f1) for x in ids):
        raise AssertionError(f"{label}: invalid face list at pixel {pid}: {pg.tolist()}")
    zs = []
    for k, gid in enumerate(ids):
        r = scene.probe(pid, gid)
        for name, g, o in (("zbuf", zg[k], r["z"]), ("dists", dg[k], r["dist"]), ("bary", bg[k], r["bary"])):
            if not _close(g, o):
                raise AssertionError(f"{label}: {name} at margin pixel {pid} slot {k} face {gid}: gpu {g} oracle {o}")
        rec[0][row, k], rec[1][row, k], rec[2][row, k], rec[3][row, k] = gid, r["z"], r["bary"], r["dist"]
        zs.append(r["z"])
    for k in range(len(ids), K):
        rec[0][row, k], rec[1][row, k], rec[2][row, k], rec[3][row, k] = -1, -1.0, -1.0, -1.0
    if np.any(np.diff(zs) < -TIE):
        raise AssertionError(f"{label}: slots not sorted by depth at margin pixel {pid}: {zs}")
    empty = ~valid
    if np.any(zg[empty] != -1) or np.any(dg[empty] != -1) or np.any(bg[empty] != -1):
        raise AssertionError(f"{label}: empty slots not -1 at margin pixel {pid}")
    # the oracle's sorted list, long enough to hold K faces that are not marginal
    K2 = K + 8
    while True:
        q = scene.fwd(K=K2, pixels=np.array([pid]), exempt=False)
        qp, qz = q[0][0], q[1][0]
        keep_q = [m for m in range(K2) if qp[m] >= 0 and not scene.marginal(pid, int(qp[m]))]
        if qp[-1] < 0 or len(keep_q) > K:
            break
        K2 *= 2
    lab = _groups(qz, qp >= 0)
    keep_g = [x for x in ids if not scene.marginal(pid, x)]
    want = min(len(keep_q), K - (len(ids) - len(keep_g)))
    if len(keep_g) != want:
        raise AssertionError(f"{label}: {len(keep_g)} non-marginal faces at margin pixel {pid}, oracle gives {want}: "
                             f"gpu {pg.tolist()} oracle {qp.tolist()}")
    for k, gid in enumerate(keep_g):
        m = keep_q[k]
        if gid not in {int(qp[x]) for x in keep_q if lab[x] == lab[m]}:
            raise AssertionError(f"{label}: non-marginal face order at margin pixel {pid}: gpu {pg.tolist()} "
                                 f"oracle {qp.tolist()}")


def compare_forward(gpu, ora, label="", scene=None, e2_max=E2_MAX):
    """gpu: (p2f, zbuf, bary, dists) tensors/arrays; ora: the oracle's tuple incl. flags.

    Returns a dict with the flagged fractions, the valid-slot count and ``rec``: the oracle's
    (p2f, zbuf, bary, dists) reconciled to the GPU's choice of faces at flagged pixels."""
    pg, zg, bg, dg = (np_(x) for x in gpu)
    po, zo, bo, do, ex = ora
    K = po.shape[-1]
    shape = po.shape
    pg, zg, dg = pg.reshape(-1, K), zg.reshape(-1, K), dg.reshape(-1, K)
    bg = bg.reshape(-1, K, 3)
    rec = [po.reshape(-1, K).copy(), np.asarray(zo, np.float64).reshape(-1, K).copy(),
           np.asarray(bo, np.float64).reshape(-1, K, 3).copy(), np.asarray(do, np.float64).reshape(-1, K).copy()]
    po_, zo_, bo_, do_ = rec[0].copy(), rec[1].copy(), rec[2].copy(), rec[3].copy()
    ex = np.asarray(ex).reshape(-1)
    e1, e2 = (ex & 1) > 0, (ex & 2) > 0
    assert e2.mean() <= e2_max, f"{label}: candidacy-margin pixels {e2.mean():.4%} of {ex.size}"
    plain = ~e1 & ~e2

    bad = (pg != po_).any(-1) & plain
    if bad.any():
        idx = np.flatnonzero(bad)[:5]
        det = [(int(i), pg[i].tolist(), po_[i].tolist(), zo_[i].tolist()) for i in idx]
        raise AssertionError(f"{label}: pix_to_face differs at {int(bad.sum())} unflagged pixels: {det}")
    valid = (po_ >= 0) & plain[:, None]
    empty = (po_ < 0) & plain[:, None]
    for name, g, o in (("zbuf", zg, zo_), ("dists", dg, do_), ("bary", bg, bo_)):
        err = np.abs(g[valid] - o[valid]) - _tol(o[valid])
        assert err.size == 0 or err.max() <= 0, f"{label}: {name} off by {err.max() + ABS:.3g}"
        assert np.all(g[empty] == -1), f"{label}: {name} empty slots not -1"

    rows1, rows2 = np.flatnonzero(e1 & ~e2), np.flatnonzero(e2)
    if (rows1.size or rows2.size) and scene is None:
        raise AssertionError(f"{label}: flagged pixels need the scene to re-ask the oracle")
    if rows1.size or rows2.size:
        ids = scene.row_ids(len(ex))
        if rows1.size:
            q = _requery(scene, ids[rows1], K)
            for t, row in enumerate(rows1):
                _check_e1_row(label, row, ids[row], (pg[row], zg[row], bg[row], dg[row]),
                              (q[0][t], q[1][t], q[2][t], q[3][t]), rec)
        for row in rows2:
            _check_e2_row(label, row, ids[row], (pg[row], zg[row], bg[row], dg[row]), scene, rec)
    rec = (rec[0].reshape(shape), rec[1].reshape(shape), rec[2].reshape(shape + (3,)), rec[3].reshape(shape))
    return dict(e1=float(e1.mean()), e2=float(e2.mean()), valid_slots=int((pg >= 0).sum()), rec=rec)


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
