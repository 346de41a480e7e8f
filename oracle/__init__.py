"""float64 CPU oracle of the mesh rasterizer hot path (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import this package.  The product path never does.

The arithmetic lives in ``oracle.c`` (plain C, float64, no SIMD, no fast-math); this
module compiles it with gcc when needed and marshals numpy arrays through ctypes.
Each function names the step of the definition (see the header of ``oracle.c``) it
follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc -O2, strict IEEE: no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                               "-shared", "-fPIC", "-pthread", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i64, i32, f64 = ctypes.c_int64, ctypes.c_int32, ctypes.c_double
        lib.oracle_rasterize_fwd.argtypes = [P, i64, P, i64, P, P, i32, i32, i32, f64, i32, i32,
                                             P, i64, P, P, P, P, P, i32]
        lib.oracle_rasterize_fwd.restype = ctypes.c_int
        lib.oracle_silhouette_fwd.argtypes = [P, P, i64, i32, f64, P]
        lib.oracle_silhouette_fwd.restype = None
        lib.oracle_silhouette_bwd.argtypes = [P, P, P, i64, i32, f64, P]
        lib.oracle_silhouette_bwd.restype = None
        lib.oracle_rasterize_bwd.argtypes = [P, i64, P, i64, P, i32, i32, i32, i32, i32, P, P, P, P, i32]
        lib.oracle_rasterize_bwd.restype = ctypes.c_int
        lib.oracle_probe.argtypes = [f64, f64, P, i32, P]
        lib.oracle_probe.restype = None
        lib.oracle_interpolate_fwd.argtypes = [P, P, i64, i32, P, P, i32, P]
        lib.oracle_interpolate_fwd.restype = None
        lib.oracle_interpolate_bwd.argtypes = [P, P, i64, i32, P, P, i64, i32, P, P, P]
        lib.oracle_interpolate_bwd.restype = None
        lib.oracle_blend_fwd.argtypes = [P, P, P, P, i64, i32, i32, P, f64, f64, f64, f64, P]
        lib.oracle_blend_fwd.restype = None
        lib.oracle_blend_bwd.argtypes = [P, P, P, P, i64, i32, i32, P, f64, f64, f64, f64, P, P, P, P]
        lib.oracle_blend_bwd.restype = None
        lib.oracle_phong_fwd.argtypes = [P, P, P, i64, P, P, P]
        lib.oracle_phong_fwd.restype = None
        lib.oracle_phong_bwd.argtypes = [P, P, P, i64, P, P, P, P, P]
        lib.oracle_phong_bwd.restype = None
        lib.oracle_phong_shade_fwd.argtypes = [P, P, i64, i32, P, P, P, P, P, P, P]
        lib.oracle_phong_shade_fwd.restype = None
        lib.oracle_phong_shade_bwd.argtypes = [P, P, i64, i32, P, P, P, P, i64, P, P, P, P, P, P]
        lib.oracle_phong_shade_bwd.restype = None
        lib.oracle_rasterize_points.argtypes = [P, i64, P, P, i32, i32, i32, f64, i32, P, P, P, P]
        lib.oracle_rasterize_points.restype = ctypes.c_int
        lib.oracle_rasterize_points_pixels.argtypes = [P, i64, P, P, i32, i32, i32, f64, i32, P, i64, P, P, P, P]
        lib.oracle_rasterize_points_pixels.restype = ctypes.c_int
        lib.oracle_rasterize_points_bwd.argtypes = [P, i64, P, i32, i32, i32, i32, P, P, P]
        lib.oracle_rasterize_points_bwd.restype = None
        lib.oracle_composite_points.argtypes = [P, P, i64, i32, P, i32, f64, i32, P]
        lib.oracle_composite_points.restype = None
        lib.oracle_composite_points_bwd.argtypes = [P, P, i64, i32, P, i64, i32, f64, i32, P, P, P]
        lib.oracle_composite_points_bwd.restype = None
        lib.oracle_knn.argtypes = [P, P, P, P, P, P, i32, i32, i32, P, P, P]
        lib.oracle_knn.restype = ctypes.c_int
        lib.oracle_knn_bwd.argtypes = [P, i64, P, i64, i32, i32, P, P, P, P]
        lib.oracle_knn_bwd.restype = None
        _lib = lib
    return _lib


def default_threads() -> int:
    return len(os.sched_getaffinity(0))


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a):
    return None if a is None else a.ctypes.data


def rasterize_fwd(verts, faces, first, num, H, W, blur_radius, K, perspective_correct=False,
                  pixels=None, nthreads=None, exempt=True):
    """Steps 1-10: per pixel the K nearest candidate faces.

    Returns ``(pix_to_face int64, zbuf f64, bary f64, dists f64, exempt uint8)`` shaped
    ``(N, H, W, K[, 3])``, or ``(P, K[, 3])`` when ``pixels`` lists flat pixel ids
    ``(n*H + i)*W + j``.  ``exempt`` bit 0 = depth near-tie (E1), bit 1 = candidacy on
    its threshold (E2).
    """
    lib = _load()
    verts = _c(verts, np.float32)
    faces = _c(faces, np.int64)
    first = _c(first, np.int64)
    num = _c(num, np.int64)
    N = int(first.shape[0])
    if pixels is None:
        lead = (N, H, W)
        pix = None
        npix = N * H * W
    else:
        pix = _c(pixels, np.int64)
        lead = (pix.shape[0],)
        npix = pix.shape[0]
    p2f = np.empty(lead + (K,), np.int64)
    zbuf = np.empty(lead + (K,), np.float64)
    bary = np.empty(lead + (K, 3), np.float64)
    dists = np.empty(lead + (K,), np.float64)
    ex = np.zeros(lead, np.uint8) if exempt else None
    rc = lib.oracle_rasterize_fwd(_ptr(verts), verts.shape[0], _ptr(faces), faces.shape[0],
                                  _ptr(first), _ptr(num), N, H, W, float(blur_radius), K,
                                  int(bool(perspective_correct)), _ptr(pix), npix,
                                  _ptr(p2f), _ptr(zbuf), _ptr(bary), _ptr(dists), _ptr(ex),
                                  nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_rasterize_fwd: invalid arguments")
    return p2f, zbuf, bary, dists, ex


def silhouette_fwd(pix_to_face, dists, sigma):
    """Step 11: alpha = 1 - prod(1 - sigmoid(-dist / sigma)) over valid slots."""
    lib = _load()
    p2f = _c(pix_to_face, np.int64)
    d = _c(dists, np.float64)
    K = p2f.shape[-1]
    alpha = np.empty(p2f.shape[:-1], np.float64)
    lib.oracle_silhouette_fwd(_ptr(p2f), _ptr(d), alpha.size, K, float(sigma), _ptr(alpha))
    return alpha


def silhouette_bwd(grad_alpha, pix_to_face, dists, sigma):
    """Step 12: dL/ddists from dL/dalpha."""
    lib = _load()
    p2f = _c(pix_to_face, np.int64)
    d = _c(dists, np.float64)
    g = _c(grad_alpha, np.float64)
    K = p2f.shape[-1]
    out = np.empty(p2f.shape, np.float64)
    lib.oracle_silhouette_bwd(_ptr(g), _ptr(p2f), _ptr(d), g.size, K, float(sigma), _ptr(out))
    return out


def rasterize_bwd(verts, faces, pix_to_face, perspective_correct=False, grad_zbuf=None,
                  grad_bary=None, grad_dists=None, nthreads=None):
    """Step 13: dL/dverts (V x 3, float64) from gradients of zbuf / bary / dists (any may be None).

    Each thread keeps a private V x 3 float64 accumulator, so the default caps threads at 16."""
    lib = _load()
    verts = _c(verts, np.float32)
    faces = _c(faces, np.int64)
    p2f = _c(pix_to_face, np.int64)
    N, H, W, K = p2f.shape
    gz = None if grad_zbuf is None else _c(grad_zbuf, np.float64)
    gb = None if grad_bary is None else _c(grad_bary, np.float64)
    gd = None if grad_dists is None else _c(grad_dists, np.float64)
    out = np.empty(verts.shape, np.float64)
    rc = lib.oracle_rasterize_bwd(_ptr(verts), verts.shape[0], _ptr(faces), faces.shape[0], _ptr(p2f),
                                  N, H, W, K, int(bool(perspective_correct)), _ptr(gz), _ptr(gb), _ptr(gd),
                                  _ptr(out), nthreads or min(default_threads(), 16))
    if rc != 0:
        raise ValueError("oracle_rasterize_bwd: invalid arguments")
    return out


def probe(px, py, abc, perspective_correct=False):
    """Steps 2-9 for one pixel centre and one face; returns a dict of every intermediate."""
    lib = _load()
    v = _c(abc, np.float64).reshape(9)
    out = np.empty(13, np.float64)
    lib.oracle_probe(float(px), float(py), _ptr(v), int(bool(perspective_correct)), _ptr(out))
    return dict(degenerate=bool(out[0]), inside=bool(out[1]), edge=int(out[2]), t=out[3], d2=out[4],
                w=out[5:8].copy(), bary=out[8:11].copy(), z=out[11], dist=out[12])


def interpolate_fwd(pix_to_face, bary, faces, attr):
    """Step 14: per-slot attributes sum_m bary_m attr[v_m]; shape p2f.shape + (D,)."""
    lib = _load()
    p2f = _c(pix_to_face, np.int64)
    b = _c(bary, np.float64)
    f = _c(faces, np.int64)
    a = _c(attr, np.float64)
    K, D = p2f.shape[-1], a.shape[1]
    npix = p2f.size // K
    out = np.empty(p2f.shape + (D,), np.float64)
    lib.oracle_interpolate_fwd(_ptr(p2f), _ptr(b), npix, K, _ptr(f), _ptr(a), D, _ptr(out))
    return out


def interpolate_bwd(pix_to_face, bary, faces, attr, grad_out):
    """Step 15: (grad_attr V x D, grad_bary like bary)."""
    lib = _load()
    p2f = _c(pix_to_face, np.int64)
    b = _c(bary, np.float64)
    f = _c(faces, np.int64)
    a = _c(attr, np.float64)
    g = _c(grad_out, np.float64)
    K, D = p2f.shape[-1], a.shape[1]
    npix = p2f.size // K
    ga = np.empty(a.shape, np.float64)
    gb = np.empty(b.shape, np.float64)
    lib.oracle_interpolate_bwd(_ptr(p2f), _ptr(b), npix, K, _ptr(f), _ptr(a), a.shape[0], D, _ptr(g), _ptr(ga),
                               _ptr(gb))
    return ga, gb


def blend_fwd(pix_to_face, colors, dists, zbuf, background, sigma, gamma, znear, zfar):
    """Step 16: soft RGB blend -> (..., D + 1) colour channels then alpha."""
    lib = _load()
    p2f = _c(pix_to_face, np.int64)
    c = _c(colors, np.float64)
    d = _c(dists, np.float64)
    z = _c(zbuf, np.float64)
    bg = _c(background, np.float64)
    K, D = p2f.shape[-1], c.shape[-1]
    npix = p2f.size // K
    out = np.empty(p2f.shape[:-1] + (D + 1,), np.float64)
    lib.oracle_blend_fwd(_ptr(p2f), _ptr(c), _ptr(d), _ptr(z), npix, K, D, _ptr(bg), float(sigma), float(gamma),
                         float(znear), float(zfar), _ptr(out))
    return out


def blend_bwd(pix_to_face, colors, dists, zbuf, background, sigma, gamma, znear, zfar, grad_rgba):
    """Step 17: (grad_colors, grad_dists, grad_zbuf)."""
    lib = _load()
    p2f = _c(pix_to_face, np.int64)
    c = _c(colors, np.float64)
    d = _c(dists, np.float64)
    z = _c(zbuf, np.float64)
    bg = _c(background, np.float64)
    g = _c(grad_rgba, np.float64)
    K, D = p2f.shape[-1], c.shape[-1]
    npix = p2f.size // K
    gc = np.empty(c.shape, np.float64)
    gd = np.empty(d.shape, np.float64)
    gz = np.empty(z.shape, np.float64)
    lib.oracle_blend_bwd(_ptr(p2f), _ptr(c), _ptr(d), _ptr(z), npix, K, D, _ptr(bg), float(sigma), float(gamma),
                         float(znear), float(zfar), _ptr(g), _ptr(gc), _ptr(gd), _ptr(gz))
    return gc, gd, gz


PHONG_PARAMS = ("light_location", "camera_position", "ambient", "diffuse", "specular", "shininess")


def phong_params(light_location, camera_position, ambient, diffuse, specular, shininess):
    """The 16 lighting numbers of steps 18-21: L, C, ambient, diffuse, specular colours, shininess."""
    return np.concatenate([np.asarray(x, np.float64).reshape(-1) for x in
                           (light_location, camera_position, ambient, diffuse, specular, [shininess])])


def phong_fwd(points, normals, albedo, params):
    """Step 18 at M points: (colours M x 3, flags M: |cos| < 1e-6)."""
    lib = _load()
    P, N, c = (_c(x, np.float64).reshape(-1, 3) for x in (points, normals, albedo))
    prm = _c(params, np.float64)
    out = np.empty(P.shape, np.float64)
    flags = np.empty(P.shape[0], np.uint8)
    lib.oracle_phong_fwd(_ptr(P), _ptr(N), _ptr(c), P.shape[0], _ptr(prm), _ptr(out), _ptr(flags))
    return out, flags.astype(bool)


def phong_bwd(points, normals, albedo, params, grad):
    """Step 19: (grad_points, grad_normals, grad_albedo), each M x 3."""
    lib = _load()
    P, N, c, g = (_c(x, np.float64).reshape(-1, 3) for x in (points, normals, albedo, grad))
    prm = _c(params, np.float64)
    gP, gN, gc = (np.empty(P.shape, np.float64) for _ in range(3))
    lib.oracle_phong_bwd(_ptr(P), _ptr(N), _ptr(c), P.shape[0], _ptr(prm), _ptr(g), _ptr(gP), _ptr(gN), _ptr(gc))
    return gP, gN, gc


def phong_shade_fwd(pix_to_face, bary, faces, points, normals, albedo, params):
    """Step 20: per-slot Phong colours (p2f.shape + (3,)) and flags (p2f.shape)."""
    lib = _load()
    p2f = _c(pix_to_face, np.int64)
    b = _c(bary, np.float64)
    f = _c(faces, np.int64)
    P, N, c = (_c(x, np.float64).reshape(-1, 3) for x in (points, normals, albedo))
    prm = _c(params, np.float64)
    K = p2f.shape[-1]
    npix = p2f.size // K
    out = np.empty(p2f.shape + (3,), np.float64)
    flags = np.empty(p2f.shape, np.uint8)
    lib.oracle_phong_shade_fwd(_ptr(p2f), _ptr(b), npix, K, _ptr(f), _ptr(P), _ptr(N), _ptr(c), _ptr(prm),
                               _ptr(out), _ptr(flags))
    return out, flags.astype(bool)


def phong_shade_bwd(pix_to_face, bary, faces, points, normals, albedo, params, grad):
    """Step 21: (grad_points, grad_normals, grad_albedo) per vertex and grad_bary."""
    lib = _load()
    p2f = _c(pix_to_face, np.int64)
    b = _c(bary, np.float64)
    f = _c(faces, np.int64)
    P, N, c = (_c(x, np.float64).reshape(-1, 3) for x in (points, normals, albedo))
    prm = _c(params, np.float64)
    g = _c(grad, np.float64)
    K = p2f.shape[-1]
    npix = p2f.size // K
    gP, gN, gc = (np.empty(P.shape, np.float64) for _ in range(3))
    gb = np.empty(b.shape, np.float64)
    lib.oracle_phong_shade_bwd(_ptr(p2f), _ptr(b), npix, K, _ptr(f), _ptr(P), _ptr(N), _ptr(c), P.shape[0],
                               _ptr(prm), _ptr(g), _ptr(gP), _ptr(gN), _ptr(gc), _ptr(gb))
    return gP, gN, gc, gb


def rasterize_points(points, cloud_first_idx, num_points_per_cloud, H, W, radius, K, pixels=None):
    """Step 22: (idx, zbuf, dists) of shape (N, H, W, K) and flags (N, H, W); with ``pixels``
    (ids n*H*W + i*W + j) only those, as (npix, K) and (npix,)."""
    lib = _load()
    pts = _c(points, np.float32)
    first = _c(cloud_first_idx, np.int64)
    num = _c(num_points_per_cloud, np.int64)
    N = first.shape[0]
    if pixels is not None:
        pix = _c(pixels, np.int64)
        n = pix.shape[0]
        idx = np.empty((n, K), np.int64)
        zbuf = np.empty((n, K), np.float64)
        dists = np.empty((n, K), np.float64)
        flags = np.empty(n, np.uint8)
        rc = lib.oracle_rasterize_points_pixels(_ptr(pts), pts.shape[0], _ptr(first), _ptr(num), N, H, W,
                                                float(radius), K, _ptr(pix), n, _ptr(idx), _ptr(zbuf), _ptr(dists),
                                                _ptr(flags))
        if rc != 0:
            raise ValueError("oracle_rasterize_points_pixels: invalid arguments")
        return idx, zbuf, dists, flags.astype(bool)
    idx = np.empty((N, H, W, K), np.int64)
    zbuf = np.empty((N, H, W, K), np.float64)
    dists = np.empty((N, H, W, K), np.float64)
    flags = np.empty((N, H, W), np.uint8)
    rc = lib.oracle_rasterize_points(_ptr(pts), pts.shape[0], _ptr(first), _ptr(num), N, H, W, float(radius), K,
                                     _ptr(idx), _ptr(zbuf), _ptr(dists), _ptr(flags))
    if rc != 0:
        raise ValueError("oracle_rasterize_points: invalid arguments")
    return idx, zbuf, dists, flags.astype(bool)


def rasterize_points_bwd(points, idx, grad_zbuf=None, grad_dists=None):
    """Step 23: grad_points (P, 3)."""
    lib = _load()
    pts = _c(points, np.float32)
    ix = _c(idx, np.int64)
    N, H, W, K = ix.shape
    gz = None if grad_zbuf is None else _c(grad_zbuf, np.float64)
    gd = None if grad_dists is None else _c(grad_dists, np.float64)
    out = np.empty((pts.shape[0], 3), np.float64)
    lib.oracle_rasterize_points_bwd(_ptr(pts), pts.shape[0], _ptr(ix), N, H, W, K, _ptr(gz), _ptr(gd), _ptr(out))
    return out


COMPOSITE_MODES = {"alpha": 0, "norm_weighted": 1}


def composite_points(idx, dists, features, radius, mode="alpha"):
    """Steps 24-25: composited features, idx.shape[:-1] + (C,)."""
    lib = _load()
    ix = _c(idx, np.int64)
    d = _c(dists, np.float64)
    f = _c(features, np.float64)
    K, C = ix.shape[-1], f.shape[1]
    npix = ix.size // K
    out = np.empty(ix.shape[:-1] + (C,), np.float64)
    lib.oracle_composite_points(_ptr(ix), _ptr(d), npix, K, _ptr(f), C, float(radius), COMPOSITE_MODES[mode],
                                _ptr(out))
    return out


def composite_points_bwd(idx, dists, features, radius, grad_out, mode="alpha"):
    """Step 26: (grad_features (P, C), grad_dists like dists)."""
    lib = _load()
    ix = _c(idx, np.int64)
    d = _c(dists, np.float64)
    f = _c(features, np.float64)
    g = _c(grad_out, np.float64)
    K, C = ix.shape[-1], f.shape[1]
    npix = ix.size // K
    gf = np.empty(f.shape, np.float64)
    gd = np.empty(d.shape, np.float64)
    lib.oracle_composite_points_bwd(_ptr(ix), _ptr(d), npix, K, _ptr(f), f.shape[0], C, float(radius),
                                    COMPOSITE_MODES[mode], _ptr(g), _ptr(gf), _ptr(gd))
    return gf, gd


def knn(p1, first1, num1, p2, first2, num2, K):
    """Step 27: (idx (P1, K) global ids into p2, dists (P1, K), flags (P1,))."""
    lib = _load()
    a = _c(p1, np.float32)
    b = _c(p2, np.float32)
    f1, n1, f2, n2 = (_c(x, np.int64) for x in (first1, num1, first2, num2))
    D = a.shape[1]
    idx = np.empty((a.shape[0], K), np.int64)
    dists = np.empty((a.shape[0], K), np.float64)
    flags = np.zeros(a.shape[0], np.uint8)
    rc = lib.oracle_knn(_ptr(a), _ptr(f1), _ptr(n1), _ptr(b), _ptr(f2), _ptr(n2), f1.shape[0], D, K, _ptr(idx),
                        _ptr(dists), _ptr(flags))
    if rc != 0:
        raise ValueError("oracle_knn: invalid arguments")
    return idx, dists, flags.astype(bool)


def knn_bwd(p1, p2, idx, grad_dists):
    """Step 28: (grad_p1, grad_p2)."""
    lib = _load()
    a = _c(p1, np.float32)
    b = _c(p2, np.float32)
    ix = _c(idx, np.int64)
    g = _c(grad_dists, np.float64)
    D, K = a.shape[1], ix.shape[1]
    g1 = np.empty(a.shape, np.float64)
    g2 = np.empty(b.shape, np.float64)
    lib.oracle_knn_bwd(_ptr(a), a.shape[0], _ptr(b), b.shape[0], D, K, _ptr(ix), _ptr(g), _ptr(g1), _ptr(g2))
    return g1, g2
