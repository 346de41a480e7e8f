"""Thin Python binding of ``libmeshrast.so`` (the sm_100a mesh rasterizer C ABI).

Argument marshalling only: every function checks shapes, dtypes and devices of torch
tensors, allocates the outputs with torch, and passes raw device pointers plus the
current CUDA stream to the C entry point of the same name (``mr_*``).  All arithmetic
runs in the library's CUDA kernels; there is no CPU path.  The library is loaded from
this directory on first use and must have been built (``python -m
differentiable_mesh_rasterization_b200.build``); every entry point raises ImportError
without it.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmeshrast.so")

MR_KMAX = 32
ERRORS = {-1: "invalid argument", -2: "out of memory", -3: "CUDA error", -4: "device index error"}

# Entry points declared by include/meshrast.h (checked by the test-suite).
EXPORTS = ("mr_rasterize_fwd", "mr_rasterize_silhouette_fwd", "mr_silhouette_blend_fwd",
           "mr_silhouette_blend_bwd", "mr_rasterize_bwd", "mr_silhouette_rasterize_bwd",
           "mr_device_status", "mr_last_error", "mr_version", "mr_profile_enable", "mr_profile_read",
           "mr_rasterize_fwd_noalloc", "mr_interpolate_fwd", "mr_interpolate_bwd", "mr_blend_fwd", "mr_blend_bwd",
           "mr_phong_fwd", "mr_phong_bwd", "mr_phong_shade_fwd", "mr_phong_shade_bwd",
           "mr_rasterize_points_fwd", "mr_rasterize_points_bwd", "mr_composite_points_fwd",
           "mr_composite_points_bwd", "mr_knn_fwd", "mr_knn_bwd", "mr_measure_fp32_peak", "mr_knn_count_pairs",
           "mr_inject_fault", "mr_scratch_in_use", "mr_scratch_peak")
STAGES = ("face_setup", "bin_count", "bin_scan", "bin_fill", "fine", "silhouette_fwd", "silhouette_bwd",
          "raster_bwd", "silhouette_raster_bwd", "epilogue", "interpolate_fwd", "interpolate_bwd", "blend_fwd",
          "blend_bwd", "phong_fwd", "phong_bwd", "phong_shade_fwd", "phong_shade_bwd",
          "points_bin", "points_fine", "points_bwd", "composite_fwd", "composite_bwd", "knn", "knn_bwd")


class MeshRastError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn}: {ERRORS.get(code, code)} ({code}): {msg}")
        self.code = code


_lib = None


def load_library() -> ctypes.CDLL:
    """Load libmeshrast.so and declare its signatures (fails loudly if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m differentiable_mesh_rasterization_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float
    sig = {
        "mr_rasterize_fwd": [P, i64, P, i64, P, P, i32, i32, i32, f32, i32, i32, P, P, P, P, P],
        "mr_rasterize_fwd_noalloc": [P, i64, P, i64, P, P, i32, i32, i32, f32, i32, i32, P, P, P, P, P],
        "mr_rasterize_silhouette_fwd": [P, i64, P, i64, P, P, i32, i32, i32, f32, i32, i32, f32, P, P, P, P, P, P],
        "mr_silhouette_blend_fwd": [P, P, i32, i32, i32, i32, f32, P, P],
        "mr_silhouette_blend_bwd": [P, P, P, i32, i32, i32, i32, f32, P, P],
        "mr_rasterize_bwd": [P, i64, P, i64, P, i32, i32, i32, i32, i32, P, P, P, P, P],
        "mr_silhouette_rasterize_bwd": [P, i64, P, i64, P, P, i32, i32, i32, i32, f32, P, P, P],
        "mr_device_status": [P],
        "mr_last_error": [],
        "mr_version": [],
        "mr_interpolate_fwd": [P, P, i64, i32, P, i64, P, i64, i32, P, P],
        "mr_interpolate_bwd": [P, P, i64, i32, P, i64, P, i64, i32, P, P, P, P],
        "mr_blend_fwd": [P, P, P, P, i64, i32, i32, P, f32, f32, f32, f32, P, P],
        "mr_blend_bwd": [P, P, P, P, i64, i32, i32, P, f32, f32, f32, f32, P, P, P, P, P],
        "mr_phong_fwd": [P, P, P, i64, P, P, P],
        "mr_phong_bwd": [P, P, P, i64, P, P, P, P, P, P],
        "mr_phong_shade_fwd": [P, P, i64, i32, P, i64, P, P, P, i64, P, P, P],
        "mr_phong_shade_bwd": [P, P, i64, i32, P, i64, P, P, P, i64, P, P, P, P, P, P, P],
        "mr_rasterize_points_fwd": [P, i64, P, P, i32, i32, i32, f32, i32, P, P, P, P],
        "mr_rasterize_points_bwd": [P, i64, P, i32, i32, i32, i32, P, P, P, P],
        "mr_composite_points_fwd": [P, P, i64, i32, P, i64, i32, f32, i32, P, P],
        "mr_composite_points_bwd": [P, P, i64, i32, P, i64, i32, f32, i32, P, P, P, P],
        "mr_knn_fwd": [P, i64, P, P, P, i64, P, P, i32, i32, i32, P, P, P],
        "mr_knn_bwd": [P, i64, P, i64, i32, i32, P, P, P, P, P],
        "mr_knn_count_pairs": [P, i64, P, P, P, i64, P, P, i32, i32, i32, P, P, P, P],
        "mr_measure_fp32_peak": [P, P],
        "mr_inject_fault": [i32, i32],
        "mr_scratch_in_use": [P],
        "mr_scratch_peak": [P, i32],
        "mr_profile_enable": [i32],
        "mr_profile_read": [P, P, i32],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    lib.mr_last_error.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _check(name: str, rc: int) -> None:
    if rc != 0:
        raise MeshRastError(name, rc, load_library().mr_last_error().decode())


def _stream(dev: torch.device) -> int:
    return torch.cuda.current_stream(dev).cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _dev(t: torch.Tensor, dtype, name: str) -> torch.Tensor:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t.contiguous()


class _Index:
    """A per-mesh (per-cloud) index array as the C ABI takes it: a 1-D int64 array in host
    memory (numpy, a list or a CPU tensor) or a CUDA tensor on the call's device, passed
    through as a device pointer (the library then reads it with one device-to-host copy on
    the call's stream)."""

    def __init__(self, a, name: str, device: torch.device):
        if isinstance(a, torch.Tensor) and a.is_cuda:
            if a.device != device:
                raise ValueError(f"{name} is on {a.device}, the call runs on {device}")
            a = a.detach().to(torch.int64).contiguous()
            self.ptr = a.data_ptr()
        else:
            if isinstance(a, torch.Tensor):
                a = a.detach().numpy()
            a = np.ascontiguousarray(a, dtype=np.int64)
            self.ptr = a.ctypes.data
        if a.ndim != 1:
            raise ValueError(f"{name} must be 1-D")
        self.keep = a
        self.n = int(a.shape[0])


def _mesh_inputs(verts, faces, mesh_to_face_first_idx, num_faces_per_mesh):
    """Checked arguments of the mesh forward: verts (V, 3) float32 and faces (F, 3) int64 on
    one CUDA device, two per-mesh index arrays of equal length.  Shapes and lengths are
    checked first: the library cannot see the extent of a buffer, so a (V, 2) verts or a
    short per-mesh array would make it read past the end of one."""
    for t, name in ((verts, "verts"), (faces, "faces")):
        if not isinstance(t, torch.Tensor) or t.ndim != 2 or t.shape[1] != 3:
            raise ValueError(f"{name} must be a tensor of shape (n, 3)")
    first = _Index(mesh_to_face_first_idx, "mesh_to_face_first_idx", verts.device)
    num = _Index(num_faces_per_mesh, "num_faces_per_mesh", verts.device)
    if first.n != num.n:
        raise ValueError("per-mesh arrays differ in length")
    verts = _dev(verts, torch.float32, "verts")
    faces = _dev(faces, torch.int64, "faces")
    if faces.device != verts.device:
        raise ValueError("verts and faces must be on the same device")
    return verts, faces, first, num


def rasterize_fwd(verts, faces, mesh_to_face_first_idx, num_faces_per_mesh, H, W, blur_radius, K,
                  perspective_correct=False, sigma=None):
    """Stage one (``mr_rasterize_fwd``); with ``sigma`` also the fused silhouette.

    verts (V, 3) float32 CUDA, faces (F, 3) int64 CUDA; the two per-mesh index arrays in
    host memory or as CUDA tensors.  Returns ``pix_to_face (N,H,W,K) int64, zbuf,
    bary (N,H,W,K,3), dists`` and, when ``sigma`` is given, ``alpha (N,H,W)``.
    """
    lib = load_library()
    verts, faces, first, num = _mesh_inputs(verts, faces, mesh_to_face_first_idx, num_faces_per_mesh)
    N = first.n
    dev = verts.device
    p2f = torch.empty((N, H, W, K), dtype=torch.int64, device=dev)
    zbuf = torch.empty((N, H, W, K), dtype=torch.float32, device=dev)
    bary = torch.empty((N, H, W, K, 3), dtype=torch.float32, device=dev)
    dists = torch.empty((N, H, W, K), dtype=torch.float32, device=dev)
    args = (_ptr(verts), verts.shape[0], _ptr(faces), faces.shape[0], first.ptr, num.ptr,
            N, H, W, float(blur_radius), K, int(bool(perspective_correct)))
    with torch.cuda.device(dev):
        if sigma is None:
            _check("mr_rasterize_fwd", lib.mr_rasterize_fwd(*args, _ptr(p2f), _ptr(zbuf), _ptr(bary), _ptr(dists),
                                                            _stream(dev)))
            return p2f, zbuf, bary, dists
        alpha = torch.empty((N, H, W), dtype=torch.float32, device=dev)
        _check("mr_rasterize_silhouette_fwd",
               lib.mr_rasterize_silhouette_fwd(*args, float(sigma), _ptr(p2f), _ptr(zbuf), _ptr(bary), _ptr(dists),
                                               _ptr(alpha), _stream(dev)))
        return p2f, zbuf, bary, dists, alpha


def rasterize_fwd_noalloc(verts, faces, mesh_to_face_first_idx, num_faces_per_mesh, H, W, blur_radius, K,
                          perspective_correct=False):
    """``mr_rasterize_fwd_noalloc``: stage one with the library's fixed scratch array, for
    callers that must not allocate device memory (the outputs here are still allocated by
    torch).  Same outputs as :func:`rasterize_fwd`; batches too large for the array raise.
    """
    lib = load_library()
    verts, faces, first, num = _mesh_inputs(verts, faces, mesh_to_face_first_idx, num_faces_per_mesh)
    N = first.n
    dev = verts.device
    p2f = torch.empty((N, H, W, K), dtype=torch.int64, device=dev)
    zbuf = torch.empty((N, H, W, K), dtype=torch.float32, device=dev)
    bary = torch.empty((N, H, W, K, 3), dtype=torch.float32, device=dev)
    dists = torch.empty((N, H, W, K), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _check("mr_rasterize_fwd_noalloc",
               lib.mr_rasterize_fwd_noalloc(_ptr(verts), verts.shape[0], _ptr(faces), faces.shape[0],
                                            first.ptr, num.ptr, N, H, W, float(blur_radius), K,
                                            int(bool(perspective_correct)), _ptr(p2f), _ptr(zbuf), _ptr(bary),
                                            _ptr(dists), _stream(dev)))
    return p2f, zbuf, bary, dists


def _nhwk(p2f: torch.Tensor):
    if p2f.ndim != 4:
        raise ValueError("pix_to_face must be (N, H, W, K)")
    return tuple(int(x) for x in p2f.shape)


def silhouette_blend_fwd(pix_to_face, dists, sigma):
    """Soft silhouette (``mr_silhouette_blend_fwd``) -> alpha (N, H, W)."""
    lib = load_library()
    p2f = _dev(pix_to_face, torch.int64, "pix_to_face")
    d = _dev(dists, torch.float32, "dists")
    N, H, W, K = _nhwk(p2f)
    if d.shape != p2f.shape:
        raise ValueError("dists must match pix_to_face")
    alpha = torch.empty((N, H, W), dtype=torch.float32, device=p2f.device)
    with torch.cuda.device(p2f.device):
        _check("mr_silhouette_blend_fwd", lib.mr_silhouette_blend_fwd(_ptr(p2f), _ptr(d), N, H, W, K, float(sigma),
                                                                      _ptr(alpha), _stream(p2f.device)))
    return alpha


def silhouette_blend_bwd(grad_alpha, pix_to_face, dists, sigma):
    """Gradient of the soft silhouette (``mr_silhouette_blend_bwd``) -> grad_dists (N, H, W, K)."""
    lib = load_library()
    p2f = _dev(pix_to_face, torch.int64, "pix_to_face")
    d = _dev(dists, torch.float32, "dists")
    g = _dev(grad_alpha, torch.float32, "grad_alpha")
    N, H, W, K = _nhwk(p2f)
    if d.shape != p2f.shape or g.shape != (N, H, W):
        raise ValueError("shape mismatch")
    out = torch.empty_like(d)
    with torch.cuda.device(p2f.device):
        _check("mr_silhouette_blend_bwd", lib.mr_silhouette_blend_bwd(_ptr(g), _ptr(p2f), _ptr(d), N, H, W, K,
                                                                      float(sigma), _ptr(out), _stream(p2f.device)))
    return out


def rasterize_bwd(verts, faces, pix_to_face, perspective_correct=False, grad_zbuf=None, grad_bary=None,
                  grad_dists=None):
    """Backward of stage one (``mr_rasterize_bwd``) -> grad_verts (V, 3) float32."""
    lib = load_library()
    verts = _dev(verts, torch.float32, "verts")
    faces = _dev(faces, torch.int64, "faces")
    p2f = _dev(pix_to_face, torch.int64, "pix_to_face")
    N, H, W, K = _nhwk(p2f)
    gz = None if grad_zbuf is None else _dev(grad_zbuf, torch.float32, "grad_zbuf")
    gb = None if grad_bary is None else _dev(grad_bary, torch.float32, "grad_bary")
    gd = None if grad_dists is None else _dev(grad_dists, torch.float32, "grad_dists")
    for t, shp in ((gz, (N, H, W, K)), (gb, (N, H, W, K, 3)), (gd, (N, H, W, K))):
        if t is not None and tuple(t.shape) != shp:
            raise ValueError(f"gradient shape {tuple(t.shape)} != {shp}")
    out = torch.empty_like(verts)
    with torch.cuda.device(verts.device):
        _check("mr_rasterize_bwd", lib.mr_rasterize_bwd(_ptr(verts), verts.shape[0], _ptr(faces), faces.shape[0],
                                                        _ptr(p2f), N, H, W, K, int(bool(perspective_correct)),
                                                        _ptr(gz), _ptr(gb), _ptr(gd), _ptr(out),
                                                        _stream(verts.device)))
    return out


def silhouette_rasterize_bwd(verts, faces, pix_to_face, dists, sigma, grad_alpha):
    """Fused silhouette + distance backward (``mr_silhouette_rasterize_bwd``) -> grad_verts (V, 3)."""
    lib = load_library()
    verts = _dev(verts, torch.float32, "verts")
    faces = _dev(faces, torch.int64, "faces")
    p2f = _dev(pix_to_face, torch.int64, "pix_to_face")
    d = _dev(dists, torch.float32, "dists")
    g = _dev(grad_alpha, torch.float32, "grad_alpha")
    N, H, W, K = _nhwk(p2f)
    if d.shape != p2f.shape or g.shape != (N, H, W):
        raise ValueError("shape mismatch")
    out = torch.empty_like(verts)
    with torch.cuda.device(verts.device):
        _check("mr_silhouette_rasterize_bwd",
               lib.mr_silhouette_rasterize_bwd(_ptr(verts), verts.shape[0], _ptr(faces), faces.shape[0], _ptr(p2f),
                                               _ptr(d), N, H, W, K, float(sigma), _ptr(g), _ptr(out),
                                               _stream(verts.device)))
    return out


def interpolate_fwd(pix_to_face, bary, faces, attr):
    """Per-slot vertex attributes (``mr_interpolate_fwd``): (N, H, W, K, D) float32."""
    lib = load_library()
    p2f = _dev(pix_to_face, torch.int64, "pix_to_face")
    b = _dev(bary, torch.float32, "bary")
    f = _dev(faces, torch.int64, "faces")
    a = _dev(attr, torch.float32, "attr")
    if a.ndim != 2 or tuple(b.shape) != tuple(p2f.shape) + (3,):
        raise ValueError("attr must be (V, D) and bary (N, H, W, K, 3)")
    K, D = p2f.shape[-1], a.shape[1]
    out = torch.empty(tuple(p2f.shape) + (D,), dtype=torch.float32, device=p2f.device)
    with torch.cuda.device(p2f.device):
        _check("mr_interpolate_fwd", lib.mr_interpolate_fwd(_ptr(p2f), _ptr(b), p2f.numel() // K, K, _ptr(f), f.shape[0],
                                                            _ptr(a), a.shape[0], D, _ptr(out), _stream(p2f.device)))
    return out


def interpolate_bwd(pix_to_face, bary, faces, attr, grad_out):
    """Gradient of the interpolation (``mr_interpolate_bwd``) -> (grad_attr (V, D), grad_bary)."""
    lib = load_library()
    p2f = _dev(pix_to_face, torch.int64, "pix_to_face")
    b = _dev(bary, torch.float32, "bary")
    f = _dev(faces, torch.int64, "faces")
    a = _dev(attr, torch.float32, "attr")
    g = _dev(grad_out, torch.float32, "grad_out")
    K, D = p2f.shape[-1], a.shape[1]
    if tuple(g.shape) != tuple(p2f.shape) + (D,):
        raise ValueError("grad_out shape mismatch")
    ga = torch.empty_like(a)
    gb = torch.empty_like(b)
    with torch.cuda.device(p2f.device):
        _check("mr_interpolate_bwd", lib.mr_interpolate_bwd(_ptr(p2f), _ptr(b), p2f.numel() // K, K, _ptr(f), f.shape[0],
                                                            _ptr(a), a.shape[0], D, _ptr(g), _ptr(ga), _ptr(gb),
                                                            _stream(p2f.device)))
    return ga, gb


PHONG_NPARAMS = 16


def phong_params(light_location, camera_position, ambient, diffuse, specular, shininess) -> np.ndarray:
    """The 16 host floats of the lighting calls: L, C, ambient, diffuse, specular colours, shininess."""
    prm = np.concatenate([np.asarray(x, np.float32).reshape(-1) for x in
                          (light_location, camera_position, ambient, diffuse, specular, [shininess])])
    if prm.shape[0] != PHONG_NPARAMS:
        raise ValueError("light/camera positions and the three colours take 3 values each")
    return np.ascontiguousarray(prm)


def _points3(name, *ts):
    out = [_dev(t, torch.float32, name) for t in ts]
    if any(t.ndim != 2 or t.shape[1] != 3 or t.shape[0] != out[0].shape[0] for t in out):
        raise ValueError(f"{name}: points, normals and albedo must all be (M, 3)")
    return out


def phong_fwd(points, normals, albedo, params):
    """Phong lighting at M points (``mr_phong_fwd``) -> colours (M, 3)."""
    lib = load_library()
    P, N, c = _points3("phong_fwd", points, normals, albedo)
    prm = np.ascontiguousarray(params, dtype=np.float32)
    out = torch.empty_like(P)
    with torch.cuda.device(P.device):
        _check("mr_phong_fwd", lib.mr_phong_fwd(_ptr(P), _ptr(N), _ptr(c), P.shape[0], prm.ctypes.data, _ptr(out),
                                                _stream(P.device)))
    return out


def phong_bwd(points, normals, albedo, params, grad_colors):
    """Gradient of the lighting (``mr_phong_bwd``) -> (grad_points, grad_normals, grad_albedo)."""
    lib = load_library()
    P, N, c, g = _points3("phong_bwd", points, normals, albedo, grad_colors)
    prm = np.ascontiguousarray(params, dtype=np.float32)
    gP, gN, gc = (torch.empty_like(P) for _ in range(3))
    with torch.cuda.device(P.device):
        _check("mr_phong_bwd", lib.mr_phong_bwd(_ptr(P), _ptr(N), _ptr(c), P.shape[0], prm.ctypes.data, _ptr(g),
                                                _ptr(gP), _ptr(gN), _ptr(gc), _stream(P.device)))
    return gP, gN, gc


def phong_shade_fwd(pix_to_face, bary, faces, points, normals, albedo, params):
    """Per-fragment Phong shading (``mr_phong_shade_fwd``) -> colours (N, H, W, K, 3)."""
    lib = load_library()
    p2f = _dev(pix_to_face, torch.int64, "pix_to_face")
    b = _dev(bary, torch.float32, "bary")
    f = _dev(faces, torch.int64, "faces")
    P, N, c = _points3("phong_shade_fwd", points, normals, albedo)
    if tuple(b.shape) != tuple(p2f.shape) + (3,):
        raise ValueError("bary must be pix_to_face.shape + (3,)")
    prm = np.ascontiguousarray(params, dtype=np.float32)
    K = p2f.shape[-1]
    out = torch.empty(tuple(p2f.shape) + (3,), dtype=torch.float32, device=p2f.device)
    with torch.cuda.device(p2f.device):
        _check("mr_phong_shade_fwd", lib.mr_phong_shade_fwd(_ptr(p2f), _ptr(b), p2f.numel() // K, K, _ptr(f),
                                                            f.shape[0], _ptr(P), _ptr(N), _ptr(c), P.shape[0],
                                                            prm.ctypes.data, _ptr(out), _stream(p2f.device)))
    return out


def phong_shade_bwd(pix_to_face, bary, faces, points, normals, albedo, params, grad_colors):
    """Gradient of the Phong shading (``mr_phong_shade_bwd``) ->
    (grad_points, grad_normals, grad_albedo, grad_bary)."""
    lib = load_library()
    p2f = _dev(pix_to_face, torch.int64, "pix_to_face")
    b = _dev(bary, torch.float32, "bary")
    f = _dev(faces, torch.int64, "faces")
    P, N, c = _points3("phong_shade_bwd", points, normals, albedo)
    g = _dev(grad_colors, torch.float32, "grad_colors")
    if tuple(b.shape) != tuple(p2f.shape) + (3,) or g.shape != b.shape:
        raise ValueError("bary and grad_colors must be pix_to_face.shape + (3,)")
    prm = np.ascontiguousarray(params, dtype=np.float32)
    K = p2f.shape[-1]
    gP, gN, gc = (torch.empty_like(P) for _ in range(3))
    gb = torch.empty_like(b)
    with torch.cuda.device(p2f.device):
        _check("mr_phong_shade_bwd", lib.mr_phong_shade_bwd(_ptr(p2f), _ptr(b), p2f.numel() // K, K, _ptr(f),
                                                            f.shape[0], _ptr(P), _ptr(N), _ptr(c), P.shape[0],
                                                            prm.ctypes.data, _ptr(g), _ptr(gP), _ptr(gN), _ptr(gc),
                                                            _ptr(gb), _stream(p2f.device)))
    return gP, gN, gc, gb


# ----------------------------------------------------------------------------- point clouds
COMPOSITE_MODES = {"alpha": 0, "norm_weighted": 1}


def rasterize_points_fwd(points, cloud_first_idx, num_points_per_cloud, H, W, radius, K):
    """K nearest points per pixel (``mr_rasterize_points_fwd``) -> (idx, zbuf, dists), each (N, H, W, K)."""
    lib = load_library()
    pts = _dev(points, torch.float32, "points")
    first = _Index(cloud_first_idx, "cloud_first_idx", pts.device)
    num = _Index(num_points_per_cloud, "num_points_per_cloud", pts.device)
    if pts.ndim != 2 or pts.shape[1] != 3 or first.n != num.n:
        raise ValueError("points must be (P, 3); cloud_first_idx and num_points_per_cloud of equal length")
    N = first.n
    dev = pts.device
    idx = torch.empty((N, H, W, K), dtype=torch.int64, device=dev)
    zbuf = torch.empty((N, H, W, K), dtype=torch.float32, device=dev)
    dists = torch.empty((N, H, W, K), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _check("mr_rasterize_points_fwd",
               lib.mr_rasterize_points_fwd(_ptr(pts), pts.shape[0], first.ptr, num.ptr, N, H, W,
                                           float(radius), K, _ptr(idx), _ptr(zbuf), _ptr(dists), _stream(dev)))
    return idx, zbuf, dists


def rasterize_points_bwd(points, idx, grad_zbuf=None, grad_dists=None):
    """Gradient of the point rasterizer (``mr_rasterize_points_bwd``) -> grad_points (P, 3)."""
    lib = load_library()
    pts = _dev(points, torch.float32, "points")
    ix = _dev(idx, torch.int64, "idx")
    N, H, W, K = ix.shape
    gz = None if grad_zbuf is None else _dev(grad_zbuf, torch.float32, "grad_zbuf")
    gd = None if grad_dists is None else _dev(grad_dists, torch.float32, "grad_dists")
    out = torch.empty_like(pts)
    with torch.cuda.device(pts.device):
        _check("mr_rasterize_points_bwd",
               lib.mr_rasterize_points_bwd(_ptr(pts), pts.shape[0], _ptr(ix), N, H, W, K, _ptr(gz), _ptr(gd),
                                           _ptr(out), _stream(pts.device)))
    return out


def composite_points_fwd(idx, dists, features, radius, mode="alpha"):
    """Alpha or norm-weighted compositing of per-point features (``mr_composite_points_fwd``) -> (N, H, W, C)."""
    lib = load_library()
    ix = _dev(idx, torch.int64, "idx")
    d = _dev(dists, torch.float32, "dists")
    f = _dev(features, torch.float32, "features")
    if d.shape != ix.shape or f.ndim != 2:
        raise ValueError("dists must match idx and features be (P, C)")
    K, C = ix.shape[-1], f.shape[1]
    out = torch.empty(tuple(ix.shape[:-1]) + (C,), dtype=torch.float32, device=ix.device)
    with torch.cuda.device(ix.device):
        _check("mr_composite_points_fwd",
               lib.mr_composite_points_fwd(_ptr(ix), _ptr(d), ix.numel() // K, K, _ptr(f), f.shape[0], C,
                                           float(radius), COMPOSITE_MODES[mode], _ptr(out), _stream(ix.device)))
    return out


def composite_points_bwd(idx, dists, features, radius, grad_out, mode="alpha"):
    """Gradient of the compositing (``mr_composite_points_bwd``) -> (grad_features, grad_dists)."""
    lib = load_library()
    ix = _dev(idx, torch.int64, "idx")
    d = _dev(dists, torch.float32, "dists")
    f = _dev(features, torch.float32, "features")
    g = _dev(grad_out, torch.float32, "grad_out")
    K, C = ix.shape[-1], f.shape[1]
    if tuple(g.shape) != tuple(ix.shape[:-1]) + (C,):
        raise ValueError("grad_out shape mismatch")
    gf = torch.empty_like(f)
    gd = torch.empty_like(d)
    with torch.cuda.device(ix.device):
        _check("mr_composite_points_bwd",
               lib.mr_composite_points_bwd(_ptr(ix), _ptr(d), ix.numel() // K, K, _ptr(f), f.shape[0], C,
                                           float(radius), COMPOSITE_MODES[mode], _ptr(g), _ptr(gf), _ptr(gd),
                                           _stream(ix.device)))
    return gf, gd


def knn_fwd(p1, first1, num1, p2, first2, num2, K):
    """Batched K nearest neighbours (``mr_knn_fwd``) -> (idx (P1, K) ids into p2, dists (P1, K))."""
    lib = load_library()
    a = _dev(p1, torch.float32, "p1")
    b = _dev(p2, torch.float32, "p2")
    f1, n1, f2, n2 = (_Index(x, nm, a.device) for x, nm in ((first1, "first1"), (num1, "num1"), (first2, "first2"),
                                                            (num2, "num2")))
    if a.ndim != 2 or b.ndim != 2 or a.shape[1] != b.shape[1] or not (f1.n == n1.n == f2.n == n2.n):
        raise ValueError("p1 (P1, D), p2 (P2, D) and four cloud arrays of equal length expected")
    idx = torch.empty((a.shape[0], K), dtype=torch.int64, device=a.device)
    dists = torch.empty((a.shape[0], K), dtype=torch.float32, device=a.device)
    with torch.cuda.device(a.device):
        _check("mr_knn_fwd", lib.mr_knn_fwd(_ptr(a), a.shape[0], f1.ptr, n1.ptr, _ptr(b), b.shape[0],
                                            f2.ptr, n2.ptr, f1.n, a.shape[1], K, _ptr(idx),
                                            _ptr(dists), _stream(a.device)))
    return idx, dists


def knn_count_pairs(p1, first1, num1, p2, first2, num2, K):
    """The (query, reference) pairs the KNN search evaluates (``mr_knn_count_pairs``): the
    search's real work, for its roofline.  Returns (pairs, idx, dists)."""
    lib = load_library()
    a = _dev(p1, torch.float32, "p1")
    b = _dev(p2, torch.float32, "p2")
    f1, n1, f2, n2 = (_Index(x, nm, a.device) for x, nm in ((first1, "first1"), (num1, "num1"), (first2, "first2"),
                                                            (num2, "num2")))
    if a.ndim != 2 or b.ndim != 2 or a.shape[1] != b.shape[1] or not (f1.n == n1.n == f2.n == n2.n):
        raise ValueError("p1 (P1, D), p2 (P2, D) and four cloud arrays of equal length expected")
    idx = torch.empty((a.shape[0], K), dtype=torch.int64, device=a.device)
    dists = torch.empty((a.shape[0], K), dtype=torch.float32, device=a.device)
    out = np.zeros(1, np.int64)
    with torch.cuda.device(a.device):
        _check("mr_knn_count_pairs",
               lib.mr_knn_count_pairs(_ptr(a), a.shape[0], f1.ptr, n1.ptr, _ptr(b), b.shape[0], f2.ptr, n2.ptr, f1.n,
                                      a.shape[1], K, _ptr(idx), _ptr(dists), out.ctypes.data, _stream(a.device)))
    return int(out[0]), idx, dists


def knn_bwd(p1, p2, idx, grad_dists):
    """Gradient of the KNN distances (``mr_knn_bwd``) -> (grad_p1, grad_p2)."""
    lib = load_library()
    a = _dev(p1, torch.float32, "p1")
    b = _dev(p2, torch.float32, "p2")
    ix = _dev(idx, torch.int64, "idx")
    g = _dev(grad_dists, torch.float32, "grad_dists")
    g1 = torch.empty_like(a)
    g2 = torch.empty_like(b)
    with torch.cuda.device(a.device):
        _check("mr_knn_bwd", lib.mr_knn_bwd(_ptr(a), a.shape[0], _ptr(b), b.shape[0], a.shape[1], ix.shape[1],
                                            _ptr(ix), _ptr(g), _ptr(g1), _ptr(g2), _stream(a.device)))
    return g1, g2


def _blend_args(pix_to_face, colors, dists, zbuf, background):
    p2f = _dev(pix_to_face, torch.int64, "pix_to_face")
    c = _dev(colors, torch.float32, "colors")
    d = _dev(dists, torch.float32, "dists")
    z = _dev(zbuf, torch.float32, "zbuf")
    K, D = p2f.shape[-1], c.shape[-1]
    if tuple(c.shape[:-1]) != tuple(p2f.shape) or d.shape != p2f.shape or z.shape != p2f.shape:
        raise ValueError("colors / dists / zbuf must match pix_to_face")
    bg = np.ascontiguousarray(np.asarray(background, dtype=np.float32).reshape(-1))
    if bg.shape[0] != D:
        raise ValueError("background must have one value per colour channel")
    return p2f, c, d, z, bg, K, D


def blend_fwd(pix_to_face, colors, dists, zbuf, background, sigma, gamma, znear, zfar):
    """Soft RGB blend (``mr_blend_fwd``) -> rgba (N, H, W, D + 1)."""
    lib = load_library()
    p2f, c, d, z, bg, K, D = _blend_args(pix_to_face, colors, dists, zbuf, background)
    out = torch.empty(tuple(p2f.shape[:-1]) + (D + 1,), dtype=torch.float32, device=p2f.device)
    with torch.cuda.device(p2f.device):
        _check("mr_blend_fwd", lib.mr_blend_fwd(_ptr(p2f), _ptr(c), _ptr(d), _ptr(z), p2f.numel() // K, K, D,
                                                bg.ctypes.data, float(sigma), float(gamma), float(znear), float(zfar),
                                                _ptr(out), _stream(p2f.device)))
    return out


def blend_bwd(pix_to_face, colors, dists, zbuf, background, sigma, gamma, znear, zfar, grad_rgba):
    """Gradient of the blend (``mr_blend_bwd``) -> (grad_colors, grad_dists, grad_zbuf)."""
    lib = load_library()
    p2f, c, d, z, bg, K, D = _blend_args(pix_to_face, colors, dists, zbuf, background)
    g = _dev(grad_rgba, torch.float32, "grad_rgba")
    gc, gd, gz = torch.empty_like(c), torch.empty_like(d), torch.empty_like(z)
    with torch.cuda.device(p2f.device):
        _check("mr_blend_bwd", lib.mr_blend_bwd(_ptr(p2f), _ptr(c), _ptr(d), _ptr(z), p2f.numel() // K, K, D,
                                                bg.ctypes.data, float(sigma), float(gamma), float(znear), float(zfar),
                                                _ptr(g), _ptr(gc), _ptr(gd), _ptr(gz), _stream(p2f.device)))
    return gc, gd, gz


INJECT = {"off": 0, "oom": 1, "cuda": 2}


def inject_fault(kind: str = "off", skip: int = 0) -> None:
    """Arm (``"oom"``, ``"cuda"``) or disarm (``"off"``) a one-shot failure of the library's
    scratch allocator after ``skip`` successful allocations (``mr_inject_fault``)."""
    _check("mr_inject_fault", load_library().mr_inject_fault(INJECT[kind], int(skip)))


def scratch_in_use(device=None) -> int:
    """Bytes allocated from the device's default memory pool (``mr_scratch_in_use``)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    out = ctypes.c_int64(0)
    with torch.cuda.device(dev):
        _check("mr_scratch_in_use", load_library().mr_scratch_in_use(ctypes.byref(out)))
    return int(out.value)


def scratch_peak(device=None, reset: bool = False) -> int:
    """High-water mark of the device's default memory pool, where the library's scratch
    comes from (``mr_scratch_peak``); ``reset`` restarts it after reading."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    out = ctypes.c_int64(0)
    with torch.cuda.device(dev):
        _check("mr_scratch_peak", load_library().mr_scratch_peak(ctypes.byref(out), int(bool(reset))))
    return int(out.value)


def measure_fp32_peak(device=None) -> float:
    """Measured FP32 instruction issue rate of the device (``mr_measure_fp32_peak``), inst/s."""
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    out = ctypes.c_double(0.0)
    with torch.cuda.device(dev):
        _check("mr_measure_fp32_peak", lib.mr_measure_fp32_peak(ctypes.byref(out), _stream(dev)))
    return float(out.value)


def device_status(device=None) -> None:
    """Synchronise and raise if an asynchronous kernel skipped an out-of-range index."""
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        _check("mr_device_status", lib.mr_device_status(_stream(dev)))


def profile_enable(on: bool = True) -> None:
    """Start (or stop) recording CUDA events around every kernel stage (``mr_profile_enable``)."""
    _check("mr_profile_enable", load_library().mr_profile_enable(int(bool(on))))


def profile_read() -> dict:
    """Summed device milliseconds and launch counts per stage since the last read."""
    n = len(STAGES)
    ms = np.zeros(n, np.float64)
    cnt = np.zeros(n, np.int64)
    _check("mr_profile_read", load_library().mr_profile_read(ms.ctypes.data, cnt.ctypes.data, n))
    return {s: (float(ms[i]), int(cnt[i])) for i, s in enumerate(STAGES)}


class SilhouetteRasterizer(torch.autograd.Function):
    """verts -> soft silhouette alpha, differentiable w.r.t. the screen-space vertices.

    Forward: ``mr_rasterize_silhouette_fwd``; backward: ``mr_silhouette_rasterize_bwd``.
    """

    @staticmethod
    def forward(ctx, verts, faces, first, num, H, W, blur_radius, K, sigma, perspective_correct=False):
        p2f, _, _, dists, alpha = rasterize_fwd(verts, faces, first, num, H, W, blur_radius, K,
                                                perspective_correct, sigma=sigma)
        ctx.save_for_backward(verts, faces, p2f, dists)
        ctx.sigma = sigma
        return alpha

    @staticmethod
    def backward(ctx, grad_alpha):
        verts, faces, p2f, dists = ctx.saved_tensors
        gv = silhouette_rasterize_bwd(verts, faces, p2f, dists, ctx.sigma, grad_alpha.contiguous())
        return gv, None, None, None, None, None, None, None, None, None
