"""The C-ABI library loads, exports every declared symbol and validates arguments (CPU only).

Only argument checks that return before any CUDA call are exercised here; nothing
touches a GPU.
"""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from differentiable_mesh_rasterization_b200 import build
    build.build()
    import differentiable_mesh_rasterization_b200 as mr
    return mr.load_library()


def declared_symbols():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(mr_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
    import differentiable_mesh_rasterization_b200 as mr
    assert set(mr.EXPORTS) == set(names)


def test_version_and_error_string(lib):
    assert lib.mr_version() >= 10000
    assert isinstance(lib.mr_last_error(), bytes)


FORWARDS = ["mr_rasterize_fwd", "mr_rasterize_fwd_noalloc"]


def _fwd(lib, entry="mr_rasterize_fwd", **kw):
    a = dict(verts=None, V=3, faces=None, F=1, first=np.array([0], np.int64), num=np.array([1], np.int64),
             N=1, H=8, W=8, blur=0.0, K=1, persp=0)
    a.update(kw)
    dummy = ctypes.c_void_p(16)   # never dereferenced: validation fails first
    return getattr(lib, entry)(dummy, a["V"], dummy, a["F"], a["first"].ctypes.data, a["num"].ctypes.data,
                               a["N"], a["H"], a["W"], a["blur"], a["K"], a["persp"], dummy, dummy, dummy, dummy,
                               None)


@pytest.mark.parametrize("entry", FORWARDS)
@pytest.mark.parametrize("kw,msg", [
    (dict(K=0), "K=0"), (dict(K=33), "K=33"), (dict(H=0), "H=0"), (dict(W=40000), "W=40000"),
    (dict(blur=-1.0), "blur_radius"), (dict(blur=float("nan")), "blur_radius"),
    (dict(num=np.array([2], np.int64)), "outside"), (dict(first=np.array([-1], np.int64)), "outside"),
    (dict(F=-1), "F=-1"), (dict(N=-1), "N=-1"),
])
def test_forward_rejects_bad_arguments(lib, entry, kw, msg):
    """Both forwards reject bad arguments before any CUDA call (the scratch-free one before
    it looks up its fixed array)."""
    rc = _fwd(lib, entry, **kw)
    assert rc == -1
    assert msg in lib.mr_last_error().decode()


@pytest.mark.parametrize("entry", FORWARDS)
def test_forward_with_no_images_is_a_no_op(lib, entry):
    assert _fwd(lib, entry, N=0, first=np.zeros(0, np.int64), num=np.zeros(0, np.int64)) == 0


@pytest.mark.parametrize("fn", ["rasterize_fwd", "rasterize_fwd_noalloc"])
def test_binding_checks_shapes_before_the_library_sees_them(fn):
    """A (V, 2) verts, an (F, 2) faces or per-mesh arrays of unequal length would make the
    kernels or the host plan read past a buffer's end; the binding refuses them."""
    import torch
    import differentiable_mesh_rasterization_b200 as mr
    call = getattr(mr, fn)
    v3, f3 = torch.zeros(3, 3), torch.zeros(1, 3, dtype=torch.int64)
    for v, f, first, num in ((torch.zeros(3, 2), f3, [0], [1]), (v3, torch.zeros(1, 2, dtype=torch.int64), [0], [1]),
                             (v3, f3, [0, 1], [1]), (v3, f3, [[0]], [[1]])):
        with pytest.raises(ValueError):
            call(v, f, first, num, 8, 8, 0.0, 1)


def test_other_entry_points_reject_bad_arguments(lib):
    d = ctypes.c_void_p(16)
    assert lib.mr_silhouette_blend_fwd(d, d, 1, 4, 4, 0, 1e-4, d, None) == -1
    assert lib.mr_silhouette_blend_fwd(d, d, 1, 4, 4, 2, 0.0, d, None) == -1
    assert lib.mr_silhouette_blend_bwd(d, d, d, 1, 4, 4, 40, 1e-4, d, None) == -1
    assert lib.mr_rasterize_bwd(d, 3, d, 1, d, 1, 4, 4, 0, 0, None, None, None, d, None) == -1
    assert lib.mr_silhouette_rasterize_bwd(d, 3, d, 1, d, d, 1, 4, 4, 2, -1.0, d, d, None) == -1
    # empty batches are valid and launch nothing
    assert lib.mr_silhouette_blend_fwd(d, d, 0, 4, 4, 2, 1e-4, d, None) == 0


def test_binding_fails_loudly_without_cuda_tensors():
    import torch
    import differentiable_mesh_rasterization_b200 as mr
    v = torch.zeros(3, 3)
    f = torch.zeros(1, 3, dtype=torch.int64)
    with pytest.raises(ValueError):
        mr.rasterize_fwd(v, f, [0], [1], 8, 8, 0.0, 1)


def test_next_row_entry_points_reject_bad_arguments(lib):
    """Stage-two shading, Phong lighting, point clouds and KNN: host-side validation only."""
    d = ctypes.c_void_p(16)
    err = lambda: lib.mr_last_error().decode()
    assert lib.mr_interpolate_fwd(d, d, 4, 2, d, 1, d, 3, 0, d, None) == -1 and "D=0" in err()
    bg = np.zeros(9, np.float32)
    assert lib.mr_blend_fwd(d, d, d, d, 4, 2, 9, bg.ctypes.data, 1e-4, 1e-2, 1.0, 10.0, d, None) == -1
    assert lib.mr_blend_fwd(d, d, d, d, 4, 2, 3, bg.ctypes.data, 0.0, 1e-2, 1.0, 10.0, d, None) == -1
    assert lib.mr_blend_bwd(d, d, d, d, 4, 2, 3, bg.ctypes.data, 1e-4, 1e-2, 10.0, 1.0, d, d, d, d, None) == -1
    prm = np.zeros(16, np.float32)
    prm[15] = 0.5                                       # shininess below 1
    assert lib.mr_phong_fwd(d, d, d, 4, prm.ctypes.data, d, None) == -1 and "shininess" in err()
    prm[15] = 8.0
    prm[0] = np.nan
    assert lib.mr_phong_bwd(d, d, d, 4, prm.ctypes.data, d, d, d, d, None) == -1 and "finite" in err()
    prm[0] = 1.0
    assert lib.mr_phong_shade_fwd(d, d, 4, 0, d, 1, d, d, d, 3, prm.ctypes.data, d, None) == -1
    first, num = np.array([0, 5], np.int64), np.array([10, 5], np.int64)     # overlapping clouds
    assert lib.mr_rasterize_points_fwd(d, 20, first.ctypes.data, num.ctypes.data, 2, 8, 8, 0.1, 4, d, d, d,
                                       None) == -1 and "not ascending" in err()
    ok_first, ok_num = np.array([0], np.int64), np.array([20], np.int64)
    assert lib.mr_rasterize_points_fwd(d, 20, ok_first.ctypes.data, ok_num.ctypes.data, 1, 8, 8, float("nan"), 4,
                                       d, d, d, None) == -1
    assert lib.mr_rasterize_points_fwd(d, 20, ok_first.ctypes.data, ok_num.ctypes.data, 1, 8, 8, 0.1, 40, d, d, d,
                                       None) == -1
    assert lib.mr_composite_points_fwd(d, d, 4, 2, d, 3, 3, 0.1, 2, d, None) == -1 and "mode=2" in err()
    assert lib.mr_composite_points_bwd(d, d, 4, 2, d, 3, 3, 0.0, 0, d, d, d, None) == -1
    assert lib.mr_knn_fwd(d, 10, ok_first.ctypes.data, ok_num.ctypes.data, d, 10, ok_first.ctypes.data,
                          ok_num.ctypes.data, 1, 5, 4, d, d, None) == -1 and "D=5" in err()
    assert lib.mr_knn_fwd(d, 20, first.ctypes.data, num.ctypes.data, d, 20, first.ctypes.data, num.ctypes.data, 2,
                          3, 4, d, d, None) == -1 and "overlap" in err()
    assert lib.mr_knn_bwd(d, 4, d, 4, 0, 2, d, d, d, d, None) == -1


@pytest.mark.parametrize("kind,code", [(1, -2), (2, -3)])
def test_injected_allocation_failure_returns_its_code_and_disarms(lib, kind, code):
    """The one-shot hook fails the library's first scratch allocation before anything is
    launched (valid arguments, so the call gets that far); the next call no longer meets it."""
    assert lib.mr_inject_fault(kind, 0) == 0
    rc = _fwd(lib)
    assert rc == code and "injected" in lib.mr_last_error().decode()
    rc = _fwd(lib)            # disarmed: without a GPU the real allocator path fails differently
    assert "injected" not in lib.mr_last_error().decode()
    assert lib.mr_inject_fault(0, 0) == 0


def test_fault_injection_rejects_bad_arguments(lib):
    assert lib.mr_inject_fault(3, 0) == -1 and "kind=3" in lib.mr_last_error().decode()
    assert lib.mr_inject_fault(1, -1) == -1
