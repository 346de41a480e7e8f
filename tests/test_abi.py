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


def _fwd(lib, **kw):
    a = dict(verts=None, V=3, faces=None, F=1, first=np.array([0], np.int64), num=np.array([1], np.int64),
             N=1, H=8, W=8, blur=0.0, K=1, persp=0)
    a.update(kw)
    dummy = ctypes.c_void_p(16)   # never dereferenced: validation fails first
    return lib.mr_rasterize_fwd(dummy, a["V"], dummy, a["F"], a["first"].ctypes.data, a["num"].ctypes.data,
                                a["N"], a["H"], a["W"], a["blur"], a["K"], a["persp"], dummy, dummy, dummy, dummy,
                                None)


@pytest.mark.parametrize("kw,msg", [
    (dict(K=0), "K=0"), (dict(K=33), "K=33"), (dict(H=0), "H=0"), (dict(W=40000), "W=40000"),
    (dict(blur=-1.0), "blur_radius"), (dict(blur=float("nan")), "blur_radius"),
    (dict(num=np.array([2], np.int64)), "outside"), (dict(first=np.array([-1], np.int64)), "outside"),
    (dict(F=-1), "F=-1"), (dict(N=-1), "N=-1"),
])
def test_forward_rejects_bad_arguments(lib, kw, msg):
    rc = _fwd(lib, **kw)
    assert rc == -1
    assert msg in lib.mr_last_error().decode()


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
