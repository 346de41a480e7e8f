"""The GPU-vs-oracle comparison rules themselves (CPU only).

A parity claim is only as strong as its comparator, so the comparator is exercised on
oracle outputs with planted differences: each must be caught exactly when it exceeds
the stated tolerance or touches a pixel the oracle does not exempt.
"""
import numpy as np
import pytest

from _parity import ABS, compare_alpha, compare_forward, compare_grad
from differentiable_mesh_rasterization_b200 import synthetic as syn


@pytest.fixture(scope="module")
def ora(oracle_mod):
    b = syn.make_batch(2, n_meshes=2)
    w = b.workload
    return oracle_mod.rasterize_fwd(b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, 48, 48,
                                    np.float32(w.blur_radius), w.K)


def as_gpu(o):
    p, z, b, d, _ = o
    return [p.copy(), z.astype(np.float32), b.astype(np.float32), d.astype(np.float32)]


def first_valid(o, exempt_ok=True):
    p, ex = o[0], o[4]
    cand = np.argwhere((p[..., 0] >= 0) & ((ex == 0) if exempt_ok else (ex != 0)))
    return tuple(cand[0])


def test_identical_outputs_pass(ora):
    info = compare_forward(as_gpu(ora), ora, "same")
    assert info["valid_slots"] > 1000


def test_a_changed_face_id_is_caught(ora):
    g = as_gpu(ora)
    g[0][first_valid(ora) + (0,)] += 1
    with pytest.raises(AssertionError, match="pix_to_face"):
        compare_forward(g, ora, "id")


def test_a_changed_face_id_at_an_exempt_pixel_is_allowed(ora):
    ex = ora[4]
    if not (ex != 0).any():
        pytest.skip("no exempt pixel in this case")
    g = as_gpu(ora)
    g[0][tuple(np.argwhere(ex != 0)[0]) + (0,)] += 1
    compare_forward(g, ora, "exempt id")


@pytest.mark.parametrize("field", [1, 2, 3])
def test_value_errors_against_the_tolerance(ora, field):
    at = first_valid(ora) + (0,)
    for delta, caught in ((0.5 * ABS, False), (3 * ABS, True)):
        g = as_gpu(ora)
        if field == 2:
            g[2][at + (1,)] += delta
        else:
            g[field][at] += delta
        if caught:
            with pytest.raises(AssertionError):
                compare_forward(g, ora, "value")
        else:
            compare_forward(g, ora, "value")


def test_empty_slot_padding_is_checked(ora):
    p = ora[0]
    at = tuple(np.argwhere((p[..., -1] < 0) & (ora[4] == 0))[0]) + (p.shape[-1] - 1,)
    g = as_gpu(ora)
    g[1][at] = 0.0
    with pytest.raises(AssertionError, match="empty"):
        compare_forward(g, ora, "pad")


def test_alpha_and_gradient_tolerances():
    a = np.linspace(0.0, 1.0, 101)
    compare_alpha(a + 0.5e-4 * a, a)
    with pytest.raises(AssertionError):
        compare_alpha(a + 2e-4 * a + 1e-6, a)
    rng = np.random.default_rng(0)
    go = rng.normal(size=(500, 3))
    rms = np.sqrt(np.mean(go ** 2))
    assert compare_grad(go * (1 + 5e-5), go) < 1e-4
    with pytest.raises(AssertionError):
        bad = go.copy()
        bad[7, 1] += 3e-4 * (abs(go[7, 1]) + rms)
        compare_grad(bad, go)
