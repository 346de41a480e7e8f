"""The GPU-vs-oracle comparison rules themselves (CPU only).

A parity claim is only as strong as its comparator, so the comparator is exercised on
oracle outputs with planted differences: each must be caught exactly when it exceeds
the stated tolerance or touches a pixel the oracle does not exempt.
"""
import numpy as np
import pytest

from _parity import ABS, Scene, compare_alpha, compare_forward, compare_grad
from differentiable_mesh_rasterization_b200 import synthetic as syn


@pytest.fixture(scope="module")
def scene(oracle_mod):
    b = syn.make_batch(2, n_meshes=2)
    w = b.workload
    return Scene(oracle_mod, b.verts, b.faces, b.mesh_to_face_first_idx, b.num_faces_per_mesh, 48, 48,
                 w.blur_radius, w.K, False)


@pytest.fixture(scope="module")
def ora(scene):
    return scene.fwd()


def as_gpu(o):
    p, z, b, d, _ = o
    return [p.copy(), z.astype(np.float32), b.astype(np.float32), d.astype(np.float32)]


def first_valid(o, exempt_ok=True):
    p, ex = o[0], o[4]
    cand = np.argwhere((p[..., 0] >= 0) & ((ex == 0) if exempt_ok else (ex != 0)))
    return tuple(cand[0])


def test_identical_outputs_pass(ora, scene):
    info = compare_forward(as_gpu(ora), ora, "same", scene=scene)
    assert info["valid_slots"] > 1000


def test_a_changed_face_id_is_caught(ora, scene):
    g = as_gpu(ora)
    g[0][first_valid(ora) + (0,)] += 1
    with pytest.raises(AssertionError, match="pix_to_face"):
        compare_forward(g, ora, "id", scene=scene)


# ------------------------------------------------ flagged pixels: ties (E1), margins (E2)
H = W = 32


def _soup(tris):
    v = np.array([p for t in tris for p in t], np.float32)
    return v, np.arange(len(v), dtype=np.int64).reshape(-1, 3)


@pytest.fixture(scope="module")
def tie_scene(oracle_mod):
    """Faces 0 and 1 cover the middle at constant depths 2 and 2 + 2 float32 ulps (< 1e-6
    apart: E1); face 2 lies behind both at depth 3."""
    a = [[-0.8, -0.7, 2.0], [0.7, -0.8, 2.0], [0.0, 0.8, 2.0]]
    z1 = float(np.nextafter(np.nextafter(np.float32(2.0), np.float32(3)), np.float32(3)))
    b = [[-0.7, 0.7, z1], [0.8, 0.6, z1], [0.1, -0.8, z1]]
    c = [[-0.9, -0.9, 3.0], [0.9, -0.9, 3.0], [0.0, 0.9, 3.0]]
    v, f = _soup([a, b, c])
    sc = Scene(oracle_mod, v, f, [0], [3], H, W, 0.0, 2, False)
    return sc, sc.fwd(), sc.fwd(K=3, exempt=False)


def _tie_pixel(o, o3):
    e1 = np.argwhere(((o[4] & 1) > 0) & ((o[4] & 2) == 0) & (o3[0][..., 2] == 2))
    assert len(e1) > 20
    return tuple(e1[len(e1) // 2])


def test_a_permutation_inside_a_depth_tie_is_allowed(tie_scene):
    sc, o, o3 = tie_scene
    at = _tie_pixel(o, o3)
    g = as_gpu(o)
    for x in g:
        x[at] = x[at][::-1]          # faces 0 and 1 swapped, each with its own values
    info = compare_forward(g, o, "tie swap", scene=sc, e2_max=1.0)
    assert info["e1"] > 0
    assert list(info["rec"][0][at]) == [1, 0]


def test_a_tie_swap_with_the_values_left_in_place_is_caught(tie_scene):
    sc, o, o3 = tie_scene
    at = _tie_pixel(o, o3)
    g = as_gpu(o)
    g[0][at] = g[0][at][::-1]        # ids swapped, bary/dists still those of the other face
    with pytest.raises(AssertionError, match="tie pixel"):
        compare_forward(g, o, "tie ids only", scene=sc, e2_max=1.0)


def test_a_face_outside_the_tie_group_is_caught(tie_scene):
    sc, o, o3 = tie_scene
    at = _tie_pixel(o, o3)
    g = as_gpu(o)
    g[0][at + (1,)] = 2              # the farther face (depth 3) in the tied slot
    g[1][at + (1,)] = np.float32(o3[1][at + (2,)])
    g[2][at + (1,)] = o3[2][at + (2,)].astype(np.float32)
    g[3][at + (1,)] = np.float32(o3[3][at + (2,)])
    with pytest.raises(AssertionError, match="tie pixel"):
        compare_forward(g, o, "outside group", scene=sc, e2_max=1.0)


def test_a_tie_across_slot_k_may_hand_the_last_slot_to_the_next_candidate(tie_scene):
    """K = 1: faces 0 and 1 tie for the only slot; the oracle keeps 0, face 1 (its second
    candidate, asked for by the comparator) is as good, face 2 is not."""
    sc, _, o3 = tie_scene
    sc1 = Scene(sc.oracle, sc.verts, sc.faces, sc.first, sc.num, H, W, 0.0, 1, False)
    o = sc1.fwd()
    at = _tie_pixel(sc.fwd(), o3)
    assert o[0][at + (0,)] == 0
    g = as_gpu(o)
    for x, y in zip(g, o3[:4]):
        x[at + (0,)] = y[at + (1,)]
    info = compare_forward(g, o, "tail", scene=sc1, e2_max=1.0)
    assert info["rec"][0][at + (0,)] == 1
    for x, y in zip(g, o3[:4]):
        x[at + (0,)] = y[at + (2,)]
    with pytest.raises(AssertionError, match="tie pixel"):
        compare_forward(g, o, "tail", scene=sc1, e2_max=1.0)


@pytest.fixture(scope="module")
def margin_scene(oracle_mod):
    """Face 0's right edge lies on x = -1/32 (column 15's centres); with blur = (2/32)^2 the
    centres of column 16 (x = 1/32) sit exactly on its blur threshold (E2). Face 1 covers every pixel
    behind it."""
    x0 = -1.0 / 32
    c = [[x0, -0.8, 3.0], [x0, 0.8, 3.0], [x0 - 0.6, 0.0, 3.0]]
    d = [[-3.0, -3.0, 4.0], [3.0, -3.0, 4.0], [0.0, 3.0, 4.0]]
    v, f = _soup([c, d])
    sc = Scene(oracle_mod, v, f, [0], [2], H, W, (2.0 / 32) ** 2, 2, False)
    return sc, sc.fwd()


def _margin_pixel(o):
    e2 = np.argwhere((o[4] & 2) > 0)
    assert len(e2) > 5 and np.all(e2[:, 2] == 16)
    at = tuple(e2[len(e2) // 2])
    assert list(o[0][at]) == [0, 1]
    return at


def test_dropping_the_marginal_face_is_allowed(margin_scene):
    sc, o = margin_scene
    at = _margin_pixel(o)
    g = as_gpu(o)
    for x in g:                       # slot 0 (the marginal face) gone, face 1 moves up
        x[at + (0,)] = x[at + (1,)]
        x[at + (1,)] = -1
    info = compare_forward(g, o, "margin drop", scene=sc, e2_max=1.0)
    assert list(info["rec"][0][at]) == [1, -1]


def test_dropping_a_face_that_is_not_marginal_is_caught(margin_scene):
    sc, o = margin_scene
    at = _margin_pixel(o)
    g = as_gpu(o)
    for x in g:
        x[at + (1,)] = -1
    with pytest.raises(AssertionError, match="non-marginal"):
        compare_forward(g, o, "margin keep", scene=sc, e2_max=1.0)


def test_wrong_values_at_a_margin_pixel_are_caught(margin_scene):
    sc, o = margin_scene
    at = _margin_pixel(o)
    g = as_gpu(o)
    g[3][at + (1,)] += 3 * ABS
    with pytest.raises(AssertionError, match="margin pixel"):
        compare_forward(g, o, "margin value", scene=sc, e2_max=1.0)


def test_too_many_margin_pixels_are_caught(margin_scene):
    sc, o = margin_scene
    with pytest.raises(AssertionError, match="candidacy-margin"):
        compare_forward(as_gpu(o), o, "margin rate", scene=sc)


@pytest.mark.parametrize("field", [1, 2, 3])
def test_value_errors_against_the_tolerance(ora, scene, field):
    at = first_valid(ora) + (0,)
    for delta, caught in ((0.5 * ABS, False), (3 * ABS, True)):
        g = as_gpu(ora)
        if field == 2:
            g[2][at + (1,)] += delta
        else:
            g[field][at] += delta
        if caught:
            with pytest.raises(AssertionError):
                compare_forward(g, ora, "value", scene=scene)
        else:
            compare_forward(g, ora, "value", scene=scene)


def test_empty_slot_padding_is_checked(ora, scene):
    p = ora[0]
    at = tuple(np.argwhere((p[..., -1] < 0) & (ora[4] == 0))[0]) + (p.shape[-1] - 1,)
    g = as_gpu(ora)
    g[1][at] = 0.0
    with pytest.raises(AssertionError, match="empty"):
        compare_forward(g, ora, "pad", scene=scene)


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
