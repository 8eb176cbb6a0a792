"""Pins for the CPU oracle: facts fixed by the pages and by mathematics, not by
the oracle itself.  CPU only.

Each test names what pins it: a value the pages print, a closed form, a
library routine that the method reduces to in a special case, or an
independent brute-force formulation.
"""
import json
import os

import numpy as np
import pytest

import oracle
from scale_deformable_attention_02_b200 import workloads as wl

RNG = np.random.default_rng(20240601)


def _one_level_value(h, w, m, d, fill):
    return np.ascontiguousarray(fill(h, w, m, d), dtype=np.float32).reshape(1, h * w, m, d)


# --------------------------------------------------------------------------
# Worked example ("Deformable DETR Samples Sparse Points", "Worked example")
# --------------------------------------------------------------------------
def _golden(golden_dir):
    with open(os.path.join(golden_dir, "worked_blend.json")) as f:
        return json.load(f)


def test_worked_example_terms_sum(golden_dir):
    g = _golden(golden_dir)
    terms = [a * v for a, v in zip(g["weights"], g["sampled_values"])]
    assert np.allclose(terms, g["terms"], atol=1e-12)
    assert abs(sum(g["terms"]) - g["blend"]) < 1e-12


def test_worked_example_four_constant_levels(golden_dir):
    """Four 28x28 levels, level l constant at the page's sampled value v_l,
    one point per level at the page's sampling locations, weights from the
    page: the blend must be 0.70 (up to the fp32 rounding of the inputs)."""
    g = _golden(golden_dir)
    h, w = g["map_hw"]
    shapes = np.array([[h, w]] * 4, dtype=np.int64)
    value = np.concatenate([np.full((1, h * w, 1, 1), v, np.float32)
                            for v in g["sampled_values"]], axis=1)
    loc = np.array(g["sample_points"], dtype=np.float32).reshape(1, 1, 1, 4, 1, 2)
    A = np.array(g["weights"], dtype=np.float64).reshape(1, 1, 1, 4, 1)
    out = oracle.forward(value, shapes, loc, A)[0, 0, 0]
    # exact value of the blend of the fp32-rounded inputs
    exact = sum(a * float(np.float32(v)) for a, v in zip(g["weights"], g["sampled_values"]))
    assert abs(out - exact) < 1e-15
    assert abs(out - g["blend"]) < 1e-7


def test_worked_example_single_map(golden_dir):
    """The page's setting taken literally: one 28x28 map, K = 4 points.  A
    bilinear map f = a + b x + c y + e x y is reproduced exactly by bilinear
    interpolation, so choosing f with f(point_i) = v_i makes the sampled
    values the page's, and the blend must again be 0.70."""
    g = _golden(golden_dir)
    h, w = g["map_hw"]
    pts = np.array(g["sample_points"], dtype=np.float64)
    px = pts[:, 0] * w - 0.5  # pixel convention x = loc*W - 0.5
    py = pts[:, 1] * h - 0.5
    cx, cy = 14.0, 13.5  # centre the basis so the stored values stay small
    Amat = np.stack([np.ones(4), px - cx, py - cy, (px - cx) * (py - cy)], axis=1)
    coef = np.linalg.solve(Amat, np.array(g["sampled_values"]))
    hh, ww = np.meshgrid(np.arange(h), np.arange(w), indexing="ij")
    f = coef[0] + coef[1] * (ww - cx) + coef[2] * (hh - cy) + coef[3] * (ww - cx) * (hh - cy)
    value = f.astype(np.float32).reshape(1, h * w, 1, 1)
    shapes = np.array([[h, w]], dtype=np.int64)
    loc = pts.reshape(1, 1, 1, 1, 4, 2)
    A = np.array(g["weights"], dtype=np.float64).reshape(1, 1, 1, 1, 4)
    out = oracle.forward(value, shapes, loc, A, loc_f32=False)[0, 0, 0]
    rounding = np.abs(value.astype(np.float64).ravel() - f.ravel()).max()
    assert abs(out - g["blend"]) <= 4 * rounding + 1e-12


# --------------------------------------------------------------------------
# Closed forms
# --------------------------------------------------------------------------
def test_level_start_index_is_prefix_sum():
    starts, S = oracle.level_start_index(wl.spatial_shapes_array(wl.ENCODER_SHAPES))
    assert starts.tolist() == [0, 13400, 16750, 17600] and S == 17821
    starts, S = oracle.level_start_index(wl.spatial_shapes_array(wl.STRESS_SHAPES))
    assert starts.tolist() == [0, 27889, 34945, 36709] and S == 37150
    starts, S = oracle.level_start_index(wl.spatial_shapes_array(wl.TINY_SHAPES))
    assert starts.tolist() == [0, 64] and S == 80


def test_constant_map_returns_constant():
    """A constant map c returns c for every sample whose four corners are in
    the map, so out = c * sum(A)."""
    shapes = np.array([[7, 9], [3, 5]], dtype=np.int64)
    S = 7 * 9 + 3 * 5
    M, D, K, Lq = 3, 4, 3, 11
    c = np.float32(0.8125)
    value = np.full((1, S, M, D), c, np.float32)
    loc = np.empty((1, Lq, M, 2, K, 2), np.float32)
    for l, (h, w) in enumerate(shapes):
        # pixel x in [0, W-1] <=> loc_x in [0.5/W, (W-0.5)/W]
        loc[..., l, :, 0] = RNG.uniform(0.5 / w, (w - 0.5) / w, size=(1, Lq, M, K))
        loc[..., l, :, 1] = RNG.uniform(0.5 / h, (h - 0.5) / h, size=(1, Lq, M, K))
    A = RNG.uniform(0, 1, size=(1, Lq, M, 2, K))
    out = oracle.forward(value, shapes, loc, A).reshape(1, Lq, M, D)
    expect = float(c) * A.sum(axis=(-1, -2))
    np.testing.assert_allclose(out, np.repeat(expect[..., None], D, -1), rtol=1e-14, atol=0)


def test_integer_centres_return_the_pixel():
    """A location at a pixel centre ((w+0.5)/W, (h+0.5)/H) returns that pixel
    exactly when W and H are powers of two (the fp32 centre is exact)."""
    shapes = np.array([[8, 8], [4, 4]], dtype=np.int64)
    S = 80
    M, D = 2, 5
    value = RNG.uniform(-1, 1, size=(1, S, M, D)).astype(np.float32)
    starts = [0, 64]
    locs, expect = [], []
    for l, (h, w) in enumerate(shapes):
        for yy in range(h):
            for xx in range(w):
                locs.append(((xx + 0.5) / w, (yy + 0.5) / h, l))
                expect.append(value[0, starts[l] + yy * w + xx])
    Lq = len(locs)
    loc = np.zeros((1, Lq, M, 2, 1, 2), np.float32)
    A = np.zeros((1, Lq, M, 2, 1))
    for q, (x, y, l) in enumerate(locs):
        loc[0, q, :, :, 0] = (x, y)  # same point on both levels ...
        A[0, q, :, l, 0] = 1.0  # ... but only level l counts
    out = oracle.forward(value, shapes, loc, A).reshape(Lq, M, D)
    np.testing.assert_array_equal(out, np.array(expect, dtype=np.float64))


def _bilinear_field(h, w, M, D, rng):
    """v(h, w) = a + b*w + c*h + e*w*h per (head, channel), integer-valued
    coefficients scaled by 1/8 so the stored fp32 values are exact."""
    a, b, c, e = (rng.integers(-8, 9, size=(4, M, D)) / 8.0)
    hh, ww = np.meshgrid(np.arange(h, dtype=np.float64), np.arange(w, dtype=np.float64),
                         indexing="ij")
    v = (a + b * ww[..., None, None] + c * hh[..., None, None]
         + e * (ww * hh)[..., None, None])
    return v.reshape(1, h * w, M, D).astype(np.float32), (a, b, c, e)


def test_bilinear_field_is_reproduced_and_its_gradient_closed_form():
    """Bilinear interpolation reproduces a bilinear field v = a + b x + c y +
    e x y exactly, so for interior samples out = A * v(x, y) and
    d out/d loc_x = A * W * (b + e y), d out/d loc_y = A * H * (c + e x)."""
    h, w, M, D, K, Lq = 6, 10, 2, 3, 5, 7
    rng = np.random.default_rng(7)
    value, (a, b, c, e) = _bilinear_field(h, w, M, D, rng)
    assert np.array_equal(value.astype(np.float64).reshape(h, w, M, D),
                          value.reshape(h, w, M, D))
    shapes = np.array([[h, w]], dtype=np.int64)
    loc = np.empty((1, Lq, M, 1, K, 2))
    loc[..., 0] = rng.uniform(0.5 / w, (w - 0.5) / w, size=(1, Lq, M, 1, K))
    loc[..., 1] = rng.uniform(0.5 / h, (h - 0.5) / h, size=(1, Lq, M, 1, K))
    A = rng.uniform(0, 1, size=(1, Lq, M, 1, K))
    g = rng.standard_normal((1, Lq, M * D))
    out = oracle.forward(value, shapes, loc, A, loc_f32=False).reshape(Lq, M, D)
    x = loc[0, :, :, 0, :, 0] * w - 0.5  # [Lq, M, K]
    y = loc[0, :, :, 0, :, 1] * h - 0.5
    Av = A[0, :, :, 0, :]
    field = (a[None, :, None, :] + b[None, :, None, :] * x[..., None]
             + c[None, :, None, :] * y[..., None] + e[None, :, None, :] * (x * y)[..., None])
    expect = (Av[..., None] * field).sum(axis=2)
    np.testing.assert_allclose(out, expect, rtol=1e-12, atol=1e-12)
    _, gl, _ = oracle.backward(value, shapes, loc, A, g, loc_f32=False)
    gg = g.reshape(Lq, M, D)
    dx = Av * w * np.einsum("qmd,qmkd->qmk", gg, b[None, :, None, :] + e[None, :, None, :] * y[..., None])
    dy = Av * h * np.einsum("qmd,qmkd->qmk", gg, c[None, :, None, :] + e[None, :, None, :] * x[..., None])
    np.testing.assert_allclose(gl[0, :, :, 0, :, 0], dx, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(gl[0, :, :, 0, :, 1], dy, rtol=1e-10, atol=1e-10)


# --------------------------------------------------------------------------
# Special cases that reduce to library routines / textbook operations
# --------------------------------------------------------------------------
def test_single_point_equals_grid_sample():
    """L = K = 1 with unit weight is plain bilinear sampling (the
    deformable-convolution degenerate case, "Deformable DETR" wiki page,
    "Multi-scale deformable attention"): per head it equals
    torch.nn.functional.grid_sample(align_corners=False, padding_mode='zeros')
    with grid = 2*loc - 1, including samples that leave the map."""
    torch = pytest.importorskip("torch")
    h, w, M, D, Lq = 9, 13, 3, 4, 50
    rng = np.random.default_rng(11)
    value = rng.uniform(-1, 1, size=(1, h * w, M, D)).astype(np.float32)
    loc = rng.uniform(-0.1, 1.1, size=(1, Lq, M, 1, 1, 2))
    A = np.ones((1, Lq, M, 1, 1))
    out = oracle.forward(value, np.array([[h, w]]), loc, A, loc_f32=False).reshape(Lq, M, D)
    img = torch.from_numpy(value.astype(np.float64).reshape(h, w, M, D)).permute(2, 3, 0, 1)
    grid = torch.from_numpy(2.0 * loc[0, :, :, 0, 0, :] - 1.0).permute(1, 0, 2)[:, :, None, :]
    ref = torch.nn.functional.grid_sample(img, grid, mode="bilinear", padding_mode="zeros",
                                          align_corners=False)  # [M, D, Lq, 1]
    ref = ref[..., 0].permute(2, 0, 1).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_multi_level_equals_weighted_grid_samples():
    """Several levels and points: the sum over (l, k) of A times per-level
    grid_sample results (the multi-scale equation read term by term)."""
    torch = pytest.importorskip("torch")
    d = wl.make_inputs(wl.TINY)
    shapes = d["spatial_shapes"]
    value = d["value"]
    loc = d["sampling_locations"].astype(np.float64)
    A = oracle.softmax(d["logits"])
    N, Lq, M, L, K, _ = loc.shape
    D = value.shape[-1]
    out = oracle.forward(value, shapes, loc, A, loc_f32=False).reshape(N, Lq, M, D)
    starts, _ = oracle.level_start_index(shapes)
    ref = np.zeros((N, Lq, M, D))
    for l, (h, w) in enumerate(shapes):
        img = torch.from_numpy(value[0, starts[l]:starts[l] + h * w].astype(np.float64)
                               .reshape(h, w, M, D)).permute(2, 3, 0, 1)
        for k in range(K):
            grid = torch.from_numpy(2.0 * loc[0, :, :, l, k, :] - 1.0).permute(1, 0, 2)[:, :, None, :]
            s = torch.nn.functional.grid_sample(img, grid, mode="bilinear",
                                                padding_mode="zeros", align_corners=False)
            s = s[..., 0].permute(2, 0, 1).numpy()  # [Lq, M, D]
            ref[0] += A[0, :, :, l, k][..., None] * s
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_points_on_every_pixel_is_dense_attention():
    """With a sampling point on every location the module reduces to ordinary
    attention ("Deformable DETR" wiki page, "Multi-scale deformable
    attention"): K = H*W points on the pixel centres of a power-of-two map
    give out[m] = A[m] @ V[:, m, :], a plain matrix-vector product."""
    h, w, M, D, Lq = 4, 8, 2, 3, 5
    rng = np.random.default_rng(3)
    value = rng.uniform(-1, 1, size=(1, h * w, M, D)).astype(np.float32)
    K = h * w
    loc = np.zeros((1, Lq, M, 1, K, 2), np.float32)
    for yy in range(h):
        for xx in range(w):
            loc[..., 0, yy * w + xx, :] = ((xx + 0.5) / w, (yy + 0.5) / h)
    logits = rng.standard_normal((1, Lq, M, 1, K)).astype(np.float32)
    A = oracle.softmax(logits)
    out = oracle.forward(value, np.array([[h, w]]), loc, A).reshape(Lq, M, D)
    V = value[0].astype(np.float64)  # [HW, M, D]
    expect = np.stack([A[0, :, m, 0, :] @ V[:, m, :] for m in range(M)], axis=1)
    np.testing.assert_allclose(out, expect, rtol=1e-13, atol=1e-14)


def test_softmax_properties():
    """sum_l sum_k A = 1 and A in [0, 1] ("Deformable DETR" wiki page,
    "Multi-scale deformable attention"); invariant to a shift of all logits;
    equal logits give 1/(LK) (the initialisation in "Hyperparameters");
    agrees with scipy.special.softmax over the joint (L, K) axes."""
    scipy_special = pytest.importorskip("scipy.special")
    z = RNG.standard_normal((3, 5, 4, 4, 4)) * 3
    A = oracle.softmax(z)
    assert np.all(A >= 0) and np.all(A <= 1)
    np.testing.assert_allclose(A.sum(axis=(-1, -2)), 1.0, rtol=0, atol=1e-14)
    np.testing.assert_allclose(oracle.softmax(z + 123.25), A, rtol=1e-12, atol=1e-15)
    flat = z.reshape(3, 5, 4, 16)
    np.testing.assert_allclose(A.reshape(3, 5, 4, 16),
                               scipy_special.softmax(flat, axis=-1), rtol=1e-13, atol=1e-16)
    same = oracle.softmax(np.full((2, 3, 8, 4, 4), 0.37))
    np.testing.assert_allclose(same, 1.0 / 16, rtol=0, atol=1e-16)
    # the 3MK projection's head split: each head normalises on its own
    big = np.zeros((1, 1, 2, 1, 4))
    big[0, 0, 0, 0, 0] = 50.0
    Ab = oracle.softmax(big)
    np.testing.assert_allclose(Ab[0, 0, 1], 0.25, rtol=0, atol=1e-16)


def test_locations_zero_offset_and_exact_steps():
    """Zero pixel offset returns the reference point bit for bit; an offset
    of j*W_l pixels moves the point by exactly j in normalised units (the
    level rescaling phi_l and the added offset, "Deformable DETR" wiki page,
    "Multi-scale deformable attention")."""
    shapes = np.array([[100, 134], [50, 67], [13, 17]], dtype=np.int64)
    N, Lq, M, L, K = 2, 9, 3, 3, 2
    ref = RNG.uniform(0, 1, size=(N, Lq, 2)).astype(np.float32)
    off = np.zeros((N, Lq, M, L, K, 2), np.float32)
    loc = oracle.locations_f32(ref, off, shapes)
    np.testing.assert_array_equal(loc, np.broadcast_to(ref[:, :, None, None, None, :], loc.shape))
    for l, (h, w) in enumerate(shapes):
        off[..., l, :, 0] = 2.0 * w
        off[..., l, :, 1] = -1.0 * h
    loc = oracle.locations_f32(ref, off, shapes)
    expx = (ref[..., 0].astype(np.float64) + 2.0).astype(np.float32)
    expy = (ref[..., 1].astype(np.float64) - 1.0).astype(np.float32)
    np.testing.assert_array_equal(loc[..., 0], np.broadcast_to(expx[:, :, None, None, None], loc.shape[:-1]))
    np.testing.assert_array_equal(loc[..., 1], np.broadcast_to(expy[:, :, None, None, None], loc.shape[:-1]))
    # fp64 variant: pixel offset d moves x by exactly d pixels at any level
    off64 = RNG.standard_normal((N, Lq, M, L, K, 2))
    loc64 = oracle.locations_f64(ref.astype(np.float64), off64, shapes)
    for l, (h, w) in enumerate(shapes):
        px = loc64[..., l, :, 0] * w - ref[:, :, None, None, 0] * w
        np.testing.assert_allclose(px, off64[..., l, :, 0], rtol=0, atol=1e-11)


def test_box_locations():
    """Box references: zero offset gives the box centre bit for bit, and an
    offset of +-1/2 box unit lands on the box edges (dyadic boxes keep every
    step exact) -- the iterative-refinement reading that offsets are scaled
    by the previous box's width and height ("Deformable DETR" wiki page,
    "Variants")."""
    N, Lq, M, L, K = 2, 5, 3, 2, 4
    cx = RNG.integers(8, 56, size=(N, Lq)) / 64.0
    cy = RNG.integers(8, 56, size=(N, Lq)) / 64.0
    w = RNG.integers(1, 8, size=(N, Lq)) / 32.0
    h = RNG.integers(1, 8, size=(N, Lq)) / 32.0
    box = np.stack([cx, cy, w, h], axis=-1).astype(np.float32)
    off = np.zeros((N, Lq, M, L, K, 2), np.float32)
    loc = oracle.locations_box_f32(box, off)
    np.testing.assert_array_equal(loc, np.broadcast_to(box[:, :, None, None, None, :2], loc.shape))
    off[..., 0] = 0.5
    off[..., 1] = -0.5
    loc = oracle.locations_box_f32(box, off)
    np.testing.assert_array_equal(loc[..., 0], np.broadcast_to((cx + w / 2)[:, :, None, None, None], loc.shape[:-1]))
    np.testing.assert_array_equal(loc[..., 1], np.broadcast_to((cy - h / 2)[:, :, None, None, None], loc.shape[:-1]))
    # general offsets: within fp32 rounding of the exact map
    off = RNG.standard_normal(off.shape).astype(np.float32)
    loc = oracle.locations_box_f32(box, off)
    exact = box[:, :, None, None, None, :2].astype(np.float64) + off * box[:, :, None, None, None, 2:].astype(np.float64)
    np.testing.assert_allclose(loc, exact, rtol=0, atol=2e-7)


# --------------------------------------------------------------------------
# Independent brute-force formulation: tent kernels over every pixel
# --------------------------------------------------------------------------
def _tent_forward(value, shapes, loc32, A):
    """Bilinear interpolation with zero padding written as a sum over every
    pixel p of max(0, 1-|x-p_x|) * max(0, 1-|y-p_y|) * v[p] (textbook tent
    kernel form).  The pixel coordinate uses the same fp32 rounding of
    x = loc*W - 0.5 as the inputs are given in; everything after is fp64."""
    N, Lq, M, L, K, _ = loc32.shape
    D = value.shape[-1]
    out = np.zeros((N, Lq, M, D))
    start = 0
    for l, (h, w) in enumerate(shapes):
        x = (loc32[..., l, :, 0] * np.float32(w) - np.float32(0.5)).astype(np.float64)
        y = (loc32[..., l, :, 1] * np.float32(h) - np.float32(0.5)).astype(np.float64)
        px = np.arange(w, dtype=np.float64)
        py = np.arange(h, dtype=np.float64)
        tx = np.maximum(0.0, 1.0 - np.abs(x[..., None] - px))  # [N,Lq,M,K,W]
        ty = np.maximum(0.0, 1.0 - np.abs(y[..., None] - py))  # [N,Lq,M,K,H]
        tx = np.nan_to_num(tx, nan=0.0)
        ty = np.nan_to_num(ty, nan=0.0)
        V = value[:, start:start + h * w].astype(np.float64).reshape(N, h, w, M, D)
        wts = np.einsum("nqmk,nqmkh,nqmkw->nqmhw", A[..., l, :], ty, tx)
        out += np.einsum("nqmhw,nhwmd->nqmd", wts, V)
        start += h * w
    return out.reshape(N, Lq, M * D)


def test_forward_matches_tent_kernel_brute_force():
    for seed in range(3):
        d = wl.make_random_problem(seed, N=2, Lq=13, M=3, D=5, K=3,
                                   shapes=((5, 7), (3, 2), (1, 4)))
        loc = d["sampling_locations"]
        A = oracle.softmax(d["logits"])
        out = oracle.forward(d["value"], d["spatial_shapes"], loc, A)
        ref = _tent_forward(d["value"], d["spatial_shapes"], loc, A)
        np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_tiny_workload_matches_tent_kernel_brute_force():
    d = wl.make_inputs(wl.TINY)
    A = oracle.softmax(d["logits"])
    out = oracle.forward(d["value"], d["spatial_shapes"], d["sampling_locations"], A)
    ref = _tent_forward(d["value"], d["spatial_shapes"], d["sampling_locations"], A)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_sample_points_enumerated_by_brute_force():
    """Every sample of the tiny workload: the corners the oracle reports are
    exactly the pixels with non-zero tent weight, in (y0,x0) (y0,x0+1)
    (y0+1,x0) (y0+1,x0+1) order, and x0 <= x < x0+1."""
    d = wl.make_inputs(wl.TINY)
    loc = d["sampling_locations"]
    shapes = d["spatial_shapes"]
    sp = oracle.sample_points(loc, shapes)
    N, Lq, M, L, K, _ = loc.shape
    starts = [0, 64]
    i = 0
    for n in range(N):
        for q in range(Lq):
            for m in range(M):
                for l in range(L):
                    h, w = shapes[l]
                    for k in range(K):
                        x = float(np.float32(loc[n, q, m, l, k, 0]) * np.float32(w) - np.float32(0.5))
                        y = float(np.float32(loc[n, q, m, l, k, 1]) * np.float32(h) - np.float32(0.5))
                        nz = set()
                        for yy in range(h):
                            for xx in range(w):
                                if abs(x - xx) < 1 and abs(y - yy) < 1:
                                    nz.add(starts[l] + yy * w + xx)
                        inside = -1 < x < w and -1 < y < h
                        assert sp["valid"][i] == int(inside)
                        rows = sp["rows"][i]
                        assert sp["x"][i] == np.float32(x) and sp["y"][i] == np.float32(y)
                        if inside:
                            x0, y0 = sp["x0"][i], sp["y0"][i]
                            assert x0 <= x < x0 + 1 and y0 <= y < y0 + 1
                            for j, (dy, dx) in enumerate(((0, 0), (0, 1), (1, 0), (1, 1))):
                                yy, xx = y0 + dy, x0 + dx
                                want = starts[l] + yy * w + xx if (0 <= yy < h and 0 <= xx < w) else -1
                                assert rows[j] == want
                            # every non-zero-weight pixel is one of the corners
                            assert nz <= {r for r in rows if r >= 0}
                        else:
                            assert (rows == -1).all() and not nz
                        i += 1


def test_non_finite_and_far_locations_contribute_nothing():
    """NaN, +-Inf and far-away locations sample nothing (zero padding) and
    carry zero gradient."""
    shapes = np.array([[4, 4]], dtype=np.int64)
    value = RNG.uniform(-1, 1, size=(1, 16, 1, 2)).astype(np.float32)
    bad = [np.nan, np.inf, -np.inf, 1e30, -1e30, 2.0, -1.0]
    K = len(bad)
    loc = np.full((1, 1, 1, 1, K, 2), 0.5, np.float32)
    loc[0, 0, 0, 0, :, 0] = bad
    A = np.ones((1, 1, 1, 1, K))
    out = oracle.forward(value, shapes, loc, A)
    assert np.all(out == 0.0)
    g = np.ones((1, 1, 2))
    gv, gl, ga = oracle.backward(value, shapes, loc, A, g)
    assert np.all(gv == 0) and np.all(gl == 0) and np.all(ga == 0)


def test_edge_band_fades_to_zero():
    """Between the last pixel centre and the map edge the sample fades
    linearly to zero: at pixel x = W - 1 + t it equals (1 - t) * v[W-1]."""
    shapes = np.array([[1, 4]], dtype=np.int64)
    value = np.array([1.0, 2.0, 3.0, 5.0], np.float32).reshape(1, 4, 1, 1)
    for t in (0.0, 0.25, 0.5, 0.75):
        xpix = 3 + t
        loc = np.array([(xpix + 0.5) / 4, 0.5]).reshape(1, 1, 1, 1, 1, 2)
        out = oracle.forward(value, shapes, loc, np.ones((1, 1, 1, 1, 1)), loc_f32=False)
        assert abs(out.item() - (1 - t) * 5.0) < 1e-12
    loc = np.array([(-1 + 0.25 + 0.5) / 4, 0.5]).reshape(1, 1, 1, 1, 1, 2)
    out = oracle.forward(value, shapes, loc, np.ones((1, 1, 1, 1, 1)), loc_f32=False)
    assert abs(out.item() - 0.25 * 1.0) < 1e-12
