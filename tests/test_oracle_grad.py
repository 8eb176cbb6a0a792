"""Pins for the oracle's backward: adjoint identities (the forward is linear
in the value and in the weights) and central finite differences for the
location gradients and for the fused chain (offsets, reference points,
logits).  CPU only."""
import numpy as np

import oracle
from scale_deformable_attention_02_b200 import workloads as wl


def _kink_mask(loc, shapes, tol):
    """True where a sample sits within tol (pixels) of a cell boundary in x
    or y, where the interpolant has a kink and a finite difference is not a
    derivative."""
    mask = np.zeros(loc.shape[:-1], bool)
    for l, (h, w) in enumerate(shapes):
        x = loc[..., l, :, 0] * w - 0.5
        y = loc[..., l, :, 1] * h - 0.5
        fx = x - np.floor(x)
        fy = y - np.floor(y)
        near = (np.minimum(fx, 1 - fx) < tol) | (np.minimum(fy, 1 - fy) < tol)
        mask[..., l, :] = near
    return mask


def test_adjoint_value_and_weights():
    """<g, F(v', A)> = <dF/dv^T g, v'> for any v' (F is linear in v), and
    <g, F(v, A')> = <dF/dA^T g, A'> for any A' (F is linear in A)."""
    for seed in range(3):
        d = wl.make_random_problem(seed, N=2, Lq=9, M=3, D=4, K=3,
                                   shapes=((6, 5), (3, 3), (2, 1)))
        shapes, value = d["spatial_shapes"], d["value"]
        loc = d["sampling_locations"]
        A = oracle.softmax(d["logits"])
        g = d["grad_out"].astype(np.float64)
        gv, gl, ga = oracle.backward(value, shapes, loc, A, g)
        rng = np.random.default_rng(100 + seed)
        v2 = rng.uniform(-1, 1, size=value.shape).astype(np.float32)
        lhs = np.sum(g * oracle.forward(v2, shapes, loc, A))
        rhs = np.sum(gv * v2.astype(np.float64))
        assert abs(lhs - rhs) <= 1e-12 * (1 + abs(lhs))
        A2 = rng.uniform(-1, 1, size=A.shape)
        lhs = np.sum(g * oracle.forward(value, shapes, loc, A2))
        rhs = np.sum(ga * A2)
        assert abs(lhs - rhs) <= 1e-12 * (1 + abs(lhs))


def test_adjoint_on_tiny_workload_bf16_value():
    d = wl.make_random_problem(5, N=1, Lq=16, M=2, D=8, K=2, shapes=wl.TINY_SHAPES,
                               value_dtype="bf16")
    shapes = d["spatial_shapes"]
    A = oracle.softmax(d["logits"])
    g = d["grad_out"].astype(np.float64)
    out_bits = oracle.forward(d["value"], shapes, d["sampling_locations"], A)
    out_f32 = oracle.forward(d["value_f32"], shapes, d["sampling_locations"], A)
    np.testing.assert_array_equal(out_bits, out_f32)  # bf16 widening is exact
    gv, _, ga = oracle.backward(d["value"], shapes, d["sampling_locations"], A, g)
    assert abs(np.sum(g * out_bits) - np.sum(ga * A)) < 1e-12


def _fd_check_loc(value, shapes, loc64, A, g, h=1e-6, kink_tol=1e-3):
    _, gl, _ = oracle.backward(value, shapes, loc64, A, g, loc_f32=False)
    skip = _kink_mask(loc64, shapes, kink_tol)
    idx = np.argwhere(~skip)
    assert len(idx) > 0
    checked = 0
    for ii in idx:
        ii = tuple(ii)
        for c in range(2):
            lp = loc64.copy()
            lm = loc64.copy()
            lp[ii + (c,)] += h
            lm[ii + (c,)] -= h
            fp = np.sum(g * oracle.forward(value, shapes, lp, A, loc_f32=False))
            fm = np.sum(g * oracle.forward(value, shapes, lm, A, loc_f32=False))
            fd = (fp - fm) / (2 * h)
            an = gl[ii + (c,)]
            assert abs(fd - an) <= 1e-6 * (1 + abs(an)), (ii, c, fd, an)
            checked += 1
    return checked


def test_finite_differences_location_gradient_tiny():
    """Central differences of <g, out> in every location coordinate of the
    tiny workload (fp64 oracle), away from cell-boundary kinks.  The
    interpolant is linear in x inside a cell, so the difference is exact up
    to rounding."""
    d = wl.make_inputs(wl.TINY)
    loc64 = d["sampling_locations"].astype(np.float64)
    A = oracle.softmax(d["logits"])
    g = d["grad_out"].astype(np.float64)
    n = _fd_check_loc(d["value"], d["spatial_shapes"], loc64, A, g)
    assert n >= 200  # 128 samples x 2 coordinates, minus kinks


def test_finite_differences_location_gradient_encoder_subsample():
    """Same check on encoder-shaped problems (D = 32, 4 levels of the
    encoder shapes) for a handful of queries; the other queries are removed
    because they do not affect the chosen queries' outputs."""
    d = wl.make_inputs(wl.ENCODER_BWD)
    rng = np.random.default_rng(44)
    qs = np.sort(rng.choice(wl.ENCODER_BWD.queries, size=6, replace=False))
    loc32 = oracle.locations_f32(d["reference_points"][:1, qs], d["offsets"][:1, qs],
                                 d["spatial_shapes"])
    A = oracle.softmax(d["logits"][:1, qs])
    g = d["grad_out"][:1, qs].astype(np.float64)
    # only one batch entry's value matters for batch entry 0
    value = np.ascontiguousarray(d["value"][:1])
    n = _fd_check_loc(value, d["spatial_shapes"], loc32.astype(np.float64), A, g)
    assert n > 6 * 8 * 16


def test_finite_differences_fused_chain():
    """The chain from sampled-point gradients to the fused inputs: central
    differences of <g, F(ref, off, logits)> with F composed in fp64."""
    d = wl.make_random_problem(9, N=1, Lq=3, M=2, D=3, K=2,
                               shapes=((5, 6), (3, 4)), offset_std=1.0)
    shapes, value = d["spatial_shapes"], d["value"]
    ref = d["reference_points"].astype(np.float64)
    off = d["offsets"].astype(np.float64)
    z = d["logits"].astype(np.float64)
    g = d["grad_out"].astype(np.float64)

    def F(ref_, off_, z_):
        loc = oracle.locations_f64(ref_, off_, shapes)
        return np.sum(g * oracle.forward(value, shapes, loc, oracle.softmax(z_), loc_f32=False))

    loc = oracle.locations_f64(ref, off, shapes)
    A = oracle.softmax(z)
    _, gl, ga = oracle.backward(value, shapes, loc, A, g, loc_f32=False)
    g_ref, g_off, g_z = oracle.fused_chain(gl, ga, A, shapes)
    h = 1e-6
    skip = _kink_mask(loc, shapes, 1e-3)
    for ii in np.ndindex(*off.shape[:-1]):
        if skip[ii]:
            continue
        for c in range(2):
            p, m = off.copy(), off.copy()
            p[ii + (c,)] += h
            m[ii + (c,)] -= h
            fd = (F(ref, p, z) - F(ref, m, z)) / (2 * h)
            assert abs(fd - g_off[ii + (c,)]) <= 1e-6 * (1 + abs(fd))
    for ii in np.ndindex(*z.shape):
        p, m = z.copy(), z.copy()
        p[ii] += h
        m[ii] -= h
        fd = (F(ref, off, p) - F(ref, off, m)) / (2 * h)
        assert abs(fd - g_z[ii]) <= 1e-6 * (1 + abs(fd))
    # moving the reference moves every sample by ~1e-5 px: only samples within
    # 1e-4 px of a cell boundary could cross a kink
    assert not _kink_mask(loc, shapes, 1e-4).any()
    for ii in np.ndindex(*ref.shape):
        p, m = ref.copy(), ref.copy()
        p[ii] += h
        m[ii] -= h
        fd = (F(p, off, z) - F(m, off, z)) / (2 * h)
        assert abs(fd - g_ref[ii]) <= 1e-6 * (1 + abs(fd))


def test_backward_mass_bounds_the_sums():
    """The absolute masses bound the gradients (|sum| <= sum of |terms|) and
    equal them when every term has the same sign (non-negative value and
    upstream gradient make every <v_j, g> >= 0, so grad_attn = its mass)."""
    d = wl.make_random_problem(21, N=1, Lq=7, M=2, D=4, K=3, shapes=((5, 6), (3, 3)))
    sh, loc = d["spatial_shapes"], d["sampling_locations"]
    A = oracle.softmax(d["logits"])
    _, gl, ga, mgl, mga = oracle.backward(d["value"], sh, loc, A, d["grad_out"], with_mass=True)
    assert np.all(np.abs(gl) <= mgl * (1 + 1e-12)) and np.all(np.abs(ga) <= mga * (1 + 1e-12))
    v = np.abs(d["value"])
    g = np.abs(d["grad_out"])
    _, _, ga2, _, mga2 = oracle.backward(v, sh, loc, A, g, with_mass=True)
    np.testing.assert_allclose(ga2, mga2, rtol=1e-13, atol=0)


def test_finite_differences_fused_chain_box():
    """Box references (cx, cy, w, h): central differences of <g, F(box, off,
    logits)> through loc = (cx, cy) + off * (w, h) match the chained
    gradients, including those of the box itself."""
    d = wl.make_random_problem(13, N=1, Lq=3, M=2, D=3, K=2,
                               shapes=((6, 7), (3, 4)), offset_std=0.3)
    shapes, value = d["spatial_shapes"], d["value"]
    rng = np.random.default_rng(14)
    box = np.concatenate([rng.uniform(0.3, 0.7, (1, 3, 2)), rng.uniform(0.1, 0.4, (1, 3, 2))],
                         axis=-1)
    off = d["offsets"].astype(np.float64)
    z = d["logits"].astype(np.float64)
    g = d["grad_out"].astype(np.float64)

    def F(box_, off_, z_):
        loc = oracle.locations_box_f64(box_, off_)
        return np.sum(g * oracle.forward(value, shapes, loc, oracle.softmax(z_), loc_f32=False))

    loc = oracle.locations_box_f64(box, off)
    A = oracle.softmax(z)
    _, gl, ga = oracle.backward(value, shapes, loc, A, g, loc_f32=False)
    g_box, g_off, g_z = oracle.fused_chain_box(gl, ga, A, box, off)
    skip = _kink_mask(loc, shapes, 1e-3)
    h = 1e-6
    for ii in np.ndindex(*off.shape[:-1]):
        if skip[ii]:
            continue
        for c in range(2):
            p_, m_ = off.copy(), off.copy()
            p_[ii + (c,)] += h
            m_[ii + (c,)] -= h
            fd = (F(box, p_, z) - F(box, m_, z)) / (2 * h)
            assert abs(fd - g_off[ii + (c,)]) <= 1e-6 * (1 + abs(fd))
    for ii in np.ndindex(*z.shape):
        p_, m_ = z.copy(), z.copy()
        p_[ii] += h
        m_[ii] -= h
        fd = (F(box, off, p_) - F(box, off, m_)) / (2 * h)
        assert abs(fd - g_z[ii]) <= 1e-6 * (1 + abs(fd))
    assert not _kink_mask(loc, shapes, 1e-4).any()
    for ii in np.ndindex(*box.shape):
        p_, m_ = box.copy(), box.copy()
        p_[ii] += h
        m_[ii] -= h
        fd = (F(p_, off, z) - F(m_, off, z)) / (2 * h)
        assert abs(fd - g_box[ii]) <= 1e-6 * (1 + abs(fd))


def test_finite_differences_grouped_locations():
    """Deformable groups: G groups of M/G heads share one set of locations.
    The gradient of a shared location is the sum over the group's heads of
    the per-head gradients (oracle.sum_groups); checked by central
    differences of <g, F(expand_groups(loc_g))> in every group coordinate."""
    d = wl.make_random_problem(61, N=1, Lq=5, M=4, D=4, K=2, shapes=((7, 6), (3, 4)))
    shapes = d["spatial_shapes"]
    G = 2
    loc_g = d["sampling_locations"][:, :, :G].astype(np.float64)
    A = oracle.softmax(d["logits"])
    g = d["grad_out"].astype(np.float64)
    loc_h = oracle.expand_groups(loc_g, 4)
    assert np.array_equal(loc_h[:, :, 1], loc_g[:, :, 0]) and np.array_equal(
        loc_h[:, :, 2], loc_g[:, :, 1])
    _, gl, _ = oracle.backward(d["value"], shapes, loc_h, A, g, loc_f32=False)
    gl_g = oracle.sum_groups(gl, G)
    assert gl_g.shape == loc_g.shape
    skip = _kink_mask(loc_h, shapes, 1e-3).reshape(1, 5, G, 2, 2, 2).any(axis=3)
    h = 1e-6
    checked = 0
    for ii in np.argwhere(~skip):
        ii = tuple(ii)
        for c in range(2):
            lp, lm = loc_g.copy(), loc_g.copy()
            lp[ii + (c,)] += h
            lm[ii + (c,)] -= h
            fp = np.sum(g * oracle.forward(d["value"], shapes, oracle.expand_groups(lp, 4), A,
                                           loc_f32=False))
            fm = np.sum(g * oracle.forward(d["value"], shapes, oracle.expand_groups(lm, 4), A,
                                           loc_f32=False))
            fd = (fp - fm) / (2 * h)
            assert abs(fd - gl_g[ii + (c,)]) <= 1e-6 * (1 + abs(fd)), (ii, c)
            checked += 1
    assert checked >= 40
    # one group per head is the ungrouped problem
    assert np.array_equal(oracle.sum_groups(gl, 4), gl)


def test_backward_without_grad_value_keeps_per_sample_gradients():
    """with_grad_value=False only drops the scatter: the per-sample
    gradients and their masses are the same numbers."""
    d = wl.make_random_problem(5, N=2, Lq=7, M=2, D=8, K=3, shapes=((5, 6), (3, 2)))
    A = oracle.softmax(d["logits"])
    full = oracle.backward(d["value"], d["spatial_shapes"], d["sampling_locations"], A,
                           d["grad_out"], with_mass=True)
    part = oracle.backward(d["value"], d["spatial_shapes"], d["sampling_locations"], A,
                           d["grad_out"], with_mass=True, with_grad_value=False)
    assert part[0] is None
    for a, b in zip(full[1:], part[1:]):
        np.testing.assert_array_equal(a, b)
