"""GPU parity: the CUDA path (called through the C ABI binding) against the
CPU oracle on the same seeded inputs, element by element.

Tolerances (|gpu - oracle| <= atol + rtol*|oracle|): fp32 outputs, weights
and the location and weight gradients (plain stores) 1e-5 / 1e-6; grad_value
(atomics) 1e-4 / 1e-5; the summed gradients also get the fp32 rounding bound
18 * 2^-24 * (sum of absolute terms), which matters only where the sum
cancels; the integer side of the path
(pixel coordinate, cell, corner rows) and the fused sampling locations bit
for bit.  Oracle inputs never come from the GPU: locations and weights that
the unfused entry points take are produced by the oracle from the generator's
raw inputs."""
import numpy as np
import pytest
import torch

import oracle
from scale_deformable_attention_02_b200 import (msda_backward, msda_debug_sample_points,
                                                msda_forward, msda_forward_fused)
from scale_deformable_attention_02_b200 import workloads as wl

from gpu_util import (F32, GRAD, PLAIN, assert_bits_equal, assert_close, cached_inputs, host,
                      to_dev, value_grad_terms)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def _unfused_inputs(d):
    """fp32 locations and weights for the unfused entry points, made by the
    oracle from the raw inputs (softmax rounded once to fp32)."""
    if "sampling_locations" in d:
        loc = d["sampling_locations"]
    else:
        loc = oracle.locations_f32(d["reference_points"], d["offsets"], d["spatial_shapes"])
    A = oracle.softmax(d["logits"]).astype(np.float32)
    return loc, A


# ---------------------------------------------------------------------------
# tiny workload: N=1, M=2, D=8, L=2 (8x8, 4x4), K=2, Lq=16
# ---------------------------------------------------------------------------
def test_tiny_forward_backward():
    d = wl.make_inputs(wl.TINY)
    loc, A = _unfused_inputs(d)
    sh = d["spatial_shapes"]
    out = msda_forward(to_dev(d["value"]), sh, None, to_dev(loc), to_dev(A))
    ora = oracle.forward(d["value"], sh, loc, A)
    assert_close(host(out), ora, **F32, what="tiny out")
    gv, gl, ga = msda_backward(to_dev(d["value"]), sh, None, to_dev(loc), to_dev(A),
                               to_dev(d["grad_out"]))
    ogv, ogl, oga, mgl, mga = oracle.backward(d["value"], sh, loc, A, d["grad_out"],
                                              with_mass=True)
    tv, mv = value_grad_terms(d["value"], sh, loc, A, d["grad_out"])
    assert_close(host(gv), ogv, **GRAD, what="tiny grad_value", mass=mv, terms=tv)
    assert_close(host(gl), ogl, **PLAIN, what="tiny grad_loc", mass=mgl)
    assert_close(host(ga), oga, **PLAIN, what="tiny grad_attn", mass=mga)


def test_tiny_fused_with_zero_offsets_equals_unfused():
    d = wl.make_inputs(wl.TINY)
    sh = d["spatial_shapes"]
    loc = d["sampling_locations"]
    N, Lq, M, L, K, _ = loc.shape
    # a point reference per query and zero offsets reproduce loc exactly only
    # if all of a query's samples share one point: use sample (0,0,0) as ref
    ref = np.ascontiguousarray(loc[:, :, 0, 0, 0, :])
    off = np.zeros_like(loc)
    out, loc_o, a_o = msda_forward_fused(to_dev(d["value"]), sh, None, to_dev(ref),
                                         to_dev(off), to_dev(d["logits"]),
                                         return_sampling=True)
    expect_loc = np.broadcast_to(ref[:, :, None, None, None, :], loc.shape)
    assert_bits_equal(host(loc_o), expect_loc, what="fused loc")
    A = oracle.softmax(d["logits"])
    assert_close(host(a_o), A, **F32, what="fused softmax")
    ora = oracle.forward(d["value"], sh, np.ascontiguousarray(expect_loc), A)
    assert_close(host(out), ora, **F32, what="fused out")
    out2 = msda_forward(to_dev(d["value"]), sh, None, loc_o, a_o)
    assert torch.equal(out, out2), "fused and unfused forward differ on identical inputs"


# ---------------------------------------------------------------------------
# index arithmetic, bit for bit
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("name", ["tiny", "decoder", "encoder", "stress"])
def test_cell_arithmetic_bit_exact(name):
    w = wl.WORKLOADS[name]
    d = wl.make_inputs(w, with_grad=False)
    if name == "stress":  # two of eight batch entries keep the test short
        for k in ("reference_points", "offsets"):
            d[k] = np.ascontiguousarray(d[k][:2])
    loc, _ = _unfused_inputs({**d, "logits": d["logits"][:1, :1]})
    sh = d["spatial_shapes"]
    g = msda_debug_sample_points(sh, None, to_dev(loc))
    o = oracle.sample_points(loc, sh)
    for k in ("valid", "x0", "y0", "x", "y", "rows"):
        assert_bits_equal(host(g[k]), o[k], what=f"{name} {k}")


# ---------------------------------------------------------------------------
# decoder-shaped fused forward (N=2, Lq=300, M=8, D=32, L=4, K=4)
# ---------------------------------------------------------------------------
def test_decoder_fused_forward():
    d = wl.make_inputs(wl.DECODER, with_grad=False)
    sh = d["spatial_shapes"]
    out, loc_o, a_o = msda_forward_fused(to_dev(d["value"]), sh, None,
                                         to_dev(d["reference_points"]), to_dev(d["offsets"]),
                                         to_dev(d["logits"]), return_sampling=True)
    ora, oloc, oA = oracle.forward_fused(d["value"], sh, d["reference_points"], d["offsets"],
                                         d["logits"])
    assert_bits_equal(host(loc_o), oloc, what="decoder loc")
    assert_close(host(a_o), oA, **F32, what="decoder softmax")
    assert_close(host(out), ora, **F32, what="decoder out")


# ---------------------------------------------------------------------------
# encoder-shaped fused forward, fp32 and bf16 value (N=2, Lq=S=17821)
# ---------------------------------------------------------------------------
def test_encoder_fused_forward_fp32():
    d = wl.make_inputs(wl.ENCODER, with_grad=False)
    sh = d["spatial_shapes"]
    out, loc_o, a_o = msda_forward_fused(to_dev(d["value"]), sh, None,
                                         to_dev(d["reference_points"]), to_dev(d["offsets"]),
                                         to_dev(d["logits"]), return_sampling=True)
    ora, oloc, oA = oracle.forward_fused(d["value"], sh, d["reference_points"], d["offsets"],
                                         d["logits"])
    assert_bits_equal(host(loc_o), oloc, what="encoder loc")
    assert_close(host(a_o), oA, **F32, what="encoder softmax")
    assert_close(host(out), ora, **F32, what="encoder out")


def test_encoder_compass_fused_forward_and_backward():
    """The encoder at the compass initialisation (uniform weights, every head
    k pixels along its own direction): a highly regular access pattern."""
    d = wl.make_inputs(wl.ENCODER_COMPASS)
    sh = d["spatial_shapes"]
    out, loc_o, a_o = msda_forward_fused(to_dev(d["value"]), sh, None,
                                         to_dev(d["reference_points"]), to_dev(d["offsets"]),
                                         to_dev(d["logits"]), return_sampling=True)
    ora, oloc, oA = oracle.forward_fused(d["value"], sh, d["reference_points"], d["offsets"],
                                         d["logits"])
    assert_bits_equal(host(loc_o), oloc, what="compass loc")
    assert np.all(host(a_o) == np.float32(1.0 / 16))  # exp(0)/16 is exact
    assert_close(host(out), ora, **F32, what="compass out")
    A = oA.astype(np.float32)
    gv, gl, ga = msda_backward(to_dev(d["value"]), sh, None, to_dev(oloc), to_dev(A),
                               to_dev(d["grad_out"]))
    ogv, ogl, oga, mgl, mga = oracle.backward(d["value"], sh, oloc, A, d["grad_out"],
                                              with_mass=True)
    tv, mv = value_grad_terms(d["value"], sh, oloc, A, d["grad_out"])
    assert_close(host(gv), ogv, **GRAD, what="compass grad_value", mass=mv, terms=tv)
    assert_close(host(gl), ogl, **PLAIN, what="compass grad_loc", mass=mgl)
    assert_close(host(ga), oga, **PLAIN, what="compass grad_attn", mass=mga)


def test_encoder_fused_forward_bf16():
    d = wl.make_inputs(wl.ENCODER_BF16, with_grad=False)
    sh = d["spatial_shapes"]
    out = msda_forward_fused(to_dev(d["value"]), sh, None, to_dev(d["reference_points"]),
                             to_dev(d["offsets"]), to_dev(d["logits"]))
    got = host(out)
    # strict: the same bf16 bits on both sides, fp32 tolerance
    ora, _, _ = oracle.forward_fused(d["value"], sh, d["reference_points"], d["offsets"],
                                     d["logits"])
    assert_close(got, ora, **F32, what="encoder bf16 (same bits)")
    # against the fp32-value oracle: 2e-2 relative, with an absolute floor of
    # 2e-2 x the rms output (rounding to bf16 moves a term by up to 2^-9 of
    # itself, so the error scales with the magnitude of the terms, not of
    # their sum)
    d32 = wl.make_inputs(wl.ENCODER, with_grad=False)
    ora32, _, _ = oracle.forward_fused(d32["value"], sh, d32["reference_points"],
                                       d32["offsets"], d32["logits"])
    rms = float(np.sqrt(np.mean(ora32 ** 2)))
    assert_close(got, ora32, rtol=2e-2, atol=2e-2 * rms, what="encoder bf16 vs fp32 value")


# ---------------------------------------------------------------------------
# encoder-shaped backward (fp32)
# ---------------------------------------------------------------------------
def test_encoder_backward():
    d = wl.make_inputs(wl.ENCODER_BWD)
    sh = d["spatial_shapes"]
    loc, A = _unfused_inputs(d)
    gv, gl, ga = msda_backward(to_dev(d["value"]), sh, None, to_dev(loc), to_dev(A),
                               to_dev(d["grad_out"]))
    ogv, ogl, oga, mgl, mga = oracle.backward(d["value"], sh, loc, A, d["grad_out"],
                                              with_mass=True)
    tv, mv = value_grad_terms(d["value"], sh, loc, A, d["grad_out"])
    assert_close(host(gv), ogv, **GRAD, what="encoder grad_value", mass=mv, terms=tv)
    assert_close(host(gl), ogl, **PLAIN, what="encoder grad_loc", mass=mgl)
    assert_close(host(ga), oga, **PLAIN, what="encoder grad_attn", mass=mga)


# ---------------------------------------------------------------------------
# high-resolution stress: N=8, S=37150, K=8, bf16 value, 5% out of range
# ---------------------------------------------------------------------------
def test_stress_forward_backward():
    w = wl.STRESS
    d = cached_inputs("stress")
    sh = d["spatial_shapes"]
    value = to_dev(d["value"])
    out, loc_o, a_o = msda_forward_fused(value, sh, None, to_dev(d["reference_points"]),
                                         to_dev(d["offsets"]), to_dev(d["logits"]),
                                         return_sampling=True)
    gv, gl, ga = msda_backward(value, sh, None, loc_o, a_o, to_dev(d["grad_out"]))
    torch.cuda.synchronize()
    # every batch entry at once: out is linear in the value map, so
    # <grad_out, out> = <grad_value, value> (fp64 sums of the GPU's results)
    g64 = torch.from_numpy(d["grad_out"]).to(value.device).double()
    lhs = float((g64 * out.double()).sum())
    rhs = float((gv.double() * value.double()).sum())
    mass = float((g64 * out.double()).abs().sum() + (gv.double() * value.double()).abs().sum())
    assert abs(lhs - rhs) <= 1e-5 * mass, ("stress adjoint", lhs, rhs, mass)
    del g64
    # oracle on three of the eight batch entries (entries are independent)
    for n in (0, w.N // 2 - 1, w.N - 1):
        sl = slice(n, n + 1)
        ref, off, z = (np.ascontiguousarray(d[k][sl]) for k in
                       ("reference_points", "offsets", "logits"))
        v = np.ascontiguousarray(d["value"][sl])
        ora, oloc, oA = oracle.forward_fused(v, sh, ref, off, z)
        assert_bits_equal(host(loc_o[sl]), oloc, what=f"stress loc n={n}")
        assert_close(host(a_o[sl]), oA, **F32, what=f"stress softmax n={n}")
        assert_close(host(out[sl]), ora, **F32, what=f"stress out n={n}")
        A32 = oA.astype(np.float32)
        # the backward takes the GPU's fp32 weights; the oracle takes its own
        # fp32-rounded softmax: they agree to a few ulp, and the location
        # gradients are linear in the weight
        ogv, ogl, oga, mgl, mga = oracle.backward(v, sh, oloc, A32, d["grad_out"][sl],
                                                  with_mass=True)
        tv, mv = value_grad_terms(v, sh, oloc, A32, d["grad_out"][sl])
        assert_close(host(gv[sl]), ogv, **GRAD, what=f"stress grad_value n={n}", mass=mv,
                     terms=tv)
        assert_close(host(gl[sl]), ogl, **PLAIN, what=f"stress grad_loc n={n}", mass=mgl)
        assert_close(host(ga[sl]), oga, **PLAIN, what=f"stress grad_attn n={n}", mass=mga)
    # at least the pushed 5% of the samples leave their level
    valid = host(msda_debug_sample_points(sh, None, loc_o[:1])["valid"])
    assert 1.0 - valid.mean() > 0.05  # pushed 5% plus natural spill at coarse levels


# ---------------------------------------------------------------------------
# ragged sizes, every lane layout, edge cases
# ---------------------------------------------------------------------------
CASES = [
    # (N, Lq, M, D, K, shapes, dtype)
    (1, 1, 1, 4, 1, ((1, 1),), "f32"),            # smallest problem, R = 1
    (2, 37, 3, 8, 3, ((5, 7), (3, 2), (1, 4)), "f32"),  # R = 2, ragged warps
    (1, 50, 2, 24, 2, ((6, 9), (3, 5)), "f32"),   # 6 chunks: lanes 6,7 idle
    (3, 19, 4, 16, 4, ((9, 11), (4, 6)), "f32"),  # R = 4
    (1, 23, 2, 64, 2, ((8, 8), (4, 4)), "f32"),   # 256-B rows, R = 16
    (1, 9, 1, 128, 1, ((7, 5),), "f32"),          # 512-B rows, R = 32
    (2, 41, 8, 32, 4, ((10, 13), (5, 7), (3, 4), (2, 2)), "bf16"),
    (1, 33, 2, 8, 2, ((6, 6), (3, 3)), "bf16"),   # 16-B rows, R = 1
    (1, 17, 3, 256, 2, ((5, 4), (2, 3)), "bf16"),  # 512-B rows
    (1, 12, 2, 32, 16, ((6, 8), (3, 4)), "f32"),  # L*K = 32: every lane a sample
    (1, 12, 2, 32, 1, tuple((2 + i, 3) for i in range(32)), "f32"),  # L = 32 levels
    (2, 15, 2, 8, 2, ((0, 4), (3, 3), (5, 0)), "f32"),  # empty levels
    # more than 32 samples per (query, head): blocks of 32, up to 4 per lane
    (1, 9, 2, 32, 16, ((6, 8), (3, 4), (2, 2)), "f32"),          # L*K = 48
    (2, 13, 3, 16, 32, ((5, 7), (3, 3), (2, 2), (1, 1)), "f32"),  # L*K = 128, R = 4
    (1, 11, 2, 32, 10, ((6, 6), (3, 3), (2, 2), (1, 2), (1, 1)), "bf16"),  # L*K = 50
    (1, 7, 2, 64, 9, ((5, 5), (3, 3), (2, 2), (1, 1)), "f32"),    # wide rows, L*K = 36
    (1, 5, 1, 128, 33, ((4, 4),), "f32"),                         # 512-B rows, tail of 1
]


# Larger problems (16800 (query, head) items, several rounds per persistent
# warp): every lane layout of the fast kernels.
LARGE_CASES = [
    (1, 4200, 4, 4, 4, ((9, 11), (5, 6), (3, 3)), "f32"),    # R = 1
    (1, 4200, 4, 8, 4, ((9, 11), (5, 6), (3, 3)), "f32"),    # R = 2
    (1, 4200, 4, 16, 4, ((9, 11), (5, 6), (3, 3)), "f32"),   # R = 4
    (1, 2100, 8, 32, 2, ((12, 14), (6, 7)), "f32"),          # R = 8, L*K = 4
    (1, 4200, 4, 16, 4, ((9, 11), (5, 6), (3, 3)), "bf16"),  # 16-byte bf16 rows
]


@pytest.mark.parametrize("case", CASES + LARGE_CASES,
                         ids=[f"case{i}" for i in range(len(CASES))] +
                             [f"large{i}" for i in range(len(LARGE_CASES))])
def test_random_problems(case):
    N, Lq, M, D, K, shapes, dt = case
    d = wl.make_random_problem(1000 + len(shapes) * 7 + D, N=N, Lq=Lq, M=M, D=D, K=K,
                               shapes=shapes, value_dtype=dt)
    sh = d["spatial_shapes"]
    loc = d["sampling_locations"]
    A = oracle.softmax(d["logits"]).astype(np.float32)
    value = to_dev(d["value"])
    out = msda_forward(value, sh, None, to_dev(loc), to_dev(A))
    assert_close(host(out), oracle.forward(d["value"], sh, loc, A), **F32, what="forward")
    fo, floc, fa = msda_forward_fused(value, sh, None, to_dev(d["reference_points"]),
                                      to_dev(d["offsets"]), to_dev(d["logits"]),
                                      return_sampling=True)
    ora, oloc, oA = oracle.forward_fused(d["value"], sh, d["reference_points"], d["offsets"],
                                         d["logits"])
    assert_bits_equal(host(floc), oloc, what="fused loc")
    assert_close(host(fa), oA, **F32, what="fused softmax")
    assert_close(host(fo), ora, **F32, what="fused out")
    gv, gl, ga = msda_backward(value, sh, None, to_dev(loc), to_dev(A), to_dev(d["grad_out"]))
    ogv, ogl, oga, mgl, mga = oracle.backward(d["value"], sh, loc, A, d["grad_out"],
                                              with_mass=True)
    tv, mv = value_grad_terms(d["value"], sh, loc, A, d["grad_out"])
    assert_close(host(gv), ogv, **GRAD, what="grad_value", mass=mv, terms=tv)
    assert_close(host(gl), ogl, **PLAIN, what="grad_loc", mass=mgl)
    assert_close(host(ga), oga, **PLAIN, what="grad_attn", mass=mga)


def test_box_reference_variant():
    """Fused forward with 4-d box references (cx, cy, w, h): the locations
    are cx + off_x * w, cy + off_y * h, one fp32 multiply and one fp32 add
    each (iterative box refinement)."""
    d = wl.make_random_problem(77, N=2, Lq=29, M=4, D=16, K=4,
                               shapes=((12, 10), (6, 5), (3, 3)))
    sh = d["spatial_shapes"]
    rng = np.random.default_rng(78)
    box = np.concatenate([rng.uniform(0.1, 0.9, (2, 29, 2)),
                          rng.uniform(0.05, 0.5, (2, 29, 2))], axis=-1).astype(np.float32)
    off = (rng.standard_normal(d["offsets"].shape) * 0.25).astype(np.float32)
    out, loc_o, a_o = msda_forward_fused(to_dev(d["value"]), sh, None, to_dev(box),
                                         to_dev(off), to_dev(d["logits"]), return_sampling=True)
    oloc = oracle.locations_box_f32(box, off)
    assert_bits_equal(host(loc_o), oloc, what="box loc")
    A = oracle.softmax(d["logits"])
    assert_close(host(out), oracle.forward(d["value"], sh, oloc, A), **F32, what="box out")


def test_out_of_range_and_non_finite_locations():
    shapes = ((4, 4), (2, 2))
    d = wl.make_random_problem(5, N=1, Lq=8, M=2, D=8, K=4, shapes=shapes)
    loc = d["sampling_locations"].copy()
    loc[0, 0] = np.nan
    loc[0, 1, :, :, :, 0] = np.inf
    loc[0, 2, :, :, :, 1] = -np.inf
    loc[0, 3] = 7.5
    loc[0, 4] = -3.0
    loc[0, 5, :, 0, :, 0] = -0.124  # just inside the fade band of level 0 (x in (-1, 0))
    A = oracle.softmax(d["logits"]).astype(np.float32)
    sh = d["spatial_shapes"]
    out = msda_forward(to_dev(d["value"]), sh, None, to_dev(loc), to_dev(A))
    ora = oracle.forward(d["value"], sh, loc, A)
    assert_close(host(out), ora, **F32, what="edge out")
    assert np.all(host(out)[0, :5] == 0)
    gv, gl, ga = msda_backward(to_dev(d["value"]), sh, None, to_dev(loc), to_dev(A),
                               to_dev(d["grad_out"]))
    ogv, ogl, oga, mgl, mga = oracle.backward(d["value"], sh, loc, A, d["grad_out"],
                                              with_mass=True)
    tv, mv = value_grad_terms(d["value"], sh, loc, A, d["grad_out"])
    assert_close(host(gv), ogv, **GRAD, what="edge grad_value", mass=mv, terms=tv)
    assert_close(host(gl), ogl, **PLAIN, what="edge grad_loc", mass=mgl)
    assert_close(host(ga), oga, **PLAIN, what="edge grad_attn", mass=mga)


def test_empty_problems():
    value = torch.zeros(2, 80, 2, 8, device="cuda")
    for Lq in (0,):
        loc = torch.zeros(2, Lq, 2, 2, 2, 2, device="cuda")
        A = torch.zeros(2, Lq, 2, 2, 2, device="cuda")
        out = msda_forward(value, wl.TINY_SHAPES, None, loc, A)
        assert out.shape == (2, 0, 16)
        g = torch.zeros(2, Lq, 16, device="cuda")
        gv = torch.full((2, 80, 2, 8), 5.0, device="cuda")
        msda_backward(value, wl.TINY_SHAPES, None, loc, A, g, grad_value=gv)
        assert torch.count_nonzero(gv).item() == 0  # zeroed even with no queries


def test_forward_deterministic_and_stream_ordered():
    d = wl.make_inputs(wl.DECODER, with_grad=False)
    sh = d["spatial_shapes"]
    args = [to_dev(d[k]) for k in ("value", "reference_points", "offsets", "logits")]
    a = msda_forward_fused(args[0], sh, None, *args[1:])
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        b = msda_forward_fused(args[0], sh, None, *args[1:])
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_forward_lane_width_follows_value_alignment():
    """fp32 rows of 32 elements are gathered in 32-byte lanes when the value
    map is 32-byte aligned and in 16-byte lanes when it is only 16-byte
    aligned: both match the oracle."""
    shapes = ((12, 15), (6, 8), (3, 4), (2, 2))
    d = wl.make_random_problem(91, N=2, Lq=77, M=4, D=32, K=4, shapes=shapes)
    sh = d["spatial_shapes"]
    ref, off, z = (to_dev(d[k]) for k in ("reference_points", "offsets", "logits"))
    ora, _, _ = oracle.forward_fused(d["value"], sh, d["reference_points"], d["offsets"],
                                     d["logits"])
    flat = torch.from_numpy(d["value"]).reshape(-1)
    buf = torch.zeros(flat.numel() + 8, device="cuda")
    for shift in (0, 4):  # 0 or 16 bytes past a 32-byte aligned base
        assert buf.data_ptr() % 32 == 0
        v = buf[shift:shift + flat.numel()]
        v.copy_(flat.to("cuda"))
        value = v.view(d["value"].shape)
        assert (value.data_ptr() % 32 == 0) == (shift == 0)
        out = msda_forward_fused(value, sh, None, ref, off, z)
        assert_close(host(out), ora, **F32, what=f"forward, value at +{4 * shift} bytes")
