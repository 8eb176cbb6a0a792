"""GPU parity of the fused backward (gradients chained to the reference
points, the pixel offsets and the logits) against the oracle's backward
followed by its chain rule (pinned by finite differences on the CPU).

Bounds: PLAIN (1e-5 relative, 1e-6 absolute) for the offsets and logits,
which the kernel writes once per sample; GRAD (1e-4 relative, 1e-5 absolute)
for grad_value and the reference points, which are summed with atomics; each
plus the fp32 rounding bound of the chained quantity, built from the oracle's
absolute masses:
  offsets   point: mass(d loc) / W_l     box: mass(d loc) * (w, h)
  logits    A_s (m_s + sum_j A_j m_j + sum_j A_j |dA_j|)  with m = mass(dA)
  reference sum over the query's samples of mass(d loc) (+ |d loc|, for the
            atomic sums over heads); box scale terms weighted by |off|."""
import numpy as np
import pytest
import torch

import oracle
from scale_deformable_attention_02_b200 import msda_backward_fused, msda_forward_fused
from scale_deformable_attention_02_b200 import workloads as wl

from gpu_util import (GRAD, KAPPA, PLAIN, U32, assert_close, cached_inputs, host, to_dev,
                      value_grad_terms)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _check(d, ref, off, logits, box: bool, got=None):
    """The fused backward of d's inputs (or `got`, its results computed by the
    caller) against the oracle's backward and chain rule."""
    sh = d["spatial_shapes"]
    g = d["grad_out"]
    if got is None:
        got = msda_backward_fused(to_dev(d["value"]), sh, None, to_dev(ref), to_dev(off),
                                  to_dev(logits), to_dev(g))
    gv, gr, go, gz = got
    loc = oracle.locations_box_f32(ref, off) if box else oracle.locations_f32(ref, off, sh)
    A = oracle.softmax(logits)
    ogv, ogl, oga, mgl, mga = oracle.backward(d["value"], sh, loc, A.astype(np.float32), g,
                                              with_mass=True)
    if box:
        ogr, ogo, ogz = oracle.fused_chain_box(ogl, oga, A, ref, off)
        mgo = mgl * np.asarray(ref, np.float64)[:, :, None, None, None, 2:]
        mref = np.stack([(mgl[..., 0] + np.abs(ogl[..., 0])).sum(axis=(2, 3, 4)),
                         (mgl[..., 1] + np.abs(ogl[..., 1])).sum(axis=(2, 3, 4)),
                         ((mgl[..., 0] + np.abs(ogl[..., 0])) * np.abs(off[..., 0])).sum(axis=(2, 3, 4)),
                         ((mgl[..., 1] + np.abs(ogl[..., 1])) * np.abs(off[..., 1])).sum(axis=(2, 3, 4))],
                        axis=-1)
    else:
        ogr, ogo, ogz = oracle.fused_chain(ogl, oga, A, sh)
        Wl = sh[:, 1].astype(np.float64)[None, None, None, :, None]
        Hl = sh[:, 0].astype(np.float64)[None, None, None, :, None]
        mgo = np.stack([mgl[..., 0] / Wl, mgl[..., 1] / Hl], axis=-1)
        mref = (mgl + np.abs(ogl)).sum(axis=(2, 3, 4))
    LK = A.shape[-1] * A.shape[-2]
    Af = A.reshape(A.shape[:3] + (LK,))
    mz_head = (Af * (mga.reshape(Af.shape) + np.abs(oga.reshape(Af.shape)))).sum(-1, keepdims=True)
    mz = (Af * (mga.reshape(Af.shape) + mz_head)).reshape(A.shape)
    tv, mv = value_grad_terms(d["value"], sh, loc, A, g)
    assert_close(host(gv), ogv, **GRAD, what="grad_value", mass=mv, terms=tv)
    assert_close(host(go), ogo, **PLAIN, what="grad_offsets", mass=mgo)
    assert_close(host(gz), ogz, **PLAIN, what="grad_logits", mass=mz)
    assert_close(host(gr), ogr, **GRAD, what="grad_reference", mass=mref)


def test_fused_backward_point_random():
    d = wl.make_random_problem(31, N=2, Lq=45, M=4, D=32, K=4,
                               shapes=((16, 20), (8, 10), (4, 5), (2, 3)))
    _check(d, d["reference_points"], d["offsets"], d["logits"], box=False)


@pytest.mark.parametrize("D,dt", [(8, "f32"), (16, "f32"), (24, "f32"), (8, "bf16"),
                                  (32, "bf16"), (36, "f32"), (64, "f32"), (128, "f32"),
                                  (64, "bf16"), (256, "bf16")])
def test_fused_backward_widths(D, dt):
    d = wl.make_random_problem(40 + D, N=1, Lq=29, M=3, D=D, K=3,
                               shapes=((9, 11), (5, 6), (3, 3)), value_dtype=dt)
    _check(d, d["reference_points"], d["offsets"], d["logits"], box=False)


@pytest.mark.parametrize("K,shapes,dt,box", [
    (16, ((6, 8), (3, 4), (2, 2)), "f32", False),              # L*K = 48
    (32, ((5, 7), (3, 3), (2, 2), (1, 1)), "f32", False),      # L*K = 128
    (10, ((6, 6), (3, 3), (2, 2), (1, 2), (1, 1)), "bf16", False),  # L*K = 50
    (12, ((8, 8), (4, 4), (2, 2)), "f32", True),               # box, L*K = 36
])
def test_fused_backward_more_than_32_samples(K, shapes, dt, box):
    """Items of more than 32 samples: the joint softmax over all blocks of
    32, and the softmax Jacobian's sum taken over every block."""
    d = wl.make_random_problem(90 + K, N=2, Lq=11, M=3, D=16, K=K, shapes=shapes,
                               value_dtype=dt)
    ref, off = d["reference_points"], d["offsets"]
    if box:
        rng = np.random.default_rng(91)
        ref = np.concatenate([rng.uniform(0.1, 0.9, (2, 11, 2)),
                              rng.uniform(0.05, 0.5, (2, 11, 2))], axis=-1).astype(np.float32)
        off = (rng.standard_normal(off.shape) * 0.25).astype(np.float32)
    _check(d, ref, off, d["logits"], box=box)


def test_fused_backward_box():
    d = wl.make_random_problem(77, N=2, Lq=29, M=4, D=16, K=4,
                               shapes=((12, 10), (6, 5), (3, 3)))
    rng = np.random.default_rng(78)
    box = np.concatenate([rng.uniform(0.1, 0.9, (2, 29, 2)),
                          rng.uniform(0.05, 0.5, (2, 29, 2))], axis=-1).astype(np.float32)
    off = (rng.standard_normal(d["offsets"].shape) * 0.25).astype(np.float32)
    _check(d, box, off, d["logits"], box=True)


def test_fused_backward_decoder():
    d = wl.make_inputs(wl.DECODER)
    _check(d, d["reference_points"], d["offsets"], d["logits"], box=False)


def test_fused_backward_encoder():
    d = wl.make_inputs(wl.ENCODER_BWD)
    _check(d, d["reference_points"], d["offsets"], d["logits"], box=False)


def test_fused_backward_matches_fused_forward_sampling():
    """The backward recomputes locations and weights exactly as the fused
    forward forms them: with grad_out = e_c (one output channel), grad_logits
    and grad_offsets vanish for samples that do not touch that channel's
    head, and grad_value of the chosen head equals sum over samples of
    A * bilinear weights, which the forward's own A and locations give."""
    d = wl.make_random_problem(5, N=1, Lq=7, M=2, D=8, K=2, shapes=((6, 6), (3, 3)))
    sh = d["spatial_shapes"]
    value = to_dev(d["value"])
    ref, off, z = (to_dev(d[k]) for k in ("reference_points", "offsets", "logits"))
    out, loc, a = msda_forward_fused(value, sh, None, ref, off, z, return_sampling=True)
    g = torch.zeros_like(out)
    g[:, :, 0] = 1.0  # head 0, channel 0
    gv, gr, go, gz = msda_backward_fused(value, sh, None, ref, off, z, g)
    # head 1 receives no gradient at all
    assert torch.count_nonzero(gz[:, :, 1]).item() == 0
    assert torch.count_nonzero(go[:, :, 1]).item() == 0
    assert torch.count_nonzero(gv[..., 1, :]).item() == 0
    # <g, out> = <grad_value, value> by linearity in the value map
    lhs = float((g * out).sum())
    rhs = float((gv * value.float()).sum())
    assert abs(lhs - rhs) <= 1e-5 * (1 + abs(lhs))


@pytest.mark.parametrize("D,K,box", [(64, 12, False), (128, 4, True), (64, 4, True)])
def test_fused_backward_wide_rows(D, K, box):
    """Rows wider than 128 bytes (one warp per item, 16-byte lanes), with more
    than 32 samples per item and with box references."""
    shapes = ((8, 8), (4, 4), (2, 2))
    d = wl.make_random_problem(120 + D + K, N=2, Lq=9, M=2, D=D, K=K, shapes=shapes)
    ref, off = d["reference_points"], d["offsets"]
    if box:
        rng = np.random.default_rng(121)
        ref = np.concatenate([rng.uniform(0.1, 0.9, (2, 9, 2)),
                              rng.uniform(0.05, 0.5, (2, 9, 2))], axis=-1).astype(np.float32)
        off = (rng.standard_normal(off.shape) * 0.25).astype(np.float32)
    _check(d, ref, off, d["logits"], box=box)


def test_fused_backward_stress():
    """The stress configuration at full size (N = 8, bf16 value, K = 8, 5% of
    the samples pushed out of range): grad_value satisfies the adjoint
    identity over every batch entry, and one middle entry matches the oracle
    in every gradient (entries are independent)."""
    w = wl.STRESS
    d = cached_inputs("stress")
    sh = d["spatial_shapes"]
    value = to_dev(d["value"])
    ref, off, z, g = (to_dev(d[k]) for k in ("reference_points", "offsets", "logits",
                                             "grad_out"))
    got = msda_backward_fused(value, sh, None, ref, off, z, g)
    out = msda_forward_fused(value, sh, None, ref, off, z)
    torch.cuda.synchronize()
    # out is linear in the value map: <grad_out, out> = <grad_value, value>
    lhs = float((g.double() * out.double()).sum())
    rhs = float((got[0].double() * value.double()).sum())
    mass = float((g.double() * out.double()).abs().sum() +
                 (got[0].double() * value.double()).abs().sum())
    assert abs(lhs - rhs) <= 1e-5 * mass, ("fused stress adjoint", lhs, rhs, mass)
    del out
    n = w.N // 2 - 1
    sl = slice(n, n + 1)
    dn = {k: (np.ascontiguousarray(v[sl]) if k != "spatial_shapes" else v) for k, v in d.items()
          if k in ("value", "spatial_shapes", "reference_points", "offsets", "logits",
                   "grad_out")}
    _check(dn, dn["reference_points"], dn["offsets"], dn["logits"], box=False,
           got=tuple(x[sl] for x in got))
