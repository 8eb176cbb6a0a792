"""GPU parity of the deformable-group entry points (msda_*_grouped): G groups
of M/G consecutive heads share one set of sampling locations (per-group
locations and offsets, per-head weights and logits).  The oracle side is the
ungrouped oracle on the per-head expansion of the group tensors, with the
location gradients summed over each group's heads (oracle.expand_groups /
oracle.sum_groups, pinned by finite differences on the CPU)."""
import numpy as np
import pytest
import torch

import oracle
from scale_deformable_attention_02_b200 import (msda_backward, msda_backward_fused,
                                                msda_forward, msda_forward_fused)
from scale_deformable_attention_02_b200 import workloads as wl

from gpu_util import (F32, GRAD, KAPPA, PLAIN, U32, assert_bits_equal, assert_close, grad_tol,
                      host, to_dev, value_grad_terms)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


# (M, G, D, K, shapes, dtype): fast, wide and more-than-32-sample kernels
CASES = [
    (8, 1, 32, 4, ((12, 14), (6, 7), (3, 4), (2, 2)), "f32"),
    (8, 2, 32, 4, ((12, 14), (6, 7), (3, 4), (2, 2)), "f32"),
    (8, 4, 32, 4, ((12, 14), (6, 7), (3, 4), (2, 2)), "bf16"),
    (6, 3, 16, 3, ((9, 11), (5, 6)), "f32"),
    (4, 2, 64, 2, ((8, 8), (4, 4)), "f32"),          # wide rows
    (4, 1, 32, 12, ((6, 8), (3, 4), (2, 2)), "f32"),  # L*K = 36
]
IDS = [f"M{c[0]}G{c[1]}D{c[2]}K{c[3]}{c[5]}" for c in CASES]


def _problem(case, seed):
    M, G, D, K, shapes, dt = case
    d = wl.make_random_problem(seed, N=2, Lq=23, M=M, D=D, K=K, shapes=shapes,
                               value_dtype=dt)
    # per-group locations and offsets: the first G head slots of the draws
    d["loc_g"] = np.ascontiguousarray(d["sampling_locations"][:, :, :G])
    d["off_g"] = np.ascontiguousarray(d["offsets"][:, :, :G])
    return d


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_grouped_forward_and_backward(case):
    M, G, D, K, shapes, dt = case
    d = _problem(case, 500 + G + D)
    sh = d["spatial_shapes"]
    A = oracle.softmax(d["logits"]).astype(np.float32)
    loc_h = oracle.expand_groups(d["loc_g"], M)
    value = to_dev(d["value"])
    out = msda_forward(value, sh, None, to_dev(d["loc_g"]), to_dev(A), groups=G)
    assert_close(host(out), oracle.forward(d["value"], sh, loc_h, A), **F32,
                 what="grouped forward")
    gv, gl, ga = msda_backward(value, sh, None, to_dev(d["loc_g"]), to_dev(A),
                               to_dev(d["grad_out"]), groups=G)
    ogv, ogl, oga, mgl, mga = oracle.backward(d["value"], sh, loc_h, A, d["grad_out"],
                                              with_mass=True)
    tv, mv = value_grad_terms(d["value"], sh, loc_h, A, d["grad_out"])
    assert_close(host(gv), ogv, **GRAD, what="grouped grad_value", mass=mv, terms=tv)
    assert_close(host(ga), oga, **PLAIN, what="grouped grad_attn", mass=mga)
    # a group's location gradient adds its heads' gradients (atomically, any order)
    assert_close(host(gl), oracle.sum_groups(ogl, G), **grad_tol(G, M), what="grouped grad_loc",
                 mass=oracle.sum_groups(mgl + np.abs(ogl), G))


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_grouped_fused_forward_and_backward(case):
    M, G, D, K, shapes, dt = case
    d = _problem(case, 700 + G + D)
    sh = d["spatial_shapes"]
    ref, off_g, z, g = d["reference_points"], d["off_g"], d["logits"], d["grad_out"]
    value = to_dev(d["value"])
    out, loc_o, a_o = msda_forward_fused(value, sh, None, to_dev(ref), to_dev(off_g),
                                         to_dev(z), return_sampling=True, groups=G)
    off_h = oracle.expand_groups(off_g, M)
    ora, oloc, oA = oracle.forward_fused(d["value"], sh, ref, off_h, z)
    assert_bits_equal(host(loc_o), np.ascontiguousarray(oloc[:, :, ::M // G]),
                      what="grouped fused loc")
    assert_close(host(a_o), oA, **F32, what="grouped fused softmax")
    assert_close(host(out), ora, **F32, what="grouped fused out")
    gv, gr, go, gz = msda_backward_fused(value, sh, None, to_dev(ref), to_dev(off_g),
                                         to_dev(z), to_dev(g), groups=G)
    A = oracle.softmax(z)
    loc = oracle.locations_f32(ref, off_h, sh)
    ogv, ogl, oga, mgl, mga = oracle.backward(d["value"], sh, loc, A.astype(np.float32), g,
                                              with_mass=True)
    ogr, ogo, ogz = oracle.fused_chain(ogl, oga, A, sh)
    Wl = sh[:, 1].astype(np.float64)[None, None, None, :, None]
    Hl = sh[:, 0].astype(np.float64)[None, None, None, :, None]
    mgo = np.stack([mgl[..., 0] / Wl, mgl[..., 1] / Hl], axis=-1) + np.abs(ogo)
    LK = A.shape[-1] * A.shape[-2]
    Af = A.reshape(A.shape[:3] + (LK,))
    mz_head = (Af * (mga.reshape(Af.shape) + np.abs(oga.reshape(Af.shape)))).sum(-1,
                                                                                keepdims=True)
    mz = (Af * (mga.reshape(Af.shape) + mz_head)).reshape(A.shape)
    mref = (mgl + np.abs(ogl)).sum(axis=(2, 3, 4))
    tv, mv = value_grad_terms(d["value"], sh, loc, A, g)
    assert_close(host(gv), ogv, **GRAD, what="grouped fused grad_value", mass=mv, terms=tv)
    assert_close(host(go), oracle.sum_groups(ogo, G), **grad_tol(G, M),
                 what="grouped grad_offsets", mass=oracle.sum_groups(mgo, G))
    assert_close(host(gz), ogz, **PLAIN, what="grouped grad_logits", mass=mz)
    assert_close(host(gr), ogr, **GRAD, what="grouped grad_reference", mass=mref)


def test_one_group_per_head_equals_ungrouped_calls():
    d = wl.make_random_problem(9, N=2, Lq=31, M=8, D=32, K=4,
                               shapes=((12, 14), (6, 7), (3, 4), (2, 2)))
    sh = d["spatial_shapes"]
    A = to_dev(oracle.softmax(d["logits"]).astype(np.float32))
    value, loc = to_dev(d["value"]), to_dev(d["sampling_locations"])
    a = msda_forward(value, sh, None, loc, A)
    b = msda_forward(value, sh, None, loc, A, groups=8)
    assert torch.equal(a, b)
    ref, off, z = (to_dev(d[k]) for k in ("reference_points", "offsets", "logits"))
    a = msda_forward_fused(value, sh, None, ref, off, z, return_sampling=True)
    b = msda_forward_fused(value, sh, None, ref, off, z, return_sampling=True, groups=8)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    g = to_dev(d["grad_out"])
    a = msda_backward(value, sh, None, loc, A, g)
    b = msda_backward(value, sh, None, loc, A, g, groups=8)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])  # no atomics: same bits


def test_grouped_rejects_bad_group_counts():
    d = wl.make_random_problem(3, N=1, Lq=4, M=6, D=8, K=2, shapes=((4, 4),))
    sh = d["spatial_shapes"]
    A = to_dev(oracle.softmax(d["logits"]).astype(np.float32))
    with pytest.raises(ValueError):
        msda_forward(to_dev(d["value"]), sh, None, to_dev(d["sampling_locations"][:, :, :4]),
                     A, groups=4)  # 4 does not divide 6
