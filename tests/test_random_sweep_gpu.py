"""A seeded sweep over random problem shapes: value dtype, row width (16 to
512 bytes), heads and deformable groups, level count and shapes (empty levels
included), points per level (L*K up to 128), point or box references, and
query counts with ragged tails.  Every case runs the four entry points
(forward, fused forward, backward, fused backward) against the oracle with
the parity tolerances."""
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

N_CASES = 40


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _case(i):
    rng = np.random.default_rng(9000 + i)
    dt = "bf16" if rng.random() < 0.4 else "f32"
    unit = 8 if dt == "bf16" else 4                 # elements of a 16-byte row unit
    D = int(unit * rng.choice([1, 2, 3, 4, 6, 8, 16, 32 if dt == "f32" else 64]))
    D = min(D, 128 if dt == "f32" else 256)         # rows of at most 512 bytes
    M = int(rng.choice([1, 2, 3, 4, 6, 8]))
    G = int(rng.choice([g for g in range(1, M + 1) if M % g == 0]))
    L = int(rng.integers(1, 5))
    # every kernel family: L*K <= 8, <= 16, 17..32, more than 32 (blocks of 32)
    K = int(rng.choice([1, 2, 3, 4, 4, 5, 8, 8, 12, 16, 33]))
    K = max(1, min(K, 128 // L))
    shapes = tuple((int(rng.integers(0 if rng.random() < 0.1 else 1, 13)),
                    int(rng.integers(1, 15))) for _ in range(L))
    if sum(h * w for h, w in shapes) == 0:
        shapes = ((3, 4),) + shapes[1:]
    N = int(rng.integers(1, 3))
    Lq = int(rng.integers(1, 40))
    box = bool(rng.random() < 0.3)
    return dict(dt=dt, D=D, M=M, G=G, L=L, K=K, shapes=shapes, N=N, Lq=Lq, box=box, seed=9000 + i)


CASES = [_case(i) for i in range(N_CASES)]
IDS = [f"{c['dt']}-D{c['D']}-M{c['M']}G{c['G']}-L{c['L']}K{c['K']}-Lq{c['Lq']}"
       f"{'-box' if c['box'] else ''}" for c in CASES]


@pytest.mark.parametrize("c", CASES, ids=IDS)
def test_random_shape(c):
    d = wl.make_random_problem(c["seed"], N=c["N"], Lq=c["Lq"], M=c["M"], D=c["D"], K=c["K"],
                               shapes=c["shapes"], value_dtype=c["dt"])
    sh = d["spatial_shapes"]
    M, G = c["M"], c["G"]
    groups = None if G == M else G
    value = to_dev(d["value"])
    # unfused: per-group locations, per-head weights
    loc_g = np.ascontiguousarray(d["sampling_locations"][:, :, :G])
    loc_h = oracle.expand_groups(loc_g, M)
    A = oracle.softmax(d["logits"]).astype(np.float32)
    out = msda_forward(value, sh, None, to_dev(loc_g), to_dev(A), groups=groups)
    assert_close(host(out), oracle.forward(d["value"], sh, loc_h, A), **F32, what="forward")
    gv, gl, ga = msda_backward(value, sh, None, to_dev(loc_g), to_dev(A), to_dev(d["grad_out"]),
                               groups=groups)
    ogv, ogl, oga, mgl, mga = oracle.backward(d["value"], sh, loc_h, A, d["grad_out"],
                                              with_mass=True)
    tv, mv = value_grad_terms(d["value"], sh, loc_h, A, d["grad_out"])
    assert_close(host(gv), ogv, **GRAD, what="grad_value", mass=mv, terms=tv)
    assert_close(host(ga), oga, **PLAIN, what="grad_attn", mass=mga)
    assert_close(host(gl), oracle.sum_groups(ogl, G), **grad_tol(G, M), what="grad_loc",
                 mass=oracle.sum_groups(mgl + np.abs(ogl), G))
    # fused: point or box references, per-group offsets
    if c["box"]:
        rng = np.random.default_rng(c["seed"] + 1)
        ref = np.concatenate([rng.uniform(0.1, 0.9, (c["N"], c["Lq"], 2)),
                              rng.uniform(0.05, 0.5, (c["N"], c["Lq"], 2))],
                             axis=-1).astype(np.float32)
        off_g = (rng.standard_normal(d["offsets"][:, :, :G].shape) * 0.25).astype(np.float32)
    else:
        ref = d["reference_points"]
        off_g = np.ascontiguousarray(d["offsets"][:, :, :G])
    off_h = oracle.expand_groups(off_g, M)
    fo, floc, fa = msda_forward_fused(value, sh, None, to_dev(ref), to_dev(off_g),
                                      to_dev(d["logits"]), return_sampling=True, groups=groups)
    if c["box"]:
        oloc = oracle.locations_box_f32(ref, off_h)
    else:
        oloc = oracle.locations_f32(ref, off_h, sh)
    assert_bits_equal(host(floc), np.ascontiguousarray(oloc[:, :, ::M // G]), what="fused loc")
    assert_close(host(fa), oracle.softmax(d["logits"]), **F32, what="fused softmax")
    assert_close(host(fo), oracle.forward(d["value"], sh, oloc, oracle.softmax(d["logits"])),
                 **F32, what="fused out")
    gv, gr, go, gz = msda_backward_fused(value, sh, None, to_dev(ref), to_dev(off_g),
                                         to_dev(d["logits"]), to_dev(d["grad_out"]),
                                         groups=groups)
    A64 = oracle.softmax(d["logits"])
    ogv, ogl, oga, mgl, mga = oracle.backward(d["value"], sh, oloc, A64.astype(np.float32),
                                              d["grad_out"], with_mass=True)
    if c["box"]:
        ogr, ogo, ogz = oracle.fused_chain_box(ogl, oga, A64, ref, off_h)
        mgo = (mgl + np.abs(ogl)) * np.asarray(ref, np.float64)[:, :, None, None, None, 2:]
        mref = np.stack([(mgl[..., 0] + np.abs(ogl[..., 0])).sum(axis=(2, 3, 4)),
                         (mgl[..., 1] + np.abs(ogl[..., 1])).sum(axis=(2, 3, 4)),
                         ((mgl[..., 0] + np.abs(ogl[..., 0])) *
                          np.abs(off_h[..., 0])).sum(axis=(2, 3, 4)),
                         ((mgl[..., 1] + np.abs(ogl[..., 1])) *
                          np.abs(off_h[..., 1])).sum(axis=(2, 3, 4))], axis=-1)
    else:
        ogr, ogo, ogz = oracle.fused_chain(ogl, oga, A64, sh)
        Wl = sh[:, 1].astype(np.float64)[None, None, None, :, None]
        Hl = sh[:, 0].astype(np.float64)[None, None, None, :, None]
        with np.errstate(divide="ignore", invalid="ignore"):
            mgo = np.stack([np.nan_to_num(mgl[..., 0] / Wl), np.nan_to_num(mgl[..., 1] / Hl)],
                           axis=-1) + np.abs(ogo)
        mref = (mgl + np.abs(ogl)).sum(axis=(2, 3, 4))
    LK = c["L"] * c["K"]
    Af = A64.reshape(A64.shape[:3] + (LK,))
    mz_head = (Af * (mga.reshape(Af.shape) + np.abs(oga.reshape(Af.shape)))).sum(-1,
                                                                                keepdims=True)
    mz = (Af * (mga.reshape(Af.shape) + mz_head)).reshape(A64.shape)
    tv, mv = value_grad_terms(d["value"], sh, oloc, A64, d["grad_out"])
    assert_close(host(gv), ogv, **GRAD, what="fused grad_value", mass=mv, terms=tv)
    assert_close(host(go), oracle.sum_groups(ogo, G), **grad_tol(G, M),
                 what="fused grad_offsets", mass=oracle.sum_groups(mgo, G))
    assert_close(host(gz), ogz, **PLAIN, what="fused grad_logits", mass=mz)
    assert_close(host(gr), ogr, **GRAD, what="fused grad_reference", mass=mref)
