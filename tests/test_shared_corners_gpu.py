"""Samples of one query, head and level that hold the same corner pixels.

The points of a level sample around one reference point, so two of them whose
cells lie within a pixel of each other share corner pixels, and so value rows:
the backward then scatters into one grad_value row from several samples of
the same item, and the forward reads the row more than once.  These cases draw
offsets a third of a pixel wide, so that most corners are shared, over the
kernels' lane shapes (rows of 2, 4 and 8 lanes; fp32 and bf16), point counts
whose levels straddle the backward's batches of eight samples (K = 3, 5, 6),
and ragged query counts, and compare every output with the oracle."""
import numpy as np
import pytest
import torch

import oracle
from scale_deformable_attention_02_b200 import (msda_backward, msda_backward_fused,
                                                msda_forward, msda_forward_fused)
from scale_deformable_attention_02_b200 import workloads as wl

from gpu_util import F32, GRAD, PLAIN, assert_close, host, to_dev, value_grad_terms

pytestmark = pytest.mark.gpu

SHAPES = {1: ((9, 11),), 2: ((9, 11), (5, 6)), 3: ((9, 11), (5, 6), (3, 3)),
          4: ((9, 11), (5, 6), (3, 3), (2, 2)), 5: ((9, 11), (5, 6), (3, 3), (2, 2), (1, 2))}

# (value dtype, D, K, L)
CASES = [("f32", 32, 4, 4), ("f32", 32, 3, 5), ("f32", 32, 5, 3), ("f32", 32, 8, 2),
         ("f32", 32, 2, 4), ("f32", 32, 1, 4), ("f32", 32, 6, 2), ("f32", 16, 4, 4),
         ("f32", 16, 3, 4), ("f32", 8, 4, 4), ("bf16", 32, 4, 4), ("bf16", 32, 3, 5),
         ("bf16", 16, 5, 3)]
IDS = [f"{dt}-D{D}-K{K}-L{L}" for dt, D, K, L in CASES]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def shared_fraction(loc, shapes):
    """Fraction of in-level corners whose pixel another point of the same
    (n, q, m, level) also holds, from the fp32 locations."""
    N, Lq, M, L, K, _ = loc.shape
    tot = shared = 0
    for lvl, (H, W) in enumerate(shapes):
        x = loc[:, :, :, lvl, :, 0].astype(np.float32) * np.float32(W) - np.float32(0.5)
        y = loc[:, :, :, lvl, :, 1].astype(np.float32) * np.float32(H) - np.float32(0.5)
        x0, y0 = np.floor(x).astype(np.int64), np.floor(y).astype(np.int64)
        keys = []
        for c in range(4):
            xx, yy = x0 + (c & 1), y0 + (c >> 1)
            ok = (xx >= 0) & (xx < W) & (yy >= 0) & (yy < H)
            keys.append(np.where(ok, yy * W + xx, -1))
        kk = np.sort(np.stack(keys, -1).reshape(-1, K * 4), axis=1)
        valid = kk >= 0
        tot += valid.sum()
        shared += (valid[:, 1:] & (kk[:, 1:] == kk[:, :-1])).sum()
    return shared / max(tot, 1)


@pytest.mark.parametrize("dt,D,K,L", CASES, ids=IDS)
def test_shared_corners_match_the_oracle(dt, D, K, L):
    shapes = SHAPES[L]
    M, N, Lq = 4, 2, 37
    d = wl.make_random_problem(700 + K * 10 + L, N=N, Lq=Lq, M=M, D=D, K=K, shapes=shapes,
                               value_dtype=dt, offset_std=0.35)
    sh = d["spatial_shapes"]
    loc = oracle.locations_f32(d["reference_points"], d["offsets"], sh)
    if K > 1:
        assert shared_fraction(loc, shapes) > 0.2, "the case shares too few corners"
    value = to_dev(d["value"])
    A64 = oracle.softmax(d["logits"])
    A = A64.astype(np.float32)

    # unfused calls on the same locations
    out = msda_forward(value, sh, None, to_dev(loc), to_dev(A))
    assert_close(host(out), oracle.forward(d["value"], sh, loc, A), **F32, what="forward")
    gv, gl, ga = msda_backward(value, sh, None, to_dev(loc), to_dev(A), to_dev(d["grad_out"]))
    ogv, ogl, oga, mgl, mga = oracle.backward(d["value"], sh, loc, A, d["grad_out"],
                                              with_mass=True)
    tv, mv = value_grad_terms(d["value"], sh, loc, A, d["grad_out"])
    assert_close(host(gv), ogv, **GRAD, what="grad_value", mass=mv, terms=tv)
    assert_close(host(gl), ogl, **PLAIN, what="grad_loc", mass=mgl)
    assert_close(host(ga), oga, **PLAIN, what="grad_attn", mass=mga)

    # fused calls
    ref, off, z, g = (to_dev(d[k]) for k in ("reference_points", "offsets", "logits",
                                             "grad_out"))
    fo = msda_forward_fused(value, sh, None, ref, off, z)
    assert_close(host(fo), oracle.forward(d["value"], sh, loc, A64), **F32, what="fused out")
    gv, gr, go, gz = msda_backward_fused(value, sh, None, ref, off, z, g)
    ogv, ogl, oga, mgl, mga = oracle.backward(d["value"], sh, loc, A, d["grad_out"],
                                              with_mass=True)
    ogr, ogo, ogz = oracle.fused_chain(ogl, oga, A64, sh)
    Wl = sh[:, 1].astype(np.float64)[None, None, None, :, None]
    Hl = sh[:, 0].astype(np.float64)[None, None, None, :, None]
    mgo = np.stack([mgl[..., 0] / Wl, mgl[..., 1] / Hl], axis=-1) + np.abs(ogo)
    LK = L * K
    Af = A64.reshape(A64.shape[:3] + (LK,))
    mza = mga.reshape(Af.shape) + np.abs(oga.reshape(Af.shape))
    mz = (Af * (mga.reshape(Af.shape) + (Af * mza).sum(-1, keepdims=True))).reshape(A64.shape)
    mref = (mgl + np.abs(ogl)).sum(axis=(2, 3, 4))
    tv, mv = value_grad_terms(d["value"], sh, loc, A64, d["grad_out"])
    assert_close(host(gv), ogv, **GRAD, what="fused grad_value", mass=mv, terms=tv)
    assert_close(host(go), ogo, **PLAIN, what="fused grad_offsets", mass=mgo)
    assert_close(host(gz), ogz, **PLAIN, what="fused grad_logits", mass=mz)
    assert_close(host(gr), ogr, **GRAD, what="fused grad_reference", mass=mref)
