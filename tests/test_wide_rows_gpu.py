"""Value rows wider than 512 bytes (D > 128 fp32, D > 256 bf16).

A warp's 32 lanes cover 512 bytes of a row at 16 bytes each, so wider rows
take passes of 32 chunks over the same corner entries: the forward stores one
slice of the output per pass, and the backward sums each corner's <v, g> over
the passes before forming the gradients of its sample.  The cases cover a
ragged last pass (640-byte rows: 40 chunks), whole passes (1 KB, 4 KB), both
value dtypes, items of at most and of more than 32 samples, deformable groups
and the fused calls, against the oracle.

Per-sample gradients (locations, weights, offsets, logits) sum one sample's
<v, g> over its corners: a lane's share of the dot product takes D / 32
roundings over all passes, then 10 more (5 adds across the lanes, the corner
weight, 2 adds over the corners, A*W and the multiply by it), so their bound
is (D / 32 + 10) * 2^-24 * mass, and never below the bound of the narrower
rows."""
import numpy as np
import pytest
import torch

import oracle
from scale_deformable_attention_02_b200 import (msda_backward, msda_backward_fused,
                                                msda_forward, msda_forward_fused)
from scale_deformable_attention_02_b200 import workloads as wl

from gpu_util import (F32, GRAD, KAPPA, PLAIN, assert_bits_equal, assert_close, host, to_dev,
                      value_grad_terms)

pytestmark = pytest.mark.gpu

# (N, Lq, M, G, D, K, shapes, dtype)
CASES = [
    (1, 13, 2, 2, 160, 2, ((6, 5), (3, 3)), "f32"),          # 640-B rows: 32 + 8 chunks
    (2, 9, 2, 2, 256, 3, ((5, 7), (3, 4), (2, 2)), "f32"),   # 1 KB rows: two whole passes
    (1, 6, 1, 1, 1024, 2, ((4, 5), (2, 3)), "f32"),          # 4 KB rows: eight passes
    (1, 11, 2, 2, 320, 4, ((5, 6), (3, 3)), "bf16"),         # 640-B bf16 rows
    (1, 7, 2, 2, 512, 2, ((4, 4), (2, 2)), "bf16"),          # 1 KB bf16 rows
    (1, 5, 2, 2, 160, 12, ((4, 4), (2, 3), (1, 2)), "f32"),  # L*K = 36: the long forward
    (1, 8, 4, 2, 192, 3, ((5, 5), (3, 2)), "f32"),           # deformable groups, 768-B rows
]
IDS = [f"{c[7]}-D{c[4]}-M{c[2]}G{c[3]}-L{len(c[6])}K{c[5]}" for c in CASES]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_wide_rows_match_the_oracle(case):
    N, Lq, M, G, D, K, shapes, dt = case
    L = len(shapes)
    d = wl.make_random_problem(3100 + D + K, N=N, Lq=Lq, M=M, D=D, K=K, shapes=shapes,
                               value_dtype=dt)
    sh = d["spatial_shapes"]
    groups = None if G == M else G
    kappa = max(KAPPA, D / 32 + 10)  # roundings of a per-sample gradient (module docstring)
    value = to_dev(d["value"])
    A64 = oracle.softmax(d["logits"])
    A = A64.astype(np.float32)

    # unfused: per-group locations, per-head weights
    loc_g = np.ascontiguousarray(d["sampling_locations"][:, :, :G])
    loc = oracle.expand_groups(loc_g, M)
    out = msda_forward(value, sh, None, to_dev(loc_g), to_dev(A), groups=groups)
    assert_close(host(out), oracle.forward(d["value"], sh, loc, A), **F32, what="forward")
    gv, gl, ga = msda_backward(value, sh, None, to_dev(loc_g), to_dev(A),
                               to_dev(d["grad_out"]), groups=groups)
    ogv, ogl, oga, mgl, mga = oracle.backward(d["value"], sh, loc, A, d["grad_out"],
                                              with_mass=True)
    tv, mv = value_grad_terms(d["value"], sh, loc, A, d["grad_out"])
    assert_close(host(gv), ogv, **GRAD, what="grad_value", mass=mv, terms=tv)
    assert_close(host(ga), oga, **PLAIN, what="grad_attn", mass=mga, terms=kappa)
    gl_tol = PLAIN if G == M else GRAD
    assert_close(host(gl), oracle.sum_groups(ogl, G), **gl_tol, what="grad_loc",
                 mass=oracle.sum_groups(mgl + np.abs(ogl), G), terms=kappa)

    # fused: point references, per-group offsets
    off_g = np.ascontiguousarray(d["offsets"][:, :, :G])
    off = oracle.expand_groups(off_g, M)
    ref, z, g = (to_dev(d[k]) for k in ("reference_points", "logits", "grad_out"))
    fo, floc, fa = msda_forward_fused(value, sh, None, ref, to_dev(off_g), z,
                                      return_sampling=True, groups=groups)
    oloc = oracle.locations_f32(d["reference_points"], off, sh)
    assert_bits_equal(host(floc), np.ascontiguousarray(oloc[:, :, ::M // G]), what="fused loc")
    assert_close(host(fa), A64, **F32, what="fused softmax")
    assert_close(host(fo), oracle.forward(d["value"], sh, oloc, A64), **F32, what="fused out")
    gv, gr, go, gz = msda_backward_fused(value, sh, None, ref, to_dev(off_g), z, g,
                                         groups=groups)
    ogv, ogl, oga, mgl, mga = oracle.backward(d["value"], sh, oloc, A, d["grad_out"],
                                              with_mass=True)
    ogr, ogo, ogz = oracle.fused_chain(ogl, oga, A64, sh)
    Wl = sh[:, 1].astype(np.float64)[None, None, None, :, None]
    Hl = sh[:, 0].astype(np.float64)[None, None, None, :, None]
    mgo = np.stack([mgl[..., 0] / Wl, mgl[..., 1] / Hl], axis=-1) + np.abs(ogo)
    Af = A64.reshape(A64.shape[:3] + (L * K,))
    mza = mga.reshape(Af.shape) + np.abs(oga.reshape(Af.shape))
    mz = (Af * (mga.reshape(Af.shape) + (Af * mza).sum(-1, keepdims=True))).reshape(A64.shape)
    mref = (mgl + np.abs(ogl)).sum(axis=(2, 3, 4))
    tv, mv = value_grad_terms(d["value"], sh, oloc, A64, d["grad_out"])
    assert_close(host(gv), ogv, **GRAD, what="fused grad_value", mass=mv, terms=tv)
    assert_close(host(go), oracle.sum_groups(ogo, G), **gl_tol, what="fused grad_offsets",
                 mass=oracle.sum_groups(mgo, G), terms=kappa)
    assert_close(host(gz), ogz, **PLAIN, what="fused grad_logits", mass=mz, terms=kappa)
    assert_close(host(gr), ogr, **GRAD, what="fused grad_reference", mass=mref, terms=kappa)
