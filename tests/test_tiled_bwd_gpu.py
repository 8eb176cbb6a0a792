"""GPU parity of the tiled backward calls (include/msda_tiled.h):
msda_backward_tiled and msda_backward_fused_tiled against the oracle's
backward (and its chain rule), element by element, with the tolerances of
the untiled calls, and against the untiled calls on the same inputs.

Per sample, the tiled kernel forms <v_j, g> from the same value bits in the
same order as the untiled kernel (a window corner outside the level reads
zero and adds nothing), so the location, weight, offset and logit gradients
equal the untiled ones bit for bit.  The value gradient is summed in another
order (per window pixel on the chip, then one reduction per pixel), so it is
compared within the atomics tolerance.  The reference-point gradient, which
the M heads add with atomics, is compared with the oracle's, with its
rounding mass (its heads' terms can cancel)."""
import numpy as np
import pytest
import torch

import oracle
from scale_deformable_attention_02_b200 import (msda_backward, msda_backward_fused,
                                                msda_backward_fused_tiled, msda_backward_tiled,
                                                msda_debug_tiled_stalls, msda_tile_plan)
from scale_deformable_attention_02_b200 import workloads as wl

from gpu_util import GRAD, PLAIN, assert_close, host, to_dev, value_grad_terms
from test_tiled_gpu import CASES, _check_plan, _refs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()
    yield
    assert msda_debug_tiled_stalls() == 0


def _fused_masses(sh, mgl, ogl, mga, oga, A):
    """Rounding masses of the chained gradients (as in the untiled fused
    backward tests): offsets = mass(d loc) / W_l, logits through the softmax
    Jacobian, reference = the query's sum of mass(d loc) and |d loc|."""
    Wl = sh[:, 1].astype(np.float64)[None, None, None, :, None]
    Hl = sh[:, 0].astype(np.float64)[None, None, None, :, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        mgo = np.stack([np.nan_to_num(mgl[..., 0] / Wl), np.nan_to_num(mgl[..., 1] / Hl)],
                       axis=-1)
    LK = A.shape[-1] * A.shape[-2]
    Af = A.reshape(A.shape[:3] + (LK,))
    mz_head = (Af * (mga.reshape(Af.shape) + np.abs(oga.reshape(Af.shape)))).sum(-1,
                                                                                keepdims=True)
    mz = (Af * (mga.reshape(Af.shape) + mz_head)).reshape(A.shape)
    mref = (mgl + np.abs(ogl)).sum(axis=(2, 3, 4))
    return mgo, mz, mref


def _check_unfused(d, halo, cps, value=None, n_sel=None):
    sh = d["spatial_shapes"]
    value = to_dev(d["value"]) if value is None else value
    ref = to_dev(d["reference_points"])
    K = d["logits"].shape[-1]
    plan = msda_tile_plan(value, sh, None, ref, K=K, halo=halo, ctas_per_sm=cps)
    loc = oracle.locations_f32(d["reference_points"], d["offsets"], sh)
    A = oracle.softmax(d["logits"]).astype(np.float32)
    dl, dA, g = to_dev(loc), to_dev(A), to_dev(d["grad_out"])
    gv, gl, ga = msda_backward_tiled(value, sh, None, dl, dA, g, plan)
    ugv, ugl, uga = msda_backward(value, sh, None, dl, dA, g)
    torch.cuda.synchronize()
    # per-sample gradients: the untiled kernel's arithmetic, bit for bit
    assert torch.equal(gl, ugl), "tiled grad_loc differs from the untiled one"
    assert torch.equal(ga, uga), "tiled grad_attn differs from the untiled one"
    tv, mv = value_grad_terms(d["value"], sh, loc, A, d["grad_out"])
    assert_close(host(gv), host(ugv), **GRAD, what="tiled vs untiled grad_value", mass=2 * mv,
                 terms=tv)
    sel = range(d["logits"].shape[0]) if n_sel is None else n_sel
    for n in sel:
        s = slice(n, n + 1)
        v = np.ascontiguousarray(d["value"][s])
        ogv, ogl, oga, mgl, mga = oracle.backward(v, sh, np.ascontiguousarray(loc[s]),
                                                  np.ascontiguousarray(A[s]),
                                                  np.ascontiguousarray(d["grad_out"][s]),
                                                  with_mass=True)
        tv, mv = value_grad_terms(v, sh, np.ascontiguousarray(loc[s]), np.ascontiguousarray(A[s]),
                                  np.ascontiguousarray(d["grad_out"][s]))
        assert_close(host(gv[s]), ogv, **GRAD, what=f"tiled grad_value n={n}", mass=mv,
                     terms=tv)
        assert_close(host(gl[s]), ogl, **PLAIN, what=f"tiled grad_loc n={n}", mass=mgl)
        assert_close(host(ga[s]), oga, **PLAIN, what=f"tiled grad_attn n={n}", mass=mga)
    return plan


def _check_fused(d, halo, cps, value=None, n_sel=None):
    sh = d["spatial_shapes"]
    value = to_dev(d["value"]) if value is None else value
    ref, off, z, g = (to_dev(d[k]) for k in ("reference_points", "offsets", "logits",
                                             "grad_out"))
    plan = msda_tile_plan(value, sh, None, ref, K=d["logits"].shape[-1], halo=halo,
                          ctas_per_sm=cps)
    gv, gr, go, gz = msda_backward_fused_tiled(value, sh, None, ref, off, z, g, plan)
    ugv, ugr, ugo, ugz = msda_backward_fused(value, sh, None, ref, off, z, g)
    torch.cuda.synchronize()
    assert torch.equal(go, ugo), "tiled grad_offsets differ from the untiled ones"
    assert torch.equal(gz, ugz), "tiled grad_logits differ from the untiled ones"
    lf = oracle.locations_f32(d["reference_points"], d["offsets"], sh)
    tv, mv = value_grad_terms(d["value"], sh, lf, oracle.softmax(d["logits"]), d["grad_out"])
    assert_close(host(gv), host(ugv), **GRAD, what="tiled vs untiled grad_value", mass=2 * mv,
                 terms=tv)
    sel = range(d["logits"].shape[0]) if n_sel is None else n_sel
    for n in sel:
        s = slice(n, n + 1)
        r_, o_, z_, g_ = (np.ascontiguousarray(d[k][s]) for k in
                          ("reference_points", "offsets", "logits", "grad_out"))
        loc = oracle.locations_f32(r_, o_, sh)
        A = oracle.softmax(z_)
        ogv, ogl, oga, mgl, mga = oracle.backward(np.ascontiguousarray(d["value"][s]), sh, loc,
                                                  A.astype(np.float32), g_, with_mass=True)
        ogr, ogo, ogz = oracle.fused_chain(ogl, oga, A, sh)
        mgo, mz, mref = _fused_masses(sh, mgl, ogl, mga, oga, A)
        tv, mv = value_grad_terms(np.ascontiguousarray(d["value"][s]), sh, loc, A, g_)
        assert_close(host(gv[s]), ogv, **GRAD, what=f"tiled fused grad_value n={n}", mass=mv,
                     terms=tv)
        assert_close(host(go[s]), ogo, **PLAIN, what=f"tiled grad_offsets n={n}", mass=mgo)
        assert_close(host(gz[s]), ogz, **PLAIN, what=f"tiled grad_logits n={n}", mass=mz)
        assert_close(host(gr[s]), ogr, **GRAD, what=f"tiled grad_reference n={n}", mass=mref)
    return plan


@pytest.mark.parametrize("name,halo,cps", [("encoder_bwd", 3, 2), ("encoder_bwd", 4, 1),
                                           ("encoder_bf16", 3, 2), ("encoder_compass", 4, 2)])
def test_tiled_encoder_backward(name, halo, cps):
    d = wl.make_inputs(wl.WORKLOADS[name])
    plan = _check_unfused(d, halo, cps)
    _check_plan(plan, d["reference_points"])


@pytest.mark.parametrize("name,halo,cps", [("encoder_bwd", 3, 2), ("encoder_bf16", 4, 1)])
def test_tiled_encoder_fused_backward(name, halo, cps):
    d = wl.make_inputs(wl.WORKLOADS[name])
    _check_fused(d, halo, cps)


def test_tiled_stress_backward():
    """N=8 bf16, 32 samples per item, 5% of the samples out of range: oracle
    on three batch entries, the untiled backward on all eight."""
    d = wl.make_inputs(wl.STRESS)
    _check_unfused(d, 8, 1, n_sel=(0, 3, 7))


@pytest.mark.parametrize("case", CASES, ids=[f"case{i}" for i in range(len(CASES))])
def test_tiled_backward_random_problems(case):
    N, Lq, M, D, K, shapes, dt, halo, cps, kind = case
    S = int(sum(h * w for h, w in shapes))
    Lq = S if Lq is None else Lq
    rng = np.random.default_rng(5000 + D + K + halo)
    d = wl.make_random_problem(5100 + Lq, N=N, Lq=Lq, M=M, D=D, K=K, shapes=shapes,
                               value_dtype=dt, offset_std=1.5)
    d["reference_points"] = _refs(case, rng)
    value = to_dev(d["value"])
    _check_unfused(d, halo, cps, value)
    # an empty level has no offset gradient to chain to (the chain divides by
    # the level's size); the unfused check above covers such levels
    if all(h > 0 and w > 0 for h, w in shapes):
        _check_fused(d, halo, cps, value)
