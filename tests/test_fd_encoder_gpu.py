"""The encoder-shaped backward (N=2, Lq=S=17821, M=8, D=32, L=4, K=4, fp32),
run at full size in the launch configuration the benchmark times, against
finite differences: on a seeded 1% subsample of the (batch, query) pairs,
every sampling-location gradient the GPU writes is compared with the central
difference of <grad_out, out> in that coordinate, evaluated one query at a
time by the fp64 oracle.  The difference is taken at the GPU's own pixel
coordinate: the kernels form x = loc*W - 0.5 in fp32, so the fp64 location
is chosen as (x + 0.5)/W with that fp32 x, and both sides differentiate the
same function at the same point.  Samples within 1e-3 px of a cell boundary
(where the interpolant has a kink) are skipped."""
import numpy as np
import pytest
import torch

import oracle
from scale_deformable_attention_02_b200 import msda_backward
from scale_deformable_attention_02_b200 import workloads as wl

from gpu_util import KAPPA, U32, host, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _at_fp32_pixel(loc_q, shapes):
    """fp64 locations whose fp64 pixel coordinates equal the fp32 pixel
    coordinates x = fl(fl(loc_x * W) - 0.5) of loc_q (float32) on each level."""
    W = shapes[None, :, None, 1].astype(np.float32)
    H = shapes[None, :, None, 0].astype(np.float32)
    x = (loc_q[..., 0] * W) - np.float32(0.5)  # numpy float32: two rounded operations
    y = (loc_q[..., 1] * H) - np.float32(0.5)
    out = np.empty(loc_q.shape, dtype=np.float64)
    out[..., 0] = (x.astype(np.float64) + 0.5) / W.astype(np.float64)
    out[..., 1] = (y.astype(np.float64) + 0.5) / H.astype(np.float64)
    return out


def _near_kink(loc_q, shapes, tol_px):
    """[M, L, K] mask: the sample's pixel coordinate lies within tol_px of an
    integer in x or y."""
    x = loc_q[..., 0] * shapes[None, :, None, 1] - 0.5
    y = loc_q[..., 1] * shapes[None, :, None, 0] - 0.5
    fx, fy = x - np.floor(x), y - np.floor(y)
    return (np.minimum(fx, 1 - fx) < tol_px) | (np.minimum(fy, 1 - fy) < tol_px)


def test_encoder_location_gradient_matches_finite_differences():
    w = wl.ENCODER_BWD
    d = wl.make_inputs(w)
    sh = d["spatial_shapes"]
    loc = oracle.locations_f32(d["reference_points"], d["offsets"], sh)
    A = oracle.softmax(d["logits"]).astype(np.float32)
    _, gl, _ = msda_backward(to_dev(d["value"]), sh, None, to_dev(loc), to_dev(A),
                             to_dev(d["grad_out"]))
    gl = host(gl)
    rng = np.random.default_rng(2024)
    pairs = rng.choice(w.N * w.queries, size=(w.N * w.queries) // 100, replace=False)
    h = 1e-6
    checked = 0
    worst = 0.0
    for nq in pairs:
        n, q = divmod(int(nq), w.queries)
        value = np.ascontiguousarray(d["value"][n:n + 1])
        loc_q = _at_fp32_pixel(loc[n:n + 1, q:q + 1], sh)
        A_q = A[n:n + 1, q:q + 1]
        g_q = d["grad_out"][n:n + 1, q:q + 1].astype(np.float64)
        _, ogl, _, mgl, _ = oracle.backward(value, sh, loc[n:n + 1, q:q + 1], A_q,
                                            d["grad_out"][n:n + 1, q:q + 1], with_mass=True)
        skip = _near_kink(loc_q[0, 0], sh.astype(np.float64), 1e-3)
        for (m, l, k) in np.argwhere(~skip):
            for c in range(2):
                lp, lm = loc_q.copy(), loc_q.copy()
                lp[0, 0, m, l, k, c] += h
                lm[0, 0, m, l, k, c] -= h
                fp = np.sum(g_q * oracle.forward(value, sh, lp, A_q, loc_f32=False))
                fm = np.sum(g_q * oracle.forward(value, sh, lm, A_q, loc_f32=False))
                fd = (fp - fm) / (2 * h)
                gpu = float(gl[n, q, m, l, k, c])
                bound = 1e-5 + 1e-4 * abs(fd) + KAPPA * U32 * float(mgl[0, 0, m, l, k, c])
                err = abs(gpu - fd)
                worst = max(worst, err / bound)
                assert err <= bound, (n, q, m, l, k, c, gpu, fd, float(ogl[0, 0, m, l, k, c]))
                checked += 1
    # about 356 queries x 128 samples x 2 coordinates, minus kinks
    assert checked > 0.9 * len(pairs) * w.M * w.L * w.K * 2 * 0.9, checked
    print(f"checked {checked} coordinates, worst error / bound = {worst:.3f}")
