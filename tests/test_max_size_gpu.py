"""Parity at the largest problems the C ABI accepts: every tensor may hold up
to 2^31 - 1 elements, and the kernels index the value map with 32-bit row
offsets inside one (n, m) map and 32-bit item indices.

Two layouts reach the limit from either side:
  * wide batch: 26214 batch entries of a 320-pixel map (8 heads, D = 32),
    2,147,450,880 value elements; the last entry's rows sit just below 2^31.
    Batch entries are independent, so entries 0 and N - 1 are checked in
    full against the oracle run on their own slices, for all four entry
    points.
  * one huge level: 16383 x 32768 pixels (one head, D = 4) plus a 3 x 5
    level, 2,147,352,636 value elements; in-map row offsets reach
    2,147,352,632.
    Only rectangular windows hold values (samples stay inside them), so the
    oracle, which reads only sampled rows, runs on the full map.  The
    forward and the per-sample gradients are checked element by element;
    grad_value, too large to mirror in fp64 on the host, is checked by the
    adjoint identity <grad_value, u> = <grad_out, forward(u)> for two value
    maps u supported on the windows, and by being zero outside them.

The device holds up to about 26 GB during these tests."""
import numpy as np
import pytest
import torch

import oracle
from scale_deformable_attention_02_b200 import (msda_backward, msda_backward_fused,
                                                msda_forward, msda_forward_fused)
from scale_deformable_attention_02_b200 import workloads as wl

from gpu_util import (F32, GRAD, KAPPA, PLAIN, U32, assert_bits_equal, assert_close, host,
                      to_dev, value_grad_terms)

pytestmark = pytest.mark.gpu

LIMIT = 2 ** 31 - 1


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    free, _ = torch.cuda.mem_get_info()
    if free < 40 * 2 ** 30:
        pytest.skip("needs about 40 GB of free device memory")


def test_wide_batch_at_the_element_limit():
    shapes = ((16, 16), (8, 8))
    M, D, K, Lq = 8, 32, 4, 3
    S = sum(h * w for h, w in shapes)
    N = LIMIT // (S * M * D)
    assert N * S * M * D <= LIMIT and (N + 1) * S * M * D > LIMIT
    d = wl.make_wide_batch_problem(2024, N=N, Lq=Lq, M=M, D=D, K=K, shapes=shapes)
    sh = d["spatial_shapes"]
    block = d["value_block"]
    value = to_dev(block).expand(N, S, M, D).contiguous()  # every entry holds the block
    loc = d["sampling_locations"]
    A = oracle.softmax(d["logits"]).astype(np.float32)
    g = d["grad_out"]
    out = msda_forward(value, sh, None, to_dev(loc), to_dev(A))
    fo, floc, fa = msda_forward_fused(value, sh, None, to_dev(d["reference_points"]),
                                      to_dev(d["offsets"]), to_dev(d["logits"]),
                                      return_sampling=True)
    gv, gl, ga = msda_backward(value, sh, None, to_dev(loc), to_dev(A), to_dev(g))
    fgv, fgr, fgo, fgz = msda_backward_fused(value, sh, None, to_dev(d["reference_points"]),
                                             to_dev(d["offsets"]), to_dev(d["logits"]),
                                             to_dev(g))
    for n in (0, N - 1):
        sl = slice(n, n + 1)
        what = f"entry {n}"
        assert_close(host(out[sl]), oracle.forward(block, sh, loc[sl], A[sl]), **F32,
                     what=f"{what} forward")
        ora, oloc, oA = oracle.forward_fused(block, sh, d["reference_points"][sl],
                                             d["offsets"][sl], d["logits"][sl])
        assert_bits_equal(host(floc[sl]), oloc, what=f"{what} fused loc")
        assert_close(host(fa[sl]), oA, **F32, what=f"{what} fused softmax")
        assert_close(host(fo[sl]), ora, **F32, what=f"{what} fused out")
        ogv, ogl, oga, mgl, mga = oracle.backward(block, sh, loc[sl], A[sl], g[sl],
                                                  with_mass=True)
        tv, mv = value_grad_terms(block, sh, loc[sl], A[sl], g[sl])
        assert_close(host(gv[sl]), ogv, **GRAD, what=f"{what} grad_value", mass=mv, terms=tv)
        assert_close(host(gl[sl]), ogl, **PLAIN, what=f"{what} grad_loc", mass=mgl)
        assert_close(host(ga[sl]), oga, **PLAIN, what=f"{what} grad_attn", mass=mga)
        # fused backward: the oracle's backward at its own locations and
        # weights, then its chain rule (bounds as in the fused-backward tests)
        oA64 = oracle.softmax(d["logits"][sl])
        fgv_o, fgl_o, fga_o, fmgl, fmga = oracle.backward(block, sh, oloc, oA64.astype(np.float32),
                                                          g[sl], with_mass=True)
        ogr, ogo, ogz = oracle.fused_chain(fgl_o, fga_o, oA64, sh)
        Wl = sh[:, 1].astype(np.float64)[None, None, None, :, None]
        Hl = sh[:, 0].astype(np.float64)[None, None, None, :, None]
        mgo = np.stack([fmgl[..., 0] / Wl, fmgl[..., 1] / Hl], axis=-1)
        mref = (fmgl + np.abs(fgl_o)).sum(axis=(2, 3, 4))
        Af = oA64.reshape(oA64.shape[:3] + (-1,))
        mz_head = (Af * (fmga.reshape(Af.shape) + np.abs(fga_o.reshape(Af.shape)))).sum(-1, keepdims=True)
        mz = (Af * (fmga.reshape(Af.shape) + mz_head)).reshape(oA64.shape)
        tv, mv = value_grad_terms(block, sh, oloc, oA64, g[sl])
        assert_close(host(fgv[sl]), fgv_o, **GRAD, what=f"{what} fused grad_value", mass=mv,
                     terms=tv)
        assert_close(host(fgo[sl]), ogo, **PLAIN, what=f"{what} grad_offsets", mass=mgo)
        assert_close(host(fgz[sl]), ogz, **PLAIN, what=f"{what} grad_logits", mass=mz)
        assert_close(host(fgr[sl]), ogr, **GRAD, what=f"{what} grad_reference", mass=mref)


def _lay_out(S, D, rows, vals, start1, other):
    """A zero [1, S, 1, D] fp32 map with the window rows and the small
    levels filled in (pages never written stay unallocated)."""
    v = np.zeros((1, S, 1, D), dtype=np.float32)
    v[0, rows, 0, :] = vals
    v[0, start1:, 0, :] = other
    return v


def test_huge_level_at_the_element_limit():
    shapes = ((16383, 32768), (3, 5))
    D, K, Lq = 4, 2, 64
    H0, W0 = shapes[0]
    S = sum(h * w for h, w in shapes)
    assert LIMIT - 2 ** 20 < S * D <= LIMIT
    windows = ((0, 0, 40, 40), (H0 - 40, W0 - 40, 40, 40), (H0 // 2, W0 // 2 - 20, 40, 40))
    d = wl.make_windowed_problem(2025, shapes, windows, Lq=Lq, K=K, D=D)
    sh = d["spatial_shapes"]
    rows = d["window_rows"]
    start1 = H0 * W0
    value_h = _lay_out(S, D, rows, d["window_values"], start1, d["other_values"])
    loc = d["sampling_locations"]
    A = oracle.softmax(d["logits"]).astype(np.float32)
    g = d["grad_out"]
    value = torch.from_numpy(value_h).to("cuda")
    out = msda_forward(value, sh, None, to_dev(loc), to_dev(A))
    assert_close(host(out), oracle.forward(value_h, sh, loc, A), **F32, what="forward")
    gv, gl, ga = msda_backward(value, sh, None, to_dev(loc), to_dev(A), to_dev(g))
    _, ogl, oga, mgl, mga = oracle.backward(value_h, sh, loc, A, g, with_mass=True,
                                            with_grad_value=False)
    assert_close(host(gl), ogl, **PLAIN, what="grad_loc", mass=mgl)
    assert_close(host(ga), oga, **PLAIN, what="grad_attn", mass=mga)
    del value
    # grad_value: zero outside the windows and the small level ...
    held = torch.from_numpy(np.concatenate([rows, np.arange(start1, S)])).to("cuda")
    gvh = gv[0, held, 0, :].double()
    nonzero = int(torch.count_nonzero(gv).item())
    assert nonzero > 0 and nonzero == int(torch.count_nonzero(gvh).item())
    # ... and the adjoint identity for the sampled map and a second one
    g64 = np.asarray(g, np.float64)
    for name, wv in (("value", d["window_values"]), ("second map", d["second_values"])):
        u = _lay_out(S, D, rows, wv, start1, d["other_values"])
        expect = float((g64 * oracle.forward(u, sh, loc, A)).sum())
        uh = torch.from_numpy(np.concatenate([wv, d["other_values"]]).astype(np.float64)).to("cuda")
        got = float((gvh * uh).sum().item())
        mass = float((gvh.abs() * uh.abs()).sum().item())
        assert abs(got - expect) <= GRAD["atol"] + GRAD["rtol"] * mass + KAPPA * U32 * mass, \
            (name, got, expect, mass)
        del u
