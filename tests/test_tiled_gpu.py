"""GPU parity of the tiled calls (include/msda_tiled.h): a tile plan sorts
the queries into cells by reference point, and the tiled kernels stage each
head's value windows around a cell in shared memory.  The results must not
depend on the schedule:

  * against the oracle, element by element, with the tolerances of the
    untiled calls (fp32 1e-5 / 1e-6; the fused locations bit for bit);
  * against the untiled call on the same inputs, within the fp32 tolerance
    (the tiled kernel sums an item's corner terms in another order), with the
    locations and weights of the fused call bit for bit;
  * the plan itself against a CPU count of the reference points' cells.

The plans cover coarse and fine grids (one to three resident CTAs per SM),
halos from 0 to 8 pixels (0: most samples fall outside their window and read
global memory), reference points outside the unit square and NaN, empty
levels and every lane layout of the fast kernels."""
import numpy as np
import pytest
import torch

import oracle
from scale_deformable_attention_02_b200 import (msda_debug_tiled_stalls, msda_forward,
                                                msda_forward_fused, msda_forward_fused_tiled,
                                                msda_forward_tiled, msda_tile_plan)
from scale_deformable_attention_02_b200 import workloads as wl

from gpu_util import F32, assert_bits_equal, assert_close, host, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()
    yield
    assert msda_debug_tiled_stalls() == 0


def _plan_cells(ref: np.ndarray, gx: int, gy: int) -> np.ndarray:
    """Cell of every reference point, as the plan defines it (fp32 products,
    clamped to the grid, NaN to the first cell)."""
    x = ref[..., 0].astype(np.float32) * np.float32(gx)
    y = ref[..., 1].astype(np.float32) * np.float32(gy)
    with np.errstate(invalid="ignore"):
        cx = np.where(x >= 0, np.minimum(np.floor(np.nan_to_num(x, posinf=gx)), gx - 1), 0)
        cy = np.where(y >= 0, np.minimum(np.floor(np.nan_to_num(y, posinf=gy)), gy - 1), 0)
    return (cy * gx + cx).astype(np.int64)


def _check_plan(plan, ref: np.ndarray):
    """cell_start is the exclusive prefix sum of the CPU's cell counts, and
    each cell's segment of perm holds exactly that cell's queries."""
    gx, gy = plan.grid
    G = gx * gy
    N, Lq = ref.shape[:2]
    buf = host(plan.buffer).view(np.int32)
    start_bytes = ((N * (G + 1) * 4 + 255) // 256) * 256
    cs = buf[:N * (G + 1)].reshape(N, G + 1)
    perm = buf[start_bytes // 4:start_bytes // 4 + N * Lq].reshape(N, Lq)
    cells = _plan_cells(ref, gx, gy)
    for n in range(N):
        counts = np.bincount(cells[n], minlength=G)
        expect = np.concatenate([[0], np.cumsum(counts)])
        assert np.array_equal(cs[n], expect), f"cell_start of entry {n}"
        assert np.array_equal(np.sort(perm[n]), np.arange(Lq)), f"perm of entry {n}"
        assert np.array_equal(cells[n][perm[n]], np.repeat(np.arange(G), counts)), \
            f"perm of entry {n} is not sorted by cell"


def _loc_equal(gpu, ora, what):
    """Locations bit for bit; NaN (from a NaN reference point) only needs to
    be NaN on both sides, since its payload is not specified."""
    g, o = np.asarray(gpu), np.asarray(ora, dtype=np.float32)
    nan = np.isnan(o)
    assert np.array_equal(np.isnan(g), nan), f"{what}: NaN positions differ"
    assert_bits_equal(np.where(nan, 0, g).astype(np.float32),
                      np.where(nan, 0, o).astype(np.float32), what=what)


def _fused_both(d, halo, cps, value=None):
    """Tiled and untiled fused forward on the same inputs."""
    sh = d["spatial_shapes"]
    value = to_dev(d["value"]) if value is None else value
    ref, off, z = (to_dev(d[k]) for k in ("reference_points", "offsets", "logits"))
    plan = msda_tile_plan(value, sh, None, ref, K=d["logits"].shape[-1], halo=halo,
                          ctas_per_sm=cps)
    tiled = msda_forward_fused_tiled(value, sh, None, ref, off, z, plan, return_sampling=True)
    untiled = msda_forward_fused(value, sh, None, ref, off, z, return_sampling=True)
    return plan, tiled, untiled


@pytest.mark.parametrize("name,halo,cps", [("encoder", 3, 2), ("encoder", 4, 1),
                                           ("encoder", 3, 3), ("encoder_bf16", 3, 2),
                                           ("encoder_compass", 4, 2)])
def test_tiled_encoder_fused_forward(name, halo, cps):
    w = wl.WORKLOADS[name]
    d = wl.make_inputs(w, with_grad=False)
    sh = d["spatial_shapes"]
    plan, (out, loc, a), (uout, uloc, ua) = _fused_both(d, halo, cps)
    _check_plan(plan, d["reference_points"])
    ora, oloc, oA = oracle.forward_fused(d["value"], sh, d["reference_points"], d["offsets"],
                                         d["logits"])
    assert_bits_equal(host(loc), oloc, what=f"{name} tiled loc")
    assert_close(host(a), oA, **F32, what=f"{name} tiled softmax")
    assert_close(host(out), ora, **F32, what=f"{name} tiled out")
    assert_close(host(out), host(uout), **F32, what=f"{name} tiled vs untiled")
    assert torch.equal(loc, uloc) and torch.equal(a, ua)


def test_tiled_stress_forward():
    """N=8, bf16 value, K=8 (32 samples per item), offsets N(0, 4) px with 5%
    pushed out of range; oracle on three batch entries, the untiled forward
    (a different kernel for 32-sample items) within the fp32 tolerance."""
    w = wl.STRESS
    d = wl.make_inputs(w, with_grad=False)
    sh = d["spatial_shapes"]
    plan, (out, loc, a), (uout, uloc, ua) = _fused_both(d, 8, 1)
    assert torch.equal(loc, uloc) and torch.equal(a, ua)
    assert_close(host(out), host(uout), **F32, what="stress tiled vs untiled")
    for n in (0, 3, w.N - 1):
        sl = slice(n, n + 1)
        ref, off, z = (np.ascontiguousarray(d[k][sl]) for k in
                       ("reference_points", "offsets", "logits"))
        ora, oloc, oA = oracle.forward_fused(np.ascontiguousarray(d["value"][sl]), sh, ref,
                                             off, z)
        assert_bits_equal(host(loc[sl]), oloc, what=f"stress tiled loc n={n}")
        assert_close(host(out[sl]), ora, **F32, what=f"stress tiled out n={n}")


# (N, Lq, M, D, K, shapes, dtype, halo, cps, ref): random problems over the
# fast kernels' lane layouts; ref "pixel" puts the queries on the pixel
# centres of the levels (the encoder layout), "uniform" draws them in the
# unit square, "wide" in [-0.3, 1.3]^2 with some NaN
CASES = [
    (2, None, 8, 32, 4, ((24, 30), (12, 15), (6, 8), (3, 4)), "f32", 3, 2, "pixel"),
    (1, None, 4, 16, 4, ((20, 18), (10, 9)), "f32", 2, 2, "pixel"),      # R = 4
    (3, None, 2, 8, 2, ((17, 23), (9, 12), (5, 6)), "f32", 1, 3, "pixel"),  # R = 2
    (1, None, 3, 4, 4, ((15, 15), (8, 8)), "f32", 0, 1, "pixel"),        # R = 1, halo 0
    (2, 700, 8, 32, 4, ((30, 40), (15, 20), (8, 10), (4, 5)), "f32", 4, 2, "uniform"),
    (1, None, 4, 32, 2, ((26, 22), (13, 11), (7, 6)), "bf16", 3, 2, "pixel"),  # bf16 16-B lanes
    (1, 400, 2, 16, 4, ((16, 16), (8, 8)), "bf16", 3, 1, "uniform"),     # bf16 8-B lanes
    (1, 300, 2, 64, 2, ((12, 14), (6, 7)), "bf16", 3, 2, "uniform"),     # 128-byte bf16 rows
    (2, 333, 4, 32, 8, ((20, 20), (10, 10), (5, 5), (3, 3)), "f32", 5, 1, "wide"),  # 32 samples
    (1, 250, 2, 32, 1, ((14, 16), (0, 5), (7, 8), (4, 0)), "f32", 3, 2, "uniform"),  # empty levels
    (2, 120, 4, 32, 3, tuple((12 - i, 10 + i) for i in range(8)), "f32", 2, 2, "wide"),  # L = 8
]


def _refs(case, rng):
    N, Lq, M, D, K, shapes, dt, halo, cps, kind = case
    if kind == "pixel":
        r = wl.pixel_centre_queries(shapes)
        return np.ascontiguousarray(np.broadcast_to(r, (N,) + r.shape)).astype(np.float32)
    lo, hi = (0.0, 1.0) if kind == "uniform" else (-0.3, 1.3)
    r = rng.uniform(lo, hi, size=(N, Lq, 2)).astype(np.float32)
    if kind == "wide":
        r[0, :3] = np.nan
        r[-1, 3:5, 0] = np.inf
    return r


@pytest.mark.parametrize("case", CASES, ids=[f"case{i}" for i in range(len(CASES))])
def test_tiled_random_problems(case):
    N, Lq, M, D, K, shapes, dt, halo, cps, kind = case
    S = int(sum(h * w for h, w in shapes))
    Lq = S if Lq is None else Lq
    rng = np.random.default_rng(4000 + D + K + halo)
    d = wl.make_random_problem(4100 + Lq, N=N, Lq=Lq, M=M, D=D, K=K, shapes=shapes,
                               value_dtype=dt, offset_std=1.5)
    d["reference_points"] = _refs(case, rng)
    sh = d["spatial_shapes"]
    value = to_dev(d["value"])
    plan, (out, loc, a), (uout, uloc, ua) = _fused_both(d, halo, cps, value)
    _check_plan(plan, d["reference_points"])
    ora, oloc, oA = oracle.forward_fused(d["value"], sh, d["reference_points"], d["offsets"],
                                         d["logits"])
    _loc_equal(host(loc), oloc, "tiled fused loc")
    assert_close(host(a), oA, **F32, what="tiled fused softmax")
    assert_close(host(out), ora, **F32, what="tiled fused out")
    assert_close(host(out), host(uout), **F32, what="tiled vs untiled")
    # the unfused tiled call on the oracle's locations and weights
    A = oA.astype(np.float32)
    t_out = msda_forward_tiled(value, sh, None, to_dev(oloc), to_dev(A), plan)
    assert_close(host(t_out), oracle.forward(d["value"], sh, oloc, A), **F32,
                 what="tiled unfused out")
    assert_close(host(t_out), host(msda_forward(value, sh, None, to_dev(oloc), to_dev(A))),
                 **F32, what="tiled vs untiled unfused")


def test_tiled_all_queries_in_one_cell():
    """Every reference point in one cell: one work unit per (entry, head)
    holds all queries; the other cells are empty."""
    shapes = ((18, 22), (9, 11))
    d = wl.make_random_problem(55, N=2, Lq=300, M=2, D=32, K=4, shapes=shapes)
    d["reference_points"][:] = np.float32(0.37)
    sh = d["spatial_shapes"]
    plan, (out, loc, a), (uout, _, _) = _fused_both(d, 3, 2)
    _check_plan(plan, d["reference_points"])
    assert_close(host(out), host(uout), **F32, what="one-cell tiled vs untiled")
    ora, _, _ = oracle.forward_fused(d["value"], sh, d["reference_points"], d["offsets"],
                                     d["logits"])
    assert_close(host(out), ora, **F32, what="one-cell out")


def test_tiled_plan_reuse_and_stream_order():
    """One plan serves repeated calls; results are deterministic and follow
    stream order on a side stream."""
    d = wl.make_inputs(wl.ENCODER, with_grad=False)
    sh = d["spatial_shapes"]
    value, ref, off, z = (to_dev(d[k]) for k in ("value", "reference_points", "offsets",
                                                 "logits"))
    plan = msda_tile_plan(value, sh, None, ref, K=4, halo=3)
    a = msda_forward_fused_tiled(value, sh, None, ref, off, z, plan)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        b = msda_forward_fused_tiled(value, sh, None, ref, off, z, plan)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
