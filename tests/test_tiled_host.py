"""The tile-plan calls of include/msda_tiled.h on the host: msda_tile_plan_init
picks the grid and windows without a GPU, and every tiled call rejects a plan
that does not belong to its problem, or that was altered, before any device
work (fake device pointers, never dereferenced)."""
import ctypes

import numpy as np
import pytest

import oracle
from scale_deformable_attention_02_b200 import _lib
from scale_deformable_attention_02_b200 import build as msda_build
from scale_deformable_attention_02_b200 import workloads as wl

OK, NULL, SHAPE, LEVELS, DTYPE, ALIGN, ALIAS, UNSUP = range(8)
BASE = 1 << 32
GAP = 1 << 28


def fake(i, off=0):
    return ctypes.c_void_p(BASE + i * GAP + off)


@pytest.fixture(scope="module")
def lib():
    msda_build.build()
    return _lib.load()


def _problem(name):
    w = wl.WORKLOADS[name]
    sh = wl.spatial_shapes_array(w.shapes)
    st, S = oracle.level_start_index(sh)
    return w, sh, st, _lib.Dims(w.N, w.queries, S, w.M, w.D, w.L, w.K)


def _init(lib, sh, st, d, dtype=0, halo=3, cps=2):
    pl = _lib.TilePlan()
    r = lib.msda_tile_plan_init(dtype, sh.ctypes.data_as(ctypes.c_void_p),
                                st.ctypes.data_as(ctypes.c_void_p), d, halo, cps,
                                ctypes.byref(pl))
    return r, pl


def _budget(cps):
    per_cta = min(233472 // cps - 1024, 232448)
    return per_cta - 14 * 1024


@pytest.mark.parametrize("name,dtype,halo,cps", [("encoder", 0, 3, 2), ("encoder", 0, 4, 1),
                                                 ("encoder_bf16", 1, 3, 3),
                                                 ("stress", 1, 8, 1), ("decoder", 0, 2, 2)])
def test_plan_windows_follow_the_cell_grid(lib, name, dtype, halo, cps):
    """Each level's window is the cell's extent on that level (ceil(W/gx)
    pixels) plus the halo and one corner on both sides, capped at the level
    and its one-pixel border; all windows fit the shared memory of `cps`
    CTAs per SM; the device buffer holds the cell starts and the sorted
    queries."""
    w, sh, st, d = _problem(name)
    r, pl = _init(lib, sh, st, d, dtype, halo, cps)
    assert r == OK
    gx, gy = pl.grid_x, pl.grid_y
    rowb = w.D * (2 if dtype else 4)
    total = 0
    for l, (H, W) in enumerate(sh):
        bw = min(-(-W // gx) + 2 * halo + 2, W + 2, 256)
        bh = min(-(-H // gy) + 2 * halo + 2, H + 2, 256)
        assert (pl.window_w[l], pl.window_h[l]) == (bw, bh)
        total += -(-bw * bh * rowb // 128) * 128
    assert pl.window_bytes == total <= _budget(cps)
    G = gx * gy
    assert pl.device_bytes == -(-(-(-(w.N * (G + 1) * 4) // 256) * 256 + w.N * w.queries * 4)
                                // 256) * 256
    # the coarsest grid that fits: one cell fewer along x does not fit, or
    # the finer grid was needed for enough work units per CTA
    assert (pl.N, pl.Lq, pl.S, pl.L, pl.D) == (w.N, w.queries, d.S, w.L, w.D)


def test_plan_init_errors(lib):
    w, sh, st, d = _problem("encoder")
    p = sh.ctypes.data_as(ctypes.c_void_p)
    s = st.ctypes.data_as(ctypes.c_void_p)
    pl = _lib.TilePlan()
    assert lib.msda_tile_plan_init(0, p, s, d, 3, 2, None) == NULL
    assert lib.msda_tile_plan_init(0, p, s, d, -1, 2, ctypes.byref(pl)) == SHAPE
    assert lib.msda_tile_plan_init(0, p, s, d, 65, 2, ctypes.byref(pl)) == SHAPE
    assert lib.msda_tile_plan_init(0, p, s, d, 3, 4, ctypes.byref(pl)) == SHAPE
    assert lib.msda_tile_plan_init(5, p, s, d, 3, 2, ctypes.byref(pl)) == DTYPE
    # beyond the tiled limits: L*K > 32, rows over 128 bytes, 9 levels
    d2 = _lib.Dims(d.N, d.Lq, d.S, d.M, d.D, d.L, 9)
    assert lib.msda_tile_plan_init(0, p, s, d2, 3, 2, ctypes.byref(pl)) == UNSUP
    d3 = _lib.Dims(d.N, d.Lq, d.S, d.M, 64, d.L, d.K)
    assert lib.msda_tile_plan_init(0, p, s, d3, 3, 2, ctypes.byref(pl)) == UNSUP
    sh9 = wl.spatial_shapes_array(tuple((4, 4) for _ in range(9)))
    st9, S9 = oracle.level_start_index(sh9)
    d9 = _lib.Dims(1, 10, S9, 2, 8, 9, 1)
    assert lib.msda_tile_plan_init(0, sh9.ctypes.data_as(ctypes.c_void_p),
                                   st9.ctypes.data_as(ctypes.c_void_p), d9, 2, 2,
                                   ctypes.byref(pl)) == UNSUP
    # a halo whose windows cannot fit even on the finest grid
    assert lib.msda_tile_plan_init(0, p, s, d, 64, 3, ctypes.byref(pl)) == UNSUP


def _fwd(lib, pl, sh, st, d, dtype=0, buf=None):
    return lib.msda_forward_fused_tiled(
        fake(0), dtype, sh.ctypes.data_as(ctypes.c_void_p), st.ctypes.data_as(ctypes.c_void_p),
        fake(1), 2, fake(2), fake(3), fake(4), None, None, d, ctypes.byref(pl) if pl else None,
        buf if buf is not None else fake(5), None)


def test_tiled_calls_reject_foreign_or_altered_plans(lib):
    w, sh, st, d = _problem("encoder")
    r, pl = _init(lib, sh, st, d)
    assert r == OK
    assert _fwd(lib, None, sh, st, d) == NULL
    assert _fwd(lib, pl, sh, st, d, buf=ctypes.c_void_p(0)) == NULL
    assert _fwd(lib, pl, sh, st, d, buf=fake(5, 8)) == ALIGN
    assert _fwd(lib, pl, sh, st, d, dtype=1) == SHAPE  # built for fp32 value
    d2 = _lib.Dims(d.N + 1, d.Lq, d.S, d.M, d.D, d.L, d.K)
    assert _fwd(lib, pl, sh, st, d2) == SHAPE  # another batch size
    for field, delta in (("window_w", 1), ("window_h", -1)):
        bad = _lib.TilePlan.from_buffer_copy(pl)
        getattr(bad, field)[0] += delta
        assert _fwd(lib, bad, sh, st, d) == SHAPE, field
    for field, value in (("grid_x", 0), ("halo", pl.halo + 1), ("window_bytes", 10 ** 6),
                         ("ctas_per_sm", 7), ("device_bytes", pl.device_bytes + 256)):
        bad = _lib.TilePlan.from_buffer_copy(pl)
        setattr(bad, field, value)
        assert _fwd(lib, bad, sh, st, d) == SHAPE, field
    # an output over the plan buffer
    assert lib.msda_forward_fused_tiled(
        fake(0), 0, sh.ctypes.data_as(ctypes.c_void_p), st.ctypes.data_as(ctypes.c_void_p),
        fake(1), 2, fake(2), fake(3), fake(5), None, None, d, ctypes.byref(pl), fake(5),
        None) == ALIAS
    # the backward calls check the same way
    assert lib.msda_backward_tiled(
        fake(0), 0, sh.ctypes.data_as(ctypes.c_void_p), st.ctypes.data_as(ctypes.c_void_p),
        fake(1), fake(2), fake(3), fake(4), None, None, d2, ctypes.byref(pl), fake(5),
        None) == SHAPE
    assert lib.msda_backward_fused_tiled(
        fake(0), 0, sh.ctypes.data_as(ctypes.c_void_p), st.ctypes.data_as(ctypes.c_void_p),
        fake(1), 3, fake(2), fake(3), fake(4), fake(6), None, None, None, d, ctypes.byref(pl),
        fake(5), None) == SHAPE


def test_plan_build_argument_errors(lib):
    w, sh, st, d = _problem("encoder")
    r, pl = _init(lib, sh, st, d)
    assert lib.msda_tile_plan_build(None, fake(1), 2, fake(5), None) == NULL
    assert lib.msda_tile_plan_build(ctypes.byref(pl), fake(1), 3, fake(5), None) == SHAPE
    assert lib.msda_tile_plan_build(ctypes.byref(pl), fake(1), 2, None, None) == NULL
    assert lib.msda_tile_plan_build(ctypes.byref(pl), fake(1, 4), 2, fake(5), None) == ALIGN
    assert lib.msda_tile_plan_build(ctypes.byref(pl), fake(1), 2, fake(1, 64), None) == ALIAS
    bad = _lib.TilePlan.from_buffer_copy(pl)
    bad.device_bytes -= 256
    assert lib.msda_tile_plan_build(ctypes.byref(bad), fake(1), 2, fake(5), None) == SHAPE
