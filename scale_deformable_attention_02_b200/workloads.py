"""Seeded synthetic inputs of the MSDeformAttn (multi-scale deformable attention) core.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no level prefix sums, no softmax, no location or sampling
math).  Both the CPU oracle tests and the CUDA path read inputs from here, so
the two sides always see identical bits.

Shapes follow the Deformable DETR encoder/decoder (Deformable DETR wiki page,
"Architecture" and "Hyperparameters": L = 4 levels at strides 8..64, C = 256,
M = 8 heads so D = C/M = 32, K = 4 points, N = 300 decoder queries).  Feature
maps for an 800x1066-class image give level shapes (100,134), (50,67),
(25,34), (13,17).  No image, dataset or trained weight is involved: values
are random normals standing in for projected feature maps.

Conventions (all readings of the pages, stated once here):
  * value is [N, S, M, D], S = sum_l H_l*W_l, levels stacked in order, each
    level row-major in (h, w).
  * spatial_shapes is [L, 2] int64 holding (H_l, W_l).
  * sampling locations / reference points are normalised (x, y) in [0, 1],
    x along the width.
  * pixel offsets are per-level pixels, last dim (dx, dy).
  * "N(0, s)" in a workload recipe means mean 0 and standard deviation s.
  * bf16 value is drawn in fp32 and rounded once to bf16 (round to nearest
    even); both sides read the same 16-bit patterns.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

ENCODER_SHAPES = ((100, 134), (50, 67), (25, 34), (13, 17))
STRESS_SHAPES = ((167, 167), (84, 84), (42, 42), (21, 21))
TINY_SHAPES = ((8, 8), (4, 4))


@dataclass(frozen=True)
class Workload:
    """One synthetic problem: dims, level shapes and the input recipe."""

    name: str
    N: int
    M: int
    D: int
    K: int
    shapes: tuple
    Lq: int | None  # None: one query per pixel of every level (encoder)
    value_dtype: str  # "f32" or "bf16"
    seed: int
    recipe: str  # "tiny", "decoder", "encoder", "stress", "compass"
    offset_std: float = 0.0
    oob_fraction: float = 0.0
    notes: str = field(default="", compare=False)

    @property
    def L(self) -> int:
        return len(self.shapes)

    @property
    def S(self) -> int:
        return int(sum(h * w for h, w in self.shapes))

    @property
    def queries(self) -> int:
        return self.S if self.Lq is None else self.Lq

    def dims(self) -> dict:
        return dict(N=self.N, Lq=self.queries, S=self.S, M=self.M, D=self.D,
                    L=self.L, K=self.K)


# The five problem sizes this library is measured and checked on.
TINY = Workload("tiny", N=1, M=2, D=8, K=2, shapes=TINY_SHAPES, Lq=16,
                value_dtype="f32", seed=1, recipe="tiny")
DECODER = Workload("decoder", N=2, M=8, D=32, K=4, shapes=ENCODER_SHAPES,
                   Lq=300, value_dtype="f32", seed=2, recipe="decoder",
                   offset_std=2.0)
ENCODER = Workload("encoder", N=2, M=8, D=32, K=4, shapes=ENCODER_SHAPES,
                   Lq=None, value_dtype="f32", seed=3, recipe="encoder",
                   offset_std=1.5)
ENCODER_BF16 = Workload("encoder_bf16", N=2, M=8, D=32, K=4,
                        shapes=ENCODER_SHAPES, Lq=None, value_dtype="bf16",
                        seed=3, recipe="encoder", offset_std=1.5)
ENCODER_BWD = Workload("encoder_bwd", N=2, M=8, D=32, K=4,
                       shapes=ENCODER_SHAPES, Lq=None, value_dtype="f32",
                       seed=4, recipe="encoder", offset_std=1.5)
STRESS = Workload("stress", N=8, M=8, D=32, K=8, shapes=STRESS_SHAPES,
                  Lq=None, value_dtype="bf16", seed=5, recipe="stress",
                  offset_std=4.0, oob_fraction=0.05)
# The encoder at initialisation: every head samples along its compass
# direction, k pixels out for point k, with uniform weights (zero logits).
ENCODER_COMPASS = Workload("encoder_compass", N=2, M=8, D=32, K=4,
                           shapes=ENCODER_SHAPES, Lq=None, value_dtype="f32",
                           seed=6, recipe="compass")

WORKLOADS = {w.name: w for w in (TINY, DECODER, ENCODER, ENCODER_BF16,
                                 ENCODER_BWD, STRESS, ENCODER_COMPASS)}

# Offset directions (dx, dy) of the eight heads at initialisation, in the
# order the "Deformable DETR" wiki page lists them ("Initialization"): head m
# samples point k (k = 1..K) at k * COMPASS[m] pixels on every level.
COMPASS = ((-1, -1), (-1, 0), (-1, 1), (0, -1), (0, 1), (1, -1), (1, 0), (1, 1))


def compass_offsets(N: int, Lq: int, M: int, L: int, K: int, scale: float = 1.0) -> np.ndarray:
    """[N,Lq,M,L,K,2] float32 offsets of the compass initialisation: head m,
    point k (0-based) at (k+1) * COMPASS[m] * scale pixels, the same for every
    query and level.  scale = 1/(2K) gives the iterative-refinement variant
    (box units).  Needs M = 8."""
    if M != len(COMPASS):
        raise ValueError("the compass pattern has one direction per head: M must be 8")
    dirs = np.asarray(COMPASS, dtype=np.float32)                      # [M, 2]
    ks = np.arange(1, K + 1, dtype=np.float32) * np.float32(scale)    # [K]
    one = dirs[:, None, None, :] * ks[None, None, :, None]           # [M, 1, K, 2]
    return np.ascontiguousarray(
        np.broadcast_to(one[None, None], (N, Lq, M, L, K, 2)).astype(np.float32))


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest, ties to even.

    Input encoding only (finite inputs): keep the top 16 bits after adding
    0x7FFF plus the lowest kept bit."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> fp32 values (exact widening)."""
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def spatial_shapes_array(shapes) -> np.ndarray:
    return np.asarray(shapes, dtype=np.int64).reshape(-1, 2)


def pixel_centre_queries(shapes) -> np.ndarray:
    """Encoder queries: one per pixel of every level, level-major then
    row-major, each with its own pixel centre as normalised (x, y) reference
    point (an encoder query refers to its own pixel: Deformable DETR wiki
    page, "Architecture / Encoder").  Computed in fp32: ((w+0.5)/W, (h+0.5)/H).
    Returns [S, 2] float32."""
    out = []
    for (h_l, w_l) in shapes:
        hh, ww = np.meshgrid(np.arange(h_l, dtype=np.float32),
                             np.arange(w_l, dtype=np.float32), indexing="ij")
        x = (ww + np.float32(0.5)) / np.float32(w_l)
        y = (hh + np.float32(0.5)) / np.float32(h_l)
        out.append(np.stack([x.ravel(), y.ravel()], axis=-1))
    return np.concatenate(out, axis=0).astype(np.float32)


def _normal(rng, shape, std=1.0):
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def make_inputs(w: Workload, with_grad: bool = True) -> dict:
    """Draw every input of workload ``w`` from PCG64(seed).

    Returns a dict of numpy arrays:
      value            [N,S,M,D] float32, or uint16 bf16 bits when bf16
      value_f32        the same values widened to float32 (bf16 only)
      spatial_shapes   [L,2] int64
      sampling_locations [N,Lq,M,L,K,2] float32   (tiny only)
      reference_points [N,Lq,2] float32            (all but tiny)
      offsets          [N,Lq,M,L,K,2] float32 pixels (all but tiny)
      logits           [N,Lq,M,L,K] float32
      grad_out         [N,Lq,M*D] float32           (if with_grad)
    """
    rng = np.random.default_rng(w.seed)
    N, M, D, K, L, S, Lq = w.N, w.M, w.D, w.K, w.L, w.S, w.queries
    d = {"spatial_shapes": spatial_shapes_array(w.shapes)}
    if w.recipe == "tiny":
        v = rng.uniform(-1.0, 1.0, size=(N, S, M, D)).astype(np.float32)
    else:
        v = _normal(rng, (N, S, M, D))
    if w.value_dtype == "bf16":
        d["value"] = round_to_bf16_bits(v)
        d["value_f32"] = bf16_bits_to_f32(d["value"])
    else:
        d["value"] = v
    if w.recipe == "tiny":
        d["sampling_locations"] = rng.uniform(
            -0.1, 1.1, size=(N, Lq, M, L, K, 2)).astype(np.float32)
    else:
        if w.recipe == "decoder":
            d["reference_points"] = rng.uniform(
                0.0, 1.0, size=(N, Lq, 2)).astype(np.float32)
        else:
            ref = pixel_centre_queries(w.shapes)
            d["reference_points"] = np.ascontiguousarray(
                np.broadcast_to(ref, (N, Lq, 2)))
        if w.recipe == "compass":
            d["offsets"] = compass_offsets(N, Lq, M, L, K)
        else:
            off = _normal(rng, (N, Lq, M, L, K, 2), w.offset_std)
            if w.oob_fraction > 0.0:
                push_offsets_out_of_range(rng, off, w.shapes, w.oob_fraction)
            d["offsets"] = off
    if w.recipe == "compass":
        d["logits"] = np.zeros((N, Lq, M, L, K), dtype=np.float32)
    else:
        d["logits"] = _normal(rng, (N, Lq, M, L, K))
    if with_grad:
        d["grad_out"] = _normal(rng, (N, Lq, M * D))
    return d


def push_offsets_out_of_range(rng, off: np.ndarray, shapes, fraction: float):
    """For a Bernoulli(fraction) subset of samples, move dx (or dy, picked at
    random) by +-(W_l + 8) (resp. +-(H_l + 8)) pixels, so the sample leaves
    its level's map.  In place on off[..., L, K, 2]."""
    L = off.shape[-3]
    hit = rng.random(size=off.shape[:-1]) < fraction
    axis = rng.integers(0, 2, size=off.shape[:-1])
    sign = np.where(rng.random(size=off.shape[:-1]) < 0.5, -1.0, 1.0)
    for lvl in range(L):
        h_l, w_l = shapes[lvl]
        sel = hit[..., lvl, :]
        ax = axis[..., lvl, :]
        sg = sign[..., lvl, :].astype(np.float32)
        ox = off[..., lvl, :, 0]
        oy = off[..., lvl, :, 1]
        ox += np.where(sel & (ax == 0), sg * np.float32(w_l + 8), 0).astype(np.float32)
        oy += np.where(sel & (ax == 1), sg * np.float32(h_l + 8), 0).astype(np.float32)


def make_random_problem(seed: int, N: int, Lq: int, M: int, D: int, K: int,
                        shapes, value_dtype: str = "f32",
                        loc_low: float = -0.1, loc_high: float = 1.1,
                        offset_std: float = 2.0) -> dict:
    """A small random problem of arbitrary dims, for edge-case and
    ragged-size tests.  Carries both unfused inputs (sampling_locations) and
    fused inputs (reference_points, offsets), plus logits and grad_out."""
    rng = np.random.default_rng(seed)
    L = len(shapes)
    S = int(sum(h * w for h, w in shapes))
    v = rng.uniform(-1.0, 1.0, size=(N, S, M, D)).astype(np.float32)
    d = {"spatial_shapes": spatial_shapes_array(shapes)}
    if value_dtype == "bf16":
        d["value"] = round_to_bf16_bits(v)
        d["value_f32"] = bf16_bits_to_f32(d["value"])
    else:
        d["value"] = v
    d["sampling_locations"] = rng.uniform(
        loc_low, loc_high, size=(N, Lq, M, L, K, 2)).astype(np.float32)
    d["reference_points"] = rng.uniform(0.0, 1.0, size=(N, Lq, 2)).astype(np.float32)
    d["offsets"] = _normal(rng, (N, Lq, M, L, K, 2), offset_std)
    d["logits"] = _normal(rng, (N, Lq, M, L, K))
    d["grad_out"] = _normal(rng, (N, Lq, M * D))
    return d


def make_wide_batch_problem(seed: int, N: int, Lq: int, M: int, D: int, K: int,
                            shapes) -> dict:
    """A problem with many batch entries that share one value block: every
    batch entry n reads value[n] = value_block[0], so the full map
    (N x the block) can be laid out on the device by repetition while a
    single block stays on the host.  Per-entry locations, reference points,
    offsets, logits and grad_out are drawn for all N entries (as in
    make_random_problem).  Used to reach value maps of close to 2^31
    elements."""
    rng = np.random.default_rng(seed)
    L = len(shapes)
    S = int(sum(h * w for h, w in shapes))
    return {
        "spatial_shapes": spatial_shapes_array(shapes),
        "value_block": rng.uniform(-1.0, 1.0, size=(1, S, M, D)).astype(np.float32),
        "sampling_locations": rng.uniform(-0.1, 1.1, size=(N, Lq, M, L, K, 2)).astype(np.float32),
        "reference_points": rng.uniform(0.0, 1.0, size=(N, Lq, 2)).astype(np.float32),
        "offsets": _normal(rng, (N, Lq, M, L, K, 2), 2.0),
        "logits": _normal(rng, (N, Lq, M, L, K)),
        "grad_out": _normal(rng, (N, Lq, M * D)),
    }


def make_windowed_problem(seed: int, shapes, windows, Lq: int, K: int, D: int) -> dict:
    """One batch entry and one head over levels that may be huge.  Only
    rectangular pixel windows of level 0 and every pixel of the other levels
    carry values; every level-0 sample of query q lies inside window
    q % len(windows), at least one and a half pixels from its edges, so all
    four corners of its cell fall inside the window.  The samples of the
    other levels are uniform over those levels.

      windows   ((row0, col0, rows, cols), ...) on level 0, each at least 4x4
    Returns the window rows as (level-0 pixel row index, values [.., D])
    pairs plus the locations, logits and grad_out; the caller lays the rows
    out in a zero map of S rows."""
    rng = np.random.default_rng(seed)
    L = len(shapes)
    H0, W0 = shapes[0]
    loc = np.empty((1, Lq, 1, L, K, 2), dtype=np.float32)
    for q in range(Lq):
        r0, c0, nr, nc = windows[q % len(windows)]
        # pixel coordinates in [c0 + 1.5, c0 + nc - 2.5]: the cell and its
        # right/lower neighbour stay inside the window
        px = rng.uniform(c0 + 1.5, c0 + nc - 2.5, size=K)
        py = rng.uniform(r0 + 1.5, r0 + nr - 2.5, size=K)
        loc[0, q, 0, 0, :, 0] = ((px + 0.5) / W0).astype(np.float32)
        loc[0, q, 0, 0, :, 1] = ((py + 0.5) / H0).astype(np.float32)
        for lvl in range(1, L):
            loc[0, q, 0, lvl] = rng.uniform(0.0, 1.0, size=(K, 2)).astype(np.float32)
    rows, vals = [], []
    for (r0, c0, nr, nc) in windows:
        rr, cc = np.meshgrid(np.arange(r0, r0 + nr), np.arange(c0, c0 + nc), indexing="ij")
        rows.append((rr * W0 + cc).ravel().astype(np.int64))
        vals.append(rng.uniform(-1.0, 1.0, size=(nr * nc, D)).astype(np.float32))
    other = int(sum(h * w for h, w in shapes[1:]))
    return {
        "spatial_shapes": spatial_shapes_array(shapes),
        "window_rows": np.concatenate(rows),
        "window_values": np.concatenate(vals),
        "other_values": rng.uniform(-1.0, 1.0, size=(other, D)).astype(np.float32),
        "sampling_locations": loc,
        "logits": _normal(rng, (1, Lq, 1, L, K)),
        "grad_out": _normal(rng, (1, Lq, D)),
        "second_values": rng.uniform(-1.0, 1.0, size=(sum(len(r) for r in rows), D)).astype(np.float32),
    }
