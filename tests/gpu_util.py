"""Helpers shared by the GPU parity tests: device transfer and the
elementwise tolerance check |gpu - oracle| <= atol + rtol * |oracle|."""
import functools

import numpy as np
import torch

# Tolerances: fp32 outputs and weights (1e-5 relative, 1e-6 absolute);
# gradients that a kernel writes once with a plain store (the location and
# weight gradients of the ungrouped calls; the offset and logit gradients of
# the ungrouped fused backward) take the same fp32 figures (PLAIN); gradients
# accumulated with atomics in an unspecified order (grad_value, the reference
# point gradient, and the location and offset gradients that the heads of a
# deformable group share) take 1e-4 relative, 1e-5 absolute (GRAD); bf16
# value against the fp32-value oracle takes 2e-2 relative.
F32 = dict(rtol=1e-5, atol=1e-6)
PLAIN = F32
GRAD = dict(rtol=1e-4, atol=1e-5)
# Gradients that are sums also get the fp32 forward-error bound of the
# kernel's evaluation order: a term that passes through at most n roundings
# leaves |fl(sum) - sum| <= n * 2^-24 * mass (to first order), where mass is
# the oracle's sum of the absolute terms.  The longest path of any kernel is
# n = 18: a 512-byte bf16 row in the wide backward (8 FMAs inside a lane,
# 5 adds across 32 lanes, the corner weight, 2 adds over the four corners,
# the product A*W and the multiply by it); the D = 32 fp32 fast path has 12
# (4 + 3 + 1 + 2 + 2).
U32 = 2.0 ** -24
KAPPA = 18


def grad_tol(groups: int, heads: int) -> dict:
    """Tolerance of a location or offset gradient: written once per group
    when every head has its own locations, else summed over the group's heads
    with atomics."""
    return PLAIN if groups == heads else GRAD


@functools.lru_cache(maxsize=2)
def cached_inputs(name: str) -> dict:
    """make_inputs of a named workload, drawn once per test session (the
    stress workload's draws take a minute of CPU).  Callers must not modify
    the arrays."""
    from scale_deformable_attention_02_b200 import workloads as wl
    return wl.make_inputs(wl.WORKLOADS[name])


def dev():
    return torch.device("cuda:0")


def to_dev(a: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:  # bf16 bit patterns
        return torch.from_numpy(a.view(np.int16)).to(dev()).view(torch.bfloat16)
    return torch.from_numpy(a).to(dev())


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").numpy()


def value_grad_terms(value, shapes, loc, attn, grad_out):
    """(terms, mass) of every grad_value element: terms is the number of
    (sample, corner) contributions it sums, counted from the oracle's corner
    rows; mass is the sum of their absolute values, which is the oracle's
    grad_value for |attention weights| and |grad_out| (corner weights are not
    negative).  A sum of n terms formed in any order is within
    n * 2^-24 * mass of the exact sum, whatever the order of the atomics."""
    import oracle
    N, Lq, M, L, K, _ = loc.shape
    S, D = value.shape[1], value.shape[3]
    rows = oracle.sample_points(loc, shapes)["rows"].reshape(N, Lq, M, L * K * 4)
    n = np.arange(N).reshape(N, 1, 1, 1)
    m = np.arange(M).reshape(1, 1, M, 1)
    ok = rows >= 0
    idx = ((n * S + rows) * M + m)[ok]
    cnt = np.bincount(idx, minlength=N * S * M).reshape(N, S, M, 1)
    terms = np.broadcast_to(cnt, (N, S, M, D)).astype(np.float64)
    mass = oracle.backward(value, shapes, loc, np.abs(np.asarray(attn, np.float64)),
                           np.abs(np.asarray(grad_out, np.float64)))[0]
    return terms, mass


def assert_close(gpu, ora, rtol, atol, what="", mass=None, terms=None):
    """|gpu - ora| <= atol + rtol*|ora| (+ KAPPA * 2^-24 * mass if given, or
    terms * 2^-24 * mass with a per-element term count)."""
    g = np.asarray(gpu, dtype=np.float64)
    o = np.asarray(ora, dtype=np.float64)
    assert g.shape == o.shape, (what, g.shape, o.shape)
    fin = np.isfinite(o)
    assert np.array_equal(np.isfinite(g), fin), f"{what}: non-finite entries differ"
    g = np.where(fin, g, 0.0)
    o = np.where(fin, o, 0.0)
    err = np.abs(g - o)
    bound = atol + rtol * np.abs(o)
    if mass is not None:
        k = KAPPA if terms is None else np.asarray(terms, dtype=np.float64)
        bound = bound + k * U32 * np.where(fin, np.asarray(mass, dtype=np.float64), 0.0)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} elements outside "
            f"atol={atol} rtol={rtol}; worst at {i}: gpu={g[i]!r} oracle={o[i]!r} "
            f"err={err[i]:.3e} bound={bound[i]:.3e}")


def assert_bits_equal(gpu, ora, what=""):
    g = np.asarray(gpu)
    o = np.asarray(ora)
    assert g.shape == o.shape, (what, g.shape, o.shape)
    if g.dtype == np.float32:
        g = g.view(np.uint32)
        o = np.asarray(o, dtype=np.float32).view(np.uint32)
    mism = g != o
    if mism.any():
        i = np.argwhere(mism)[0]
        raise AssertionError(f"{what}: {int(mism.sum())} mismatches; first at {tuple(i)}: "
                             f"gpu={g[tuple(i)]} oracle={o[tuple(i)]}")
