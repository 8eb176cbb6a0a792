"""The bounds-checked build (libmsda_checked.so, -DMSDA_CHECKED) on the GPU.

1. With the default bound (the whole value map) every entry point returns OK
   and matches the oracle as the product build does: the checks change no
   arithmetic.
2. With the bound lowered to a pixel boundary inside the value map, the
   kernels skip every gather and scatter at or beyond it, count them, and the
   call returns MSDA_ERR_DEVICE_CHECK.  The outputs are then exactly the
   method on a value map whose pixels beyond the bound are zero (which the
   oracle computes), and grad_value beyond the bound stays zero.  Every access
   that is made stays inside the caller's buffers: the lowered bound only
   removes accesses.
3. The device word is cleared after a report: the next call returns OK.
"""
import numpy as np
import pytest
import torch

import oracle
from scale_deformable_attention_02_b200 import (MsdaError, checked_library, last_violation,
                                                msda_backward, msda_backward_fused,
                                                msda_forward, msda_forward_fused)
from scale_deformable_attention_02_b200 import workloads as wl

from gpu_util import F32, GRAD, PLAIN, assert_close, host, to_dev, value_grad_terms

pytestmark = pytest.mark.gpu

DEVICE_CHECK = 9


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


# (N, Lq, M, D, K, shapes, dtype): fast and wide kernels of both dtypes
CASES = [
    (2, 41, 8, 32, 4, ((10, 13), (5, 7), (3, 4), (2, 2)), "f32"),  # fast, R = 8
    (2, 41, 8, 32, 4, ((10, 13), (5, 7), (3, 4), (2, 2)), "bf16"),  # fast bf16
    (1, 50, 2, 24, 2, ((6, 9), (3, 5)), "f32"),                      # idle chunk lanes
    (1, 23, 2, 64, 2, ((8, 8), (4, 4)), "f32"),                      # wide, 256-B rows
    (1, 17, 3, 256, 2, ((5, 4), (2, 3)), "bf16"),                    # wide, 512-B rows
    (1, 12, 2, 32, 16, ((6, 8), (3, 4)), "f32"),                     # L*K = 32
    (1, 9, 2, 32, 16, ((6, 8), (3, 4), (2, 2)), "f32"),              # L*K = 48, blocks
    (1, 7, 2, 64, 9, ((5, 5), (3, 3), (2, 2), (1, 1)), "f32"),       # wide, L*K = 36
    (1, 9, 2, 160, 2, ((5, 4), (2, 3)), "f32"),                      # 640-B rows, two passes
]
IDS = [f"case{i}" for i in range(len(CASES))]


def _problem(case):
    N, Lq, M, D, K, shapes, dt = case
    return wl.make_random_problem(4000 + D + K, N=N, Lq=Lq, M=M, D=D, K=K, shapes=shapes,
                                  value_dtype=dt)


def _oracle_all(value, d, A):
    sh = d["spatial_shapes"]
    loc = d["sampling_locations"]
    out = oracle.forward(value, sh, loc, A)
    fo, _, _ = oracle.forward_fused(value, sh, d["reference_points"], d["offsets"],
                                    d["logits"])
    bwd = oracle.backward(value, sh, loc, A, d["grad_out"], with_mass=True)
    return out, fo, bwd


def _run_all(d, A, value_dev):
    """Forward, fused forward and backward through the current library,
    outputs preallocated so that a call that raises still leaves them."""
    sh = d["spatial_shapes"]
    N, Lq, M, L, K = d["logits"].shape
    D = d["grad_out"].shape[-1] // M
    outs = {"out": torch.zeros(N, Lq, M * D, device="cuda"),
            "fout": torch.zeros(N, Lq, M * D, device="cuda"),
            "gv": torch.zeros(value_dev.shape, device="cuda", dtype=torch.float32),
            "gl": torch.zeros(d["sampling_locations"].shape, device="cuda"),
            "ga": torch.zeros(d["logits"].shape, device="cuda")}
    codes = []
    calls = [
        lambda: msda_forward(value_dev, sh, None, to_dev(d["sampling_locations"]), to_dev(A),
                             out=outs["out"]),
        lambda: msda_forward_fused(value_dev, sh, None, to_dev(d["reference_points"]),
                                   to_dev(d["offsets"]), to_dev(d["logits"]),
                                   out=outs["fout"]),
        lambda: msda_backward(value_dev, sh, None, to_dev(d["sampling_locations"]), to_dev(A),
                              to_dev(d["grad_out"]), grad_value=outs["gv"],
                              grad_sampling_locations=outs["gl"],
                              grad_attention_weights=outs["ga"]),
    ]
    for call in calls:
        try:
            call()
            codes.append((0, 0, -1))
        except MsdaError as e:
            codes.append((e.status, e.violations, e.first_element))
    torch.cuda.synchronize()
    return outs, codes


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_checked_build_default_bound_matches_oracle(case):
    d = _problem(case)
    A = oracle.softmax(d["logits"]).astype(np.float32)
    with checked_library():
        outs, codes = _run_all(d, A, to_dev(d["value"]))
    assert codes == [(0, 0, -1)] * 3
    out, fo, (ogv, ogl, oga, mgl, mga) = _oracle_all(d["value"], d, A)
    # bf16 value bits are widened exactly on both sides: the fp32 bound holds
    assert_close(host(outs["out"]), out, **F32, what="checked forward")
    assert_close(host(outs["fout"]), fo, **F32, what="checked fused forward")
    tv, mv = value_grad_terms(d["value"], d["spatial_shapes"], d["sampling_locations"], A,
                              d["grad_out"])
    assert_close(host(outs["gv"]), ogv, **GRAD, what="checked grad_value", mass=mv, terms=tv)
    assert_close(host(outs["gl"]), ogl, **PLAIN, what="checked grad_loc", mass=mgl)
    assert_close(host(outs["ga"]), oga, **PLAIN, what="checked grad_attn", mass=mga)


def _zero_beyond(value: np.ndarray, limit: int) -> np.ndarray:
    z = value.copy()
    z.reshape(-1)[limit:] = 0
    return z


def _skipped_pairs(d, limit: int) -> int:
    """(sample, corner) pairs whose corner row starts at or beyond `limit`
    value elements: each is at least one skipped access."""
    sh = d["spatial_shapes"]
    loc = d["sampling_locations"]
    N, Lq, M, L, K, _ = loc.shape
    D = d["grad_out"].shape[-1] // M
    S = int(sum(h * w for h, w in sh))
    rec = oracle.sample_points(loc, sh)
    rows = rec["rows"].reshape(N, Lq, M, L, K, 4)
    n = np.arange(N).reshape(N, 1, 1, 1, 1, 1)
    m = np.arange(M).reshape(1, 1, M, 1, 1, 1)
    first = ((n * S + rows) * M + m) * D
    return int(((rows >= 0) & (first >= limit)).sum())


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_checked_build_skips_and_reports_beyond_lowered_bound(case):
    d = _problem(case)
    N, Lq, M, D, K, shapes, dt = case
    S = int(sum(h * w for h, w in shapes))
    A = oracle.softmax(d["logits"]).astype(np.float32)
    pixels = N * S
    limit = (pixels * 3 // 5) * M * D  # a pixel boundary inside the map
    pairs = _skipped_pairs(d, limit)
    assert pairs > 0
    with checked_library(limit=limit):
        outs, codes = _run_all(d, A, to_dev(d["value"]))
    total = N * S * M * D
    for (st, cnt, first), what in zip(codes, ("forward", "fused forward", "backward")):
        assert st == DEVICE_CHECK, what
        assert limit <= first < total, (what, first)
    # the unfused calls skip at least one access per (sample, corner) pair
    # beyond the bound, and no more than one per lane and pass of 32 chunks
    esz = 2 if dt == "bf16" else 4
    npass = -(-(D * esz // 16) // 32)
    for st, cnt, first in (codes[0], codes[2]):
        assert pairs <= cnt <= 32 * npass * pairs
    # outputs: the method on the value map with the pixels beyond the bound zeroed
    vz = _zero_beyond(d["value"], limit)
    out, fo, (ogv, ogl, oga, mgl, mga) = _oracle_all(vz, d, A)
    assert_close(host(outs["out"]), out, **F32, what="forward, lowered bound")
    assert_close(host(outs["fout"]), fo, **F32, what="fused forward, lowered bound")
    gv = host(outs["gv"])
    assert not gv.reshape(-1)[limit:].any(), "a scatter beyond the bound was made"
    assert_close(gv.reshape(-1)[:limit], ogv.reshape(-1)[:limit], **GRAD,
                 what="grad_value below the bound")
    assert_close(host(outs["gl"]), ogl, **PLAIN, what="grad_loc, lowered bound", mass=mgl)
    assert_close(host(outs["ga"]), oga, **PLAIN, what="grad_attn, lowered bound", mass=mga)
    # the word was cleared: the next call with the default bound is clean, and
    # the thread's last report is still the backward's
    with checked_library():
        outs2, codes2 = _run_all(d, A, to_dev(d["value"]))
    assert codes2 == [(0, 0, -1)] * 3
    assert last_violation() == codes[2][1:]


def test_checked_fused_backward_lowered_bound():
    """msda_backward_fused in the checked build: the same skip-and-report
    contract, checked against the product build run on the zeroed map."""
    case = CASES[0]
    d = _problem(case)
    N, Lq, M, D, K, shapes, dt = case
    S = int(sum(h * w for h, w in shapes))
    limit = (N * S // 2) * M * D
    sh = d["spatial_shapes"]
    args = (to_dev(d["reference_points"]), to_dev(d["offsets"]), to_dev(d["logits"]),
            to_dev(d["grad_out"]))
    g = [torch.zeros(N, S, M, D, device="cuda"), torch.zeros(N, Lq, 2, device="cuda"),
         torch.zeros(d["offsets"].shape, device="cuda"),
         torch.zeros(d["logits"].shape, device="cuda")]
    with checked_library(limit=limit):
        with pytest.raises(MsdaError) as ei:
            msda_backward_fused(to_dev(d["value"]), sh, None, *args, grad_value=g[0],
                                grad_reference_points=g[1], grad_offsets=g[2],
                                grad_logits=g[3])
    assert ei.value.status == DEVICE_CHECK and ei.value.violations > 0
    torch.cuda.synchronize()
    vz = to_dev(_zero_beyond(d["value"], limit))
    pv, pr, po, pz = msda_backward_fused(vz, sh, None, *args)
    gv = host(g[0]).reshape(-1)
    assert not gv[limit:].any(), "a scatter beyond the bound was made"
    assert_close(gv[:limit], host(pv).reshape(-1)[:limit], **GRAD, what="fused grad_value")
    assert_close(host(g[2]), host(po), **GRAD, what="fused grad_offsets")
    assert_close(host(g[3]), host(pz), **GRAD, what="fused grad_logits")
    assert_close(host(g[1]), host(pr), **GRAD, what="fused grad_ref")
