"""The allocation-free tiled forward, msda_forward_fused_tiled_noalloc
(include/msda_tiled.h), through the C ABI.

It serves callers that cannot hand the library device memory beyond their
inputs and outputs: it keeps the tile plan in a device array of the
library's own, so the caller allocates no plan buffer.  Its results must
match msda_forward_fused_tiled given a plan buffer by the caller, within the
fp32 tolerance (locations and weights bit for bit), and two calls in a row
with different inputs must each match, since every call rebuilds the plan in
the shared array."""
import ctypes

import numpy as np
import pytest
import torch

from scale_deformable_attention_02_b200 import _lib, msda_forward_fused_tiled, msda_tile_plan
from scale_deformable_attention_02_b200 import workloads as wl

from gpu_util import F32, assert_close, host, to_dev

pytestmark = pytest.mark.gpu

SHAPES = ((26, 34), (13, 17), (7, 9), (4, 5))
HALO, CTAS = 3, 2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def _problem(seed, dtype):
    S = sum(h * w for h, w in SHAPES)
    d = wl.make_random_problem(seed, N=2, Lq=S, M=4, D=32, K=4, shapes=SHAPES, value_dtype=dtype,
                               offset_std=1.5)
    # the encoder layout: one query per pixel, at its own pixel centre
    d["reference_points"] = np.ascontiguousarray(
        np.broadcast_to(wl.pixel_centre_queries(SHAPES), (2, S, 2)))
    return d


def _noalloc(value, sh, starts, ref, off, logits):
    N, S, M, D = value.shape
    L, K = logits.shape[3], logits.shape[4]
    dims = _lib.Dims(N, ref.shape[1], S, M, D, L, K)
    out = torch.empty((N, ref.shape[1], M * D), device=value.device)
    loc = torch.empty_like(off)
    attn = torch.empty_like(logits)
    dt = _lib.MSDA_BF16 if value.dtype == torch.bfloat16 else _lib.MSDA_F32
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = _lib.load().msda_forward_fused_tiled_noalloc(
        p(value), dt, sh.ctypes.data_as(ctypes.c_void_p), starts.ctypes.data_as(ctypes.c_void_p),
        p(ref), 2, p(off), p(logits), p(out), p(loc), p(attn), dims, HALO, CTAS,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, _lib.status_string(st)
    return out, loc, attn


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_noalloc_matches_the_caller_plan_call_twice_in_a_row(dtype):
    sh = wl.spatial_shapes_array(SHAPES)
    starts = np.concatenate([[0], np.cumsum([h * w for h, w in SHAPES])[:-1]]).astype(np.int64)
    for seed in (11, 12):  # two calls in a row, different inputs
        d = _problem(seed, dtype)
        value, ref, off, z = (to_dev(d[k]) for k in ("value", "reference_points", "offsets",
                                                     "logits"))
        got = _noalloc(value, sh, starts, ref, off, z)
        plan = msda_tile_plan(value, sh, starts, ref, K=4, halo=HALO, ctas_per_sm=CTAS)
        want = msda_forward_fused_tiled(value, sh, starts, ref, off, z, plan,
                                        return_sampling=True)
        torch.cuda.synchronize()
        assert_close(host(got[0]), host(want[0]), **F32, what=f"out, call {seed}")
        assert torch.equal(got[1], want[1]), "sampling locations differ"
        assert torch.equal(got[2], want[2]), "attention weights differ"


def test_noalloc_rejects_plans_beyond_its_array():
    """A problem whose plan exceeds the 4 MiB array is refused up front."""
    shapes = ((1000, 1100),)
    sh = wl.spatial_shapes_array(shapes)
    starts = np.zeros(1, dtype=np.int64)
    S = 1000 * 1100
    dims = _lib.Dims(2, S, S, 1, 32, 1, 4)
    fake = ctypes.c_void_p(1 << 32)
    st = _lib.load().msda_forward_fused_tiled_noalloc(
        fake, 0, sh.ctypes.data_as(ctypes.c_void_p), starts.ctypes.data_as(ctypes.c_void_p),
        fake, 2, fake, fake, fake, None, None, dims, HALO, CTAS, None)
    assert _lib.STATUS_NAMES[st] == "MSDA_ERR_UNSUPPORTED"
