"""Python binding of the C ABI: argument marshalling only.

Each function takes torch CUDA tensors, checks that their dtypes, devices,
shapes and contiguity agree, allocates missing outputs with torch, and calls
the C entry point of the same name on the current (or given) CUDA stream.
Every step of the computation runs in libmsda.so's kernels; there is no
other code path.  Inside `with checked_library():` the calls of the current
thread go to libmsda_checked.so instead (the bounds-checked build of the same
sources, include/msda_checked.h).

Layouts (see include/msda.h):
  value [N,S,M,D] float32 | bfloat16, sampling_locations [N,Lq,M,L,K,2],
  attention_weights / logits [N,Lq,M,L,K], reference_points [N,Lq,2|4],
  offsets [N,Lq,M,L,K,2], out / grad_out [N,Lq,M*D] (all float32 except value),
  spatial_shapes [L,2] int64 (H, W) and level_start_index [L] int64 on the host.
"""
from __future__ import annotations

import contextlib
import ctypes

import numpy as np
import torch

from . import _lib


class MsdaError(RuntimeError):
    """A non-OK status from libmsda.so.  For MSDA_ERR_DEVICE_CHECK (checked
    build), `violations` and `first_element` say what the kernel skipped."""

    def __init__(self, status: int, where: str):
        self.status = int(status)
        self.violations = 0
        self.first_element = -1
        msg = f"{where}: {_lib.status_string(status)}"
        if self.status == 8:
            msg += f" (cudaError {_lib.load().msda_last_cuda_error()})"
        if self.status == 9:
            self.violations, self.first_element = last_violation()
            msg += (f" ({self.violations} accesses skipped, first at value element "
                    f"{self.first_element})")
        super().__init__(msg)


@contextlib.contextmanager
def checked_library(limit: int | None = None):
    """Route this thread's calls to libmsda_checked.so, where every value-map
    gather and grad_value scatter is bounds-checked on the device and a call
    that skipped one raises MsdaError(MSDA_ERR_DEVICE_CHECK).  `limit` lowers
    the bound to that many value elements (a test of the checks themselves)."""
    lib = _lib.load(checked=True)
    prev = getattr(_lib._route, "checked", False)
    _lib._route.checked = True
    if limit is not None:
        lib.msda_checked_set_limit(int(limit))
    try:
        yield lib
    finally:
        if limit is not None:
            lib.msda_checked_set_limit(-1)
        _lib._route.checked = prev


def last_violation() -> tuple[int, int]:
    """(accesses skipped, first element index) of this thread's last
    MSDA_ERR_DEVICE_CHECK in the checked build."""
    cnt, first = ctypes.c_int64(0), ctypes.c_int64(-1)
    _lib.load(checked=True).msda_checked_last_violation(ctypes.byref(cnt), ctypes.byref(first))
    return cnt.value, first.value


def _check(status: int, where: str) -> None:
    if status != 0:
        raise MsdaError(status, where)


def _host_i64(x, name: str) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        x = x.detach().to("cpu").numpy()
    a = np.ascontiguousarray(np.asarray(x, dtype=np.int64))
    if a.ndim == 0:
        raise ValueError(f"{name} must be an array")
    return a


def _hptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _dptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(device: torch.device, stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    if isinstance(stream, torch.cuda.Stream):
        stream = stream.cuda_stream
    return ctypes.c_void_p(int(stream))


def _value_dtype(value: torch.Tensor) -> int:
    if value.dtype == torch.float32:
        return _lib.MSDA_F32
    if value.dtype == torch.bfloat16:
        return _lib.MSDA_BF16
    raise TypeError(f"value must be float32 or bfloat16, got {value.dtype}")


def _need(t: torch.Tensor, name: str, shape, device, dtype=torch.float32):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _levels(spatial_shapes, level_start_index):
    shapes = _host_i64(spatial_shapes, "spatial_shapes").reshape(-1, 2)
    if level_start_index is None:
        starts, _ = msda_level_start_index(shapes)
    else:
        starts = _host_i64(level_start_index, "level_start_index").reshape(-1)
    return shapes, starts


def msda_level_start_index(spatial_shapes) -> tuple[np.ndarray, int]:
    """Level start rows (exclusive prefix sum of H*W) and S, from the C ABI."""
    shapes = _host_i64(spatial_shapes, "spatial_shapes").reshape(-1, 2)
    starts = np.zeros(shapes.shape[0], dtype=np.int64)
    S = ctypes.c_int64(0)
    _check(_lib.load().msda_level_start_index(_hptr(shapes), shapes.shape[0], _hptr(starts),
                                              ctypes.byref(S)), "msda_level_start_index")
    return starts, int(S.value)


def _value_dims(value: torch.Tensor, shapes: np.ndarray, lead):
    """Dims from value [N,S,M,D] and a per-head tensor's shape [N,Lq,M,L,K]."""
    if value.dim() != 4:
        raise ValueError("value must be [N, S, M, D]")
    N, S, M, D = value.shape
    L = shapes.shape[0]
    if len(lead) < 5:
        raise ValueError("per-sample tensors must be [N, Lq, M, L, K(, 2)]")
    if lead[0] != N or lead[2] != M or lead[3] != L:
        raise ValueError(f"per-sample tensor shape {tuple(lead)} disagrees with value "
                         f"{tuple(value.shape)} and L={L}")
    Lq, K = lead[1], lead[4]
    return _lib.Dims(N, Lq, S, M, D, L, K)


def _groups(d, groups) -> int:
    """Deformable groups: None means one group per head (the ungrouped calls)."""
    if groups is None:
        return d.M
    g = int(groups)
    if g < 1 or d.M % g != 0:
        raise ValueError(f"groups={g} must divide the {d.M} heads")
    return g


def msda_forward(value: torch.Tensor, spatial_shapes, level_start_index,
                 sampling_locations: torch.Tensor, attention_weights: torch.Tensor,
                 out: torch.Tensor | None = None, groups: int | None = None,
                 stream=None) -> torch.Tensor:
    """out[n,q,m*D:(m+1)*D] = sum_{l,k} A * bilinear(value level l, head m, loc).
    With `groups` G, sampling_locations is [N,Lq,G,L,K,2], shared by the M/G
    heads of each group (msda_forward_grouped)."""
    dev = value.device
    shapes, starts = _levels(spatial_shapes, level_start_index)
    d = _value_dims(value, shapes, tuple(attention_weights.shape))
    G = _groups(d, groups)
    _need(sampling_locations, "sampling_locations", (d.N, d.Lq, G, d.L, d.K, 2), dev)
    _need(attention_weights, "attention_weights", (d.N, d.Lq, d.M, d.L, d.K), dev)
    if not value.is_contiguous():
        raise ValueError("value must be contiguous")
    if out is None:
        out = torch.empty((d.N, d.Lq, d.M * d.D), device=dev, dtype=torch.float32)
    _need(out, "out", (d.N, d.Lq, d.M * d.D), dev)
    args = (_dptr(value), _value_dtype(value), _hptr(shapes), _hptr(starts),
            _dptr(sampling_locations), _dptr(attention_weights), _dptr(out), d)
    if groups is None:
        _check(_lib.load().msda_forward(*args, _stream_handle(dev, stream)), "msda_forward")
    else:
        _check(_lib.load().msda_forward_grouped(*args, G, _stream_handle(dev, stream)),
               "msda_forward_grouped")
    return out


def msda_forward_fused(value: torch.Tensor, spatial_shapes, level_start_index,
                       reference_points: torch.Tensor, offsets: torch.Tensor,
                       logits: torch.Tensor, out: torch.Tensor | None = None,
                       sampling_locations_out: torch.Tensor | None = None,
                       attention_weights_out: torch.Tensor | None = None,
                       return_sampling: bool = False, groups: int | None = None,
                       stream=None):
    """Fused forward: softmax over the L*K logits of each head and the
    location map (ref + off/W_l, or box: (cx,cy) + off*(w,h)) inside the
    kernel.  Returns out, or (out, sampling_locations, attention_weights) when
    return_sampling is true (those outputs are then allocated if not given).
    With `groups` G, offsets (and sampling_locations_out) are [N,Lq,G,L,K,2]
    (msda_forward_fused_grouped)."""
    dev = value.device
    shapes, starts = _levels(spatial_shapes, level_start_index)
    d = _value_dims(value, shapes, tuple(logits.shape))
    G = _groups(d, groups)
    rdim = reference_points.shape[-1] if reference_points.dim() == 3 else -1
    if rdim not in (2, 4):
        raise ValueError("reference_points must be [N, Lq, 2] or [N, Lq, 4]")
    _need(reference_points, "reference_points", (d.N, d.Lq, rdim), dev)
    _need(offsets, "offsets", (d.N, d.Lq, G, d.L, d.K, 2), dev)
    _need(logits, "logits", (d.N, d.Lq, d.M, d.L, d.K), dev)
    if not value.is_contiguous():
        raise ValueError("value must be contiguous")
    if out is None:
        out = torch.empty((d.N, d.Lq, d.M * d.D), device=dev, dtype=torch.float32)
    _need(out, "out", (d.N, d.Lq, d.M * d.D), dev)
    if return_sampling:
        if sampling_locations_out is None:
            sampling_locations_out = torch.empty_like(offsets)
        if attention_weights_out is None:
            attention_weights_out = torch.empty_like(logits)
    if sampling_locations_out is not None:
        _need(sampling_locations_out, "sampling_locations_out", tuple(offsets.shape), dev)
    if attention_weights_out is not None:
        _need(attention_weights_out, "attention_weights_out", tuple(logits.shape), dev)
    args = (_dptr(value), _value_dtype(value), _hptr(shapes), _hptr(starts),
            _dptr(reference_points), int(rdim), _dptr(offsets), _dptr(logits), _dptr(out),
            _dptr(sampling_locations_out), _dptr(attention_weights_out), d)
    if groups is None:
        _check(_lib.load().msda_forward_fused(*args, _stream_handle(dev, stream)),
               "msda_forward_fused")
    else:
        _check(_lib.load().msda_forward_fused_grouped(*args, G, _stream_handle(dev, stream)),
               "msda_forward_fused_grouped")
    if return_sampling:
        return out, sampling_locations_out, attention_weights_out
    return out


def msda_backward(value: torch.Tensor, spatial_shapes, level_start_index,
                  sampling_locations: torch.Tensor, attention_weights: torch.Tensor,
                  grad_out: torch.Tensor, grad_value: torch.Tensor | None = None,
                  grad_sampling_locations: torch.Tensor | None = None,
                  grad_attention_weights: torch.Tensor | None = None,
                  need_sampling_grad: bool = True, need_weight_grad: bool = True,
                  groups: int | None = None, stream=None):
    """Gradients of msda_forward.  Returns (grad_value [fp32], grad_loc or
    None, grad_attn or None).  With `groups`, the locations and their
    gradient are per group (msda_backward_grouped)."""
    dev = value.device
    shapes, starts = _levels(spatial_shapes, level_start_index)
    d = _value_dims(value, shapes, tuple(attention_weights.shape))
    G = _groups(d, groups)
    _need(sampling_locations, "sampling_locations", (d.N, d.Lq, G, d.L, d.K, 2), dev)
    _need(attention_weights, "attention_weights", (d.N, d.Lq, d.M, d.L, d.K), dev)
    _need(grad_out, "grad_out", (d.N, d.Lq, d.M * d.D), dev)
    if not value.is_contiguous():
        raise ValueError("value must be contiguous")
    if grad_value is None:
        grad_value = torch.empty(tuple(value.shape), device=dev, dtype=torch.float32)
    _need(grad_value, "grad_value", tuple(value.shape), dev)
    if grad_sampling_locations is None and need_sampling_grad:
        grad_sampling_locations = torch.empty_like(sampling_locations)
    if grad_attention_weights is None and need_weight_grad:
        grad_attention_weights = torch.empty_like(attention_weights)
    if grad_sampling_locations is not None:
        _need(grad_sampling_locations, "grad_sampling_locations",
              tuple(sampling_locations.shape), dev)
    if grad_attention_weights is not None:
        _need(grad_attention_weights, "grad_attention_weights",
              tuple(attention_weights.shape), dev)
    args = (_dptr(value), _value_dtype(value), _hptr(shapes), _hptr(starts),
            _dptr(sampling_locations), _dptr(attention_weights), _dptr(grad_out),
            _dptr(grad_value), _dptr(grad_sampling_locations), _dptr(grad_attention_weights), d)
    if groups is None:
        _check(_lib.load().msda_backward(*args, _stream_handle(dev, stream)), "msda_backward")
    else:
        _check(_lib.load().msda_backward_grouped(*args, G, _stream_handle(dev, stream)),
               "msda_backward_grouped")
    return grad_value, grad_sampling_locations, grad_attention_weights


def msda_backward_fused(value: torch.Tensor, spatial_shapes, level_start_index,
                        reference_points: torch.Tensor, offsets: torch.Tensor,
                        logits: torch.Tensor, grad_out: torch.Tensor,
                        grad_value: torch.Tensor | None = None,
                        grad_reference_points: torch.Tensor | None = None,
                        grad_offsets: torch.Tensor | None = None,
                        grad_logits: torch.Tensor | None = None,
                        need_reference_grad: bool = True, need_offset_grad: bool = True,
                        need_logit_grad: bool = True, groups: int | None = None,
                        stream=None):
    """Gradients of msda_forward_fused with respect to the value map, the
    reference points, the offsets and the logits.  Returns (grad_value,
    grad_reference_points or None, grad_offsets or None, grad_logits or None).
    With `groups`, offsets and their gradient are per group
    (msda_backward_fused_grouped)."""
    dev = value.device
    shapes, starts = _levels(spatial_shapes, level_start_index)
    d = _value_dims(value, shapes, tuple(logits.shape))
    G = _groups(d, groups)
    rdim = reference_points.shape[-1] if reference_points.dim() == 3 else -1
    if rdim not in (2, 4):
        raise ValueError("reference_points must be [N, Lq, 2] or [N, Lq, 4]")
    _need(reference_points, "reference_points", (d.N, d.Lq, rdim), dev)
    _need(offsets, "offsets", (d.N, d.Lq, G, d.L, d.K, 2), dev)
    _need(logits, "logits", (d.N, d.Lq, d.M, d.L, d.K), dev)
    _need(grad_out, "grad_out", (d.N, d.Lq, d.M * d.D), dev)
    if not value.is_contiguous():
        raise ValueError("value must be contiguous")
    if grad_value is None:
        grad_value = torch.empty(tuple(value.shape), device=dev, dtype=torch.float32)
    _need(grad_value, "grad_value", tuple(value.shape), dev)
    if grad_reference_points is None and need_reference_grad:
        grad_reference_points = torch.empty_like(reference_points)
    if grad_offsets is None and need_offset_grad:
        grad_offsets = torch.empty_like(offsets)
    if grad_logits is None and need_logit_grad:
        grad_logits = torch.empty_like(logits)
    if grad_reference_points is not None:
        _need(grad_reference_points, "grad_reference_points", tuple(reference_points.shape), dev)
    if grad_offsets is not None:
        _need(grad_offsets, "grad_offsets", tuple(offsets.shape), dev)
    if grad_logits is not None:
        _need(grad_logits, "grad_logits", tuple(logits.shape), dev)
    args = (_dptr(value), _value_dtype(value), _hptr(shapes), _hptr(starts),
            _dptr(reference_points), int(rdim), _dptr(offsets), _dptr(logits), _dptr(grad_out),
            _dptr(grad_value), _dptr(grad_reference_points), _dptr(grad_offsets),
            _dptr(grad_logits), d)
    if groups is None:
        _check(_lib.load().msda_backward_fused(*args, _stream_handle(dev, stream)),
               "msda_backward_fused")
    else:
        _check(_lib.load().msda_backward_fused_grouped(*args, G, _stream_handle(dev, stream)),
               "msda_backward_fused_grouped")
    return grad_value, grad_reference_points, grad_offsets, grad_logits


class TilePlan:
    """A tile plan (include/msda_tiled.h): the host description `desc` (an
    msda_tile_plan) and the device buffer `buffer` that msda_tile_plan_build
    filled.  Valid while the reference points it was built from do not
    change."""

    def __init__(self, desc, buffer: torch.Tensor):
        self.desc = desc
        self.buffer = buffer

    @property
    def grid(self) -> tuple[int, int]:
        return self.desc.grid_x, self.desc.grid_y

    @property
    def windows(self) -> list[tuple[int, int]]:
        return [(self.desc.window_w[i], self.desc.window_h[i]) for i in range(self.desc.L)]


def msda_tile_plan(value: torch.Tensor, spatial_shapes, level_start_index,
                   reference_points: torch.Tensor, K: int, M: int | None = None,
                   halo: int = 4, ctas_per_sm: int = 0, stream=None) -> TilePlan:
    """Describe (msda_tile_plan_init), allocate and build (msda_tile_plan_build)
    the tile plan of a problem: value [N,S,M,D] gives N, S, D, M and the value
    dtype, reference_points [N,Lq,2|4] gives Lq and the points to sort."""
    dev = value.device
    shapes, starts = _levels(spatial_shapes, level_start_index)
    if value.dim() != 4:
        raise ValueError("value must be [N, S, M, D]")
    N, S, Mv, D = value.shape
    rdim = reference_points.shape[-1] if reference_points.dim() == 3 else -1
    if rdim not in (2, 4):
        raise ValueError("reference_points must be [N, Lq, 2] or [N, Lq, 4]")
    Lq = reference_points.shape[1]
    _need(reference_points, "reference_points", (N, Lq, rdim), dev)
    d = _lib.Dims(N, Lq, S, Mv if M is None else M, D, shapes.shape[0], K)
    desc = _lib.TilePlan()
    _check(_lib.load().msda_tile_plan_init(_value_dtype(value), _hptr(shapes), _hptr(starts), d,
                                           int(halo), int(ctas_per_sm), ctypes.byref(desc)),
           "msda_tile_plan_init")
    buf = torch.empty(max(int(desc.device_bytes), 16), device=dev, dtype=torch.uint8)
    _check(_lib.load().msda_tile_plan_build(ctypes.byref(desc), _dptr(reference_points),
                                            int(rdim), _dptr(buf), _stream_handle(dev, stream)),
           "msda_tile_plan_build")
    return TilePlan(desc, buf)


def msda_tile_plan_rebuild(plan: TilePlan, reference_points: torch.Tensor,
                           buffer: torch.Tensor | None = None, stream=None) -> None:
    """Sort `reference_points` into the plan's cells again (msda_tile_plan_build),
    into the plan's own buffer or into `buffer` (another uint8 device tensor
    of at least plan.desc.device_bytes)."""
    buf = plan.buffer if buffer is None else buffer
    dev = buf.device
    rdim = reference_points.shape[-1] if reference_points.dim() == 3 else -1
    if rdim not in (2, 4):
        raise ValueError("reference_points must be [N, Lq, 2] or [N, Lq, 4]")
    _need(reference_points, "reference_points", (plan.desc.N, plan.desc.Lq, rdim), dev)
    if buf.numel() < plan.desc.device_bytes or buf.dtype != torch.uint8:
        raise ValueError("the plan buffer must be uint8 of at least plan.desc.device_bytes")
    _check(_lib.load().msda_tile_plan_build(ctypes.byref(plan.desc), _dptr(reference_points),
                                            int(rdim), _dptr(buf), _stream_handle(dev, stream)),
           "msda_tile_plan_build")


def msda_forward_tiled(value: torch.Tensor, spatial_shapes, level_start_index,
                       sampling_locations: torch.Tensor, attention_weights: torch.Tensor,
                       plan: TilePlan, out: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
    """msda_forward on a tile plan (the same result, cell by cell with the
    value windows in shared memory)."""
    dev = value.device
    shapes, starts = _levels(spatial_shapes, level_start_index)
    d = _value_dims(value, shapes, tuple(attention_weights.shape))
    _need(sampling_locations, "sampling_locations", (d.N, d.Lq, d.M, d.L, d.K, 2), dev)
    _need(attention_weights, "attention_weights", (d.N, d.Lq, d.M, d.L, d.K), dev)
    if not value.is_contiguous():
        raise ValueError("value must be contiguous")
    if out is None:
        out = torch.empty((d.N, d.Lq, d.M * d.D), device=dev, dtype=torch.float32)
    _need(out, "out", (d.N, d.Lq, d.M * d.D), dev)
    _check(_lib.load().msda_forward_tiled(
        _dptr(value), _value_dtype(value), _hptr(shapes), _hptr(starts),
        _dptr(sampling_locations), _dptr(attention_weights), _dptr(out), d,
        ctypes.byref(plan.desc), _dptr(plan.buffer), _stream_handle(dev, stream)),
        "msda_forward_tiled")
    return out


def msda_forward_fused_tiled(value: torch.Tensor, spatial_shapes, level_start_index,
                             reference_points: torch.Tensor, offsets: torch.Tensor,
                             logits: torch.Tensor, plan: TilePlan,
                             out: torch.Tensor | None = None,
                             sampling_locations_out: torch.Tensor | None = None,
                             attention_weights_out: torch.Tensor | None = None,
                             return_sampling: bool = False, stream=None):
    """msda_forward_fused on a tile plan."""
    dev = value.device
    shapes, starts = _levels(spatial_shapes, level_start_index)
    d = _value_dims(value, shapes, tuple(logits.shape))
    rdim = reference_points.shape[-1] if reference_points.dim() == 3 else -1
    if rdim not in (2, 4):
        raise ValueError("reference_points must be [N, Lq, 2] or [N, Lq, 4]")
    _need(reference_points, "reference_points", (d.N, d.Lq, rdim), dev)
    _need(offsets, "offsets", (d.N, d.Lq, d.M, d.L, d.K, 2), dev)
    _need(logits, "logits", (d.N, d.Lq, d.M, d.L, d.K), dev)
    if not value.is_contiguous():
        raise ValueError("value must be contiguous")
    if out is None:
        out = torch.empty((d.N, d.Lq, d.M * d.D), device=dev, dtype=torch.float32)
    _need(out, "out", (d.N, d.Lq, d.M * d.D), dev)
    if return_sampling:
        if sampling_locations_out is None:
            sampling_locations_out = torch.empty_like(offsets)
        if attention_weights_out is None:
            attention_weights_out = torch.empty_like(logits)
    if sampling_locations_out is not None:
        _need(sampling_locations_out, "sampling_locations_out", tuple(offsets.shape), dev)
    if attention_weights_out is not None:
        _need(attention_weights_out, "attention_weights_out", tuple(logits.shape), dev)
    _check(_lib.load().msda_forward_fused_tiled(
        _dptr(value), _value_dtype(value), _hptr(shapes), _hptr(starts),
        _dptr(reference_points), int(rdim), _dptr(offsets), _dptr(logits), _dptr(out),
        _dptr(sampling_locations_out), _dptr(attention_weights_out), d,
        ctypes.byref(plan.desc), _dptr(plan.buffer), _stream_handle(dev, stream)),
        "msda_forward_fused_tiled")
    if return_sampling:
        return out, sampling_locations_out, attention_weights_out
    return out


def msda_backward_tiled(value: torch.Tensor, spatial_shapes, level_start_index,
                        sampling_locations: torch.Tensor, attention_weights: torch.Tensor,
                        grad_out: torch.Tensor, plan: TilePlan,
                        grad_value: torch.Tensor | None = None,
                        grad_sampling_locations: torch.Tensor | None = None,
                        grad_attention_weights: torch.Tensor | None = None,
                        need_sampling_grad: bool = True, need_weight_grad: bool = True,
                        stream=None):
    """msda_backward on a tile plan.  Returns (grad_value, grad_loc or None,
    grad_attn or None)."""
    dev = value.device
    shapes, starts = _levels(spatial_shapes, level_start_index)
    d = _value_dims(value, shapes, tuple(attention_weights.shape))
    _need(sampling_locations, "sampling_locations", (d.N, d.Lq, d.M, d.L, d.K, 2), dev)
    _need(attention_weights, "attention_weights", (d.N, d.Lq, d.M, d.L, d.K), dev)
    _need(grad_out, "grad_out", (d.N, d.Lq, d.M * d.D), dev)
    if not value.is_contiguous():
        raise ValueError("value must be contiguous")
    if grad_value is None:
        grad_value = torch.empty(tuple(value.shape), device=dev, dtype=torch.float32)
    _need(grad_value, "grad_value", tuple(value.shape), dev)
    if grad_sampling_locations is None and need_sampling_grad:
        grad_sampling_locations = torch.empty_like(sampling_locations)
    if grad_attention_weights is None and need_weight_grad:
        grad_attention_weights = torch.empty_like(attention_weights)
    if grad_sampling_locations is not None:
        _need(grad_sampling_locations, "grad_sampling_locations",
              tuple(sampling_locations.shape), dev)
    if grad_attention_weights is not None:
        _need(grad_attention_weights, "grad_attention_weights",
              tuple(attention_weights.shape), dev)
    _check(_lib.load().msda_backward_tiled(
        _dptr(value), _value_dtype(value), _hptr(shapes), _hptr(starts),
        _dptr(sampling_locations), _dptr(attention_weights), _dptr(grad_out), _dptr(grad_value),
        _dptr(grad_sampling_locations), _dptr(grad_attention_weights), d,
        ctypes.byref(plan.desc), _dptr(plan.buffer), _stream_handle(dev, stream)),
        "msda_backward_tiled")
    return grad_value, grad_sampling_locations, grad_attention_weights


def msda_backward_fused_tiled(value: torch.Tensor, spatial_shapes, level_start_index,
                              reference_points: torch.Tensor, offsets: torch.Tensor,
                              logits: torch.Tensor, grad_out: torch.Tensor, plan: TilePlan,
                              grad_value: torch.Tensor | None = None,
                              grad_reference_points: torch.Tensor | None = None,
                              grad_offsets: torch.Tensor | None = None,
                              grad_logits: torch.Tensor | None = None,
                              need_reference_grad: bool = True, need_offset_grad: bool = True,
                              need_logit_grad: bool = True, stream=None):
    """msda_backward_fused on a tile plan.  Returns (grad_value,
    grad_reference_points or None, grad_offsets or None, grad_logits or None)."""
    dev = value.device
    shapes, starts = _levels(spatial_shapes, level_start_index)
    d = _value_dims(value, shapes, tuple(logits.shape))
    rdim = reference_points.shape[-1] if reference_points.dim() == 3 else -1
    if rdim not in (2, 4):
        raise ValueError("reference_points must be [N, Lq, 2] or [N, Lq, 4]")
    _need(reference_points, "reference_points", (d.N, d.Lq, rdim), dev)
    _need(offsets, "offsets", (d.N, d.Lq, d.M, d.L, d.K, 2), dev)
    _need(logits, "logits", (d.N, d.Lq, d.M, d.L, d.K), dev)
    _need(grad_out, "grad_out", (d.N, d.Lq, d.M * d.D), dev)
    if not value.is_contiguous():
        raise ValueError("value must be contiguous")
    if grad_value is None:
        grad_value = torch.empty(tuple(value.shape), device=dev, dtype=torch.float32)
    _need(grad_value, "grad_value", tuple(value.shape), dev)
    if grad_reference_points is None and need_reference_grad:
        grad_reference_points = torch.empty_like(reference_points)
    if grad_offsets is None and need_offset_grad:
        grad_offsets = torch.empty_like(offsets)
    if grad_logits is None and need_logit_grad:
        grad_logits = torch.empty_like(logits)
    if grad_reference_points is not None:
        _need(grad_reference_points, "grad_reference_points", tuple(reference_points.shape), dev)
    if grad_offsets is not None:
        _need(grad_offsets, "grad_offsets", tuple(offsets.shape), dev)
    if grad_logits is not None:
        _need(grad_logits, "grad_logits", tuple(logits.shape), dev)
    _check(_lib.load().msda_backward_fused_tiled(
        _dptr(value), _value_dtype(value), _hptr(shapes), _hptr(starts),
        _dptr(reference_points), int(rdim), _dptr(offsets), _dptr(logits), _dptr(grad_out),
        _dptr(grad_value), _dptr(grad_reference_points), _dptr(grad_offsets),
        _dptr(grad_logits), d, ctypes.byref(plan.desc), _dptr(plan.buffer),
        _stream_handle(dev, stream)),
        "msda_backward_fused_tiled")
    return grad_value, grad_reference_points, grad_offsets, grad_logits


def msda_debug_sample_points(spatial_shapes, level_start_index,
                             sampling_locations: torch.Tensor, stream=None) -> dict:
    """Per-sample cell record computed by the kernels' own cell arithmetic."""
    dev = sampling_locations.device
    shapes, starts = _levels(spatial_shapes, level_start_index)
    if sampling_locations.dim() != 6:
        raise ValueError("sampling_locations must be [N, Lq, M, L, K, 2]")
    N, Lq, M, L, K, _ = sampling_locations.shape
    S = int(sum(int(h) * int(w) for h, w in shapes))
    d = _lib.Dims(N, Lq, S, M, 4, L, K)
    _need(sampling_locations, "sampling_locations", (N, Lq, M, L, K, 2), dev)
    n = N * Lq * M * L * K
    r = {
        "valid": torch.empty(n, device=dev, dtype=torch.int32),
        "x0": torch.empty(n, device=dev, dtype=torch.int32),
        "y0": torch.empty(n, device=dev, dtype=torch.int32),
        "x": torch.empty(n, device=dev, dtype=torch.float32),
        "y": torch.empty(n, device=dev, dtype=torch.float32),
        "rows": torch.empty((n, 4), device=dev, dtype=torch.int64),
    }
    _check(_lib.load().msda_debug_sample_points(
        _hptr(shapes), _hptr(starts), _dptr(sampling_locations), d, _dptr(r["valid"]),
        _dptr(r["x0"]), _dptr(r["y0"]), _dptr(r["x"]), _dptr(r["y"]), _dptr(r["rows"]),
        _stream_handle(dev, stream)), "msda_debug_sample_points")
    return r


def msda_debug_row_traffic(mode: int, rows: torch.Tensor, value: torch.Tensor | None = None,
                           grad: torch.Tensor | None = None, sink: torch.Tensor | None = None,
                           depth: int = 0, ctas: int = 0, stream=None) -> None:
    """Replay 32-element rows (int32 element offsets `rows`) as bare gathers
    of fp32 or bf16 `value` (mode 0), vector reductions of a row of ones into
    the fp32 `grad` (mode 1), or both (mode 2): the memory-system floor of
    the kernels (include/msda_debug.h)."""
    ref = value if value is not None else grad
    if ref is None:
        raise ValueError("value or grad is required")
    dev = ref.device
    n_value = ref.numel()
    vdt = _lib.MSDA_F32
    if value is not None:
        vdt = _value_dtype(value)
        _need(value, "value", tuple(value.shape), dev, dtype=value.dtype)
    if grad is not None:
        _need(grad, "grad", tuple(grad.shape), dev)
        if grad.numel() != n_value:
            raise ValueError("value and grad must have the same number of elements")
    _need(rows, "rows", tuple(rows.shape), dev, dtype=torch.int32)
    if sink is not None:
        _need(sink, "sink", tuple(sink.shape), dev)
    _check(_lib.load().msda_debug_row_traffic(
        int(mode), _dptr(value), vdt, _dptr(grad), n_value, _dptr(rows), rows.numel(),
        _dptr(sink), 0 if sink is None else sink.numel(), int(depth), int(ctas),
        _stream_handle(dev, stream)),
        "msda_debug_row_traffic")


def msda_debug_tiled_stalls() -> int:
    """Bounded waits of the tiled kernels that ran out since the last call
    (synchronises the device; include/msda_debug.h)."""
    c = ctypes.c_int64(0)
    _check(_lib.load().msda_debug_tiled_stalls(ctypes.byref(c)), "msda_debug_tiled_stalls")
    return int(c.value)
