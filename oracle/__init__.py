"""CPU oracle of the MSDeformAttn (multi-scale deformable attention) core.

TEST INFRASTRUCTURE ONLY: the test suite, the package smoke check and the
benchmark's CPU-baseline leg are the only users.  The product path (the CUDA
library and its Python binding) never imports this package.

The arithmetic lives in ``msda_oracle.c`` (plain loops, fp64 accumulation);
this module compiles it with gcc on first use and marshals numpy arrays.
Every function follows the definition on the "Deformable DETR" wiki page
("Multi-scale deformable attention" equation and "Deformable attention
module"); the C file states each reading of a point the pages leave open.

Pinning: every function here is checked against facts the pages and plain
mathematics fix (worked example, closed forms, library special cases,
adjoint identities, finite differences) in tests/test_oracle_pins.py and
tests/test_oracle_grad.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "msda_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libmsda_oracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-shared",
          "-fPIC", "-std=c11"]


class Dims(ctypes.Structure):
    _fields_ = [(k, ctypes.c_int64) for k in ("N", "Lq", "S", "M", "D", "L", "K")]


def build(force: bool = False) -> str:
    """Compile the oracle into oracle/_build/libmsda_oracle.so (if stale)."""
    os.makedirs(_BUILD, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            _lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            I = ctypes.c_int
            _lib.ora_level_start_index.restype = I64
            _lib.ora_level_start_index.argtypes = [P, I64, P]
            _lib.ora_forward.restype = None
            _lib.ora_forward.argtypes = [P, I, P, P, P, I, P, P, Dims, I64, I64]
            _lib.ora_softmax.restype = None
            _lib.ora_softmax.argtypes = [P, P, I64, I64]
            _lib.ora_locations_f32.restype = None
            _lib.ora_locations_f32.argtypes = [P, P, P, Dims, P]
            _lib.ora_locations_box_f32.restype = None
            _lib.ora_locations_box_f32.argtypes = [P, P, Dims, P]
            _lib.ora_locations_f64.restype = None
            _lib.ora_locations_f64.argtypes = [P, P, P, Dims, P]
            _lib.ora_backward.restype = None
            _lib.ora_backward.argtypes = [P, I, P, P, P, I, P, P, P, P, P, P, P, Dims]
            _lib.ora_fused_chain.restype = None
            _lib.ora_fused_chain.argtypes = [P, P, P, P, Dims, P, P, P]
            _lib.ora_fused_chain_box.restype = None
            _lib.ora_fused_chain_box.argtypes = [P, P, P, P, P, Dims, P, P, P]
            _lib.ora_locations_box_f64.restype = None
            _lib.ora_locations_box_f64.argtypes = [P, P, Dims, P]
            _lib.ora_sample_points_f32.restype = None
            _lib.ora_sample_points_f32.argtypes = [P, P, P, Dims, P, P, P, P, P, P]
            _lib.ora_set_threads.restype = None
            _lib.ora_set_threads.argtypes = [I]
            _lib.ora_max_threads.restype = I
            _lib.ora_max_threads.argtypes = []
        return _lib


def set_threads(n: int) -> None:
    lib().ora_set_threads(int(n))


def max_threads() -> int:
    return int(lib().ora_max_threads())


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _value_arg(value: np.ndarray):
    """fp32 array, or uint16 bf16 bit patterns."""
    if value.dtype == np.uint16:
        return np.ascontiguousarray(value), 1
    return np.ascontiguousarray(value, dtype=np.float32), 0


def dims_of(value: np.ndarray, shapes: np.ndarray, loc_or_logits_shape) -> Dims:
    N, S, M, D = value.shape
    L = shapes.shape[0]
    Lq = loc_or_logits_shape[1]
    K = loc_or_logits_shape[4]
    return Dims(N, Lq, S, M, D, L, K)


def level_start_index(shapes: np.ndarray) -> tuple[np.ndarray, int]:
    shapes = np.ascontiguousarray(shapes, dtype=np.int64).reshape(-1, 2)
    starts = np.zeros(shapes.shape[0], dtype=np.int64)
    S = lib().ora_level_start_index(_ptr(shapes), shapes.shape[0], _ptr(starts))
    return starts, int(S)


def softmax(logits: np.ndarray) -> np.ndarray:
    """Joint softmax over the trailing (L, K) axes, fp64."""
    z = np.ascontiguousarray(logits, dtype=np.float64)
    LK = z.shape[-1] * z.shape[-2]
    a = np.empty_like(z)
    lib().ora_softmax(_ptr(z), _ptr(a), z.size // LK, LK)
    return a


def locations_f32(ref: np.ndarray, off: np.ndarray, shapes: np.ndarray) -> np.ndarray:
    ref = np.ascontiguousarray(ref, dtype=np.float32)
    off = np.ascontiguousarray(off, dtype=np.float32)
    shapes = np.ascontiguousarray(shapes, dtype=np.int64)
    N, Lq, M, L, K, _ = off.shape
    loc = np.empty_like(off)
    lib().ora_locations_f32(_ptr(ref), _ptr(off), _ptr(shapes),
                            Dims(N, Lq, 0, M, 0, L, K), _ptr(loc))
    return loc


def locations_box_f32(box: np.ndarray, off: np.ndarray) -> np.ndarray:
    """Box references (cx, cy, w, h): loc = (cx, cy) + off * (w, h), fp32."""
    box = np.ascontiguousarray(box, dtype=np.float32)
    off = np.ascontiguousarray(off, dtype=np.float32)
    N, Lq, M, L, K, _ = off.shape
    assert box.shape == (N, Lq, 4)
    loc = np.empty_like(off)
    lib().ora_locations_box_f32(_ptr(box), _ptr(off), Dims(N, Lq, 0, M, 0, L, K), _ptr(loc))
    return loc


def locations_f64(ref: np.ndarray, off: np.ndarray, shapes: np.ndarray) -> np.ndarray:
    ref = np.ascontiguousarray(ref, dtype=np.float64)
    off = np.ascontiguousarray(off, dtype=np.float64)
    shapes = np.ascontiguousarray(shapes, dtype=np.int64)
    N, Lq, M, L, K, _ = off.shape
    loc = np.empty_like(off)
    lib().ora_locations_f64(_ptr(ref), _ptr(off), _ptr(shapes),
                            Dims(N, Lq, 0, M, 0, L, K), _ptr(loc))
    return loc


def forward(value, shapes, loc, attn, loc_f32: bool = True, q_range=None) -> np.ndarray:
    """out [N,Lq,M*D] float64.  ``loc`` fp32 values (loc_f32) or fp64."""
    v, bf = _value_arg(value)
    shapes = np.ascontiguousarray(shapes, dtype=np.int64)
    starts, S = level_start_index(shapes)
    assert S == v.shape[1], "value rows must equal the sum of H*W"
    loc64 = np.ascontiguousarray(loc, dtype=np.float64)
    a64 = np.ascontiguousarray(attn, dtype=np.float64)
    d = dims_of(v, shapes, loc64.shape)
    out = np.zeros((d.N, d.Lq, d.M * d.D), dtype=np.float64)
    q0, q1 = (0, d.Lq) if q_range is None else q_range
    lib().ora_forward(_ptr(v), bf, _ptr(shapes), _ptr(starts), _ptr(loc64),
                      1 if loc_f32 else 0, _ptr(a64), _ptr(out), d, q0, q1)
    return out


def forward_fused(value, shapes, ref, off, logits):
    """Fused path: A = softmax(logits), loc = ref + off/W (fp32), then the
    forward.  Returns (out fp64, loc fp32, A fp64)."""
    loc = locations_f32(ref, off, shapes)
    a = softmax(logits)
    return forward(value, shapes, loc, a, loc_f32=True), loc, a


def backward(value, shapes, loc, attn, grad_out, loc_f32: bool = True, with_mass=False,
             with_grad_value: bool = True):
    """Returns (grad_value [N,S,M,D], grad_loc like loc, grad_attn like attn),
    all float64; with_mass=True appends (grad_loc_mass, grad_attn_mass), the
    sums of absolute terms that scale a finite-precision rounding bound.
    with_grad_value=False skips the scatter (grad_value is returned as None),
    for value maps too large to mirror in fp64."""
    v, bf = _value_arg(value)
    shapes = np.ascontiguousarray(shapes, dtype=np.int64)
    starts, S = level_start_index(shapes)
    assert S == v.shape[1]
    loc64 = np.ascontiguousarray(loc, dtype=np.float64)
    a64 = np.ascontiguousarray(attn, dtype=np.float64)
    g64 = np.ascontiguousarray(grad_out, dtype=np.float64)
    d = dims_of(v, shapes, loc64.shape)
    gv = np.empty(v.shape, dtype=np.float64) if with_grad_value else None
    gl = np.empty(loc64.shape, dtype=np.float64)
    ga = np.empty(a64.shape, dtype=np.float64)
    glm = np.empty(loc64.shape, dtype=np.float64) if with_mass else None
    gam = np.empty(a64.shape, dtype=np.float64) if with_mass else None
    lib().ora_backward(_ptr(v), bf, _ptr(shapes), _ptr(starts), _ptr(loc64),
                       1 if loc_f32 else 0, _ptr(a64), _ptr(g64),
                       None if gv is None else _ptr(gv),
                       _ptr(gl), _ptr(ga), None if glm is None else _ptr(glm),
                       None if gam is None else _ptr(gam), d)
    if with_mass:
        return gv, gl, ga, glm, gam
    return gv, gl, ga


def fused_chain(grad_loc, grad_attn, attn, shapes):
    """Chain the sampled-point gradients back to (ref, off, logits)."""
    gl = np.ascontiguousarray(grad_loc, dtype=np.float64)
    ga = np.ascontiguousarray(grad_attn, dtype=np.float64)
    a = np.ascontiguousarray(attn, dtype=np.float64)
    shapes = np.ascontiguousarray(shapes, dtype=np.int64)
    N, Lq, M, L, K = a.shape
    g_ref = np.empty((N, Lq, 2), dtype=np.float64)
    g_off = np.empty(gl.shape, dtype=np.float64)
    g_z = np.empty(a.shape, dtype=np.float64)
    lib().ora_fused_chain(_ptr(gl), _ptr(ga), _ptr(a), _ptr(shapes),
                          Dims(N, Lq, 0, M, 0, L, K), _ptr(g_ref), _ptr(g_off), _ptr(g_z))
    return g_ref, g_off, g_z


def fused_chain_box(grad_loc, grad_attn, attn, box, off):
    """Chain for box references: returns (grad_box [N,Lq,4], grad_off, grad_logits)."""
    gl = np.ascontiguousarray(grad_loc, dtype=np.float64)
    ga = np.ascontiguousarray(grad_attn, dtype=np.float64)
    a = np.ascontiguousarray(attn, dtype=np.float64)
    bx = np.ascontiguousarray(box, dtype=np.float64)
    of = np.ascontiguousarray(off, dtype=np.float64)
    N, Lq, M, L, K = a.shape
    g_box = np.empty((N, Lq, 4), dtype=np.float64)
    g_off = np.empty(gl.shape, dtype=np.float64)
    g_z = np.empty(a.shape, dtype=np.float64)
    lib().ora_fused_chain_box(_ptr(gl), _ptr(ga), _ptr(a), _ptr(bx), _ptr(of),
                              Dims(N, Lq, 0, M, 0, L, K), _ptr(g_box), _ptr(g_off), _ptr(g_z))
    return g_box, g_off, g_z


def locations_box_f64(box: np.ndarray, off: np.ndarray) -> np.ndarray:
    box = np.ascontiguousarray(box, dtype=np.float64)
    off = np.ascontiguousarray(off, dtype=np.float64)
    N, Lq, M, L, K, _ = off.shape
    loc = np.empty_like(off)
    lib().ora_locations_box_f64(_ptr(box), _ptr(off), Dims(N, Lq, 0, M, 0, L, K), _ptr(loc))
    return loc


def sample_points(loc: np.ndarray, shapes: np.ndarray) -> dict:
    """Per-sample cell record (fp32 arithmetic): valid, the pixel
    coordinates x, y, the cell x0, y0 and the four corner rows (-1 outside
    the map)."""
    loc = np.ascontiguousarray(loc, dtype=np.float32)
    shapes = np.ascontiguousarray(shapes, dtype=np.int64)
    starts, S = level_start_index(shapes)
    N, Lq, M, L, K, _ = loc.shape
    cnt = N * Lq * M * L * K
    out = {
        "valid": np.empty(cnt, dtype=np.int32),
        "x0": np.empty(cnt, dtype=np.int32),
        "y0": np.empty(cnt, dtype=np.int32),
        "x": np.empty(cnt, dtype=np.float32),
        "y": np.empty(cnt, dtype=np.float32),
        "rows": np.empty((cnt, 4), dtype=np.int64),
    }
    lib().ora_sample_points_f32(_ptr(loc), _ptr(shapes), _ptr(starts),
                                Dims(N, Lq, S, M, 0, L, K), _ptr(out["valid"]),
                                _ptr(out["x0"]), _ptr(out["y0"]), _ptr(out["x"]),
                                _ptr(out["y"]), _ptr(out["rows"]))
    return out


def expand_groups(x: np.ndarray, M: int) -> np.ndarray:
    """Deformable groups ("Deformable Attention" glossary page, multi-head
    paragraph: the heads of a group look up the same key locations): a per-group
    tensor [N, Lq, G, ...] as the per-head tensor [N, Lq, M, ...] it stands
    for, head m reading group m // (M/G)."""
    G = x.shape[2]
    if M % G != 0:
        raise ValueError("groups must divide the heads")
    return np.ascontiguousarray(np.repeat(x, M // G, axis=2))


def sum_groups(g: np.ndarray, G: int) -> np.ndarray:
    """Gradient with respect to a per-group input shared by M/G heads: the sum
    of the per-head gradients over each group.  [N, Lq, M, ...] -> [N, Lq, G, ...]."""
    N, Lq, M = g.shape[:3]
    return g.reshape((N, Lq, G, M // G) + g.shape[3:]).sum(axis=3)
