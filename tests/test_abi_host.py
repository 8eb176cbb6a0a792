"""The C ABI on the host: both builds of the library (libmsda.so and the
bounds-checked libmsda_checked.so) load, export exactly the symbols their
headers declare, compute the level metadata, and reject bad arguments with
the documented status codes before any device work.  CPU only: every call
here returns before touching CUDA (pointers are fake and never dereferenced)."""
import ctypes
import glob
import os
import re

import numpy as np
import pytest

import oracle
from scale_deformable_attention_02_b200 import _lib
from scale_deformable_attention_02_b200 import build as msda_build
from scale_deformable_attention_02_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

OK, NULL, SHAPE, LEVELS, DTYPE, ALIGN, ALIAS, UNSUP = range(8)

PRODUCT_HEADERS = ("msda.h", "msda_tiled.h", "msda_debug.h")
CHECKED_HEADERS = PRODUCT_HEADERS + ("msda_checked.h",)


@pytest.fixture(scope="module", params=[False, True], ids=["libmsda", "libmsda_checked"])
def lib(request):
    msda_build.build()
    return _lib.load(checked=request.param)


def declared_functions(headers=PRODUCT_HEADERS):
    names = []
    for h in headers:
        text = open(os.path.join(ROOT, "include", h)).read()
        names += re.findall(r"^MSDA_API\s+[\w\s\*]*?\b(msda_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_every_header_is_covered():
    assert sorted(os.path.basename(h) for h in glob.glob(os.path.join(ROOT, "include", "*.h"))) \
        == sorted(CHECKED_HEADERS)


def test_headers_declare_the_entry_points():
    names = declared_functions()
    for must in ("msda_forward", "msda_forward_fused", "msda_backward", "msda_backward_fused",
                 "msda_level_start_index", "msda_status_string", "msda_debug_sample_points"):
        assert must in names
    assert set(declared_functions(CHECKED_HEADERS)) - set(names) == {
        "msda_checked_set_limit", "msda_checked_last_violation"}


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, f"binding lacks {name}"


@pytest.mark.parametrize("path,headers", [(_lib.LIB_PATH, PRODUCT_HEADERS),
                                          (_lib.LIB_CHECKED_PATH, CHECKED_HEADERS)])
def test_library_exports_nothing_else(path, headers):
    import subprocess
    msda_build.build()
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True,
                         text=True, check=True).stdout
    exported = sorted({ln.split()[-1] for ln in out.splitlines() if " T " in ln})
    assert exported == declared_functions(headers)
    for name in exported:
        assert name in _lib.SIGNATURES or name in _lib.CHECKED_SIGNATURES


def test_status_strings_and_version(lib):
    for code, name in _lib.STATUS_NAMES.items():
        assert lib.msda_status_string(code).decode().startswith(name)
    assert lib.msda_abi_version() == 10300


def test_checked_build_host_calls():
    """The checked build's own entry points: a fresh thread has seen no
    violation; setting and restoring the limit needs no device."""
    import threading
    msda_build.build()
    lib = _lib.load(checked=True)
    out = {}

    def fresh():
        cnt, first = ctypes.c_int64(7), ctypes.c_int64(7)
        out["st"] = lib.msda_checked_last_violation(ctypes.byref(cnt), ctypes.byref(first))
        out["v"] = (cnt.value, first.value)
        out["null"] = lib.msda_checked_last_violation(None, None)

    t = threading.Thread(target=fresh)
    t.start()
    t.join()
    assert out == {"st": OK, "v": (0, -1), "null": OK}
    assert lib.msda_checked_set_limit(1000) == OK
    assert lib.msda_checked_set_limit(-5) == OK


@pytest.mark.parametrize("shapes", [wl.TINY_SHAPES, wl.ENCODER_SHAPES, wl.STRESS_SHAPES,
                                    ((0, 5), (3, 0), (1, 1)), ((7, 3),)])
def test_level_start_index_bit_exact_with_oracle(lib, shapes):
    from scale_deformable_attention_02_b200 import msda_level_start_index
    s = wl.spatial_shapes_array(shapes)
    starts, S = msda_level_start_index(s)
    ostarts, oS = oracle.level_start_index(s)
    assert starts.tolist() == ostarts.tolist() and S == oS


def test_level_start_index_errors(lib):
    s = np.array([[3, -1]], dtype=np.int64)
    out = np.zeros(1, dtype=np.int64)
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)  # noqa: E731
    assert lib.msda_level_start_index(p(s), 1, p(out), None) == SHAPE
    assert lib.msda_level_start_index(None, 1, p(out), None) == NULL
    assert lib.msda_level_start_index(p(s), 0, p(out), None) == SHAPE


# ---------------------------------------------------------------------------
# Argument checks of the compute entry points (fake device pointers).
# ---------------------------------------------------------------------------
BASE = 1 << 32  # fake, 256-byte aligned device addresses, far apart
GAP = 1 << 28


def fake(i, off=0):
    return ctypes.c_void_p(BASE + i * GAP + off)


class Prob:
    def __init__(self, N=2, Lq=5, M=2, D=8, K=2, shapes=((4, 6), (2, 3)), dtype=0):
        self.shapes = np.array(shapes, dtype=np.int64).reshape(-1, 2)
        self.starts, S = oracle.level_start_index(self.shapes)
        self.dims = _lib.Dims(N, Lq, S, M, D, len(shapes), K)
        self.dtype = dtype

    def sp(self):
        return self.shapes.ctypes.data_as(ctypes.c_void_p)

    def st(self):
        return self.starts.ctypes.data_as(ctypes.c_void_p)


def fwd(lib, pr, value=None, loc=None, attn=None, out=None, dims=None, dtype=None,
        shapes=None, starts=None):
    return lib.msda_forward(value or fake(0), pr.dtype if dtype is None else dtype,
                            shapes or pr.sp(), starts or pr.st(), loc or fake(1),
                            attn or fake(2), out or fake(3), dims or pr.dims, None)


def test_forward_argument_errors(lib):
    pr = Prob()
    assert fwd(lib, pr, dtype=7) == DTYPE
    bad = Prob()
    bad.dims.M = 0
    assert fwd(lib, bad) == SHAPE
    bad = Prob()
    bad.dims.N = -1
    assert fwd(lib, bad) == SHAPE
    # L*K beyond four samples per lane, more than 32 levels
    assert fwd(lib, Prob(K=65)) == UNSUP
    assert fwd(lib, Prob(K=1, shapes=tuple((1, 1) for _ in range(33)))) == UNSUP
    # level metadata that disagrees with S or with the prefix sum
    bad = Prob()
    bad.dims.S += 1
    assert fwd(lib, bad) == LEVELS
    bad = Prob()
    bad.starts[1] += 1
    assert fwd(lib, bad) == LEVELS
    bad = Prob(shapes=((4, -6), (2, 3)))
    assert fwd(lib, bad) == SHAPE
    # row sizes: fp32 D = 3 (12 B), bf16 D = 4 (8 B) are not 16-byte multiples
    assert fwd(lib, Prob(D=3)) == ALIGN
    assert fwd(lib, Prob(D=4, dtype=1)) == ALIGN
    # int32 head offsets: M*D must stay below 2^31 (any row width below that)
    assert fwd(lib, Prob(M=2, D=1 << 30)) == UNSUP
    # pointers
    assert lib.msda_forward(fake(0), 0, None, pr.st(), fake(1), fake(2), fake(3), pr.dims,
                            None) == NULL
    assert fwd(lib, pr, value=fake(0, 8)) == ALIGN
    assert fwd(lib, pr, out=fake(3, 4)) == ALIGN
    assert fwd(lib, pr, loc=fake(1, 4)) == ALIGN
    assert fwd(lib, pr, attn=fake(2, 2)) == ALIGN
    assert lib.msda_forward(fake(0), 0, pr.sp(), pr.st(), None, fake(2), fake(3), pr.dims,
                            None) == NULL
    # out overlapping an input
    assert fwd(lib, pr, out=fake(1)) == ALIAS
    assert fwd(lib, pr, out=fake(0, 64)) == ALIAS
    # int32 row offsets: S*M*D must stay below 2^31
    huge = Prob(M=8, D=32, shapes=((4096, 2049),))
    assert fwd(lib, huge) == UNSUP
    # 32-bit item indices: N*Lq*M must stay below 2^31 (here exactly 2^31)
    many = Prob(N=2, Lq=1 << 29, M=2)
    assert fwd(lib, many) == UNSUP
    assert lib.msda_backward(fake(0), 0, many.sp(), many.st(), fake(1), fake(2), fake(3),
                             fake(4), None, None, many.dims, None) == UNSUP


def test_empty_problems_are_no_ops(lib):
    """N = 0 or Lq = 0: nothing to compute, null tensors allowed, no launch."""
    for N, Lq in ((0, 5), (2, 0)):
        pr = Prob(N=N, Lq=Lq)
        assert lib.msda_forward(None, 0, pr.sp(), pr.st(), None, None, None, pr.dims,
                                None) == OK
        assert lib.msda_forward_fused(None, 0, pr.sp(), pr.st(), None, 2, None, None, None,
                                      None, None, pr.dims, None) == OK
    pr = Prob(N=0)
    assert lib.msda_backward(None, 0, pr.sp(), pr.st(), None, None, None, None, None, None,
                             pr.dims, None) == OK


def test_fused_argument_errors(lib):
    pr = Prob()

    def call(ref=None, rdim=2, off=None, logits=None, out=None, loc_out=None, attn_out=None):
        return lib.msda_forward_fused(fake(0), 0, pr.sp(), pr.st(), ref or fake(1), rdim,
                                      off or fake(2), logits or fake(4), out or fake(3),
                                      loc_out, attn_out, pr.dims, None)

    assert call(rdim=3) == SHAPE
    assert call(ref=fake(1, 4)) == ALIGN
    assert call(off=fake(2, 4)) == ALIGN
    assert call(loc_out=fake(5, 4)) == ALIGN
    assert call(loc_out=fake(2)) == ALIAS          # writes over the offsets
    assert call(attn_out=fake(3, 16)) == ALIAS     # overlaps out
    assert call(out=fake(5), loc_out=fake(5, 32)) == ALIAS
    assert lib.msda_forward_fused(fake(0), 0, pr.sp(), pr.st(), None, 2, fake(2), fake(4),
                                  fake(3), None, None, pr.dims, None) == NULL


def test_backward_argument_errors(lib):
    pr = Prob()

    def call(gv=None, gl=None, ga=None, g=None, loc=None):
        return lib.msda_backward(fake(0), 0, pr.sp(), pr.st(), loc or fake(1), fake(2),
                                 g or fake(3), gv or fake(4), gl, ga, pr.dims, None)

    assert call(gv=fake(4, 8)) == ALIGN
    assert call(gl=fake(5, 4)) == ALIGN
    assert call(gv=fake(3)) == ALIAS          # grad_value over grad_out
    assert call(gl=fake(4, 64)) == ALIAS      # grad_loc inside grad_value
    assert call(ga=fake(1)) == ALIAS          # grad_attn over the locations
    assert lib.msda_backward(fake(0), 0, pr.sp(), pr.st(), fake(1), fake(2), fake(3), None,
                             None, None, pr.dims, None) == NULL


def test_binding_rejects_mismatched_tensors():
    torch = pytest.importorskip("torch")
    from scale_deformable_attention_02_b200 import msda_forward
    value = torch.zeros(1, 80, 2, 8)
    loc = torch.zeros(1, 4, 2, 2, 2, 2)
    attn = torch.zeros(1, 4, 2, 2, 3)  # K mismatch
    with pytest.raises(ValueError):
        msda_forward(value, wl.TINY_SHAPES, None, loc, attn)


def test_backward_fused_argument_errors(lib):
    pr = Prob()

    def call(rdim=2, gv=None, gr=None, go=None, gz=None, ref=None, dims=None):
        return lib.msda_backward_fused(fake(0), 0, pr.sp(), pr.st(), ref or fake(1), rdim,
                                       fake(2), fake(3), fake(4), gv or fake(5), gr, go, gz,
                                       dims or pr.dims, None)

    assert call(rdim=3) == SHAPE
    assert call(gv=fake(5, 8)) == ALIGN
    assert call(gr=fake(6, 4)) == ALIGN
    assert call(go=fake(2)) == ALIAS           # grad_offsets over the offsets
    assert call(gz=fake(5, 64)) == ALIAS       # grad_logits inside grad_value
    assert call(gr=fake(6), go=fake(6, 8)) == ALIAS
    assert lib.msda_backward_fused(fake(0), 0, pr.sp(), pr.st(), None, 2, fake(2), fake(3),
                                   fake(4), fake(5), None, None, None, pr.dims, None) == NULL


def test_grouped_argument_errors(lib):
    """Group counts must divide M (MSDA_ERR_SHAPE); per-group tensors are
    G/M the size of per-head ones in the alias check."""
    pr = Prob(M=4)

    def fwd_g(G, loc=None, out=None):
        return lib.msda_forward_grouped(fake(0), 0, pr.sp(), pr.st(), loc or fake(1), fake(2),
                                        out or fake(3), pr.dims, G, None)

    for G in (0, -1, 3, 5, 8):
        assert fwd_g(G) == SHAPE, G
    # a grouped location tensor of G=1 spans N*Lq*1*L*K*2 floats: an output
    # placed right after it does not alias, one inside it does
    n_loc = 2 * 5 * 1 * 2 * 2 * 2 * 4  # bytes, G = 1
    assert lib.msda_forward_grouped(fake(0), 0, pr.sp(), pr.st(), fake(1), fake(2),
                                    fake(1, n_loc - 16), pr.dims, 1, None) == ALIAS
    assert lib.msda_backward_grouped(fake(0), 0, pr.sp(), pr.st(), fake(1), fake(2), fake(3),
                                     fake(4), None, None, pr.dims, 3, None) == SHAPE
    assert lib.msda_forward_fused_grouped(fake(0), 0, pr.sp(), pr.st(), fake(1), 2, fake(2),
                                          fake(4), fake(3), None, None, pr.dims, 0,
                                          None) == SHAPE
    assert lib.msda_backward_fused_grouped(fake(0), 0, pr.sp(), pr.st(), fake(1), 2, fake(2),
                                           fake(3), fake(4), fake(5), None, None, None,
                                           pr.dims, 6, None) == SHAPE


def test_row_traffic_argument_errors(lib):
    """msda_debug_row_traffic rejects bad modes, depths, sizes, pointers and
    aliasing before any device work."""
    def f(mode, value, grad, n_value, rows, n_rows, sink=None, sink_len=0, depth=0, dt=0):
        return lib.msda_debug_row_traffic(mode, value, dt, grad, n_value, rows, n_rows, sink,
                                          sink_len, depth, 0, None)

    assert f(3, fake(0), fake(1), 64, fake(2), 10) == SHAPE
    assert f(0, fake(0), None, 16, fake(2), 10) == SHAPE
    assert f(0, fake(0), None, 64, fake(2), -1) == SHAPE
    assert f(0, fake(0), None, 64, fake(2), 10, depth=3) == SHAPE
    assert f(0, None, None, 64, fake(2), 10) == NULL
    assert f(1, fake(0), None, 64, fake(2), 10) == NULL
    assert f(0, fake(0), None, 64, None, 10) == NULL
    assert f(0, fake(0, 8), None, 64, fake(2), 10) == ALIGN
    assert f(2, fake(0), fake(0, 64), 64, fake(2), 10) == ALIAS
    assert f(2, fake(0), fake(1), 64, fake(2), 10, fake(1, 16), 8) == ALIAS
    assert f(2, fake(0), fake(1), 64, fake(2), 0) == OK  # nothing to do
    assert f(0, fake(0), None, 64, fake(2), 10, dt=2) == DTYPE
    # a bf16 value map of 64 elements is 128 bytes: a grad 128 bytes on does not overlap it
    assert f(2, fake(0), fake(0, 128), 64, fake(2), 0, dt=1) == OK
    assert f(2, fake(0), fake(0, 112), 64, fake(2), 0, dt=1) == ALIAS
