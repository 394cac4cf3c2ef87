"""CPU checks of the C-ABI library: it builds, loads, exports every declared
symbol, and its host-side logic (sizes, argument validation) is right.  No call
here reaches a CUDA kernel: every invalid argument is rejected before launch.
"""
from __future__ import annotations

import math
import os
import re

import pytest

from oracle import bcq_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lutgemm.h")


@pytest.fixture(scope="module")
def L():
    from weight_only_quantized_bcq_b200 import build, lutgemm
    build.build()
    return lutgemm


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lutgemm_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("lutgemm_pack_bcq", "lutgemm_uniform_to_bcq", "lutgemm_run",
                 "lutgemm_packed_bytes", "lutgemm_workspace_size", "lutgemm_status_string"):
        assert must in names


def test_library_exports_every_declared_symbol(L):
    lib = L.lib()
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_version_and_status_strings(L):
    lib = L.lib()
    assert lib.lutgemm_version() >= 10000
    for st in range(7):
        assert len(L.status_string(st)) > 5
    assert L.status_string(99) == "unknown status"


@pytest.mark.parametrize("q,m,n", [(1, 1, 8), (3, 512, 512), (3, 49152, 12288), (2, 33, 1032),
                                   (8, 100, 5000), (4, 5120, 5120)])
def test_packed_bytes_matches_oracle(L, q, m, n):
    assert L.packed_bytes(q, m, n) == O.packed_nbytes(q, m, n)


@pytest.mark.parametrize("q,m,n", [(0, 32, 1024), (9, 32, 1024), (3, 0, 1024), (3, 32, 0), (3, 32, 12)])
def test_packed_bytes_rejects_bad_shapes(L, q, m, n):
    assert L.packed_bytes(q, m, n) == 0


def test_workspace_size(L):
    m, n, b = 49152, 12288, 1
    ns, mt = math.ceil(n / 1024), math.ceil(m / 32)
    part = b * ns * mt * 32 * 4
    rup = lambda v: (v + 255) // 256 * 256
    assert L.workspace_size(m, n, b, 3, 128) == 256 + 4096 + rup(part)   # status word, tile counters, partials
    assert L.workspace_size(m, n, 0, 3, 128) == 0
    assert L.workspace_size(m, n, 1, 3, 100) == 0          # g % 8 != 0
    assert L.workspace_size(m, 12288, 1, 3, 5000) == 0     # n % g != 0


FAKE = 1 << 20           # 16-byte aligned, never dereferenced: validation fails first


def _run(L, m=64, n=1024, batch=1, q=3, g=128, packed=FAKE, alpha=FAKE, offset=None, x=FAKE, y=FAKE,
         flags=0, ws=FAKE, ws_bytes=None):
    lib = L.lib()
    if ws_bytes is None:
        ws_bytes = 1 << 30
    return lib.lutgemm_run(m, n, batch, q, g, packed, alpha, offset, x, y, flags, ws, ws_bytes, None)


def test_run_rejects_null(L):
    assert _run(L, packed=None) == L.ERR_NULL
    assert _run(L, alpha=None) == L.ERR_NULL
    assert _run(L, x=None) == L.ERR_NULL
    assert _run(L, y=None) == L.ERR_NULL
    assert _run(L, ws=None) == L.ERR_NULL


@pytest.mark.parametrize("kw", [dict(m=0), dict(n=0), dict(n=1028), dict(batch=0), dict(q=0), dict(q=9),
                                dict(g=100), dict(g=0), dict(n=1024, g=384), dict(n=12),
                                # batch * ceil(n / 1024) must stay below 2^31
                                dict(batch=1 << 20, n=1 << 21)])
def test_run_rejects_bad_shapes(L, kw):
    assert _run(L, **kw) == L.ERR_SHAPE


def test_run_rejects_misaligned(L):
    assert _run(L, packed=FAKE + 8) == L.ERR_ALIGN
    assert _run(L, x=FAKE + 8) == L.ERR_ALIGN
    assert _run(L, alpha=FAKE + 1) == L.ERR_ALIGN
    assert _run(L, offset=FAKE + 2) == L.ERR_ALIGN
    assert _run(L, y=FAKE + 2) == L.ERR_ALIGN
    assert _run(L, ws=FAKE + 4) == L.ERR_ALIGN


def test_run_rejects_bad_flags_and_small_workspace(L):
    assert _run(L, flags=8) == L.ERR_VALUE
    assert _run(L, flags=16 | L.Y_F16) == L.ERR_VALUE
    assert _run(L, flags=8 | L.ALLOW_TENSOR_CORES) == L.ERR_VALUE
    # Unit-major scales need g % 128 == 0 or g == 64 and a 16-byte aligned scale buffer.
    assert _run(L, n=1024, g=32, flags=L.SCALES_PACKED) == L.ERR_VALUE
    assert _run(L, n=1024, g=64, flags=L.SCALES_PACKED, alpha=FAKE + 2) == L.ERR_ALIGN
    assert _run(L, alpha=FAKE + 2, flags=L.SCALES_PACKED) == L.ERR_ALIGN
    need = L.workspace_size(64, 1024, 1, 3, 128)
    assert _run(L, ws_bytes=need - 1) == L.ERR_WORKSPACE


def test_scales_bytes(L):
    for q, m, n, g in [(3, 40, 2048, 128), (5, 70, 2048, 256), (2, 33, 640, 128), (8, 1, 1024, 1024),
                       (2, 40, 2048, 64), (6, 33, 640, 64)]:
        assert L.scales_bytes(q, m, n, g) == O.scales_nbytes(q, m, n, g)
    assert L.scales_bytes(3, 64, 1024, 32) == 0        # neither g % 128 == 0 nor g == 64
    assert L.scales_bytes(3, 64, 1000, 128) == 0       # n % g != 0
    assert L.scales_bytes(9, 64, 1024, 128) == 0


def test_run_tc_validation(L):
    lib = L.lib()
    ok = [256, 1024, 16, 3, 128, FAKE, FAKE, None, FAKE, FAKE, 0, None]
    def call(**kw):
        a = list(ok)
        for k, v in kw.items():
            a[["m", "n", "batch", "q", "g", "packed", "alpha", "offset", "x", "y", "flags", "stream"].index(k)] = v
        return lib.lutgemm_run_tc(*a)
    assert call(packed=None) == L.ERR_NULL
    assert call(y=None) == L.ERR_NULL
    assert call(g=32) == L.ERR_SHAPE             # needs g % 64 == 0
    assert call(n=1032, g=8) == L.ERR_SHAPE      # needs n % 128 == 0
    assert call(batch=0) == L.ERR_SHAPE
    assert call(flags=2) == L.ERR_VALUE
    assert call(x=FAKE + 8) == L.ERR_ALIGN
    assert call(packed=FAKE + 8) == L.ERR_ALIGN
    assert call(y=FAKE + 2) == L.ERR_ALIGN
    assert call(offset=FAKE + 2) == L.ERR_ALIGN  # offsets are fp32


def test_fit_validation(L):
    lib = L.lib()
    ok = [FAKE, 3, 32, 1024, 128, 3, FAKE, FAKE, None, None]
    def call(**kw):
        a = list(ok)
        for k, v in kw.items():
            a[["w", "q", "m", "n", "g", "iters", "signs", "alpha", "err", "stream"].index(k)] = v
        return lib.lutgemm_fit_bcq(*a)
    assert call(w=None) == L.ERR_NULL
    assert call(signs=None) == L.ERR_NULL
    assert call(alpha=None) == L.ERR_NULL
    assert call(q=9) == L.ERR_SHAPE
    assert call(g=96) == L.ERR_SHAPE             # n % g != 0
    assert call(n=4096, g=2048) == L.ERR_SHAPE   # groups above 1024 inputs
    assert call(iters=-1) == L.ERR_VALUE
    assert call(iters=65) == L.ERR_VALUE
    assert call(w=FAKE + 8) == L.ERR_ALIGN
    assert call(signs=FAKE + 4) == L.ERR_ALIGN
    assert call(alpha=FAKE + 1) == L.ERR_ALIGN
    assert call(err=FAKE + 2) == L.ERR_ALIGN


def test_fit_grid_validation(L):
    lib = L.lib()
    names = ["w", "q", "m", "n", "g", "iters", "signs", "alpha", "offset", "err", "stream"]
    ok = [FAKE, 3, 32, 1024, 128, 3, FAKE, FAKE, FAKE, None, None]
    def call(**kw):
        a = list(ok)
        for k, v in kw.items():
            a[names.index(k)] = v
        return lib.lutgemm_fit_bcq_grid(*a)
    assert call(w=None) == L.ERR_NULL
    assert call(offset=None) == L.ERR_NULL       # the grid's constant is an output
    assert call(signs=None) == L.ERR_NULL
    assert call(q=0) == L.ERR_SHAPE
    assert call(g=96) == L.ERR_SHAPE
    assert call(n=4096, g=2048) == L.ERR_SHAPE
    assert call(iters=65) == L.ERR_VALUE
    assert call(w=FAKE + 8) == L.ERR_ALIGN
    assert call(offset=FAKE + 2) == L.ERR_ALIGN
    assert call(err=FAKE + 2) == L.ERR_ALIGN


def test_pack_scales_validation(L):
    lib = L.lib()
    assert lib.lutgemm_pack_scales(None, 3, 32, 1024, 128, FAKE, None) == L.ERR_NULL
    assert lib.lutgemm_pack_scales(FAKE, 3, 32, 1024, 128, None, None) == L.ERR_NULL
    assert lib.lutgemm_pack_scales(FAKE, 3, 32, 1024, 32, FAKE, None) == L.ERR_SHAPE
    assert lib.lutgemm_pack_scales(FAKE, 0, 32, 1024, 128, FAKE, None) == L.ERR_SHAPE
    assert lib.lutgemm_pack_scales(FAKE + 1, 3, 32, 1024, 128, FAKE, None) == L.ERR_ALIGN
    assert lib.lutgemm_pack_scales(FAKE, 3, 32, 1024, 128, FAKE + 8, None) == L.ERR_ALIGN


def test_pack_and_convert_validation(L):
    lib = L.lib()
    assert lib.lutgemm_pack_bcq(None, 3, 32, 1024, FAKE, None, None) == L.ERR_NULL
    assert lib.lutgemm_pack_bcq(FAKE, 3, 32, 1020, FAKE, None, None) == L.ERR_SHAPE
    assert lib.lutgemm_pack_bcq(FAKE + 4, 3, 32, 1024, FAKE, None, None) == L.ERR_ALIGN
    assert lib.lutgemm_pack_bcq(FAKE, 3, 32, 1024, FAKE + 8, None, None) == L.ERR_ALIGN
    args = [FAKE, FAKE, FAKE, 4, 32, 1024, 128, FAKE, FAKE, FAKE, None, None]
    bad = list(args); bad[1] = None
    assert lib.lutgemm_uniform_to_bcq(*bad) == L.ERR_NULL
    bad = list(args); bad[6] = 96
    assert lib.lutgemm_uniform_to_bcq(*bad) == L.ERR_SHAPE
    bad = list(args); bad[9] = FAKE + 2
    assert lib.lutgemm_uniform_to_bcq(*bad) == L.ERR_ALIGN


def test_product_has_no_cpu_fallback(L, monkeypatch):
    """Without the library the binding raises instead of computing anything."""
    monkeypatch.setattr(L, "_lib", None)
    monkeypatch.setattr(L, "LIB_PATH", os.path.join(ROOT, "does-not-exist.so"))
    with pytest.raises(RuntimeError):
        L.lib()


def test_product_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "weight_only_quantized_bcq_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle\b", text, re.M), f
                assert "bcq_oracle" not in text, f


def test_tensor_core_plan_matches_the_measured_choices(L):
    """lutgemm_tc_plan on 148 SMs picks, for each measured (shape, batch), the
    path and split count that measured fastest on a B200 (OPT-175B and
    LLaMA-70B linears; see the config sweep): QKV and FC1 one split, out-proj
    and FC2 three; at batch 8 the LLaMA-70B up-projection one split and its
    8192-wide q/k/v/o and down projections two."""
    sms = 148
    want = {  # (m, n, q): {batch: splits}
        (36864, 12288, 3): {8: 1, 16: 1, 32: 1, 256: 1},
        (49152, 12288, 3): {8: 1, 16: 1, 32: 1, 256: 1},
        (12288, 49152, 3): {8: 3, 16: 3, 32: 3, 256: 3},
        (12288, 12288, 3): {256: 3},
        (8192, 8192, 2): {8: 2},
        (28672, 8192, 2): {8: 1},
        (8192, 28672, 2): {8: 2},
    }
    for (m, n, q), cases in want.items():
        for batch, splits in cases.items():
            assert L.tc_plan(m, n, batch, q, sms) == splits, (m, n, q, batch)
    # Below batch 8, and with splitting disallowed, the plan never splits.
    assert L.tc_plan(49152, 12288, 7, 3, sms) == 0
    assert L.tc_plan(12288, 49152, 32, 3, sms, max_split=1) == 1
    # Splits are whole 1024-input slices: never more splits than slices.
    for batch in (8, 64, 256):
        assert 0 <= L.tc_plan(12288, 3072, batch, 3, sms) <= 3


def test_binding_signatures_match_the_header(L):
    """Every function the binding declares has the header's argument count and
    a return type of the same kind (int status, size_t size, const char*)."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    decls = {}
    for ret, name, args in re.findall(r"(\w[\w\s\*]*?)\s*\b(lutgemm_\w+)\s*\(([^)]*)\)\s*;", text, flags=re.S):
        args = args.strip()
        n = 0 if args in ("", "void") else len([a for a in args.split(",") if a.strip()])
        decls[name] = (ret.split()[-1] if ret.split() else ret, n)
    import ctypes
    kinds = {"int": ctypes.c_int, "size_t": ctypes.c_size_t, "char*": ctypes.c_char_p}
    for name, (argtypes, restype) in L._SIGNATURES.items():
        assert name in decls, name
        ret, n = decls[name]
        assert len(argtypes) == n, (name, len(argtypes), n)
        want = kinds.get(ret.replace("const", "").strip())
        if want is not None:
            assert restype is want, (name, ret, restype)


# ---------------------------------------------------------------------------
# The launch plan query and the status-word calls' host-side validation.
# ---------------------------------------------------------------------------
def _plan(L, m, n, batch, sms=148):
    return L.launch_plan(m, n, batch, sms)


def test_launch_plan_matches_the_kernels_grouping(L):
    # 37 batch columns x 4 slices = 148 segments, one CTA each: 64 row tiles
    # per segment, 32 of them static, so 32 per segment come from the counters.
    assert _plan(L, 2048, 4096, 37) == (148, 1, 148 * 32)
    # OPT-175B FC1 at batch 1: 12 segments of 12 CTAs (144 launched), 384
    # static tiles and 1152 dynamic ones per segment.
    assert _plan(L, 49152, 12288, 1) == (144, 1, 12 * 1152)
    # Two tiles: one CTA per tile, no counters needed.
    assert _plan(L, 64, 1024, 1) == (2, 1, 0)
    # More segments than SMs: the unit list is cut into contiguous ranges.
    assert _plan(L, 64, 1024, 200) == (148, 0, 0)


def test_launch_plan_group_sizes_are_the_kernels():
    """The dynamic count is the sum over segments of mt - 32 * (CTAs of the
    segment), with the kernel's own rule for a segment's CTA count."""
    from weight_only_quantized_bcq_b200 import lutgemm as L
    L.lib()
    for (m, n, b) in [(2048, 4096, 37), (12600, 12288, 1), (40000, 2048, 3)]:
        grid, aligned, dyn = _plan(L, m, n, b)
        segs = b * math.ceil(n / 1024)
        mt = math.ceil(m / 32)
        if aligned:
            want = sum(max(0, mt - 32 * ((grid - z + segs - 1) // segs)) for z in range(segs))
            assert dyn == want


def test_launch_plan_rejects_bad_arguments(L):
    lib = L.lib()
    import ctypes
    a = ctypes.c_int(0)
    assert lib.lutgemm_launch_plan(64, 1024, 1, 148, None, ctypes.byref(a), ctypes.byref(a)) == L.ERR_NULL
    for args in [(0, 1024, 1, 148), (64, 12, 1, 148), (64, 1024, 0, 148), (64, 1024, 1, 0)]:
        assert lib.lutgemm_launch_plan(*args, ctypes.byref(a), ctypes.byref(a), ctypes.byref(a)) == L.ERR_SHAPE


def test_status_calls_validate_before_touching_the_device(L):
    lib = L.lib()
    import ctypes
    v = ctypes.c_uint32(0)
    assert lib.lutgemm_workspace_status(None, 1 << 20, ctypes.byref(v), 1, None) == L.ERR_NULL
    assert lib.lutgemm_workspace_status(FAKE, 1 << 20, None, 1, None) == L.ERR_NULL
    assert lib.lutgemm_workspace_status(FAKE + 4, 1 << 20, ctypes.byref(v), 1, None) == L.ERR_ALIGN
    assert lib.lutgemm_workspace_status(FAKE, 256 + 4095, ctypes.byref(v), 1, None) == L.ERR_WORKSPACE
    assert lib.lutgemm_library_status(None, 1, None) == L.ERR_NULL


def test_test_stall_flag_is_accepted_by_validation_only_with_valid_arguments(L):
    # The flag passes flag validation (the call then fails on the null pointer).
    assert _run(L, flags=L.TEST_STALL, packed=None) == L.ERR_NULL
    assert _run(L, flags=L.TEST_STALL | 8) == L.ERR_VALUE
