"""Thin ctypes binding over ``liblutgemm.so`` (declared in ``include/lutgemm.h``).

The functions here only marshal torch tensors (device memory, the current CUDA
stream) into the C calls; every step of the computation runs in the library's
CUDA kernels.  If the library is missing the calls raise: there is no fallback.
"""
from __future__ import annotations

import ctypes
import functools
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblutgemm.so")

OK, ERR_NULL, ERR_SHAPE, ERR_ALIGN, ERR_WORKSPACE, ERR_VALUE, ERR_CUDA = range(7)
FLAG_BAD_SIGN, FLAG_BAD_CODE, FLAG_BAD_ZERO = 1, 2, 4
STATUS_WINDOW, STATUS_TIMEOUT, STATUS_FORMAT = 1, 2, 4
FLAG_BAD_BLOCK = 8
Y_F16 = 1
SCALES_PACKED = 2
ALLOW_TENSOR_CORES = 4
TEST_STALL = 0x80000000

_lib = None

_c_int, _c_uint, _c_size, _vp = ctypes.c_int, ctypes.c_uint, ctypes.c_size_t, ctypes.c_void_p
_SIGNATURES = {
    "lutgemm_version": ([], _c_int),
    "lutgemm_status_string": ([_c_int], ctypes.c_char_p),
    "lutgemm_packed_bytes": ([_c_int, _c_int, _c_int], _c_size),
    "lutgemm_workspace_size": ([_c_int, _c_int, _c_int, _c_int, _c_int], _c_size),
    "lutgemm_scales_bytes": ([_c_int, _c_int, _c_int, _c_int], _c_size),
    "lutgemm_tc_plan": ([_c_int, _c_int, _c_int, _c_int, _c_int, _c_int], _c_int),
    "lutgemm_pack_scales": ([_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp], _c_int),
    "lutgemm_fit_bcq": ([_vp, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp], _c_int),
    "lutgemm_fit_bcq_grid": ([_vp, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp], _c_int),
    "lutgemm_run_tc": ([_c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp, _c_uint, _vp], _c_int),
    "lutgemm_pack_bcq": ([_vp, _c_int, _c_int, _c_int, _vp, _vp, _vp], _c_int),
    "lutgemm_uniform_to_bcq": ([_vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp],
                               _c_int),
    "lutgemm_run": ([_c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp, _c_uint, _vp, _c_size,
                     _vp], _c_int),
    "lutgemm_run_noalloc": ([_c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp, _c_uint, _vp],
                            _c_int),
    "lutgemm_workspace_status": ([_vp, _c_size, _vp, _c_int, _vp], _c_int),
    "lutgemm_mixed_offsets": ([_vp, _c_int, _c_int, _c_int, _vp], _c_int),
    "lutgemm_pack_outliers": ([_vp, _vp, _vp, _c_int, _c_int, _c_int, _vp, _vp], _c_int),
    "lutgemm_pack_bcq_mixed": ([_vp, _vp, _c_int, _c_int, _c_int, _vp, _c_size, _vp, _vp], _c_int),
    "lutgemm_pack_scales_mixed": ([_vp, _vp, _c_int, _c_int, _c_int, _c_int, _vp, _c_size, _vp, _vp], _c_int),
    "lutgemm_run_mixed": ([_c_int, _c_int, _c_int, _c_int, _c_int, _vp, _c_size, _vp, _vp, _vp, _vp, _c_int, _vp,
                           _vp, _c_uint, _vp, _c_size, _vp], _c_int),
    "lutgemm_library_status": ([_vp, _c_int, _vp], _c_int),
    "lutgemm_launch_plan": ([_c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp], _c_int),
}


class LutgemmError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        super().__init__(f"{call}: {status_string(status)} (status {status})")


def lib() -> ctypes.CDLL:
    """Load the library once; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m weight_only_quantized_bcq_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.argtypes = args
            fn.restype = res
        _lib = handle
    return _lib


class LutgemmDeviceError(RuntimeError):
    """A kernel failed while it ran: its sticky status word has bits set."""

    def __init__(self, bits: int, where: str):
        self.bits = bits
        names = [n for b, n in ((STATUS_WINDOW, "shared-memory window"), (STATUS_TIMEOUT, "wait timed out"),
                                (STATUS_FORMAT, "mixed-storage entry out of range")) if bits & b]
        super().__init__(f"{where}: device status 0x{bits:x} ({', '.join(names) or 'unknown bits'}): "
                         "the outputs are not valid")


def status_string(status: int) -> str:
    return lib().lutgemm_status_string(int(status)).decode()


def _check(status: int, call: str):
    if status != OK:
        raise LutgemmError(status, call)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, dtype, name, numel=None):
    """Host checks of one tensor argument: dtype, contiguity and size.

    ``numel`` is the element count the call reads or writes through the
    pointer; the library sees only the pointer, so a smaller tensor would be
    accessed past its end on the GPU.  Devices are checked by ``_one_device``
    once every argument has passed these checks."""
    if t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} tensor")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} elements; the call needs {numel}")


def _one_device(stream, **named):
    """Every tensor argument (None: absent) on one CUDA device, which is the
    current device (the library launches there) and, when given, the stream's."""
    dev = None
    for name, t in named.items():
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device}, other arguments on {dev}: all must be on one device")
    cur = torch.cuda.current_device()
    if dev.index != cur:
        raise ValueError(f"arguments on {dev} but the current device is cuda:{cur}: "
                         f"call under torch.cuda.device({dev.index})")
    if stream is not None and stream.device != dev:
        raise ValueError(f"stream on {stream.device}, arguments on {dev}")


def _groups(n: int, g: int) -> int:
    return n // g if g > 0 else 0


def _batch_of(x, n: int) -> int:
    """x is [n] (batch 1) or [batch][n]."""
    if x.dim() not in (1, 2) or x.shape[-1] != n:
        raise ValueError(f"x must be [n] or [batch][n] with n = {n}; got {tuple(x.shape)}")
    return x.shape[0] if x.dim() == 2 else 1


def workspace_status(workspace: torch.Tensor, clear: bool = True, stream=None) -> int:
    """The LUTGEMM_STATUS_* bits of a lutgemm_run workspace (waits for the
    stream's work so far); cleared afterwards when ``clear``."""
    _need(workspace, torch.uint8, "workspace")
    _one_device(stream, workspace=workspace)
    v = ctypes.c_uint32(0)
    _check(lib().lutgemm_workspace_status(_ptr(workspace), workspace.numel(), ctypes.byref(v), int(clear),
                                          _stream(stream)),
           "lutgemm_workspace_status")
    return int(v.value)


def library_status(clear: bool = True, stream=None) -> int:
    """The LUTGEMM_STATUS_* bits of the words lutgemm_run_tc and
    lutgemm_run_noalloc use on the current device; cleared when ``clear``."""
    v = ctypes.c_uint32(0)
    _check(lib().lutgemm_library_status(ctypes.byref(v), int(clear), _stream(stream)), "lutgemm_library_status")
    return int(v.value)


def launch_plan(m: int, n: int, batch: int, sm_count: int):
    """(grid, seg_aligned, dynamic_tiles) of the lookup kernel, as lutgemm_run chooses it."""
    grid, aligned, dyn = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    _check(lib().lutgemm_launch_plan(m, n, batch, sm_count, ctypes.byref(grid), ctypes.byref(aligned),
                                     ctypes.byref(dyn)),
           "lutgemm_launch_plan")
    return grid.value, aligned.value, dyn.value


def _raise_if_bits(bits: int, where: str):
    if bits:
        raise LutgemmDeviceError(bits, where)


@functools.lru_cache(maxsize=256)
def packed_bytes(q: int, m: int, n: int) -> int:
    return int(lib().lutgemm_packed_bytes(q, m, n))


@functools.lru_cache(maxsize=256)
def workspace_size(m: int, n: int, batch: int, q: int, g: int) -> int:
    return int(lib().lutgemm_workspace_size(m, n, batch, q, g))


def tc_plan(m: int, n: int, batch: int, q: int, sm_count: int, max_split: int = None) -> int:
    """K splits lutgemm_run would run the tensor cores with under
    LUTGEMM_ALLOW_TENSOR_CORES (0: the lookup kernel), by lutgemm_tc_plan."""
    if max_split is None:
        max_split = -(-n // 1024)
    return int(lib().lutgemm_tc_plan(m, n, batch, q, max_split, sm_count))


def new_workspace(m: int, n: int, batch: int, q: int, g: int, device=None) -> torch.Tensor:
    """A zero-filled workspace, as lutgemm_run requires before first use."""
    nbytes = workspace_size(m, n, batch, q, g)
    if nbytes == 0:
        raise ValueError("invalid shape for lutgemm_workspace_size")
    return torch.zeros(nbytes, dtype=torch.uint8, device=device or "cuda")


@functools.lru_cache(maxsize=256)
def scales_bytes(q: int, m: int, n: int, g: int) -> int:
    """Bytes of the unit-major scale buffer (0 unless g % 128 == 0 or g == 64, or for an invalid shape)."""
    return lib().lutgemm_scales_bytes(q, m, n, g)


def pack_scales(alpha: torch.Tensor, m: int, n: int, g: int, stream=None) -> torch.Tensor:
    """fp16 alpha [q][n/g][m] on the GPU -> unit-major scales (fp16, 1-D), for
    ``run(..., scales_packed=True)``; needs g % 128 == 0 or g == 64."""
    q = alpha.shape[0] if alpha.dim() else 0
    _need(alpha, torch.float16, "alpha", q * _groups(n, g) * m)
    _one_device(stream, alpha=alpha)
    nbytes = scales_bytes(q, m, n, g)
    if nbytes == 0:
        raise LutgemmError(ERR_SHAPE, "lutgemm_scales_bytes")
    scales = torch.empty(nbytes // 2, dtype=torch.float16, device=alpha.device)
    _check(lib().lutgemm_pack_scales(_ptr(alpha), q, m, n, g, _ptr(scales), _stream(stream)),
           "lutgemm_pack_scales")
    return scales


def fit_bcq(w: torch.Tensor, q: int, g: int, iters: int = 3, with_error: bool = False, stream=None):
    """fp16 weights [m][n] on the GPU -> (int8 signs [q][m][n], fp16 alpha [q][n/g][m]
    [, fp32 squared error per group [n/g][m]]) by lutgemm_fit_bcq."""
    _need(w, torch.float16, "w")
    _one_device(stream, w=w)
    m, n = w.shape
    signs = torch.empty((q, m, n), dtype=torch.int8, device=w.device)
    alpha = torch.empty((q, n // g if g > 0 else 0, m), dtype=torch.float16, device=w.device)
    err = torch.empty((n // g if g > 0 else 0, m), dtype=torch.float32, device=w.device) if with_error else None
    _check(lib().lutgemm_fit_bcq(_ptr(w), q, m, n, g, iters, _ptr(signs), _ptr(alpha), _ptr(err), _stream(stream)),
           "lutgemm_fit_bcq")
    return (signs, alpha, err) if with_error else (signs, alpha)


def fit_bcq_grid(w: torch.Tensor, q: int, g: int, iters: int = 3, with_error: bool = False, stream=None):
    """fp16 weights [m][n] on the GPU -> (int8 signs [q][m][n], fp16 alpha [q][n/g][m],
    fp32 offset [n/g][m] [, fp32 squared error per group [n/g][m]]) by lutgemm_fit_bcq_grid:
    the variable grid offset + sum_i alpha_i beta_i, run with ``run(..., offset=offset)``."""
    _need(w, torch.float16, "w")
    _one_device(stream, w=w)
    m, n = w.shape
    ng = n // g if g > 0 else 0
    signs = torch.empty((q, m, n), dtype=torch.int8, device=w.device)
    alpha = torch.empty((q, ng, m), dtype=torch.float16, device=w.device)
    offset = torch.empty((ng, m), dtype=torch.float32, device=w.device)
    err = torch.empty((ng, m), dtype=torch.float32, device=w.device) if with_error else None
    _check(lib().lutgemm_fit_bcq_grid(_ptr(w), q, m, n, g, iters, _ptr(signs), _ptr(alpha), _ptr(offset), _ptr(err),
                                      _stream(stream)),
           "lutgemm_fit_bcq_grid")
    return (signs, alpha, offset, err) if with_error else (signs, alpha, offset)


def pack_bcq(signs: torch.Tensor, packed: torch.Tensor = None, status_flags: torch.Tensor = None,
             stream=None) -> torch.Tensor:
    """int8 signs [q][m][n] (+-1) on the GPU -> packed uint8 planes."""
    _need(signs, torch.int8, "signs")
    q, m, n = signs.shape
    if packed is not None:
        _need(packed, torch.uint8, "packed", packed_bytes(q, m, n))
    if status_flags is not None:
        _need(status_flags, torch.int32, "status_flags", 1)
    _one_device(stream, signs=signs, packed=packed, status_flags=status_flags)
    if packed is None:
        packed = torch.empty(max(packed_bytes(q, m, n), 16), dtype=torch.uint8, device=signs.device)
    _check(lib().lutgemm_pack_bcq(_ptr(signs), q, m, n, _ptr(packed), _ptr(status_flags), _stream(stream)),
           "lutgemm_pack_bcq")
    return packed


def uniform_to_bcq(codes: torch.Tensor, scale: torch.Tensor, zero: torch.Tensor, q: int, g: int,
                   status_flags: torch.Tensor = None, stream=None):
    """Uniform codes [m][n], scale fp16 [n/g][m], zero uint8 [n/g][m] -> (packed, alpha, offset)."""
    _need(codes, torch.uint8, "codes")
    m, n = codes.shape
    _need(scale, torch.float16, "scale", _groups(n, g) * m)
    _need(zero, torch.uint8, "zero", _groups(n, g) * m)
    if status_flags is not None:
        _need(status_flags, torch.int32, "status_flags", 1)
    _one_device(stream, codes=codes, scale=scale, zero=zero, status_flags=status_flags)
    dev = codes.device
    packed = torch.empty(max(packed_bytes(q, m, n), 16), dtype=torch.uint8, device=dev)
    alpha = torch.empty((q, n // g, m), dtype=torch.float16, device=dev)
    offset = torch.empty((n // g, m), dtype=torch.float32, device=dev)
    _check(lib().lutgemm_uniform_to_bcq(_ptr(codes), _ptr(scale), _ptr(zero), q, m, n, g, _ptr(packed),
                                        _ptr(alpha), _ptr(offset), _ptr(status_flags), _stream(stream)),
           "lutgemm_uniform_to_bcq")
    return packed, alpha, offset


def _check_product_args(packed, alpha, x, offset, y, workspace, m, n, q, g, y_f16, scales_packed, stream) -> int:
    """The checks shared by the product calls; returns the batch."""
    batch = _batch_of(x, n)
    _need(packed, torch.uint8, "packed", packed_bytes(q, m, n))
    a_need = scales_bytes(q, m, n, g) // 2 if scales_packed else q * _groups(n, g) * m
    _need(alpha, torch.float16, "alpha", a_need)
    _need(x, torch.float16, "x")
    if offset is not None:
        _need(offset, torch.float32, "offset", _groups(n, g) * m)
    if y is not None:
        _need(y, torch.float16 if y_f16 else torch.float32, "y", batch * m)
    if workspace is not None:
        _need(workspace, torch.uint8, "workspace")
    _one_device(stream, x=x, packed=packed, alpha=alpha, offset=offset, y=y, workspace=workspace)
    return batch


def run(packed: torch.Tensor, alpha: torch.Tensor, x: torch.Tensor, m: int, n: int, q: int, g: int,
        offset: torch.Tensor = None, y: torch.Tensor = None, workspace: torch.Tensor = None,
        y_f16: bool = False, scales_packed: bool = False, allow_tensor_cores: bool = False,
        check: bool = False, stream=None, _flags: int = 0) -> torch.Tensor:
    """y[b] = W x[b] for a packed BCQ weight W (m x n), computed by lutgemm_run.
    With ``scales_packed`` alpha is the output of ``pack_scales``; with
    ``allow_tensor_cores`` the library may take the tensor-core path (batch >= 8).
    With ``check`` the call waits for the kernels and raises LutgemmDeviceError
    if the workspace's status word has bits set (and clears them)."""
    batch = _check_product_args(packed, alpha, x, offset, y, workspace, m, n, q, g, y_f16, scales_packed, stream)
    if y is None:
        y = torch.empty((batch, m), dtype=torch.float16 if y_f16 else torch.float32, device=x.device)
    if workspace is None:
        workspace = new_workspace(m, n, batch, q, g, device=x.device)
    flags = (Y_F16 if y_f16 else 0) | (SCALES_PACKED if scales_packed else 0) | \
        (ALLOW_TENSOR_CORES if allow_tensor_cores else 0) | _flags
    _check(lib().lutgemm_run(m, n, batch, q, g, _ptr(packed), _ptr(alpha), _ptr(offset), _ptr(x), _ptr(y),
                             flags, _ptr(workspace), workspace.numel(), _stream(stream)),
           "lutgemm_run")
    if check:
        _raise_if_bits(workspace_status(workspace, clear=True, stream=stream), "lutgemm_run")
    return y


def run_tc(packed: torch.Tensor, alpha: torch.Tensor, x: torch.Tensor, m: int, n: int, q: int, g: int,
           y: torch.Tensor = None, y_f16: bool = False, offset: torch.Tensor = None, check: bool = False,
           stream=None) -> torch.Tensor:
    """``run`` on the tensor cores (lutgemm_run_tc), for large batches;
    n % 128 == 0 and g % 64 == 0, [q][n/g][m] scales, optional fp32 offsets."""
    batch = _check_product_args(packed, alpha, x, offset, y, None, m, n, q, g, y_f16, False, stream)
    if y is None:
        y = torch.empty((batch, m), dtype=torch.float16 if y_f16 else torch.float32, device=x.device)
    _check(lib().lutgemm_run_tc(m, n, batch, q, g, _ptr(packed), _ptr(alpha), _ptr(offset), _ptr(x), _ptr(y),
                                Y_F16 if y_f16 else 0, _stream(stream)),
           "lutgemm_run_tc")
    if check:
        _raise_if_bits(library_status(clear=True, stream=stream), "lutgemm_run_tc")
    return y


def run_noalloc(packed: torch.Tensor, alpha: torch.Tensor, x: torch.Tensor, m: int, n: int, q: int, g: int,
                offset: torch.Tensor = None, y: torch.Tensor = None, y_f16: bool = False,
                scales_packed: bool = False, allow_tensor_cores: bool = False, check: bool = False,
                stream=None, _flags: int = 0) -> torch.Tensor:
    """``run`` through lutgemm_run_noalloc, for callers that cannot allocate a
    workspace: the library uses its own fixed 16 MiB device scratch instead.
    Only ``y`` is allocated here, and only when the caller passes none.  Calls
    that overlap on the GPU share that scratch and race."""
    batch = _check_product_args(packed, alpha, x, offset, y, None, m, n, q, g, y_f16, scales_packed, stream)
    if y is None:
        y = torch.empty((batch, m), dtype=torch.float16 if y_f16 else torch.float32, device=x.device)
    flags = (Y_F16 if y_f16 else 0) | (SCALES_PACKED if scales_packed else 0) | \
        (ALLOW_TENSOR_CORES if allow_tensor_cores else 0) | _flags
    _check(lib().lutgemm_run_noalloc(m, n, batch, q, g, _ptr(packed), _ptr(alpha), _ptr(offset), _ptr(x),
                                     _ptr(y), flags, _stream(stream)),
           "lutgemm_run_noalloc")
    if check:
        _raise_if_bits(library_status(clear=True, stream=stream), "lutgemm_run_noalloc")
    return y


# ---------------------------------------------------------------------------
# Mixed storage (2/4/16-bit in one matrix): per-block plane counts, sparse
# fp16 outliers.  The format is described in include/lutgemm.h.
# ---------------------------------------------------------------------------
def mixed_offsets(block_planes: torch.Tensor, q_max: int, m: int, n: int) -> torch.Tensor:
    """Host uint8 plane counts [ceil(n/1024)][ceil(m/32)] -> the block table
    (exclusive prefix sums, 4096-byte units) as a host int32 tensor holding
    the uint32 values, by lutgemm_mixed_offsets."""
    ns, mt = -(-n // 1024), -(-m // 32)
    bp = block_planes.contiguous()
    if bp.dtype != torch.uint8 or bp.is_cuda or tuple(bp.shape) != (ns, mt):
        raise ValueError(f"block_planes must be a host uint8 tensor [{ns}][{mt}]")
    out = torch.empty(ns * mt + 1, dtype=torch.int32)
    _check(lib().lutgemm_mixed_offsets(_ptr(bp), q_max, m, n, _ptr(out)), "lutgemm_mixed_offsets")
    return out


def pack_outliers(row_ptr: torch.Tensor, col: torch.Tensor, val: torch.Tensor, m: int, n: int):
    """Host row-CSR outliers (int32 row_ptr [m+1], int32 col, fp16 val) ->
    (optr, oent) host int32 tensors holding the kernel's uint32 layout."""
    rp, c, v = row_ptr.contiguous(), col.contiguous(), val.contiguous()
    if rp.dtype != torch.int32 or c.dtype != torch.int32 or v.dtype != torch.float16 or rp.numel() != m + 1 \
            or rp.is_cuda or c.is_cuda or v.is_cuda or c.numel() != v.numel():
        raise ValueError("outliers must be host tensors: int32 row_ptr [m+1], int32 col [nnz], fp16 val [nnz]")
    nnz = c.numel()
    optr = torch.empty(-(-n // 1024) * m + 1, dtype=torch.int32)
    oent = torch.empty(max(nnz, 1), dtype=torch.int32)
    _check(lib().lutgemm_pack_outliers(_ptr(rp), _ptr(c), _ptr(v), m, n, nnz, _ptr(optr), _ptr(oent)),
           "lutgemm_pack_outliers")
    return optr, oent[:nnz]


def pack_bcq_mixed(signs: torch.Tensor, block_off: torch.Tensor, status_flags: torch.Tensor = None,
                   stream=None) -> torch.Tensor:
    """int8 signs [q_max][m][n] and the block table (int32, on the device) ->
    the mixed packed planes, by lutgemm_pack_bcq_mixed."""
    _need(signs, torch.int8, "signs")
    q_max, m, n = signs.shape
    _need(block_off, torch.int32, "block_off", -(-n // 1024) * -(-m // 32) + 1)
    if status_flags is not None:
        _need(status_flags, torch.int32, "status_flags", 1)
    _one_device(stream, signs=signs, block_off=block_off, status_flags=status_flags)
    nbytes = int(block_off[-1].item()) * 4096
    packed = torch.empty(nbytes, dtype=torch.uint8, device=signs.device)
    _check(lib().lutgemm_pack_bcq_mixed(_ptr(signs), _ptr(block_off), q_max, m, n, _ptr(packed), nbytes,
                                        _ptr(status_flags), _stream(stream)),
           "lutgemm_pack_bcq_mixed")
    return packed


def pack_scales_mixed(alpha: torch.Tensor, block_off: torch.Tensor, m: int, n: int, g: int,
                      status_flags: torch.Tensor = None, stream=None) -> torch.Tensor:
    """fp16 alpha [q_max][n/g][m] and the block table (device) -> the unit-major
    mixed scales (fp16, 1-D), for ``run_mixed(..., scales_packed=True)``;
    needs g % 128 == 0 or g == 64."""
    q_max = alpha.shape[0] if alpha.dim() else 0
    _need(alpha, torch.float16, "alpha", q_max * _groups(n, g) * m)
    _need(block_off, torch.int32, "block_off", -(-n // 1024) * -(-m // 32) + 1)
    if status_flags is not None:
        _need(status_flags, torch.int32, "status_flags", 1)
    _one_device(stream, alpha=alpha, block_off=block_off, status_flags=status_flags)
    nbytes = int(block_off[-1].item()) * (1024 if g == 64 else 512)
    scales = torch.empty(max(nbytes // 2, 8), dtype=torch.float16, device=alpha.device)
    _check(lib().lutgemm_pack_scales_mixed(_ptr(alpha), _ptr(block_off), q_max, m, n, g, _ptr(scales), nbytes,
                                           _ptr(status_flags), _stream(stream)),
           "lutgemm_pack_scales_mixed")
    return scales


def run_mixed(packed: torch.Tensor, block_off: torch.Tensor, alpha: torch.Tensor, x: torch.Tensor, m: int, n: int,
              q_max: int, g: int, optr: torch.Tensor = None, oent: torch.Tensor = None, y: torch.Tensor = None,
              workspace: torch.Tensor = None, y_f16: bool = False, scales_packed: bool = False, check: bool = False,
              stream=None, _flags: int = 0) -> torch.Tensor:
    """y[b] = W x[b] for a mixed matrix, by lutgemm_run_mixed (outliers optional;
    with ``scales_packed`` alpha is the output of ``pack_scales_mixed``)."""
    batch = _batch_of(x, n)
    _need(packed, torch.uint8, "packed")
    _need(block_off, torch.int32, "block_off", -(-n // 1024) * -(-m // 32) + 1)
    _need(alpha, torch.float16, "alpha",
          (packed.numel() // 4096) * (512 if g == 64 else 256) if scales_packed else q_max * _groups(n, g) * m)
    _need(x, torch.float16, "x")
    nnz = 0
    if oent is not None:
        _need(oent, torch.int32, "oent")
        _need(optr, torch.int32, "optr", -(-n // 1024) * m + 1)
        nnz = oent.numel()
    if y is not None:
        _need(y, torch.float16 if y_f16 else torch.float32, "y", batch * m)
    if workspace is not None:
        _need(workspace, torch.uint8, "workspace")
    _one_device(stream, x=x, packed=packed, block_off=block_off, alpha=alpha, optr=optr, oent=oent, y=y,
                workspace=workspace)
    if y is None:
        y = torch.empty((batch, m), dtype=torch.float16 if y_f16 else torch.float32, device=x.device)
    if workspace is None:
        workspace = new_workspace(m, n, batch, q_max, g, device=x.device)
    flags = (Y_F16 if y_f16 else 0) | (SCALES_PACKED if scales_packed else 0) | _flags
    _check(lib().lutgemm_run_mixed(m, n, batch, q_max, g, _ptr(packed), packed.numel(), _ptr(block_off),
                                   _ptr(alpha), _ptr(optr) if nnz else None, _ptr(oent) if nnz else None, nnz,
                                   _ptr(x), _ptr(y), flags, _ptr(workspace), workspace.numel(), _stream(stream)),
           "lutgemm_run_mixed")
    if check:
        _raise_if_bits(workspace_status(workspace, clear=True, stream=stream), "lutgemm_run_mixed")
    return y
