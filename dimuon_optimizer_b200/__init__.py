"""Python binding of libdimuon.so (the B200 Muon / Dimuon optimizer step).

Argument marshalling only: every step of the method runs in the CUDA kernels
of the shared library.  The names mirror the C ABI in include/dimuon.h.
PyTorch supplies device memory and streams.

    import torch, dimuon_optimizer_b200 as dm
    mats = [dm.dm_matrix(W, G, M)]                      # torch CUDA tensors
    hp = dm.dm_default_hparams()
    ws = torch.empty(dm.dm_workspace_size(mats, hp, 0), dtype=torch.uint8,
                     device="cuda")
    dm.check(dm.dm_muon_step(mats, hp, ws))

The shared library must have been built (python dimuon_optimizer_b200/build.py,
or __graft_entry__.build()); importing fails loudly otherwise.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import c_float, c_int, c_int32, c_int64, c_size_t, c_uint32, c_void_p

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdimuon.so")

DM_OK = 0
DM_ERR_INVALID_ARG = 1
DM_ERR_UNSUPPORTED = 2
DM_ERR_WORKSPACE = 3
DM_ERR_CUDA = 4
DM_ERR_DEVICE_TIMEOUT = 5
DM_ERR_NONFINITE = 6
DM_ERR_CANARY = 7

DM_BF16 = 0
DM_FP32 = 1
DM_PREC_FP32 = 0
DM_PREC_BF16_TC = 1
DM_SCALE_NONE = 0
DM_SCALE_MOONSHOT = 1
DM_SCALE_JORDAN = 2
DM_SCALE_BERNSTEIN = 3
DM_THIN_MAX = 32
DM_MAX_NS_STEPS = 64
DM_DBG_NO_THIN = 0x1
DM_DBG_TC_SINGLE = 0x2
DM_DBG_TC_PAIR = 0x4
DM_DBG_FORCE_TIMEOUT = 0x8
DM_DBG_THIN_REGS = 0x10
DM_DBG_THIN_STAGED = 0x20
DM_DBG_CANARY = 0x40
DM_DBG_THIN_CLUSTER = 0x80
DM_DBG_CANARY_SELFTEST = 0x100

DM_NOALLOC_MAX_BYTES = 32 * 1024 * 1024

EXPORTED = ("dm_default_hparams", "dm_workspace_size", "dm_step_launches", "dm_muon_step",
            "dm_dimuon_step", "dm_read_device_status", "dm_step_noalloc", "dm_status_string",
            "dm_version")


class dm_matrix_t(ctypes.Structure):
    _fields_ = [("rows", c_int64), ("cols", c_int64), ("weight", c_void_p),
                ("weight_dtype", c_int32), ("grad_dtype", c_int32), ("grad", c_void_p),
                ("momentum", c_void_p), ("momentum_dtype", c_int32), ("reserved0", c_int32),
                ("row_energy", c_void_p), ("col_energy", c_void_p), ("update_out", c_void_p)]


class dm_hparams_t(ctypes.Structure):
    _fields_ = [("mu", c_float), ("lr", c_float), ("weight_decay", c_float),
                ("ns_steps", c_int32), ("a", c_float), ("b", c_float), ("c", c_float),
                ("cond_eps", c_float), ("scale_mode", c_int32), ("scale_coef", c_float),
                ("precision", c_int32), ("debug_flags", c_uint32), ("nesterov", c_int32),
                ("reserved", c_int32 * 3), ("ns_coeffs", ctypes.POINTER(c_float))]


class DimuonError(RuntimeError):
    def __init__(self, code):
        super().__init__(f"libdimuon status {code}: {dm_status_string(code)}")
        self.code = code


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python dimuon_optimizer_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER
    lib.dm_default_hparams.argtypes = [P(dm_hparams_t)]
    lib.dm_default_hparams.restype = None
    lib.dm_workspace_size.argtypes = [P(dm_matrix_t), c_int, P(dm_hparams_t), c_int,
                                      P(c_size_t)]
    lib.dm_workspace_size.restype = c_int
    lib.dm_step_launches.argtypes = [P(dm_matrix_t), c_int, P(dm_hparams_t), c_int,
                                     P(c_int64)]
    lib.dm_step_launches.restype = c_int
    for name in ("dm_muon_step", "dm_dimuon_step"):
        fn = getattr(lib, name)
        fn.argtypes = [P(dm_matrix_t), c_int, P(dm_hparams_t), c_void_p, c_size_t, c_void_p]
        fn.restype = c_int
    lib.dm_step_noalloc.argtypes = [P(dm_matrix_t), c_int, P(dm_hparams_t), c_int, c_void_p,
                                    c_void_p]
    lib.dm_step_noalloc.restype = c_int
    lib.dm_read_device_status.argtypes = [c_void_p, c_void_p, P(c_int32)]
    lib.dm_read_device_status.restype = c_int
    lib.dm_status_string.argtypes = [c_int32]
    lib.dm_status_string.restype = ctypes.c_char_p
    lib.dm_version.argtypes = []
    lib.dm_version.restype = ctypes.c_char_p
    return lib


_lib = _load()


# ----------------------------------------------------------------------------
# marshalling helpers
# ----------------------------------------------------------------------------
def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return DM_BF16
    if t.dtype == torch.float32:
        return DM_FP32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _ptr(t):
    return None if t is None else c_void_p(t.data_ptr())


def dm_matrix(weight, grad, momentum, row_energy=None, col_energy=None, update_out=None):
    """A dm_matrix_t over torch CUDA tensors (row-major, contiguous)."""
    rows, cols = weight.shape
    for t in (weight, grad, momentum):
        if t.shape != (rows, cols) or not t.is_contiguous():
            raise ValueError("weight, grad and momentum must be contiguous rows x cols")
    for t, n in ((row_energy, rows), (col_energy, cols)):
        if t is not None and (t.numel() != n or t.dtype.itemsize != 4 or not t.is_contiguous()):
            raise ValueError("energies must be contiguous fp32 vectors of rows / cols")
    if update_out is not None and (update_out.shape != (rows, cols)
                                   or not update_out.is_contiguous()):
        raise ValueError("update_out must be a contiguous fp32 rows x cols tensor")
    m = dm_matrix_t()
    m.rows, m.cols = rows, cols
    m.weight, m.weight_dtype = weight.data_ptr(), _dtype_code(weight)
    m.grad, m.grad_dtype = grad.data_ptr(), _dtype_code(grad)
    m.momentum, m.momentum_dtype = momentum.data_ptr(), _dtype_code(momentum)
    m.row_energy = None if row_energy is None else row_energy.data_ptr()
    m.col_energy = None if col_energy is None else col_energy.data_ptr()
    m.update_out = None if update_out is None else update_out.data_ptr()
    return m


def _array(mats):
    if isinstance(mats, ctypes.Array):
        return mats, len(mats)
    mats = list(mats)
    arr = (dm_matrix_t * max(1, len(mats)))(*mats)
    return arr, len(mats)


def _stream_handle(stream):
    if stream is None:
        import torch
        return c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return c_void_p(stream)
    return c_void_p(stream.cuda_stream)


def _ws(workspace):
    if hasattr(workspace, "data_ptr"):
        return c_void_p(workspace.data_ptr()), workspace.numel() * workspace.element_size()
    ptr, nbytes = workspace
    return c_void_p(ptr), nbytes


# ----------------------------------------------------------------------------
# the C ABI, by name
# ----------------------------------------------------------------------------
def dm_default_hparams(**overrides):
    """dm_hparams_t with the library's defaults and the given fields set.
    `ns_coeffs` takes a sequence of (a_k, b_k, c_k) triples, one per
    Newton-Schulz iteration (it also sets ns_steps to its length)."""
    hp = dm_hparams_t()
    _lib.dm_default_hparams(ctypes.byref(hp))
    coeffs = overrides.pop("ns_coeffs", None)
    for k, v in overrides.items():
        setattr(hp, k, v)
    if coeffs is not None:
        set_ns_coeffs(hp, coeffs)
    return hp


def set_ns_coeffs(hp, coeffs):
    """Points hp.ns_coeffs at a host float array holding the triples (kept
    alive on the struct) and sets hp.ns_steps to their count; None restores
    the fixed (a, b, c)."""
    if coeffs is None:
        hp.ns_coeffs = None
        hp._ns_coeffs_keep = None
        return hp
    flat = [float(v) for triple in coeffs for v in triple]
    if len(flat) == 0 or len(flat) % 3:
        raise ValueError("ns_coeffs must be a non-empty sequence of (a, b, c) triples")
    arr = (c_float * len(flat))(*flat)
    hp._ns_coeffs_keep = arr
    hp.ns_coeffs = ctypes.cast(arr, ctypes.POINTER(c_float))
    hp.ns_steps = len(flat) // 3
    return hp


def dm_workspace_size(mats, hp, conditioned):
    arr, n = _array(mats)
    out = c_size_t(0)
    st = _lib.dm_workspace_size(arr, n, ctypes.byref(hp), int(conditioned), ctypes.byref(out))
    if st != DM_OK:
        raise DimuonError(st)
    return out.value


def dm_step_launches(mats, hp, conditioned):
    """Kernel launches one step enqueues (host-only query)."""
    arr, n = _array(mats)
    out = c_int64(0)
    st = _lib.dm_step_launches(arr, n, ctypes.byref(hp), int(conditioned), ctypes.byref(out))
    if st != DM_OK:
        raise DimuonError(st)
    return out.value


def dm_muon_step(mats, hp, workspace, stream=None):
    arr, n = _array(mats)
    ptr, nbytes = _ws(workspace)
    return _lib.dm_muon_step(arr, n, ctypes.byref(hp), ptr, nbytes, _stream_handle(stream))


def dm_dimuon_step(mats, hp, workspace, stream=None):
    arr, n = _array(mats)
    ptr, nbytes = _ws(workspace)
    return _lib.dm_dimuon_step(arr, n, ctypes.byref(hp), ptr, nbytes, _stream_handle(stream))


def dm_step_noalloc(mats, hp, conditioned, device_status_out=None, stream=None):
    """The step with the library's own fixed scratch array instead of a
    workspace (for callers that cannot allocate device memory); see
    include/dimuon.h.  device_status_out: optional int32 CUDA tensor."""
    arr, n = _array(mats)
    return _lib.dm_step_noalloc(arr, n, ctypes.byref(hp), int(conditioned),
                                _ptr(device_status_out), _stream_handle(stream))


def dm_read_device_status(workspace, stream=None):
    ptr, _ = _ws(workspace)
    out = c_int32(0)
    st = _lib.dm_read_device_status(ptr, _stream_handle(stream), ctypes.byref(out))
    if st != DM_OK:
        raise DimuonError(st)
    return out.value


def dm_status_string(code):
    return _lib.dm_status_string(int(code)).decode()


def dm_version():
    return _lib.dm_version().decode()


def check(status):
    """Raises DimuonError for a non-zero status."""
    if status != DM_OK:
        raise DimuonError(status)
    return status


def vector_matrix_shape(length, width):
    """Shape (rows, width) of the matrix a 1-D parameter of `length`
    variables is laid out in ("From PCG to Muon", section 6 "Muon
    Reshaping"): the variables in order, row-major, the cells past the end
    zero.  Give the library the padded matrices with zero gradient in the
    padding: the padded momentum cells then stay zero, and the padded weight
    cells (which the update does write) are simply not read back."""
    length, width = int(length), int(width)
    if length < 1 or width < 1:
        raise ValueError("length and width must be positive")
    return (-(-length // width), width)
