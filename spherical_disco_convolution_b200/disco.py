"""Thin ctypes binding of libdisco (the C ABI declared in include/disco.h).

Every function here marshals arguments and calls the entry point of the same
name; all arithmetic of the DISCO convolution runs in the library's CUDA
kernels.  Pointers are passed as Python ints (device pointers from
``tensor.data_ptr()``, streams from ``torch.cuda.Stream.cuda_stream``).  The
library must have been built (``python -m spherical_disco_convolution_b200.build``);
if it is missing, importing this module raises: there is no fallback.
"""

from __future__ import annotations

import ctypes
import os
import re

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdisco.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "disco.h")

DISCO_OK = 0
DISCO_ERR_INVALID_ARG = 1
DISCO_ERR_UNSUPPORTED = 2
DISCO_ERR_CUDA = 3
DISCO_ERR_ALLOC = 4
DISCO_ERR_TIMEOUT = 5
DISCO_ERR_GEOMETRY = 6
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "CUDA", 4: "ALLOC", 5: "TIMEOUT", 6: "GEOMETRY"}

DISCO_F32 = 0
DISCO_BF16 = 1
DISCO_GRID_EQUIANGULAR = 0
DISCO_GRID_LEGENDRE_GAUSS = 1
DISCO_GRID_LOBATTO = 2
DISCO_GRID_EQUIANGULAR_TRAPEZOIDAL = 3
GRID_CODES = {"equiangular": DISCO_GRID_EQUIANGULAR, "legendre-gauss": DISCO_GRID_LEGENDRE_GAUSS,
              "lobatto": DISCO_GRID_LOBATTO, "equiangular-trapezoidal": DISCO_GRID_EQUIANGULAR_TRAPEZOIDAL}
DISCO_BASIS_PIECEWISE_LINEAR = 0
DISCO_NORM_NODAL = 0

DISCO_OP_FWD = 0
DISCO_OP_FWD_FUSED = 1
DISCO_OP_BWD_INPUT = 2
DISCO_OP_BWD_WEIGHT = 3
DISCO_OP_BWD_WEIGHT_RECOMPUTE = 4
DISCO_OP_EINSUM_ADJOINT = 5


class DiscoError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"disco status {STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class disco_spec_t(ctypes.Structure):
    _fields_ = [
        ("nlat_in", ctypes.c_int), ("nlon_in", ctypes.c_int),
        ("nlat_out", ctypes.c_int), ("nlon_out", ctypes.c_int),
        ("grid_in", ctypes.c_int), ("grid_out", ctypes.c_int),
        ("kernel_shape", ctypes.c_int * 2),
        ("basis_type", ctypes.c_int), ("basis_norm_mode", ctypes.c_int),
        ("theta_cutoff", ctypes.c_double),
    ]


def make_spec(nlat_in, nlon_in, nlat_out, nlon_out, kernel_shape, theta_cutoff,
              grid_in=DISCO_GRID_EQUIANGULAR, grid_out=DISCO_GRID_EQUIANGULAR,
              basis_type=DISCO_BASIS_PIECEWISE_LINEAR, basis_norm_mode=DISCO_NORM_NODAL) -> disco_spec_t:
    ks = (kernel_shape, 1) if isinstance(kernel_shape, int) else tuple(kernel_shape)
    if len(ks) == 1:
        ks = (ks[0], 1)
    s = disco_spec_t()
    s.nlat_in, s.nlon_in, s.nlat_out, s.nlon_out = nlat_in, nlon_in, nlat_out, nlon_out
    s.grid_in, s.grid_out = grid_in, grid_out
    s.kernel_shape[0], s.kernel_shape[1] = ks
    s.basis_type, s.basis_norm_mode = basis_type, basis_norm_mode
    s.theta_cutoff = float(theta_cutoff)
    return s


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libdisco.so not built at {LIB_PATH}; run python -m spherical_disco_convolution_b200.build")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, LL, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t
    IP = ctypes.POINTER(ctypes.c_int)
    DP = ctypes.POINTER(ctypes.c_double)
    sig = {
        "disco_psi_build": [ctypes.POINTER(disco_spec_t), I, ctypes.POINTER(P)],
        "disco_psi_build_band": [ctypes.POINTER(disco_spec_t), I, I, I, ctypes.POINTER(P), IP, IP],
        "disco_psi_build_inputs": [ctypes.POINTER(disco_spec_t), I, I, I, ctypes.POINTER(P)],
        "disco_psi_destroy": [P],
        "disco_psi_info": [P, IP, ctypes.POINTER(LL)],
        "disco_psi_export": [P, IP, IP, IP, IP, DP],
        "disco_workspace_size": [P, I, I, I, I, I, I, ctypes.POINTER(Z)],
        "disco_contract": [P, I, I, I, P, P, P],
        "disco_einsum": [P, I, I, I, I, I, P, P, P, P, P],
        "disco_fwd": [P, I, I, I, I, I, P, P, P, P, P, P, Z, P],
        "disco_fwd_fused": [P, I, I, I, I, I, P, P, P, P, P, Z, P],
        "disco_bwd_input": [P, I, I, I, I, I, P, P, P, P, Z, P],
        "disco_einsum_adjoint": [P, I, I, I, I, I, P, P, P, P, Z, P],
        "disco_contract_adjoint": [P, I, I, I, P, P, P],
        "disco_bwd_weight": [P, I, I, I, I, I, P, P, P, P, P, P, Z, P],
        "disco_bwd_weight_noalloc": [P, I, I, I, I, I, P, P, P, P, P],
        "disco_mix_workspace_size": [I, I, I, I, I, I, LL, I, ctypes.POINTER(Z)],
        "disco_mix": [I, I, I, I, I, LL, I, P, P, P, P, P],
        "disco_mix_adjoint": [I, I, I, I, I, LL, I, P, P, P, P, Z, P],
        "disco_mix_weight": [I, I, I, I, I, LL, I, P, P, P, P, P, Z, P],
        "disco_plan_info": [P, I, IP],
        "disco_sync_status": [P],
        "disco_wait_selftest": [ctypes.c_uint, P],
        "disco_plan_export": [P, I, IP, IP, IP, ctypes.POINTER(ctypes.c_float), IP],
        "disco_toeplitz_info": [P, I, IP],
        "disco_toeplitz_export": [P, I, IP, IP, ctypes.POINTER(ctypes.c_ushort)],
        "disco_ring_info": [P, I, IP],
        "disco_ring_export": [P, I, IP, IP, IP, IP, ctypes.POINTER(ctypes.c_ushort)],
        "disco_tile_info": [P, I, IP],
        "disco_tile_export": [P, I, IP, IP, IP, ctypes.POINTER(ctypes.c_uint), IP, IP, ctypes.POINTER(ctypes.c_ushort)],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    lib.disco_launch_count.argtypes = []
    lib.disco_launch_count.restype = ctypes.c_ulonglong
    lib.disco_last_error.argtypes = []
    lib.disco_last_error.restype = ctypes.c_char_p
    return lib


_lib = _load()


def header_functions() -> list:
    """Names of every function that include/disco.h declares."""
    text = open(HEADER_PATH).read()
    return sorted(set(re.findall(r"^\s*(?:disco_status|const char\*|unsigned long long)\s+(disco_\w+)\s*\(",
                                 text, re.M)))


def library():
    return _lib


def _check(status: int):
    if status != DISCO_OK:
        raise DiscoError(status, _lib.disco_last_error().decode())


def disco_sync_status(stream) -> None:
    _check(_lib.disco_sync_status(stream))


def disco_wait_selftest(limit_us: int, stream) -> None:
    _check(_lib.disco_wait_selftest(limit_us, stream))


def disco_launch_count() -> int:
    return int(_lib.disco_launch_count())


def disco_last_error() -> str:
    return _lib.disco_last_error().decode()


def disco_psi_build(spec: disco_spec_t, device: int) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check(_lib.disco_psi_build(ctypes.byref(spec), device, ctypes.byref(h)))
    return h


def disco_psi_build_band(spec: disco_spec_t, j_begin: int, j_end: int, device: int):
    """(handle, i_begin, i_end): Psi of output rows [j_begin, j_end) over input rows [i_begin, i_end)."""
    h = ctypes.c_void_p()
    ib, ie = ctypes.c_int(), ctypes.c_int()
    _check(_lib.disco_psi_build_band(ctypes.byref(spec), j_begin, j_end, device, ctypes.byref(h), ctypes.byref(ib),
                                     ctypes.byref(ie)))
    return h, ib.value, ie.value


def disco_psi_build_inputs(spec: disco_spec_t, i_begin: int, i_end: int, device: int):
    """Psi of input rows [i_begin, i_end) (re-indexed from 0) over every output row."""
    h = ctypes.c_void_p()
    _check(_lib.disco_psi_build_inputs(ctypes.byref(spec), i_begin, i_end, device, ctypes.byref(h)))
    return h


def disco_psi_destroy(psi) -> None:
    _check(_lib.disco_psi_destroy(psi))


def disco_psi_info(psi):
    K = ctypes.c_int()
    nnz = ctypes.c_longlong()
    _check(_lib.disco_psi_info(psi, ctypes.byref(K), ctypes.byref(nnz)))
    return K.value, nnz.value


def disco_psi_export(psi):
    """(k, j, i, p, val) host arrays sorted by (j, k, i, p)."""
    _, nnz = disco_psi_info(psi)
    k, j, i, p = (np.empty(nnz, dtype=np.int32) for _ in range(4))
    v = np.empty(nnz, dtype=np.float64)
    ip = lambda a: a.ctypes.data_as(ctypes.POINTER(ctypes.c_int))  # noqa: E731
    _check(_lib.disco_psi_export(psi, ip(k), ip(j), ip(i), ip(p), v.ctypes.data_as(ctypes.POINTER(ctypes.c_double))))
    return k, j, i, p, v


def disco_plan_export(psi, which: int):
    """Plan arrays of the forward (which=0) or adjoint (which=1) gather kernels."""
    dims = np.zeros(9, dtype=np.int32)
    _check(_lib.disco_plan_info(psi, which, dims.ctypes.data_as(ctypes.POINTER(ctypes.c_int))))
    n_rows, n_src, n_chunks, n_vals, nk, step, residues, row_ints, n_rings = (int(v) for v in dims)
    rows = np.zeros((n_rows, row_ints), dtype=np.int32)
    srcs = np.zeros((n_src, 4), dtype=np.int32)
    chunks = np.zeros((n_chunks, 4), dtype=np.int32)
    vals = np.zeros(n_vals, dtype=np.float32)
    rings = np.zeros((max(n_rings, 1), 4), dtype=np.int32)
    ip = lambda a: a.ctypes.data_as(ctypes.POINTER(ctypes.c_int))  # noqa: E731
    _check(_lib.disco_plan_export(psi, which, ip(rows), ip(srcs), ip(chunks),
                                  vals.ctypes.data_as(ctypes.POINTER(ctypes.c_float)), ip(rings)))
    ring_v = rings[:n_rings, 2].copy().view(np.float32)
    return dict(rows=rows, srcs=srcs, chunks=chunks, vals=vals, nk=nk, step=step, residues=residues,
                rings=rings[:n_rings], ring_v=ring_v)


def disco_toeplitz_export(psi, which: int):
    """Toeplitz plan of the tensor-core kernels: which=0 forward, which=1 adjoint."""
    dims = np.zeros(8, dtype=np.int32)
    _check(_lib.disco_toeplitz_info(psi, which, dims.ctypes.data_as(ctypes.POINTER(ctypes.c_int))))
    K, parts, N, n_slabs, n_rows, n_b, kslab, ksteps = (int(v) for v in dims)
    slabs = np.zeros((n_slabs, 4), dtype=np.int32)
    slots = np.zeros((n_rows, 4), dtype=np.int32)
    b = np.zeros(n_b, dtype=np.uint16)
    ip = lambda a: a.ctypes.data_as(ctypes.POINTER(ctypes.c_int))  # noqa: E731
    _check(_lib.disco_toeplitz_export(psi, which, ip(slabs), ip(slots),
                                      b.ctypes.data_as(ctypes.POINTER(ctypes.c_ushort))))
    return dict(K=K, parts=parts, N=N, slabs=slabs, slots=slots, b=b, kslab=kslab, ksteps=ksteps)


RING_DIMS = ("K", "N", "mirror", "nb", "wmax", "ns", "nrb", "bk", "nbs", "src_order", "n_strips", "n_loads",
             "n_items", "n_rows", "n_b", "mmas")


def disco_ring_info(psi, which: int) -> dict:
    """Shape of a ring plan: which = 0/1 forward (mirror rows / plane pairs), 2/3 adjoint."""
    dims = np.zeros(16, dtype=np.int32)
    _check(_lib.disco_ring_info(psi, which, dims.ctypes.data_as(ctypes.POINTER(ctypes.c_int))))
    return dict(zip(RING_DIMS, (int(v) for v in dims)))


TILE_DIMS = ("K", "N", "mirror", "nb", "ns", "nrb", "nbs", "bslot_bytes", "src_order", "n_strips", "n_qt",
             "n_ctas", "n_loads", "n_copies", "n_cmds", "n_rows", "n_b", "mmas", "boxes", "n_cta_ints")


def disco_tile_info(psi, which: int) -> dict:
    """Shape of a tile-script plan: which = 0/1 forward (mirror rows / plane pairs), 2/3 adjoint."""
    dims = np.zeros(20, dtype=np.int32)
    _check(_lib.disco_tile_info(psi, which, dims.ctypes.data_as(ctypes.POINTER(ctypes.c_int))))
    return dict(zip(TILE_DIMS, (int(v) for v in dims)))


def disco_tile_export(psi, which: int) -> dict:
    """Tile-script plan records (see include/disco.h) as NumPy arrays."""
    d = disco_tile_info(psi, which)
    tiles = np.zeros((d["n_strips"] * d["n_qt"], 16), dtype=np.int32)
    loads = np.zeros((d["n_loads"], 4), dtype=np.int32)
    copies = np.zeros((d["n_copies"], 4), dtype=np.int32)
    cmds = np.zeros(max(d["n_cmds"], 1), dtype=np.uint32)
    rows = np.zeros((d["n_rows"], 2), dtype=np.int32)
    cta = np.zeros(d["n_cta_ints"], dtype=np.int32)
    b = np.zeros(max(d["n_b"], 1), dtype=np.uint16)
    ip = lambda a: a.ctypes.data_as(ctypes.POINTER(ctypes.c_int))  # noqa: E731
    _check(_lib.disco_tile_export(psi, which, ip(tiles), ip(loads), ip(copies),
                                  cmds.ctypes.data_as(ctypes.POINTER(ctypes.c_uint)), ip(rows), ip(cta),
                                  b.ctypes.data_as(ctypes.POINTER(ctypes.c_ushort))))
    d.update(tiles=tiles, loads=loads, copies=copies, cmds=cmds[:d["n_cmds"]], rows=rows, cta_tiles=cta,
             b=b[:d["n_b"]])
    return d


def disco_ring_export(psi, which: int) -> dict:
    """Ring plan records (see include/disco.h) as NumPy arrays."""
    d = disco_ring_info(psi, which)
    strips = np.zeros((d["n_strips"], 8), dtype=np.int32)
    loads = np.zeros((d["n_loads"], 2), dtype=np.int32)
    items = np.zeros((d["n_items"], 4), dtype=np.int32)
    rows = np.zeros((d["n_rows"], 2), dtype=np.int32)
    b = np.zeros(max(d["n_b"], 1), dtype=np.uint16)
    ip = lambda a: a.ctypes.data_as(ctypes.POINTER(ctypes.c_int))  # noqa: E731
    _check(_lib.disco_ring_export(psi, which, ip(strips), ip(loads), ip(items), ip(rows),
                                  b.ctypes.data_as(ctypes.POINTER(ctypes.c_ushort))))
    d.update(strips=strips, loads=loads, items=items, rows=rows, b=b[:d["n_b"]])
    return d


def disco_workspace_size(psi, op, B, C_in, C_out, groups, dtype) -> int:
    n = ctypes.c_size_t()
    _check(_lib.disco_workspace_size(psi, op, B, C_in, C_out, groups, dtype, ctypes.byref(n)))
    return n.value


def disco_contract(psi, B, C, dtype, x, y, stream) -> None:
    _check(_lib.disco_contract(psi, B, C, dtype, x, y, stream))


def disco_einsum(psi, B, C_in, C_out, groups, dtype, y, w, bias, out, stream) -> None:
    _check(_lib.disco_einsum(psi, B, C_in, C_out, groups, dtype, y, w, bias, out, stream))


def disco_fwd(psi, B, C_in, C_out, groups, dtype, x, w, bias, y, out, workspace, ws_bytes, stream) -> None:
    _check(_lib.disco_fwd(psi, B, C_in, C_out, groups, dtype, x, w, bias, y, out, workspace, ws_bytes, stream))


def disco_fwd_fused(psi, B, C_in, C_out, groups, dtype, x, w, bias, out, workspace, ws_bytes, stream) -> None:
    _check(_lib.disco_fwd_fused(psi, B, C_in, C_out, groups, dtype, x, w, bias, out, workspace, ws_bytes, stream))


def disco_bwd_input(psi, B, C_in, C_out, groups, dtype, dout, w, dx, workspace, ws_bytes, stream) -> None:
    _check(_lib.disco_bwd_input(psi, B, C_in, C_out, groups, dtype, dout, w, dx, workspace, ws_bytes, stream))


def disco_einsum_adjoint(psi, B, C_in, C_out, groups, dtype, dout, w, dy, workspace, ws_bytes, stream) -> None:
    _check(_lib.disco_einsum_adjoint(psi, B, C_in, C_out, groups, dtype, dout, w, dy, workspace, ws_bytes, stream))


def disco_contract_adjoint(psi, B, C, dtype, dy, dx, stream) -> None:
    _check(_lib.disco_contract_adjoint(psi, B, C, dtype, dy, dx, stream))


def disco_bwd_weight(psi, B, C_in, C_out, groups, dtype, dout, y, x, dw, dbias, workspace, ws_bytes, stream) -> None:
    _check(_lib.disco_bwd_weight(psi, B, C_in, C_out, groups, dtype, dout, y, x, dw, dbias, workspace, ws_bytes,
                                 stream))


def disco_bwd_weight_noalloc(psi, B, C_in, C_out, groups, dtype, dout, y, dw, dbias, stream) -> None:
    _check(_lib.disco_bwd_weight_noalloc(psi, B, C_in, C_out, groups, dtype, dout, y, dw, dbias, stream))


def disco_mix_workspace_size(op, B, C_in, C_out, groups, K, npts, dtype) -> int:
    n = ctypes.c_size_t()
    _check(_lib.disco_mix_workspace_size(op, B, C_in, C_out, groups, K, npts, dtype, ctypes.byref(n)))
    return n.value


def disco_mix(B, C_in, C_out, groups, K, npts, dtype, y, w, bias, out, stream) -> None:
    _check(_lib.disco_mix(B, C_in, C_out, groups, K, npts, dtype, y, w, bias, out, stream))


def disco_mix_adjoint(B, C_in, C_out, groups, K, npts, dtype, dout, w, dy, workspace, ws_bytes, stream) -> None:
    _check(_lib.disco_mix_adjoint(B, C_in, C_out, groups, K, npts, dtype, dout, w, dy, workspace, ws_bytes, stream))


def disco_mix_weight(B, C_in, C_out, groups, K, npts, dtype, dout, y, dw, dbias, workspace, ws_bytes,
                     stream) -> None:
    _check(_lib.disco_mix_weight(B, C_in, C_out, groups, K, npts, dtype, dout, y, dw, dbias, workspace, ws_bytes,
                                 stream))
