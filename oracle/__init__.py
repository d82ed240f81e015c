"""CPU oracle for the spherical DISCO convolution (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path never does; the two
share no code.  The oracle is a plain fp64 C++ program (``disco_oracle.cpp``)
driven through ctypes, plus a NumPy brute force (``brute.py``) that checks it
on tiny grids.

What it computes follows the forward equation and the definition of Psi on
the page "torch_harmonics.DiscreteContinuousConvS2"; the readings taken where
that page is silent are listed at the top of ``disco_oracle.cpp``.  The
absolute Psi values are parity unpinned against the pages (no worked values
are printed there); the test suite pins them by mathematics instead.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "disco_oracle.cpp")
_LIB = os.path.join(_HERE, "_build", "liboracle.so")


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (fp64, OpenMP, no fast-math)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp])
    os.replace(tmp, _LIB)
    return _LIB


class _Spec(ctypes.Structure):
    _fields_ = [
        ("nlat_in", ctypes.c_int), ("nlon_in", ctypes.c_int),
        ("nlat_out", ctypes.c_int), ("nlon_out", ctypes.c_int),
        ("n_r", ctypes.c_int), ("n_alpha", ctypes.c_int),
        ("theta_cutoff", ctypes.c_double),
        ("th_in", ctypes.POINTER(ctypes.c_double)), ("w_in", ctypes.POINTER(ctypes.c_double)),
        ("th_out", ctypes.POINTER(ctypes.c_double)),
    ]


_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        D = ctypes.POINTER(ctypes.c_double)
        I = ctypes.POINTER(ctypes.c_int)
        S = ctypes.POINTER(_Spec)
        lib.orc_num_basis.argtypes = [S]
        lib.orc_cc_weights.argtypes = [ctypes.c_int, D]
        lib.orc_geodesic.argtypes = [ctypes.c_double] * 3 + [D, D]
        lib.orc_basis.argtypes = [S, ctypes.c_int, ctypes.c_double, ctypes.c_double]
        lib.orc_basis.restype = ctypes.c_double
        lib.orc_psi_dense_row.argtypes = [S, ctypes.c_int, D]
        lib.orc_psi_build.argtypes = [S, I]
        lib.orc_psi_build.restype = P
        lib.orc_psi_free.argtypes = [P]
        lib.orc_psi_nnz.argtypes = [P]
        lib.orc_psi_nnz.restype = ctypes.c_longlong
        lib.orc_psi_export.argtypes = [P, I, I, I, I, D]
        lib.orc_contract.argtypes = [P, ctypes.c_int, ctypes.c_int, D, D]
        lib.orc_mix.argtypes = [P] + [ctypes.c_int] * 4 + [D, D, D, D]
        lib.orc_forward.argtypes = [P] + [ctypes.c_int] * 4 + [D, D, D, D, D]
        lib.orc_backward_input.argtypes = [P] + [ctypes.c_int] * 4 + [D, D, D]
        lib.orc_backward_weight.argtypes = [P] + [ctypes.c_int] * 4 + [D, D, D, D]
        lib.orc_contract_dense_samples.argtypes = [S, ctypes.c_int, ctypes.c_int, D, ctypes.c_int] + [I] * 5 + [D]
        lib.orc_num_threads.restype = ctypes.c_int
        lib.orc_set_num_threads.argtypes = [ctypes.c_int]
        lib.orc_set_num_threads.restype = None
        _lib = lib
    return _lib


def _d(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double)) if a is not None else None


def _i(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int))


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


GRIDS = ("equiangular", "legendre-gauss", "lobatto", "equiangular-trapezoidal")
_GRID_CACHE: dict = {}


def latitude_grid(name: str, nlat: int):
    """(theta, w): colatitudes north to south and quadrature weights on t = cos(theta), summing to 2.

    The DISCO constructor takes grid_in / grid_out (page "torch_harmonics.DiscreteContinuousConvS2",
    signature); the four names are listed on the page of the module
    "torch_harmonics.distributed.distributed_spectral_convolution" (class docstring, Parameters).
    Neither page defines them, so each is read as the textbook rule of that name:
      - equiangular: theta_i = pi*i/(nlat-1), poles included, Clenshaw-Curtis weights;
      - legendre-gauss: Gauss-Legendre nodes, here by Golub-Welsch (the eigenvalues of the
        Jacobi matrix of the Legendre recurrence), weights 2 / ((1 - t^2) P_n'(t)^2);
      - lobatto: Gauss-Lobatto-Legendre: t = +-1 and the n-2 roots of P'_{n-1}, which are the
        Gauss nodes of the weight 1 - t^2 (Golub-Welsch on its recurrence), weights
        2 / (m (m+1) P_m(t)^2) with m = n-1;
      - equiangular-trapezoidal: equiangular nodes, the trapezoidal rule in t (the integral of
        the piecewise-linear interpolant in t).
    """
    key = (name, nlat)
    if key in _GRID_CACHE:
        return _GRID_CACHE[key]
    n = nlat
    if n < 2:
        raise ValueError("a latitude grid needs nlat >= 2")
    if name in ("equiangular", "equiangular-trapezoidal"):
        theta = np.pi * np.arange(n) / (n - 1)
        if name == "equiangular":
            w = cc_weights(n)
        else:
            t = np.cos(theta)
            w = np.empty(n)
            for i in range(n):
                w[i] = 0.5 * (t[max(i - 1, 0)] - t[min(i + 1, n - 1)])
    elif name == "legendre-gauss":
        k = np.arange(1, n, dtype=np.float64)
        off = k / np.sqrt(4.0 * k * k - 1.0)
        t = np.sort(np.linalg.eigvalsh(np.diag(off, 1) + np.diag(off, -1)))[::-1]
        dP = np.polynomial.legendre.legval(t, np.polynomial.legendre.legder(np.eye(n + 1)[n]))
        w = 2.0 / ((1.0 - t * t) * dP ** 2)
        theta = np.arccos(np.clip(t, -1.0, 1.0))
    elif name == "lobatto":
        m = n - 1
        if n > 2:
            k = np.arange(1, n - 2, dtype=np.float64)
            off = np.sqrt(k * (k + 2.0) / ((2.0 * k + 1.0) * (2.0 * k + 3.0)))
            inner = np.linalg.eigvalsh(np.diag(off, 1) + np.diag(off, -1)) if n > 3 else np.zeros(1)
        else:
            inner = np.zeros(0)
        t = np.concatenate([[1.0], np.sort(inner)[::-1], [-1.0]])
        Pm = np.polynomial.legendre.legval(t, np.eye(m + 1)[m])
        w = 2.0 / (m * (m + 1.0) * Pm ** 2)
        theta = np.arccos(np.clip(t, -1.0, 1.0))
    else:
        raise ValueError(f"unknown grid {name!r}; one of {GRIDS}")
    out = (np.ascontiguousarray(theta, dtype=np.float64), np.ascontiguousarray(w, dtype=np.float64))
    _GRID_CACHE[key] = out
    return out


@dataclass(frozen=True)
class Spec:
    """Layer geometry: in/out grid shapes, kernel_shape (n_r, n_alpha), theta_cutoff, latitude grids."""

    nlat_in: int
    nlon_in: int
    nlat_out: int
    nlon_out: int
    n_r: int
    n_alpha: int
    theta_cutoff: float
    grid_in: str = "equiangular"
    grid_out: str = "equiangular"

    @property
    def K(self) -> int:
        return self.n_r if self.n_alpha == 1 else 1 + (self.n_r - 1) * self.n_alpha

    @property
    def stride(self) -> int:
        return self.nlon_in // self.nlon_out

    def _c(self):
        # non-equiangular grids pass their arrays (kept alive by the grid cache)
        th_in = w_in = th_out = None
        if self.grid_in != "equiangular":
            th_in, w_in = latitude_grid(self.grid_in, self.nlat_in)
        if self.grid_out != "equiangular":
            th_out = latitude_grid(self.grid_out, self.nlat_out)[0]
        return ctypes.byref(_Spec(self.nlat_in, self.nlon_in, self.nlat_out, self.nlon_out,
                                  self.n_r, self.n_alpha, float(self.theta_cutoff),
                                  _d(th_in), _d(w_in), _d(th_out)))


class OracleError(RuntimeError):
    pass


def num_threads() -> int:
    return _L().orc_num_threads()


def set_num_threads(n: int) -> None:
    """Threads of the oracle's OpenMP loops from now on (for timing it on one core or on all)."""
    _L().orc_set_num_threads(int(n))


def cc_weights(nlat: int) -> np.ndarray:
    """Clenshaw-Curtis weights on cos(theta) at theta_i = pi*i/(nlat-1); they sum to 2."""
    w = np.empty(nlat)
    _L().orc_cc_weights(nlat, _d(w))
    return w


def geodesic(th_out: float, th_in: float, dlam: float):
    """(r, alpha): distance and bearing east of north of (th_in, dlam) seen from (th_out, 0)."""
    r = ctypes.c_double()
    a = ctypes.c_double()
    _L().orc_geodesic(th_out, th_in, dlam, ctypes.byref(r), ctypes.byref(a))
    return r.value, a.value


def basis(spec: Spec, k: int, r: float, alpha: float) -> float:
    return _L().orc_basis(spec._c(), k, r, alpha)


def psi_dense_row(spec: Spec, j: int) -> np.ndarray:
    """Dense normalised Psi row j as an array (K, nlat_in, nlon_in)."""
    out = np.empty((spec.K, spec.nlat_in, spec.nlon_in))
    st = _L().orc_psi_dense_row(spec._c(), j, _d(out))
    if st:
        raise OracleError(f"dense Psi row {j}: status {st}")
    return out


class Psi:
    """Sparse Psi: every input point evaluated, exact zeros dropped."""

    def __init__(self, spec: Spec):
        st = ctypes.c_int(0)
        h = _L().orc_psi_build(spec._c(), ctypes.byref(st))
        if not h:
            raise OracleError(f"Psi build failed with status {st.value}")
        self.spec = spec
        self._h = ctypes.c_void_p(h)

    def __del__(self):
        if getattr(self, "_h", None) and _lib is not None:
            _lib.orc_psi_free(self._h)
            self._h = None

    @property
    def K(self) -> int:
        return self.spec.K

    @property
    def nnz(self) -> int:
        return _L().orc_psi_nnz(self._h)

    def entries(self):
        """(k, j, i, p, val) arrays sorted by (j, k, i, p); p in [0, nlon_in)."""
        n = self.nnz
        k, j, i, p = (np.empty(n, dtype=np.int32) for _ in range(4))
        v = np.empty(n)
        _L().orc_psi_export(self._h, _i(k), _i(j), _i(i), _i(p), _d(v))
        return k, j, i, p, v

    def contract(self, x: np.ndarray) -> np.ndarray:
        """x (B, C, nlat_in, nlon_in) -> y (B, C, K, nlat_out, nlon_out)."""
        x = _f64(x)
        B, C = x.shape[:2]
        s = self.spec
        y = np.empty((B, C, self.K, s.nlat_out, s.nlon_out))
        _L().orc_contract(self._h, B, C, _d(x), _d(y))
        return y

    def forward(self, x, w, bias=None, groups: int = 1, return_y: bool = False):
        """out[b,o,j,q] = sum_{c in group(o), k} w[o,c',k] y[b,c,k,j,q] + bias[o]."""
        x, w = _f64(x), _f64(w)
        bias = _f64(bias) if bias is not None else None
        B, C_in = x.shape[:2]
        C_out = w.shape[0]
        s = self.spec
        out = np.empty((B, C_out, s.nlat_out, s.nlon_out))
        y = np.empty((B, C_in, self.K, s.nlat_out, s.nlon_out)) if return_y else None
        _L().orc_forward(self._h, B, C_in, C_out, groups, _d(x), _d(w), _d(bias), _d(y), _d(out))
        return (out, y) if return_y else out

    def mix(self, y, w, bias=None, groups: int = 1):
        y, w = _f64(y), _f64(w)
        bias = _f64(bias) if bias is not None else None
        B, C_in = y.shape[:2]
        C_out = w.shape[0]
        s = self.spec
        out = np.empty((B, C_out, s.nlat_out, s.nlon_out))
        _L().orc_mix(self._h, B, C_in, C_out, groups, _d(y), _d(w), _d(bias), _d(out))
        return out

    def backward_input(self, dout, w, C_in: int, groups: int = 1):
        dout, w = _f64(dout), _f64(w)
        B, C_out = dout.shape[:2]
        s = self.spec
        dx = np.empty((B, C_in, s.nlat_in, s.nlon_in))
        _L().orc_backward_input(self._h, B, C_in, C_out, groups, _d(dout), _d(w), _d(dx))
        return dx

    def backward_weight(self, dout, x, groups: int = 1):
        """(dw (C_out, C_in/G, K), dbias (C_out,))."""
        dout, x = _f64(dout), _f64(x)
        B, C_out = dout.shape[:2]
        C_in = x.shape[1]
        dw = np.empty((C_out, C_in // groups, self.K))
        db = np.empty(C_out)
        _L().orc_backward_weight(self._h, B, C_in, C_out, groups, _d(dout), _d(x), _d(dw), _d(db))
        return dw, db


def contract_dense_samples(spec: Spec, x: np.ndarray, samples: np.ndarray) -> np.ndarray:
    """y at (b, c, k, j, q) samples, summed densely over every input point."""
    x = _f64(x)
    B, C = x.shape[:2]
    smp = np.ascontiguousarray(np.asarray(samples, dtype=np.int32))
    n = smp.shape[0]
    cols = [np.ascontiguousarray(smp[:, t]) for t in range(5)]
    out = np.empty(n)
    st = _L().orc_contract_dense_samples(spec._c(), B, C, _d(x), n, *[_i(c) for c in cols], _d(out))
    if st:
        raise OracleError(f"dense samples: status {st}")
    return out
