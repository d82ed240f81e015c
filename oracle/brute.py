"""NumPy brute force for tiny grids (test infrastructure).

An independent second route to the DISCO forward map on the page
"torch_harmonics.DiscreteContinuousConvS2" (forward equation and the
definition of Psi): for EVERY output point (theta'_j, lambda'_q), rotate the
sphere so that point sits at the north pole, evaluate the filter basis at
every input point in Cartesian coordinates, weight by the quadrature and
normalise that point's own basis rows.  There is no p-shift, no sparse
structure and no shared code with the C++ oracle; it agrees with the oracle
only if the p-shift reduction, the longitude index map, the bearing
convention and the normalisation are all right.

Readings (the same as the oracle's, taken from the pages' silence): grids
with poles and Clenshaw-Curtis weights by default (the other latitude grids
take the oracle's nodes and weights), bearing east of local north, radial and
azimuthal hats, inclusive cutoff with tie threshold 1e-10, nodal rows that
sum to one.  The Clenshaw-Curtis weights here come from a linear solve of the
exactness conditions on polynomials of degree <= n, not from the closed form.
"""

from __future__ import annotations

import numpy as np

TAU = 1e-10


def cc_weights_vandermonde(nlat: int) -> np.ndarray:
    """Interpolatory quadrature on t_i = cos(pi*i/n), found by solving the
    exactness conditions sum_i w_i T_m(t_i) = int_{-1}^{1} T_m(t) dt for the
    Chebyshev polynomials T_m, m = 0..n (a well-conditioned Vandermonde)."""
    n = nlat - 1
    th = np.pi * np.arange(nlat) / n
    m = np.arange(nlat)
    V = np.cos(m[:, None] * th[None, :])
    rhs = np.zeros(nlat)
    even = m % 2 == 0
    rhs[even] = 2.0 / (1.0 - m[even].astype(np.float64) ** 2)
    return np.linalg.solve(V, rhs)


def _grid(name: str, nlat: int):
    """Nodes and weights of the non-equiangular grids: the oracle's (pinned on their own by the
    tests against closed forms and numpy's Gauss-Legendre rule); this module re-checks what is
    built from them."""
    from . import latitude_grid

    return latitude_grid(name, nlat)


def _unit(theta, lam):
    theta, lam = np.broadcast_arrays(theta, lam)
    return np.stack([np.sin(theta) * np.cos(lam), np.sin(theta) * np.sin(lam), np.cos(theta)], axis=-1)


def _to_pole(theta_o: float, lam_o: float) -> np.ndarray:
    """Rotation matrix taking the point (theta_o, lam_o) to the north pole."""
    cz, sz = np.cos(-lam_o), np.sin(-lam_o)
    Rz = np.array([[cz, -sz, 0.0], [sz, cz, 0.0], [0.0, 0.0, 1.0]])
    cy, sy = np.cos(-theta_o), np.sin(-theta_o)
    Ry = np.array([[cy, 0.0, sy], [0.0, 1.0, 0.0], [-sy, 0.0, cy]])
    return Ry @ Rz


def basis_values(r, alpha, n_r: int, n_alpha: int, theta_c: float) -> np.ndarray:
    """Array (K, ...) of basis values; zero outside the cutoff."""
    d = theta_c / (n_r - 1)
    inside = r <= theta_c + TAU

    def hat(c):
        return np.maximum(0.0, 1.0 - np.abs(r - c) / d)

    if n_alpha == 1:
        vals = [hat(k * d) for k in range(n_r)]
    else:
        h = 2 * np.pi / n_alpha
        vals = [hat(0.0)]
        for kr in range(1, n_r):
            for l in range(n_alpha):
                da = np.angle(np.exp(1j * (alpha - l * h)))
                vals.append(hat(kr * d) * np.maximum(0.0, 1.0 - np.abs(da) / h))
    v = np.stack(vals) * inside
    return np.where(v > TAU, v, 0.0)


def psi_point(spec, j: int, q: int) -> np.ndarray:
    """Normalised basis x quadrature at every input point for output point (j, q):
    array (K, nlat_in, nlon_in) indexed by ABSOLUTE input longitude."""
    grid_in = getattr(spec, "grid_in", "equiangular")
    grid_out = getattr(spec, "grid_out", "equiangular")
    if grid_out == "equiangular":
        th_o = np.pi * j / (spec.nlat_out - 1)
    else:
        th_o = _grid(grid_out, spec.nlat_out)[0][j]
    la_o = 2 * np.pi * q / spec.nlon_out
    if grid_in == "equiangular":
        th = np.pi * np.arange(spec.nlat_in) / (spec.nlat_in - 1)
        qw = cc_weights_vandermonde(spec.nlat_in)
    else:
        th, qw = _grid(grid_in, spec.nlat_in)
    la = 2 * np.pi * np.arange(spec.nlon_in) / spec.nlon_in
    P = _unit(th[:, None], la[None, :]) @ _to_pole(th_o, la_o).T
    r = np.arctan2(np.hypot(P[..., 0], P[..., 1]), P[..., 2])
    # rotated frame: local north of the output point lies along -x, east along +y
    alpha = np.arctan2(P[..., 1], -P[..., 0])
    phi = basis_values(r, alpha, spec.n_r, spec.n_alpha, spec.theta_cutoff)
    phi = phi * (qw * 2 * np.pi / spec.nlon_in)[None, :, None]
    s = phi.sum(axis=(1, 2), keepdims=True)
    assert np.all(s > 0)
    return phi / s


def forward(spec, x, w, bias=None, groups: int = 1):
    """(out, y) by brute force; x (B,C_in,nlat_in,nlon_in), w (C_out, C_in/G, K)."""
    x = np.asarray(x, dtype=np.float64)
    B, C_in = x.shape[:2]
    C_out = w.shape[0]
    K = w.shape[2]
    y = np.zeros((B, C_in, K, spec.nlat_out, spec.nlon_out))
    for j in range(spec.nlat_out):
        for q in range(spec.nlon_out):
            psi = psi_point(spec, j, q)
            y[:, :, :, j, q] = np.einsum("kil,bcil->bck", psi, x)
    cg, og = C_in // groups, C_out // groups
    out = np.zeros((B, C_out, spec.nlat_out, spec.nlon_out))
    for o in range(C_out):
        g = o // og
        out[:, o] = np.einsum("ck,bckjq->bjq", w[o], y[:, g * cg:(g + 1) * cg])
        if bias is not None:
            out[:, o] += bias[o]
    return out, y
