"""Pins for the CPU oracle against mathematics, not against itself.

Every check here follows from the DISCO definition on the page
"torch_harmonics.DiscreteContinuousConvS2" (forward equation, Psi as basis
values at rotated positions times quadrature weights, p-shift symmetry) or
from plain mathematics (exact quadrature, partition of unity, adjoints,
Euler's identity for a linear map), or compares against an independent route
(the NumPy brute force without the p-shift, Cartesian geometry).
"""

import math
import os

import numpy as np
import pytest

import oracle
from oracle import brute
from spherical_disco_convolution_b200.workloads import WORKLOADS, make_inputs

HERE = os.path.dirname(os.path.abspath(__file__))


def spec_of(wl):
    return oracle.Spec(wl.nlat_in, wl.nlon_in, wl.nlat_out, wl.nlon_out, wl.kernel_shape[0],
                       wl.kernel_shape[1], wl.theta_cutoff)


TINY = spec_of(WORKLOADS["tiny"])
ANISO = oracle.Spec(9, 16, 9, 16, 3, 4, 3 * math.pi / 16)
DOWN = oracle.Spec(9, 16, 5, 8, 3, 4, 3 * math.pi / 16)
DOWN_ISO = oracle.Spec(13, 24, 7, 12, 3, 1, 2 * math.pi / 12)
# the other latitude grids of the constructor's grid_in / grid_out
GAUSS = oracle.Spec(10, 16, 8, 16, 3, 1, 3 * math.pi / 16, "legendre-gauss", "legendre-gauss")
LOBATTO_DOWN = oracle.Spec(11, 24, 6, 12, 3, 4, 2 * math.pi / 10, "lobatto", "equiangular-trapezoidal")
TRAP_GAUSS = oracle.Spec(9, 16, 7, 8, 3, 1, 3 * math.pi / 16, "equiangular-trapezoidal", "legendre-gauss")


# ---------------------------------------------------------------- quadrature

def test_cc_weights_golden():
    for line in open(os.path.join(HERE, "golden", "cc_weights.txt")):
        if line.startswith("#") or not line.strip():
            continue
        n, rest = line.split(":")
        nums, den = rest.split("/")
        want = np.array([float(v) for v in nums.split()]) / float(den)
        np.testing.assert_allclose(oracle.cc_weights(int(n) + 1), want, rtol=0, atol=1e-15)


@pytest.mark.parametrize("nlat", [3, 5, 8, 17, 91, 181])
def test_cc_weights_integrate_polynomials_exactly(nlat):
    n = nlat - 1
    w = oracle.cc_weights(nlat)
    t = np.cos(np.pi * np.arange(nlat) / n)
    assert abs(w.sum() - 2.0) < 1e-13
    np.testing.assert_allclose(w, w[::-1], atol=1e-15)
    for m in range(0, min(n, 24) + 1):
        exact = 2.0 / (m + 1) if m % 2 == 0 else 0.0
        assert abs(np.dot(w, t ** m) - exact) < 1e-13, m


@pytest.mark.parametrize("nlat", [5, 9, 17, 33, 721])
def test_cc_weights_match_linear_solve(nlat):
    np.testing.assert_allclose(oracle.cc_weights(nlat), brute.cc_weights_vandermonde(nlat), atol=1e-14)


def _monomial_integral(m: int) -> float:
    return 2.0 / (m + 1) if m % 2 == 0 else 0.0


@pytest.mark.parametrize("nlat", [2, 3, 7, 16, 91, 361, 721])
def test_legendre_gauss_grid_matches_numpy(nlat):
    """Golub-Welsch nodes and their weights against numpy's Gauss-Legendre rule (a library
    routine), ordered north to south."""
    theta, w = oracle.latitude_grid("legendre-gauss", nlat)
    t_np, w_np = np.polynomial.legendre.leggauss(nlat)
    order = np.argsort(-t_np)
    np.testing.assert_allclose(np.cos(theta), t_np[order], rtol=0, atol=1e-13)
    # numpy's own weights drift from the exact ones by up to ~3e-9 relative at 721 points (measured
    # against a Newton solve in 80-bit precision; this grid is closer), hence the tolerance
    np.testing.assert_allclose(w, w_np[order], rtol=1e-8, atol=0)


def test_lobatto_grid_closed_forms():
    """Gauss-Lobatto-Legendre rules with 3, 4 and 5 points, from their textbook closed forms."""
    cases = {
        3: ([1.0, 0.0, -1.0], [1 / 3, 4 / 3, 1 / 3]),
        4: ([1.0, 1 / math.sqrt(5), -1 / math.sqrt(5), -1.0], [1 / 6, 5 / 6, 5 / 6, 1 / 6]),
        5: ([1.0, math.sqrt(3 / 7), 0.0, -math.sqrt(3 / 7), -1.0], [1 / 10, 49 / 90, 32 / 45, 49 / 90, 1 / 10]),
    }
    for n, (t, w) in cases.items():
        theta, wq = oracle.latitude_grid("lobatto", n)
        np.testing.assert_allclose(np.cos(theta), t, rtol=0, atol=1e-15)
        np.testing.assert_allclose(wq, w, rtol=0, atol=1e-15)


def test_trapezoidal_grid_closed_forms():
    """Equiangular nodes with trapezoidal weights in cos(theta): 3 and 4 points by hand."""
    theta, w = oracle.latitude_grid("equiangular-trapezoidal", 3)
    np.testing.assert_allclose(theta, [0.0, math.pi / 2, math.pi], atol=0)
    np.testing.assert_allclose(w, [0.5, 1.0, 0.5], atol=1e-16)
    theta, w = oracle.latitude_grid("equiangular-trapezoidal", 4)
    np.testing.assert_allclose(w, [0.25, 0.75, 0.75, 0.25], atol=1e-15)


# degree up to which each rule integrates polynomials in t exactly
_EXACT = {"equiangular": lambda n: n - 1, "legendre-gauss": lambda n: 2 * n - 1,
          "lobatto": lambda n: 2 * n - 3, "equiangular-trapezoidal": lambda n: 1}


@pytest.mark.parametrize("grid", oracle.GRIDS)
@pytest.mark.parametrize("nlat", [2, 3, 6, 17, 64])
def test_latitude_grids_are_quadrature_rules(grid, nlat):
    """Every grid: colatitudes rise from north to south inside [0, pi], mirror-symmetric about the
    equator, positive weights summing to 2, exact on the polynomials its rule is exact for, and
    (a degree beyond that) not exact, so the exactness check has teeth."""
    theta, w = oracle.latitude_grid(grid, nlat)
    assert theta.shape == w.shape == (nlat,)
    assert np.all(np.diff(theta) > 0) and theta[0] >= 0 and theta[-1] <= math.pi
    np.testing.assert_allclose(theta + theta[::-1], math.pi, atol=1e-13)
    np.testing.assert_allclose(w, w[::-1], rtol=1e-12, atol=0)
    assert np.all(w > 0)
    t = np.cos(theta)
    deg = min(_EXACT[grid](nlat), 40)
    for m in range(deg + 1):
        assert abs(np.dot(w, t ** m) - _monomial_integral(m)) < 1e-12, (grid, nlat, m)
    if _EXACT[grid](nlat) < 40:
        m = _EXACT[grid](nlat) + 1
        m += m % 2  # odd monomials vanish by symmetry for every rule
        assert abs(np.dot(w, t ** m) - _monomial_integral(m)) > 1e-11, (grid, nlat, m)


def test_trapezoidal_grid_converges_at_second_order():
    errs = []
    for n in (33, 65, 129):
        theta, w = oracle.latitude_grid("equiangular-trapezoidal", n)
        errs.append(abs(np.dot(w, np.exp(np.cos(theta))) - (math.e - 1 / math.e)))
    assert 3.5 < errs[0] / errs[1] < 4.5 and 3.5 < errs[1] / errs[2] < 4.5


def test_equiangular_grid_is_the_default():
    theta, w = oracle.latitude_grid("equiangular", 9)
    np.testing.assert_array_equal(w, oracle.cc_weights(9))
    np.testing.assert_allclose(theta, np.pi * np.arange(9) / 8, atol=0)
    a = oracle.Psi(oracle.Spec(9, 16, 9, 16, 3, 1, 3 * math.pi / 16)).entries()
    b = oracle.Psi(oracle.Spec(9, 16, 9, 16, 3, 1, 3 * math.pi / 16, "equiangular", "equiangular")).entries()
    for u, v in zip(a, b):
        np.testing.assert_array_equal(u, v)


# ------------------------------------------------------------------ geometry

def _cartesian(theta, lam):
    return np.array([np.sin(theta) * np.cos(lam), np.sin(theta) * np.sin(lam), np.cos(theta)])


def test_geodesic_special_cases():
    for th_o, th_i in [(0.3, 0.5), (1.2, 0.4), (math.pi / 2, math.pi / 2 + 0.01)]:
        r, a = oracle.geodesic(th_o, th_i, 0.0)
        assert abs(r - abs(th_i - th_o)) < 1e-14
        # same meridian: due north (alpha = 0) when the input is nearer the north pole
        assert abs(a - (0.0 if th_i < th_o else math.pi)) < 1e-12 or abs(abs(a) - math.pi) < 1e-12
        r, a = oracle.geodesic(th_o, th_i, math.pi)
        assert abs(r - min(th_i + th_o, 2 * math.pi - th_i - th_o)) < 1e-14
    # on the equator, a point slightly east lies due east
    r, a = oracle.geodesic(math.pi / 2, math.pi / 2, 0.01)
    assert abs(r - 0.01) < 1e-14 and abs(a - math.pi / 2) < 1e-12


def test_geodesic_matches_cartesian_route():
    rng = np.random.default_rng(1)
    for _ in range(200):
        th_o, th_i = rng.uniform(0.05, math.pi - 0.05, 2)
        dl = rng.uniform(-math.pi, math.pi)
        r, a = oracle.geodesic(th_o, th_i, dl)
        P, Q = _cartesian(th_o, 0.0), _cartesian(th_i, dl)
        r_ref = math.atan2(np.linalg.norm(np.cross(P, Q)), np.dot(P, Q))
        north = np.array([-math.cos(th_o), 0.0, math.sin(th_o)])  # tangent toward the north pole
        east = np.array([0.0, 1.0, 0.0])
        t = Q - np.dot(P, Q) * P
        a_ref = math.atan2(np.dot(t, east), np.dot(t, north))
        assert abs(r - r_ref) < 1e-13
        assert abs(math.remainder(a - a_ref, 2 * math.pi)) < 1e-10


# --------------------------------------------------------------------- basis

def test_basis_partition_of_unity():
    iso = oracle.Spec(9, 16, 9, 16, 3, 1, 0.4)
    an = oracle.Spec(9, 16, 9, 16, 3, 4, 0.4)
    for r in np.linspace(0, 0.4, 41):
        assert abs(sum(oracle.basis(iso, k, r, 0.0) for k in range(3)) - 1.0) < 1e-14
        for alpha in np.linspace(-math.pi, math.pi, 13):
            vals = [oracle.basis(an, k, r, alpha) for k in range(an.K)]
            assert abs(sum(vals) - 1.0) < 1e-14
            # azimuthal hats of one radial ring add up to that ring's radial hat
            for kr in (1, 2):
                ring = sum(vals[1 + (kr - 1) * 4: 1 + kr * 4])
                assert abs(ring - oracle.basis(iso, kr, r, 0.0)) < 1e-14
    assert oracle.basis(iso, 2, 0.4 + 1e-6, 0.0) == 0.0


# ----------------------------------------------------------------------- Psi

@pytest.mark.parametrize("spec", [TINY, ANISO, DOWN, DOWN_ISO, GAUSS, LOBATTO_DOWN],
                         ids=["tiny", "aniso", "down", "down_iso", "gauss", "lobatto_down"])
def test_psi_rows_sum_to_one_and_sparse_matches_dense(spec):
    P = oracle.Psi(spec)
    k, j, i, p, v = P.entries()
    assert np.all(v > 0)
    sums = np.zeros((spec.K, spec.nlat_out))
    np.add.at(sums, (k, j), v)
    np.testing.assert_allclose(sums, 1.0, atol=1e-13)
    for jj in range(spec.nlat_out):
        dense = oracle.psi_dense_row(spec, jj)
        sel = j == jj
        rebuilt = np.zeros_like(dense)
        rebuilt[k[sel], i[sel], p[sel]] = v[sel]
        assert np.array_equal(rebuilt, dense)


@pytest.mark.parametrize("spec", [TINY, ANISO, DOWN, DOWN_ISO, GAUSS, LOBATTO_DOWN, TRAP_GAUSS],
                         ids=["tiny", "aniso", "down", "down_iso", "gauss", "lobatto_down", "trap_gauss"])
def test_forward_matches_brute_force_without_p_shift(spec):
    rng = np.random.default_rng(0)
    G, C_in, C_out = 2, 4, 6
    x = rng.standard_normal((2, C_in, spec.nlat_in, spec.nlon_in))
    w = rng.standard_normal((C_out, C_in // G, spec.K))
    b = rng.standard_normal(C_out)
    out, y = oracle.Psi(spec).forward(x, w, b, groups=G, return_y=True)
    out_b, y_b = brute.forward(spec, x, w, b, groups=G)
    np.testing.assert_allclose(y, y_b, rtol=0, atol=1e-12)
    np.testing.assert_allclose(out, out_b, rtol=0, atol=1e-12)
    # the oracle's weight einsum on its own, from the brute force's y: the group index, the
    # (c, k) pairing and the bias are fixed by the brute force's independent einsum
    np.testing.assert_allclose(oracle.Psi(spec).mix(y_b, w, b, groups=G), out_b, rtol=0, atol=1e-12)


def test_constant_field_and_impulse_response():
    for spec in (TINY, DOWN):
        P = oracle.Psi(spec)
        y = P.contract(np.ones((1, 1, spec.nlat_in, spec.nlon_in)))
        np.testing.assert_allclose(y, 1.0, atol=1e-13)
        w = np.random.default_rng(2).standard_normal((3, 1, spec.K))
        b = np.array([0.1, -0.2, 0.3])
        out = P.forward(np.ones((1, 1, spec.nlat_in, spec.nlon_in)), w, b)
        np.testing.assert_allclose(out, (b + w.sum(axis=(1, 2)))[None, :, None, None] + 0 * out, atol=1e-12)
        # impulse at (i0, l0): y[k, j, q] = Psi[k, j, (i0, (l0 - q*s) mod nlon_in)], zero beyond the cutoff
        i0, l0 = spec.nlat_in // 3, 5
        x = np.zeros((1, 1, spec.nlat_in, spec.nlon_in))
        x[0, 0, i0, l0] = 1.0
        y = P.contract(x)[0, 0]
        k, j, i, p, v = P.entries()
        want = np.zeros_like(y)
        s = spec.stride
        for q in range(spec.nlon_out):
            sel = (i == i0) & (p == (l0 - q * s) % spec.nlon_in)
            want[k[sel], j[sel], q] = v[sel]
        assert np.array_equal(y, want)
        th_o = np.pi * np.arange(spec.nlat_out) / (spec.nlat_out - 1)
        for jj in range(spec.nlat_out):
            for q in range(spec.nlon_out):
                r, _ = oracle.geodesic(th_o[jj], np.pi * i0 / (spec.nlat_in - 1),
                                       2 * np.pi * ((l0 - q * s) % spec.nlon_in) / spec.nlon_in)
                if r > spec.theta_cutoff + 1e-9:
                    assert not np.any(y[:, jj, q])


def test_roll_equivariance_is_exact():
    for spec in (TINY, ANISO, DOWN):
        P = oracle.Psi(spec)
        rng = np.random.default_rng(3)
        x = rng.standard_normal((1, 2, spec.nlat_in, spec.nlon_in))
        w = rng.standard_normal((2, 2, spec.K))
        out = P.forward(x, w)
        for m in (1, 3):
            out_r = P.forward(np.roll(x, spec.stride * m, axis=-1), w)
            assert np.array_equal(out_r, np.roll(out, m, axis=-1))


def test_pole_and_equator_symmetries():
    P = oracle.Psi(TINY)
    x = np.random.default_rng(4).standard_normal((1, 2, TINY.nlat_in, TINY.nlon_in))
    y = P.contract(x)
    for jj in (0, TINY.nlat_out - 1):
        np.testing.assert_allclose(y[..., jj, :], y[..., jj, :1] + 0 * y[..., jj, :], rtol=1e-12, atol=1e-12)
    n = TINY.nlat_out - 1
    for jj in range(TINY.nlat_out):
        a = oracle.psi_dense_row(TINY, jj)
        b = oracle.psi_dense_row(TINY, n - jj)[:, ::-1, :]
        np.testing.assert_allclose(a, b, atol=1e-13)


def test_linearity():
    P = oracle.Psi(ANISO)
    rng = np.random.default_rng(5)
    x1, x2 = rng.standard_normal((2, 1, 3, ANISO.nlat_in, ANISO.nlon_in))
    w = rng.standard_normal((2, 3, ANISO.K))
    lhs = P.forward(2.5 * x1 - 0.75 * x2, w)
    rhs = 2.5 * P.forward(x1, w) - 0.75 * P.forward(x2, w)
    np.testing.assert_allclose(lhs, rhs, rtol=0, atol=1e-12 * np.abs(rhs).max())


# ------------------------------------------------------------------ backward

@pytest.mark.parametrize("spec", [TINY, ANISO, DOWN, DOWN_ISO], ids=["tiny", "aniso", "down", "down_iso"])
def test_backward_input_is_the_adjoint(spec):
    P = oracle.Psi(spec)
    rng = np.random.default_rng(6)
    G, C_in, C_out = 2, 4, 6
    x = rng.standard_normal((2, C_in, spec.nlat_in, spec.nlon_in))
    w = rng.standard_normal((C_out, C_in // G, spec.K))
    dout = rng.standard_normal((2, C_out, spec.nlat_out, spec.nlon_out))
    lhs = np.vdot(dout, P.forward(x, w, groups=G))
    rhs = np.vdot(P.backward_input(dout, w, C_in, groups=G), x)
    assert abs(lhs - rhs) < 1e-12 * max(1.0, abs(lhs))


@pytest.mark.parametrize("spec", [TINY, DOWN], ids=["tiny", "down"])
def test_backward_weight_euler_and_finite_difference(spec):
    P = oracle.Psi(spec)
    rng = np.random.default_rng(7)
    G, C_in, C_out = 2, 4, 6
    x = rng.standard_normal((2, C_in, spec.nlat_in, spec.nlon_in))
    w = rng.standard_normal((C_out, C_in // G, spec.K))
    b = rng.standard_normal(C_out)
    dout = rng.standard_normal((2, C_out, spec.nlat_out, spec.nlon_out))
    dw, db = P.backward_weight(dout, x, groups=G)
    out = P.forward(x, w, b, groups=G)
    # out is linear in w: <dw, w> = <dout, out - bias>
    lhs = np.vdot(dw, w)
    rhs = np.vdot(dout, out - b[None, :, None, None])
    assert abs(lhs - rhs) < 1e-11 * max(1.0, abs(rhs))
    np.testing.assert_allclose(db, dout.sum(axis=(0, 2, 3)), atol=1e-11)
    # directional derivative of L(w) = <dout, out(w)> along a random direction
    v = rng.standard_normal(w.shape)
    eps = 1e-3
    fd = (np.vdot(dout, P.forward(x, w + eps * v, b, groups=G))
          - np.vdot(dout, P.forward(x, w - eps * v, b, groups=G))) / (2 * eps)
    assert abs(fd - np.vdot(dw, v)) < 1e-8 * max(1.0, abs(fd))


# ------------------------------------------------------ samples, ties, sizes

def test_dense_samples_match_sparse_contraction():
    for spec in (TINY, DOWN):
        rng = np.random.default_rng(8)
        x = rng.standard_normal((2, 3, spec.nlat_in, spec.nlon_in))
        y = oracle.Psi(spec).contract(x)
        smp = np.stack([rng.integers(0, 2, 50), rng.integers(0, 3, 50), rng.integers(0, spec.K, 50),
                        rng.integers(0, spec.nlat_out, 50), rng.integers(0, spec.nlon_out, 50)], axis=1)
        got = oracle.contract_dense_samples(spec, x, smp)
        np.testing.assert_allclose(got, y[tuple(smp.T)], atol=1e-13)


@pytest.mark.slow
@pytest.mark.parametrize("name", ["downsample", "weather", "grouped"])
def test_dense_samples_match_sparse_contraction_at_full_size(name):
    # the sparse Psi of a full-size layer against the dense quadrature sum over every input point,
    # on 16 output rows: both poles, the two rows next to each pole, the equator and random rows
    spec = spec_of(WORKLOADS[name])
    rng = np.random.default_rng(11)
    x = rng.standard_normal((1, 2, spec.nlat_in, spec.nlon_in))
    y = oracle.Psi(spec).contract(x)
    n = spec.nlat_out
    rows = [0, 1, 2, n - 3, n - 2, n - 1, n // 2]
    rows += [int(r) for r in rng.choice(np.setdiff1d(np.arange(n), rows), 16 - len(rows), replace=False)]
    m = len(rows) * 3
    smp = np.stack([np.zeros(m, int), rng.integers(0, 2, m), rng.integers(0, spec.K, m),
                    np.repeat(rows, 3), rng.integers(0, spec.nlon_out, m)], axis=1)
    got = oracle.contract_dense_samples(spec, x, smp)
    np.testing.assert_allclose(got, y[tuple(smp.T)], rtol=0, atol=1e-12)


def test_near_tie_cutoff_is_rejected():
    # a cutoff 5e-11 above a grid distance puts computed r - theta_c inside the gap band
    spec = oracle.Spec(17, 32, 17, 32, 3, 1, 2 * math.pi / 16 - 5e-11)
    with pytest.raises(oracle.OracleError):
        oracle.Psi(spec)


def test_invalid_specs_are_rejected():
    with pytest.raises(oracle.OracleError):
        oracle.Psi(oracle.Spec(17, 32, 17, 24, 3, 1, 0.3))  # nlon_in not a multiple of nlon_out
    with pytest.raises(oracle.OracleError):
        oracle.Psi(oracle.Spec(17, 32, 17, 32, 3, 1, 0.0))


@pytest.mark.slow
@pytest.mark.parametrize("name,nnz", [("tiny", 899), ("mid", 7381), ("downsample", 119747),
                                      ("weather", 79931), ("grouped", 147425)])
def test_full_size_psi_builds(name, nnz):
    P = oracle.Psi(spec_of(WORKLOADS[name]))
    assert P.nnz == nnz
    k, j, i, p, v = P.entries()
    sums = np.zeros((P.K, P.spec.nlat_out))
    np.add.at(sums, (k, j), v)
    np.testing.assert_allclose(sums, 1.0, atol=1e-12)


def test_workload_inputs_are_seeded_and_rounded():
    wl = WORKLOADS["tiny"]
    a, b = make_inputs(wl, 0), make_inputs(wl, 0)
    for key in ("x", "w", "bias", "dout"):
        assert np.array_equal(a[key], b[key])
    wl16 = wl.scaled(dtype="bf16")
    x16 = make_inputs(wl16, 0)["x"]
    assert np.all((x16.view(np.uint32) & 0xFFFF) == 0)
