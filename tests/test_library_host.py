"""Host-side checks of libdisco (no GPU): symbols, Psi builder vs oracle, plans, status codes."""

import ctypes
import math
import subprocess

import numpy as np
import pytest

import oracle
from spherical_disco_convolution_b200 import disco as D
from spherical_disco_convolution_b200.workloads import WORKLOADS, make_inputs
from tests import plan_emulator


def spec_pair(wl):
    s = D.make_spec(wl.nlat_in, wl.nlon_in, wl.nlat_out, wl.nlon_out, wl.kernel_shape, wl.theta_cutoff)
    o = oracle.Spec(wl.nlat_in, wl.nlon_in, wl.nlat_out, wl.nlon_out, wl.kernel_shape[0], wl.kernel_shape[1],
                    wl.theta_cutoff)
    return s, o


def test_library_exports_every_declared_symbol():
    names = D.header_functions()
    assert len(names) >= 10
    out = subprocess.run(["nm", "-D", "--defined-only", D.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in names:
        assert n in exported, n
        assert getattr(D.library(), n) is not None


QUICK = ["tiny", "mid", "downsample"]


@pytest.mark.parametrize("name", QUICK + [pytest.param(n, marks=pytest.mark.slow) for n in ("weather", "grouped")])
def test_psi_export_matches_oracle(name):
    s, o = spec_pair(WORKLOADS[name])
    h = D.disco_psi_build(s, -1)
    try:
        k, j, i, p, v = D.disco_psi_export(h)
    finally:
        D.disco_psi_destroy(h)
    ko, jo, io, po, vo = oracle.Psi(o).entries()
    # same non-zero pattern, bit for bit, in the same (j, k, i, p) order
    assert np.array_equal(k, ko) and np.array_equal(j, jo) and np.array_equal(i, io) and np.array_equal(p, po)
    # values: the two distance routes differ by rounding (~1e-17 rad); a small phi near a hat end
    # point turns that into an absolute error of ~1e-16/width, so the bound is 1e-12 relative plus
    # 1e-11 of the largest entry
    np.testing.assert_allclose(v, vo, rtol=1e-12, atol=1e-11 * np.abs(vo).max())


GRID_LAYERS = [
    # (nlat_in, nlon_in, nlat_out, nlon_out, kernel_shape, theta_cutoff, grid_in, grid_out)
    (24, 48, 24, 48, (3, 1), 2 * math.pi / 24, "legendre-gauss", "legendre-gauss"),
    (25, 48, 13, 24, (3, 4), 2 * math.pi / 20, "lobatto", "equiangular-trapezoidal"),
    (21, 40, 17, 40, (4, 1), 3 * math.pi / 32, "equiangular-trapezoidal", "legendre-gauss"),
    (33, 64, 33, 64, (3, 1), 2 * math.pi / 32, "legendre-gauss", "lobatto"),
]


@pytest.mark.parametrize("layer", GRID_LAYERS, ids=lambda l: f"{l[6]}->{l[7]}")
def test_psi_export_matches_oracle_on_other_grids(layer):
    """The library's latitude grids (Newton on the Legendre recurrence) give the oracle's Psi
    (Golub-Welsch nodes): the same pattern bit for bit, the values to rounding."""
    nli, nlo_i, nlo, nlo_o, ks, tc, gi, go = layer
    s = D.make_spec(nli, nlo_i, nlo, nlo_o, ks, tc, D.GRID_CODES[gi], D.GRID_CODES[go])
    o = oracle.Spec(nli, nlo_i, nlo, nlo_o, ks[0], ks[1], tc, gi, go)
    h = D.disco_psi_build(s, -1)
    try:
        k, j, i, p, v = D.disco_psi_export(h)
    finally:
        D.disco_psi_destroy(h)
    ko, jo, io, po, vo = oracle.Psi(o).entries()
    assert np.array_equal(k, ko) and np.array_equal(j, jo) and np.array_equal(i, io) and np.array_equal(p, po)
    np.testing.assert_allclose(v, vo, rtol=1e-11, atol=1e-11 * np.abs(vo).max())


@pytest.mark.parametrize("grid", ["legendre-gauss", "lobatto", "equiangular-trapezoidal"])
def test_full_size_grid_rows_match_oracle(grid):
    """721 x 1440 latitude grids (the weather layer's size, where a node solve that loses digits
    or lands on the wrong root would show): sampled Psi rows, poles and equator included,
    against the oracle's dense rows."""
    wl = WORKLOADS["weather"]
    s = D.make_spec(wl.nlat_in, wl.nlon_in, wl.nlat_out, wl.nlon_out, wl.kernel_shape, wl.theta_cutoff,
                    D.GRID_CODES[grid], D.GRID_CODES[grid])
    o = oracle.Spec(wl.nlat_in, wl.nlon_in, wl.nlat_out, wl.nlon_out, wl.kernel_shape[0], wl.kernel_shape[1],
                    wl.theta_cutoff, grid, grid)
    h = D.disco_psi_build(s, -1)
    try:
        k, j, i, p, v = D.disco_psi_export(h)
    finally:
        D.disco_psi_destroy(h)
    for jj in (0, 1, 180, wl.nlat_out // 2, wl.nlat_out - 2, wl.nlat_out - 1):
        dense = oracle.psi_dense_row(o, jj)
        sel = j == jj
        got = np.zeros_like(dense)
        got[k[sel], i[sel], p[sel]] = v[sel]
        assert np.array_equal(got != 0, dense != 0), (grid, jj)
        np.testing.assert_allclose(got, dense, rtol=0, atol=1e-9 * np.abs(dense).max())


def test_grids_change_psi_and_unknown_grids_are_rejected():
    base = D.make_spec(24, 48, 24, 48, (3, 1), 2 * math.pi / 24)
    h = D.disco_psi_build(base, -1)
    try:
        v0 = D.disco_psi_export(h)[4]
    finally:
        D.disco_psi_destroy(h)
    gauss = D.make_spec(24, 48, 24, 48, (3, 1), 2 * math.pi / 24, D.DISCO_GRID_LEGENDRE_GAUSS,
                        D.DISCO_GRID_LEGENDRE_GAUSS)
    h = D.disco_psi_build(gauss, -1)
    try:
        v1 = D.disco_psi_export(h)[4]
    finally:
        D.disco_psi_destroy(h)
    assert v0.shape != v1.shape or not np.allclose(v0, v1)
    for gi, go in ((4, 0), (0, 4), (-1, 0)):
        bad = D.make_spec(24, 48, 24, 48, (3, 1), 2 * math.pi / 24, gi, go)
        with pytest.raises(D.DiscoError) as e:
            D.disco_psi_build(bad, -1)
        assert e.value.status == D.DISCO_ERR_UNSUPPORTED


def _bc(x):
    return x.reshape((-1,) + x.shape[2:])


@pytest.mark.parametrize("which", [0, 2], ids=["rows", "bands"])
@pytest.mark.parametrize("name", ["tiny", "downsample", "mid"])
def test_forward_plan_reproduces_oracle_contraction(name, which):
    wl = WORKLOADS[name].scaled(B=1, C_in=2)
    s, o = spec_pair(wl)
    h = D.disco_psi_build(s, -1)
    plan = D.disco_plan_export(h, which)
    D.disco_psi_destroy(h)
    x = make_inputs(wl, 1)["x"].astype(np.float64)
    y_ref = oracle.Psi(o).contract(x)
    y = plan_emulator.forward(plan, _bc(x), wl.nlat_out, wl.nlon_out, wl.K)
    # plan values are fp32: relative rounding 6e-8 per entry
    np.testing.assert_allclose(y, _bc(y_ref), rtol=0, atol=1e-6 * np.abs(y_ref).max())


@pytest.mark.parametrize("which", [1, 3], ids=["rows", "bands"])
@pytest.mark.parametrize("name", ["tiny", "downsample", "mid"])
def test_adjoint_plan_reproduces_oracle_backward(name, which):
    wl = WORKLOADS[name].scaled(B=1, C_in=2, C_out=3)
    s, o = spec_pair(wl)
    h = D.disco_psi_build(s, -1)
    plan = D.disco_plan_export(h, which)
    D.disco_psi_destroy(h)
    assert plan["residues"] == wl.stride
    P = oracle.Psi(o)
    rng = np.random.default_rng(3)
    dout = rng.standard_normal((1, wl.C_out, wl.nlat_out, wl.nlon_out))
    w = rng.standard_normal((wl.C_out, wl.C_in, wl.K))
    dx_ref = P.backward_input(dout, w, wl.C_in)
    dy = np.einsum("ock,bojq->bckjq", w, dout).reshape(1 * wl.C_in, wl.K * wl.nlat_out, wl.nlon_out)
    dx = plan_emulator.adjoint(plan, dy, wl.nlat_in, wl.nlon_in, wl.stride)
    np.testing.assert_allclose(dx, _bc(dx_ref), rtol=0, atol=1e-6 * np.abs(dx_ref).max())


def test_plans_respect_kernel_limits():
    for name in QUICK:
        s, _ = spec_pair(WORKLOADS[name])
        h = D.disco_psi_build(s, -1)
        for which in (0, 1):
            plan = D.disco_plan_export(h, which)
            chunks = plan["chunks"]
            assert np.all((chunks[:, 3] & 0xFF) >= 1) and np.all((chunks[:, 3] & 0xFF) <= 8)
            assert np.all(chunks[:, 3] >> 8 > 0)
            rows = plan["rows"]
            assert np.all(rows[:, 2] - rows[:, 1] <= 512)
            # every chunk's columns lie inside its source row's span
            for r in rows:
                for ch in range(r[3], r[7 + plan["residues"] - 1]):
                    src, t0, _, wk = chunks[ch]
                    assert 0 <= src < r[2] - r[1]
                    assert t0 + (wk & 0xFF) <= plan["srcs"][r[1] + src][2]
        D.disco_psi_destroy(h)


def test_status_codes():
    lib = D.library()
    h = ctypes.c_void_p()
    bad = D.make_spec(17, 32, 17, 32, 3, 0.0)
    assert lib.disco_psi_build(ctypes.byref(bad), -1, ctypes.byref(h)) == D.DISCO_ERR_INVALID_ARG
    assert "theta_cutoff" in D.disco_last_error()
    assert not h.value
    bad = D.make_spec(17, 32, 17, 24, 3, 0.3)
    assert lib.disco_psi_build(ctypes.byref(bad), -1, ctypes.byref(h)) == D.DISCO_ERR_UNSUPPORTED
    bad = D.make_spec(17, 32, 17, 32, 3, 0.3, grid_in=4)  # no such grid
    assert lib.disco_psi_build(ctypes.byref(bad), -1, ctypes.byref(h)) == D.DISCO_ERR_UNSUPPORTED
    bad = D.make_spec(1, 32, 17, 32, 3, 0.3)
    assert lib.disco_psi_build(ctypes.byref(bad), -1, ctypes.byref(h)) == D.DISCO_ERR_INVALID_ARG
    bad = D.make_spec(17, 32, 17, 32, (1, 1), 0.3)
    assert lib.disco_psi_build(ctypes.byref(bad), -1, ctypes.byref(h)) == D.DISCO_ERR_INVALID_ARG
    # a cutoff 5e-11 below a grid distance: the tie is too close to call
    tie = D.make_spec(17, 32, 17, 32, 3, 2 * math.pi / 16 - 5e-11)
    assert lib.disco_psi_build(ctypes.byref(tie), -1, ctypes.byref(h)) == D.DISCO_ERR_GEOMETRY
    ok = D.make_spec(17, 32, 17, 32, 3, 2 * math.pi / 16)
    h = D.disco_psi_build(ok, -1)
    try:
        # host-only handle: compute calls refuse
        st = lib.disco_fwd(h, 1, 4, 4, 1, D.DISCO_F32, None, None, None, None, None, None, 0, None)
        assert st == D.DISCO_ERR_INVALID_ARG
        n = D.disco_workspace_size(h, D.DISCO_OP_FWD, 1, 4, 4, 1, D.DISCO_F32)
        assert n == 0
        n_bi = D.disco_workspace_size(h, D.DISCO_OP_BWD_INPUT, 2, 4, 6, 2, D.DISCO_BF16)
        assert n_bi >= 2 * 4 * 3 * 17 * 32 * 2
        n_bw = D.disco_workspace_size(h, D.DISCO_OP_BWD_WEIGHT_RECOMPUTE, 2, 4, 6, 2, D.DISCO_F32)
        assert n_bw > D.disco_workspace_size(h, D.DISCO_OP_BWD_WEIGHT, 2, 4, 6, 2, D.DISCO_F32)
        with pytest.raises(D.DiscoError):
            D.disco_workspace_size(h, D.DISCO_OP_FWD, 1, 4, 6, 4, D.DISCO_F32)  # groups do not divide C_in
    finally:
        D.disco_psi_destroy(h)
    assert lib.disco_psi_destroy(None) == D.DISCO_OK


# bf16 layers with nlon_in == nlon_out take the tensor-core kernels: their Toeplitz plans must
# reproduce the contraction and its adjoint (Psi as bf16 hi + lo: relative error <= 2^-17)
TZ_LAYERS = {
    "iso_k3": WORKLOADS["tiny"],
    "aniso_k9": WORKLOADS["tiny"].scaled(nlat_in=21, nlon_in=40, nlat_out=21, nlon_out=40, kernel_shape=(3, 4),
                                         theta_cutoff=0.5),
    "iso_k5": WORKLOADS["tiny"].scaled(nlat_in=25, nlon_in=64, nlat_out=25, nlon_out=64, kernel_shape=(5, 1),
                                       theta_cutoff=0.45),
}


@pytest.mark.parametrize("name", list(TZ_LAYERS))
def test_toeplitz_plan_reproduces_oracle_contraction(name):
    wl = TZ_LAYERS[name].scaled(B=1, C_in=3)
    s, o = spec_pair(wl)
    h = D.disco_psi_build(s, -1)
    try:
        plan = D.disco_toeplitz_export(h, 0)
    finally:
        D.disco_psi_destroy(h)
    assert plan["K"] == wl.K and plan["parts"] == (1 if 16 * wl.K <= 128 else 2)
    assert np.all((plan["slabs"][:, 2] >= 1) & (plan["slabs"][:, 2] <= plan["kslab"]))
    assert np.all(plan["slabs"][:, 1] % 8 == 0)  # windows start on 16-byte boundaries
    assert sorted(plan["slots"][:, 0].tolist()) == list(range(wl.nlat_out))
    x = make_inputs(wl, 1)["x"].astype(np.float64)
    y_ref = oracle.Psi(o).contract(x)
    y = plan_emulator.toeplitz(plan, _bc(x), wl.nlat_out)
    np.testing.assert_allclose(y, _bc(y_ref), rtol=0, atol=2e-5 * np.abs(y_ref).max())


@pytest.mark.parametrize("name", list(TZ_LAYERS))
def test_adjoint_toeplitz_plan_reproduces_oracle_backward(name):
    wl = TZ_LAYERS[name].scaled(B=1, C_in=2, C_out=3)
    s, o = spec_pair(wl)
    h = D.disco_psi_build(s, -1)
    try:
        plan = D.disco_toeplitz_export(h, 1)
    finally:
        D.disco_psi_destroy(h)
    assert plan["K"] == 1 and plan["N"] == 16
    rng = np.random.default_rng(5)
    dout = rng.standard_normal((1, wl.C_out, wl.nlat_out, wl.nlon_out))
    w = rng.standard_normal((wl.C_out, wl.C_in, wl.K))
    dx_ref = oracle.Psi(o).backward_input(dout, w, wl.C_in)
    dy = np.einsum("ock,bojq->bckjq", w, dout).reshape(wl.C_in, wl.K * wl.nlat_out, wl.nlon_out)
    dx = plan_emulator.toeplitz(plan, dy, wl.nlat_in)[:, 0]
    np.testing.assert_allclose(dx, _bc(dx_ref), rtol=0, atol=2e-5 * np.abs(dx_ref).max())


def test_toeplitz_plan_absent_for_stride_two():
    s, _ = spec_pair(WORKLOADS["downsample"])
    h = D.disco_psi_build(s, -1)
    try:
        with pytest.raises(D.DiscoError) as e:
            D.disco_toeplitz_export(h, 0)
        assert e.value.status == D.DISCO_ERR_UNSUPPORTED
    finally:
        D.disco_psi_destroy(h)


def test_layer_rejects_unknown_grid_names_before_building():
    from spherical_disco_convolution_b200 import conv

    with pytest.raises(ValueError, match="grids are one of"):
        conv.Psi(17, 32, 17, 32, (3, 1), 0.3, "cuda:0", grid_in="gaussian")
    with pytest.raises(ValueError, match="grids are one of"):
        conv.Psi(17, 32, 17, 32, (3, 1), 0.3, "cuda:0", grid_out="healpix")
    assert sorted(D.GRID_CODES) == sorted(oracle.GRIDS)


@pytest.mark.parametrize("grids", [("legendre-gauss", "legendre-gauss"), ("lobatto", "equiangular-trapezoidal")])
def test_tensor_core_plans_on_other_grids_reproduce_oracle(grids):
    """The Toeplitz and ring plans depend on Psi only; on the other latitude grids they still
    reproduce the oracle (re-enacted on CPU; the ring plan's blocks hold Psi rounded to bf16, so
    its bound is 2^-8 max|x|, the rounding of entries that are >= 0 and sum to one per row)."""
    gi, go = grids
    nli, nlo, nlon, tc = 40, 40, 64, 2 * math.pi / 36
    s = D.make_spec(nli, nlon, nlo, nlon, (3, 1), tc, D.GRID_CODES[gi], D.GRID_CODES[go])
    o = oracle.Spec(nli, nlon, nlo, nlon, 3, 1, tc, gi, go)
    h = D.disco_psi_build(s, -1)
    try:
        tz = D.disco_toeplitz_export(h, 0)
        rp = D.disco_ring_export(h, 1)
    finally:
        D.disco_psi_destroy(h)
    rng = np.random.default_rng(9)
    x = rng.standard_normal((1, 2, nli, nlon))
    ref = _bc(oracle.Psi(o).contract(x))
    got = plan_emulator.toeplitz(tz, _bc(x), nlo)
    np.testing.assert_allclose(got, ref, rtol=0, atol=2e-5 * np.abs(ref).max())
    got = plan_emulator.ring(rp, _bc(x), nlo)
    assert np.abs(got - ref).max() <= 1.05 * 2.0 ** -8 * np.abs(x).max()
