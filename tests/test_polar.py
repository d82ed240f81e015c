"""Polar-band ("halo-exchange") distribution on CPU: band Psi, plans, and gloo ranks.

The band handles are host-only (no GPU), so the per-rank contraction here is the band's exported
Psi applied in NumPy; what is checked is everything around it: that a band's Psi is exactly the
full Psi's rows, that its plans still reproduce the oracle, and that the halo gather, the
reverse halo sum and the weight-gradient all-reduce reassemble the global oracle's out, dx and
dw on 2, 3 and 4 ranks.
"""

import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from spherical_disco_convolution_b200 import disco as D
from spherical_disco_convolution_b200 import polar
from tests import plan_emulator

# (nlat_in, nlon_in, nlat_out, nlon_out, kernel_shape, theta_cutoff, grid_in, grid_out)
LAYERS = {
    "iso": (33, 64, 33, 64, (3, 1), 2 * math.pi / 32, "equiangular", "equiangular"),
    "aniso_down": (37, 48, 19, 24, (3, 4), 2 * math.pi / 24, "equiangular", "equiangular"),
    "gauss": (30, 48, 30, 48, (3, 1), 2 * math.pi / 28, "legendre-gauss", "legendre-gauss"),
}


def _spec(layer):
    nli, nloi, nlo, nloo, ks, tc, gi, go = layer
    return D.make_spec(nli, nloi, nlo, nloo, ks, tc, D.GRID_CODES[gi], D.GRID_CODES[go])


def _ospec(layer):
    nli, nloi, nlo, nloo, ks, tc, gi, go = layer
    return oracle.Spec(nli, nloi, nlo, nloo, ks[0], ks[1], tc, gi, go)


def _export(h):
    try:
        return D.disco_psi_export(h)
    finally:
        D.disco_psi_destroy(h)


def test_split_rows_is_balanced_and_contiguous():
    for n, p in ((10, 3), (721, 8), (8, 8), (5, 1)):
        parts = polar.split_rows(n, p)
        assert parts[0][0] == 0 and parts[-1][1] == n
        assert all(a[1] == b[0] for a, b in zip(parts, parts[1:]))
        sizes = [e - b for b, e in parts]
        assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)
    with pytest.raises(ValueError):
        polar.split_rows(3, 4)


@pytest.mark.parametrize("name", list(LAYERS))
def test_band_psi_is_the_full_psi_rows(name):
    layer = LAYERS[name]
    s = _spec(layer)
    k, j, i, p, v = _export(D.disco_psi_build(s, -1))
    nlat_out = layer[2]
    for jb, je in polar.split_rows(nlat_out, 3) + [(0, 1), (nlat_out - 1, nlat_out), (0, nlat_out)]:
        h, ib, ie = D.disco_psi_build_band(s, jb, je, -1)
        kb, jbb, ibb, pb, vb = _export(h)
        sel = (j >= jb) & (j < je)
        assert ib == i[sel].min() and ie == i[sel].max() + 1
        # the same entries, re-indexed, bit for bit
        assert np.array_equal(kb, k[sel]) and np.array_equal(jbb, j[sel] - jb)
        assert np.array_equal(ibb, i[sel] - ib) and np.array_equal(pb, p[sel]) and np.array_equal(vb, v[sel])


def test_band_rejects_bad_row_ranges():
    s = _spec(LAYERS["iso"])
    for jb, je in ((-1, 3), (3, 3), (5, 2), (0, 34)):
        with pytest.raises(D.DiscoError) as e:
            D.disco_psi_build_band(s, jb, je, -1)
        assert e.value.status == D.DISCO_ERR_INVALID_ARG


def test_band_toeplitz_plan_reproduces_the_oracle_rows():
    """A band's tensor-core plan (re-indexed rows) still reproduces the oracle's contraction."""
    layer = LAYERS["iso"]
    s = _spec(layer)
    rng = np.random.default_rng(3)
    x = rng.standard_normal((1, 2, layer[0], layer[1]))
    y_ref = oracle.Psi(_ospec(layer)).contract(x)
    for jb, je in polar.split_rows(layer[2], 4):
        h, ib, ie = D.disco_psi_build_band(s, jb, je, -1)
        try:
            plan = D.disco_toeplitz_export(h, 0)
        finally:
            D.disco_psi_destroy(h)
        xb = x[:, :, ib:ie].reshape((-1, ie - ib, layer[1]))
        y = plan_emulator.toeplitz(plan, xb, je - jb)
        want = y_ref[:, :, :, jb:je].reshape((-1,) + y_ref.shape[2:3] + (je - jb, layer[3]))
        np.testing.assert_allclose(y, want, rtol=0, atol=2e-5 * np.abs(y_ref).max())


def test_band_adjoint_toeplitz_plan_reproduces_the_oracle():
    """A band's adjoint plan (source rows (k, j) of the band's dy, output rows the reached input
    rows) gives the oracle's dx for a dout that is zero outside the band."""
    layer = LAYERS["iso"]
    s = _spec(layer)
    nli, nloi, nlo, nloo = layer[:4]
    P = oracle.Psi(_ospec(layer))
    K = P.K
    rng = np.random.default_rng(4)
    w = rng.standard_normal((3, 2, K))
    for jb, je in polar.split_rows(nlo, 4):
        dout = np.zeros((1, 3, nlo, nloo))
        dout[:, :, jb:je] = rng.standard_normal((1, 3, je - jb, nloo))
        dx_ref = P.backward_input(dout, w, 2)
        h, ib, ie = D.disco_psi_build_band(s, jb, je, -1)
        try:
            plan = D.disco_toeplitz_export(h, 1)
        finally:
            D.disco_psi_destroy(h)
        dy = np.einsum("ock,bojq->bckjq", w, dout[:, :, jb:je]).reshape(2, K * (je - jb), nloo)
        dx = plan_emulator.toeplitz(plan, dy, ie - ib)[:, 0]
        # nothing outside the reached rows, and the reached rows match
        assert np.abs(dx_ref[0, :, :ib]).max(initial=0) == 0 and np.abs(dx_ref[0, :, ie:]).max(initial=0) == 0
        np.testing.assert_allclose(dx, dx_ref[0, :, ib:ie], rtol=0, atol=2e-5 * np.abs(dx_ref).max())


@pytest.mark.parametrize("world", [2, 3, 5, 8])
@pytest.mark.parametrize("cut", [1, 2, 3])
def test_exchange_plan_covers_each_reach_exactly(world, cut):
    """For every rank: its own rows plus what it borrows tile its reach with no overlap; every
    borrowed range is a neighbour's own rows; sends mirror receives."""
    nlat = 65
    try:
        bands = polar.PolarBands(nlat, 64, nlat, 64, (3, 1), cut * math.pi / (nlat - 1) + 1e-3, world)
    except ValueError:
        assert world * (cut + 1) > nlat  # refused only when bands are thinner than the reach
        return
    for r in range(world):
        ib, ie = bands.reach[r]
        ob, oe = bands.in_rows[r]
        covered = np.zeros(ie - ib, dtype=int)
        lo, hi = max(ib, ob), min(ie, oe)
        if lo < hi:
            covered[lo - ib:hi - ib] += 1
        for src, lo, hi in bands.recv[r]:
            assert abs(src - r) == 1
            sb, se = bands.in_rows[src]
            assert sb <= lo < hi <= se
            covered[lo - ib:hi - ib] += 1
            assert (r, lo, hi) in bands.send[src]
        assert np.all(covered == 1)
    assert sum(len(x) for x in bands.send) == sum(len(x) for x in bands.recv)


def test_too_wide_filter_is_refused():
    """A cutoff that reaches past the neighbouring rank's latitudes raises at construction."""
    nli, nloi, nlo, nloo, ks, _, gi, go = LAYERS["iso"]
    polar.PolarBands(nli, nloi, nlo, nloo, ks, 2 * math.pi / 32, 4)  # fine: 8 rows per rank
    with pytest.raises(ValueError, match="too wide"):
        polar.PolarBands(nli, nloi, nlo, nloo, ks, 0.6, 8)


# ------------------------------------------------------------------ gloo ranks

def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _band_ops(entries, n_out_rows, nlon_in, nlon_out, K):
    """Dense band operator A[(k, jl, q), (il, l)] from exported entries (the definition, q*s + p)."""
    k, j, i, p, v = entries
    s = nlon_in // nlon_out
    n_in = (i.max() + 1) * nlon_in
    A = np.zeros((K * n_out_rows * nlon_out, n_in))
    for q in range(nlon_out):
        rows = (k * n_out_rows + j) * nlon_out + q
        cols = i * nlon_in + (q * s + p) % nlon_in
        np.add.at(A, (rows, cols), v)
    return A


def _worker(rank, world, port, name, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        layer = LAYERS[name]
        nli, nloi, nlo, nloo, ks, tc, gi, go = layer
        bands = polar.PolarBands(nli, nloi, nlo, nloo, ks, tc, world, gi, go)
        B, C_in, C_out, G = 2, 4, 6, 2
        P = oracle.Psi(_ospec(layer))
        K = P.K
        rng = np.random.default_rng(11)
        x = rng.standard_normal((B, C_in, nli, nloi))
        w = rng.standard_normal((C_out, C_in // G, K))
        bias = rng.standard_normal(C_out)
        dout = rng.standard_normal((B, C_out, nlo, nloo))
        out_ref = P.forward(x, w, bias, groups=G)
        dx_ref = P.backward_input(dout, w, C_in, groups=G)
        dw_ref, db_ref = P.backward_weight(dout, x, groups=G)

        ob, oe = bands.in_rows[rank]
        jb, je = bands.out_rows[rank]
        ib, ie = bands.reach[rank]
        x_band = polar.halo_gather(bands, rank, torch.from_numpy(x[:, :, ob:oe].copy())).numpy()
        np.testing.assert_array_equal(x_band, x[:, :, ib:ie])  # the halo is the neighbours' rows

        h, ib2, ie2 = D.disco_psi_build_band(bands.spec, jb, je, -1)
        ent = _export(h)
        assert (ib2, ie2) == (ib, ie)
        A = _band_ops(ent, je - jb, nloi, nloo, K)
        A = np.pad(A, ((0, 0), (0, (ie - ib) * nloi - A.shape[1])))
        y = np.einsum("ra,bca->bcr", A, x_band.reshape(B, C_in, -1)).reshape(B, C_in, K, je - jb, nloo)
        cg, og = C_in // G, C_out // G
        out = np.empty((B, C_out, je - jb, nloo))
        for o in range(C_out):
            g = o // og
            out[:, o] = np.einsum("ck,bckjq->bjq", w[o], y[:, g * cg:(g + 1) * cg]) + bias[o]
        np.testing.assert_allclose(out, out_ref[:, :, jb:je], rtol=0, atol=1e-11)

        # backward: dy = w^T dout on the band, dx_band = A^T dy, then the reverse halo sum
        d = dout[:, :, jb:je]
        dy = np.zeros((B, C_in, K, je - jb, nloo))
        for o in range(C_out):
            g = o // og
            dy[:, g * cg:(g + 1) * cg] += np.einsum("ck,bjq->bckjq", w[o], d[:, o])
        dx_band = np.einsum("ra,bcr->bca", A, dy.reshape(B, C_in, -1)).reshape(B, C_in, ie - ib, nloi)
        dx_own = polar.halo_reduce(bands, rank, torch.from_numpy(dx_band)).numpy()
        np.testing.assert_allclose(dx_own, dx_ref[:, :, ob:oe], rtol=0, atol=1e-11)

        dw = np.zeros_like(w)
        for o in range(C_out):
            g = o // og
            dw[o] = np.einsum("bjq,bckjq->ck", d[:, o], y[:, g * cg:(g + 1) * cg])
        dw_t = torch.from_numpy(dw)
        db_t = torch.from_numpy(d.sum(axis=(0, 2, 3)))
        dist.all_reduce(dw_t)
        dist.all_reduce(db_t)
        np.testing.assert_allclose(dw_t.numpy(), dw_ref, rtol=0, atol=1e-10)
        np.testing.assert_allclose(db_t.numpy(), db_ref, rtol=0, atol=1e-10)
        q.put((rank, "ok"))
    except Exception as e:  # reported to the parent, which fails the test
        q.put((rank, f"{type(e).__name__}: {e}"))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world,name", [(2, "iso"), (3, "aniso_down"), (3, "gauss"), (4, "iso")])
def test_halo_exchange_reassembles_the_oracle(world, name):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, name, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [m for _, m in res] == ["ok"] * world, res
