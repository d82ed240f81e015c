"""The "reduce-scatter" polar mode on CPU: input-band Psi and gloo ranks.

Every rank holds one band of input latitudes and computes a partial sum over every output
latitude; a reduce-scatter completes the sums and splits them by output band (page
"torch_harmonics.distributed.DistributedDiscreteContinuousConvS2", parameter polar_mode).  The
band handles are host-only here, so each rank applies its band's exported Psi in NumPy; what is
checked is that a band's Psi is exactly the full Psi's entries of those input rows, and that the
reduce-scatter of the partial out, the all-gather of dout, each band's adjoint and the
all-reduce of dw reassemble the global oracle's out, dx and dw on 2, 3 and 4 ranks (the
reduce-scatter both as one collective on equal padded chunks and as the sum-then-slice that
gloo runs).
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
from tests.test_polar import LAYERS, _band_ops, _export, _ospec, _spec

WIDE = ("wide", (33, 64, 33, 64, (3, 1), 0.9, "equiangular", "equiangular"))  # beyond any halo


def _layer(name):
    return WIDE[1] if name == "wide" else LAYERS[name]


@pytest.mark.parametrize("name", list(LAYERS) + ["wide"])
def test_input_band_psi_is_the_full_psi_entries(name):
    layer = _layer(name)
    full = _export(D.disco_psi_build(_spec(layer), -1))
    nli = layer[0]
    for ib, ie in [(0, nli // 3), (nli // 3, 2 * nli // 3 + 1), (nli - 2, nli)]:
        band = _export(D.disco_psi_build_inputs(_spec(layer), ib, ie, -1))
        keep = (full[2] >= ib) & (full[2] < ie)
        got = sorted(zip(band[0].tolist(), band[1].tolist(), (band[2] + ib).tolist(), band[3].tolist(), band[4].tolist()))
        ref = sorted(zip(full[0][keep].tolist(), full[1][keep].tolist(), full[2][keep].tolist(), full[3][keep].tolist(),
                         full[4][keep].tolist()))
        assert got == ref


def test_input_band_rejects_bad_row_ranges():
    spec = _spec(LAYERS["iso"])
    for ib, ie in [(-1, 3), (3, 3), (5, 2), (0, 34)]:
        with pytest.raises(D.DiscoError):
            D.disco_psi_build_inputs(spec, ib, ie, -1)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, name, padded, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        if padded:
            # the one-collective path on equal padded chunks, its reduce-scatter emulated by a sum
            # and the rank's chunk (gloo has no reduce-scatter of its own)
            def rs(out, inp, group=None):
                s = inp.clone()
                dist.all_reduce(s)
                out.copy_(s.reshape((world, -1) + tuple(out.shape[1:]))[rank].reshape(out.shape))

            polar.dist.get_backend = lambda *a: "nccl"
            polar.dist.reduce_scatter_tensor = rs
        layer = _layer(name)
        nli, nloi, nlo, nloo, ks, tc, gi, go = layer
        bands = polar.InputBands(nli, nloi, nlo, nloo, ks, tc, world, gi, go)
        B, C_in, C_out, G = 2, 4, 6, 2
        P = oracle.Psi(_ospec(layer))
        K = P.K
        rng = np.random.default_rng(17)
        x = rng.standard_normal((B, C_in, nli, nloi))
        w = rng.standard_normal((C_out, C_in // G, K))
        bias = rng.standard_normal(C_out)
        dout = rng.standard_normal((B, C_out, nlo, nloo))
        out_ref = P.forward(x, w, bias, groups=G)
        dx_ref = P.backward_input(dout, w, C_in, groups=G)
        dw_ref, db_ref = P.backward_weight(dout, x, groups=G)

        ib, ie = bands.in_rows[rank]
        jb, je = bands.out_rows[rank]
        ent = _export(D.disco_psi_build_inputs(bands.spec, ib, ie, -1))
        A = _band_ops(ent, nlo, nloi, nloo, K)
        A = np.pad(A, ((0, 0), (0, (ie - ib) * nloi - A.shape[1])))
        x_own = x[:, :, ib:ie]
        y = np.einsum("ra,bca->bcr", A, x_own.reshape(B, C_in, -1)).reshape(B, C_in, K, nlo, nloo)
        cg, og = C_in // G, C_out // G
        out_part = np.empty((B, C_out, nlo, nloo))
        for o in range(C_out):
            g = o // og
            out_part[:, o] = np.einsum("ck,bckjq->bjq", w[o], y[:, g * cg:(g + 1) * cg])
        out_own = polar.reduce_scatter_rows(bands.out_rows, rank, torch.from_numpy(out_part)).numpy()
        out_own = out_own + bias[None, :, None, None]
        np.testing.assert_allclose(out_own, out_ref[:, :, jb:je], rtol=0, atol=1e-10)

        # backward: dout gathered onto every output row, the band's adjoint, dw summed over ranks
        d = polar.all_gather_rows(bands.out_rows, rank, torch.from_numpy(dout[:, :, jb:je].copy())).numpy()
        np.testing.assert_array_equal(d, dout)
        dy = np.zeros((B, C_in, K, nlo, nloo))
        for o in range(C_out):
            g = o // og
            dy[:, g * cg:(g + 1) * cg] += np.einsum("ck,bjq->bckjq", w[o], d[:, o])
        dx_own = np.einsum("ra,bcr->bca", A, dy.reshape(B, C_in, -1)).reshape(B, C_in, ie - ib, nloi)
        np.testing.assert_allclose(dx_own, dx_ref[:, :, ib:ie], rtol=0, atol=1e-10)
        dw = np.zeros_like(w)
        for o in range(C_out):
            g = o // og
            dw[o] = np.einsum("bjq,bckjq->ck", d[:, o], y[:, g * cg:(g + 1) * cg])
        dw_t = torch.from_numpy(dw)
        db_t = torch.from_numpy(dout[:, :, jb:je].sum(axis=(0, 2, 3)))
        dist.all_reduce(dw_t)
        dist.all_reduce(db_t)
        np.testing.assert_allclose(dw_t.numpy(), dw_ref, rtol=0, atol=1e-9)
        np.testing.assert_allclose(db_t.numpy(), db_ref, rtol=0, atol=1e-9)
        q.put((rank, "ok"))
    except Exception as e:  # reported to the parent, which fails the test
        q.put((rank, f"{type(e).__name__}: {e}"))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world,name,padded", [(2, "iso", False), (3, "aniso_down", True), (3, "gauss", False),
                                               (4, "wide", True), (2, "wide", False)])
def test_reduce_scatter_mode_reassembles_the_oracle(world, name, padded):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, name, padded, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [m for _, m in res] == ["ok"] * world, res


def test_wide_filter_needs_the_reduce_scatter_mode():
    # the halo mode refuses a reach past the neighbours; the reduce-scatter mode has no bound
    nli, nloi, nlo, nloo, ks, tc, gi, go = WIDE[1]
    with pytest.raises(ValueError, match="too wide"):
        polar.PolarBands(nli, nloi, nlo, nloo, ks, tc, 4, gi, go)
    bands = polar.InputBands(nli, nloi, nlo, nloo, ks, tc, 4, gi, go)
    assert bands.in_rows[0] == (0, 9) and bands.out_rows[-1] == (25, 33)
