"""The polar x azimuth distributed layer on CPU: gloo ranks, the layer's own forward and backward.

DistributedDiscoConvS2 (page "torch_harmonics.distributed.DistributedDiscreteContinuousConvS2")
runs here end to end through autograd on 2 to 4 gloo ranks, with every collective of the real
layer (the azimuth all-to-alls, the halo exchange, the reduce-scatters and all-gathers, the
gradient all-reduces).  The per-rank kernels are replaced by CpuOps below: each rank's Psi is
the exported host-only handle of its band (full, halo band or input band) applied as a dense
matrix in fp64, and the einsums are written out with torch.einsum.  out, dx, dw and dbias of
every rank's shard are compared with the global oracle's.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from spherical_disco_convolution_b200 import disco as D
from spherical_disco_convolution_b200 import distributed, polar
from tests.test_polar import LAYERS, _band_ops, _export, _ospec, _spec

LAYERS = dict(LAYERS)
# longitudes that no rank count divides evenly (40 -> 14/13/13 and 20 -> 7/7/6 on 3 ranks)
LAYERS["odd"] = (25, 40, 13, 20, (3, 2), 0.6, "equiangular", "equiangular")
# a cutoff wider than any halo of 2 polar ranks: the reduce-scatter mode's case
LAYERS["wide"] = (33, 64, 33, 64, (3, 1), 0.9, "equiangular", "equiangular")


class _HostPsi:
    def __init__(self, A, K, n_out, n_in, nlon_in, nlon_out):
        self.A = torch.from_numpy(A)
        self.K, self.n_out, self.n_in, self.nlon_in, self.nlon_out = K, n_out, n_in, nlon_in, nlon_out


class CpuOps:
    """The layer's per-rank steps in fp64 on the CPU, for gloo ranks: exported band Psi as a dense
    matrix, einsums written out."""

    def psi(self, geometry, rows=None, inputs=None):
        nli, nloi, nlo, nloo = geometry[:4]
        spec = _spec(geometry)
        if rows is not None:
            h, ib, ie = D.disco_psi_build_band(spec, rows[0], rows[1], -1)
            n_out, n_in = rows[1] - rows[0], ie - ib
        elif inputs is not None:
            h = D.disco_psi_build_inputs(spec, inputs[0], inputs[1], -1)
            n_out, n_in = nlo, inputs[1] - inputs[0]
        else:
            h = D.disco_psi_build(spec, -1)
            n_out, n_in = nlo, nli
        K, _ = D.disco_psi_info(h)
        A = _band_ops(_export(h), n_out, nloi, nloo, K)
        A = np.pad(A, ((0, 0), (0, n_in * nloi - A.shape[1])))
        return _HostPsi(A, K, n_out, n_in, nloi, nloo)

    def contract(self, psi, x):
        B, C = x.shape[:2]
        y = torch.einsum("ra,na->nr", psi.A, x.reshape(B * C, -1))
        return y.reshape(B, C, psi.K, psi.n_out, psi.nlon_out)

    def contract_adjoint(self, psi, dy):
        B, C = dy.shape[:2]
        dx = torch.einsum("ra,nr->na", psi.A, dy.reshape(B * C, -1))
        return dx.reshape(B, C, psi.n_in, psi.nlon_in)

    def mix(self, y, w, bias, groups):
        B, C, K = y.shape[:3]
        pts = y.shape[3:]
        Co = w.shape[0]
        out = torch.einsum("gock,bgckn->bgon", w.reshape(groups, Co // groups, C // groups, K),
                           y.reshape(B, groups, C // groups, K, -1)).reshape((B, Co) + pts)
        return out if bias is None else out + bias.view((1, Co) + (1,) * len(pts))

    def mix_adjoint(self, dout, w, C_in, groups):
        B, Co = dout.shape[:2]
        pts = dout.shape[2:]
        K = w.shape[2]
        dy = torch.einsum("gock,bgon->bgckn", w.reshape(groups, Co // groups, C_in // groups, K),
                          dout.reshape(B, groups, Co // groups, -1))
        return dy.reshape((B, C_in, K) + pts)

    def mix_weight(self, dout, y, groups, need_bias):
        B, Co = dout.shape[:2]
        C, K = y.shape[1:3]
        dw = torch.einsum("bgon,bgckn->gock", dout.reshape(B, groups, Co // groups, -1),
                          y.reshape(B, groups, C // groups, K, -1)).reshape(Co, C // groups, K)
        db = dout.sum(dim=[0] + list(range(2, dout.dim()))) if need_bias else None
        return dw, db

    def forward_fused(self, psi, x, w, bias):
        return self.mix(self.contract(psi, x), w, bias, 1)

    def backward_input(self, psi, dout, w, C_in):
        return self.contract_adjoint(psi, self.mix_adjoint(dout, w, C_in, 1))

    def backward_weight_x(self, psi, dout, x, need_bias):
        return self.mix_weight(dout, self.contract(psi, x), 1, need_bias)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, case, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        n_polar, n_az, mode, fused, name, padded = case
        if padded:
            # the one-collective path on equal padded chunks (as NCCL runs it), its reduce-scatter
            # emulated by a sum and the rank's chunk (gloo has no reduce-scatter of its own)
            def rs(out, inp, group=None):
                s = inp.clone()
                dist.all_reduce(s, group=group)
                n = dist.get_world_size(group)
                r = dist.get_rank(group)
                out.copy_(s.reshape((n, -1) + tuple(out.shape[1:]))[r].reshape(out.shape))

            polar.dist.get_backend = lambda *a: "nccl"
            polar.dist.reduce_scatter_tensor = rs
        layer = LAYERS[name]
        nli, nloi, nlo, nloo, ks, tc, gi, go = layer
        B, C_in, C_out, G = 2, 4, 6, 2
        P = oracle.Psi(_ospec(layer))
        rng = np.random.default_rng(29)
        x = rng.standard_normal((B, C_in, nli, nloi))
        w = rng.standard_normal((C_out, C_in // G, P.K))
        bias = rng.standard_normal(C_out)
        dout = rng.standard_normal((B, C_out, nlo, nloo))
        out_ref = P.forward(x, w, bias, groups=G)
        dx_ref = P.backward_input(dout, w, C_in, groups=G)
        dw_ref, db_ref = P.backward_weight(dout, x, groups=G)

        m = distributed.DistributedDiscoConvS2(C_in, C_out, (nli, nloi), (nlo, nloo), ks, tc, polar_size=n_polar,
                                               azimuth_size=n_az, polar_mode=mode, groups=G, grid_in=gi, grid_out=go,
                                               fused=fused, dtype=torch.float64, ops=CpuOps())
        with torch.no_grad():
            m.weight.copy_(torch.from_numpy(w))
            m.bias.copy_(torch.from_numpy(bias))
        ob, oe = m.bands.in_rows[m.p]
        jb, je = m.bands.out_rows[m.p]
        lb, le = m.shards.lon_in[m.a]
        qb, qe = m.shards.lon_out[m.a]
        x_own = torch.from_numpy(x[:, :, ob:oe, lb:le].copy()).requires_grad_()
        out = m(x_own)
        np.testing.assert_allclose(out.detach().numpy(), out_ref[:, :, jb:je, qb:qe], rtol=0, atol=1e-10)
        out.backward(torch.from_numpy(dout[:, :, jb:je, qb:qe].copy()))
        np.testing.assert_allclose(x_own.grad.numpy(), dx_ref[:, :, ob:oe, lb:le], rtol=0, atol=1e-10)
        np.testing.assert_allclose(m.weight.grad.numpy(), dw_ref, rtol=0, atol=1e-9)
        np.testing.assert_allclose(m.bias.grad.numpy(), db_ref, rtol=0, atol=1e-9)
        q.put((rank, "ok"))
    except Exception as e:  # reported to the parent, which fails the test
        q.put((rank, f"{type(e).__name__}: {e}"))
    finally:
        dist.barrier()
        dist.destroy_process_group()


CASES = [
    (1, 2, "halo-exchange", False, "iso", False),         # azimuth all-to-all alone
    (1, 3, "halo-exchange", True, "odd", False),          # reordered all-to-all, uneven longitudes and channels
    (1, 3, "halo-exchange", True, "odd", True),           # ... its reduce-scatter on padded chunks
    (2, 2, "halo-exchange", False, "aniso_down", False),  # halo rows and the azimuth all-to-all together
    (2, 2, "halo-exchange", True, "gauss", False),
    (2, 2, "reduce-scatter", False, "wide", False),
    (2, 2, "reduce-scatter", True, "odd", True),
    (3, 1, "reduce-scatter", True, "wide", False),
]


@pytest.mark.parametrize("case", CASES, ids=["x".join(map(str, c[:2])) + f"-{c[2]}-{'fused' if c[3] else 'std'}-{c[4]}"
                                             + ("-padded" if c[5] else "") for c in CASES])
def test_distributed_layer_reassembles_the_oracle(case):
    world = case[0] * case[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [m for _, m in res] == ["ok"] * world, res


def test_all_to_all_pair_is_a_permutation_on_one_rank():
    # on one rank both swaps are the identity, and the shard tables cover every index once
    sh = distributed.AzimuthShards(40, 20, 5, 3)
    assert sh.lon_in == [(0, 14), (14, 27), (27, 40)] and sh.lon_out == [(0, 7), (7, 14), (14, 20)]
    assert sh.chans == [(0, 2), (2, 4), (4, 5)]
    t = torch.arange(2 * 3 * 4 * 5, dtype=torch.float64).reshape(2, 3, 4, 5)
    assert torch.equal(distributed.lon_to_chan(t, [(0, 5)], [(0, 3)], 0), t)
    assert torch.equal(distributed.chan_to_lon(t, [(0, 5)], [(0, 3)], 0), t)
    with pytest.raises(ValueError):
        distributed.AzimuthShards(40, 20, 2, 3)
