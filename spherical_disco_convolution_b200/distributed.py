"""The DISCO layer with its grid split over ranks in both the polar and the azimuth direction.

Follows the page "torch_harmonics.distributed.DistributedDiscreteContinuousConvS2" (class
description; parameters polar_mode and fused).  The data is split in latitude (polar) and in
longitude (azimuth).  In the azimuth direction an all-to-all swaps the longitude shard for a
channel shard, so that the sparse Psi contraction runs on full rows of nlon_in points, and a
second all-to-all swaps back.  In the polar direction `polar_mode` chooses between a halo of
borrowed input rows ("halo-exchange": each rank computes its own output rows outright) and
partial sums over every output row completed by a reduce-scatter ("reduce-scatter").  `fused`
picks where the weight einsum runs:

  * fused=False: contraction on the channel shard, all-to-all of the K-expanded y back to
    longitude shards, then the einsum; y is saved for backward;
  * fused=True: the fused contraction + einsum on the channel shard gives each rank a partial out
    (its channels' share of the sum over input channels) on full rows, and the collective that
    returns to longitude shards is a reduce-scatter of out, K times smaller than y when C_in =
    C_out; x's channel shard is saved and y is recomputed in backward.

Readings where the page is silent:

  * the ranks form a polar_size x azimuth_size grid, rank = p * azimuth_size + a; rank (p, a)
    holds the p-th band of latitudes and the a-th shard of longitudes;
  * latitudes, longitudes and input channels are each split into contiguous parts as evenly as
    possible, the first (n mod P) parts one longer; input and output grids are split alike;
  * the azimuth all-to-all gives rank a the a-th shard of the input channels;
  * fused=True with groups > 1: the channel shard's weight is the dense block w[o, c, k] for the
    shard's channels c, zero where o and c lie in different groups;
  * the bias is added once: by the einsum on every rank when each rank owns its output points
    outright, else by the partial sum of the ranks with a = 0 (and p = 0 in the reduce-scatter
    mode), which the reduce-scatters then add once;
  * backward is the adjoint of each step: all-to-alls run in reverse, a reduce-scatter's adjoint
    is an all-gather, the halo's adjoint sums borrowed rows' gradients onto their owners; dw is
    summed over all ranks, dbias over the ranks whose dout it has not seen.

Every rank runs the same collective steps in the same order; torch.distributed carries them
(NCCL on GPUs, gloo on CPU).  The kernels come from a KernelOps object, the libdisco CUDA calls.
"""

from __future__ import annotations

import math

import torch
import torch.distributed as dist

from . import conv
from . import polar

POLAR_MODES = ("halo-exchange", "reduce-scatter")


class KernelOps:
    """The per-rank compute steps of the layer: libdisco's kernels on the current CUDA device."""

    def __init__(self, device=None):
        self.device = device

    def psi(self, geometry, rows=None, inputs=None):
        nli, nloi, nlo, nloo, ks, tc, gi, go = geometry
        return conv.Psi(nli, nloi, nlo, nloo, ks, tc, self.device, gi, go, rows=rows, inputs=inputs)

    def contract(self, psi, x):
        return conv.disco_contract(psi, x)

    def contract_adjoint(self, psi, dy):
        return conv.disco_contract_adjoint(psi, dy)

    def forward_fused(self, psi, x, w, bias):
        return conv.disco_forward(psi, x, w, bias, 1, fused=True)[0]

    def backward_input(self, psi, dout, w, C_in):
        return conv.disco_backward_input(psi, dout, w, C_in, 1)

    def backward_weight_x(self, psi, dout, x, need_bias):
        return conv.disco_backward_weight(psi, dout, x=x, groups=1, need_bias=need_bias)

    def mix(self, y, w, bias, groups):
        return conv.mix(y, w, bias, groups)

    def mix_adjoint(self, dout, w, C_in, groups):
        return conv.mix_adjoint(dout, w, C_in, groups)

    def mix_weight(self, dout, y, groups, need_bias):
        return conv.mix_weight(dout, y, groups, need_bias)


# ------------------------------------------------------------------ the azimuth all-to-all

def _all_to_all(sends, recv_shapes, group):
    """sends[s] goes to rank s of `group`; returns the blocks received from each rank, shaped."""
    flat_in = torch.cat([t.reshape(-1) for t in sends])
    in_splits = [t.numel() for t in sends]
    out_splits = [math.prod(sh) for sh in recv_shapes]
    flat_out = flat_in.new_empty(sum(out_splits))
    dist.all_to_all_single(flat_out, flat_in, out_splits, in_splits, group=group)
    return [c.view(sh) for c, sh in zip(flat_out.split(out_splits), recv_shapes)]


def lon_to_chan(t, lon, chans, rank: int, group=None) -> torch.Tensor:
    """t (B, C, ..., w) on rank's longitudes lon[rank] -> (B, C_a, ..., nlon) on rank's channels
    chans[rank] and every longitude."""
    if len(lon) == 1:
        return t.contiguous()
    cb, ce = chans[rank]
    sends = [t[:, b:e].contiguous() for b, e in chans]
    shapes = [(t.shape[0], ce - cb) + tuple(t.shape[2:-1]) + (e - b,) for b, e in lon]
    return torch.cat(_all_to_all(sends, shapes, group), dim=-1).contiguous()


def chan_to_lon(t, lon, chans, rank: int, group=None) -> torch.Tensor:
    """The inverse of lon_to_chan (and its adjoint): (B, C_a, ..., nlon) on rank's channels ->
    (B, C, ..., w) on rank's longitudes."""
    if len(lon) == 1:
        return t.contiguous()
    lb, le = lon[rank]
    sends = [t[..., b:e].contiguous() for b, e in lon]
    shapes = [(t.shape[0], e - b) + tuple(t.shape[2:-1]) + (le - lb,) for b, e in chans]
    return torch.cat(_all_to_all(sends, shapes, group), dim=1).contiguous()


class AzimuthShards:
    """Longitudes (input and output grid) and input channels each rank of the azimuth group owns."""

    def __init__(self, nlon_in, nlon_out, in_channels, size: int):
        if in_channels < size:
            raise ValueError(f"{in_channels} input channels cannot be split over {size} azimuth ranks")
        self.lon_in = polar.split_rows(nlon_in, size)
        self.lon_out = polar.split_rows(nlon_out, size)
        self.chans = polar.split_rows(in_channels, size)


def channel_shard(in_channels: int, out_channels: int, groups: int, span):
    """Where the input channels span = (begin, end) sit in a weight w (C_out, C_in/groups, K):
    column cols[i] of the rows o with mask[o, i] (the rows of channel begin + i's group)."""
    cs = torch.arange(span[0], span[1])
    cg, og = in_channels // groups, out_channels // groups
    gs = cs // cg
    return cs - gs * cg, torch.arange(out_channels)[:, None] // og == gs[None, :]


def shard_weight(w, cols, mask):
    """(C_out, C_a, K): the dense weight of a channel shard, zero across groups."""
    cols, mask = cols.to(w.device), mask.to(w.device)
    return (w[:, cols, :] * mask[..., None].to(w.dtype)).contiguous()


def unshard_weight_grad(dws, cols, mask, out_channels: int, cols_per_group: int):
    """The adjoint of shard_weight: (C_out, C_a, K) -> (C_out, C_in/groups, K)."""
    cols, mask = cols.to(dws.device), mask.to(dws.device)
    dw = dws.new_zeros((out_channels, cols_per_group, dws.shape[2]))
    return dw.index_add_(1, cols, dws * mask[..., None].to(dws.dtype))


# ------------------------------------------------------------------ the layer

class _DistributedFn(torch.autograd.Function):

    @staticmethod
    def forward(ctx, x_own, w, bias, layer):
        L, ops, sh = layer, layer.ops, layer.shards
        x = x_own
        if L.halo:
            x = polar.halo_gather(L.bands, L.p, x, L.polar_group)
        xc = lon_to_chan(x, sh.lon_in, sh.chans, L.a, L.azimuth_group)
        if not L.fused:
            yc = ops.contract(L.psi, xc)
            y = chan_to_lon(yc, sh.lon_out, sh.chans, L.a, L.azimuth_group)
            # each rank owns its points outright unless the polar mode sums partials
            b = bias if (not L.rs or L.p == 0) else None
            out = ops.mix(y, w, b, L.groups)
            if L.rs:
                out = polar.reduce_scatter_rows(L.bands.out_rows, L.p, out, L.polar_group)
            ctx.save_for_backward(y, w)
        else:
            ws = L.shard_weight(w)
            b = bias if (L.a == 0 and (not L.rs or L.p == 0)) else None
            part = ops.forward_fused(L.psi, xc, ws, b)
            out = polar.reduce_scatter_dim(sh.lon_out, L.a, part, -1, L.azimuth_group)
            if L.rs:
                out = polar.reduce_scatter_rows(L.bands.out_rows, L.p, out, L.polar_group)
            ctx.save_for_backward(xc, w)
        ctx.layer = layer
        ctx.has_bias = bias is not None
        return out

    @staticmethod
    def backward(ctx, dout_own):
        saved, w = ctx.saved_tensors
        L, ops, sh = ctx.layer, ctx.layer.ops, ctx.layer.shards
        d = dout_own.contiguous()
        C_in = L.in_channels
        db = None
        if not L.fused:
            if L.rs:
                d = polar.all_gather_rows(L.bands.out_rows, L.p, d, L.polar_group)
            dy = ops.mix_adjoint(d, w, C_in, L.groups)
            dw, db = ops.mix_weight(d, saved, L.groups, ctx.has_bias)
            dyc = lon_to_chan(dy, sh.lon_out, sh.chans, L.a, L.azimuth_group)
            dxc = ops.contract_adjoint(L.psi, dyc)
            # dbias has seen this rank's longitudes and, in the reduce-scatter mode, every row
            db_group = L.azimuth_group if L.rs else None
        else:
            d = polar.all_gather_dim(sh.lon_out, L.a, d, -1, L.azimuth_group)
            if L.rs:
                d = polar.all_gather_rows(L.bands.out_rows, L.p, d, L.polar_group)
            ws = L.shard_weight(w)
            dxc = ops.backward_input(L.psi, d, ws, sh.chans[L.a][1] - sh.chans[L.a][0])
            dws, db = ops.backward_weight_x(L.psi, d, saved, ctx.has_bias)
            dw = L.unshard_weight_grad(dws)
            # dbias has seen every longitude and, in the reduce-scatter mode, every row
            db_group = "none" if L.rs else L.polar_group
        dx = chan_to_lon(dxc, sh.lon_in, sh.chans, L.a, L.azimuth_group)
        if L.halo:
            dx = polar.halo_reduce(L.bands, L.p, dx, L.polar_group)
        if L.world > 1:
            dist.all_reduce(dw)
            if db is not None and db_group != "none":
                dist.all_reduce(db, group=db_group)
        return dx, dw, db, None


class DistributedDiscoConvS2(torch.nn.Module):
    """DISCO convolution on a polar_size x azimuth_size grid of ranks (the default process group).

    Rank r = p * azimuth_size + a passes x (B, C_in, rows, lons) on its input latitudes
    bands.in_rows[p] and longitudes shards.lon_in[a], and gets out on its output latitudes
    bands.out_rows[p] and longitudes shards.lon_out[a].  Weights and bias are replicated (the
    same seed on every rank, or a broadcast, is the caller's business); their gradients are the
    full sums on every rank.
    """

    def __init__(self, in_channels, out_channels, in_shape, out_shape, kernel_shape, theta_cutoff, polar_size=None,
                 azimuth_size=1, polar_mode="halo-exchange", groups=1, grid_in="equiangular", grid_out="equiangular",
                 bias=True, fused=False, device=None, dtype=torch.float32, ops=None):
        super().__init__()
        if in_channels % groups or out_channels % groups:
            raise ValueError("groups must divide in_channels and out_channels")
        if polar_mode not in POLAR_MODES:
            raise ValueError(f"polar_mode is one of {POLAR_MODES}")
        self.world, rank = dist.get_world_size(), dist.get_rank()
        if polar_size is None:
            polar_size = self.world // azimuth_size
        if polar_size * azimuth_size != self.world:
            raise ValueError(f"polar_size {polar_size} x azimuth_size {azimuth_size} != world size {self.world}")
        self.P, self.A = polar_size, azimuth_size
        self.p, self.a = divmod(rank, azimuth_size)
        self.in_channels, self.out_channels, self.groups, self.fused = in_channels, out_channels, groups, fused
        self.polar_mode = polar_mode
        self.halo = polar_mode == "halo-exchange" and polar_size > 1
        self.rs = polar_mode == "reduce-scatter" and polar_size > 1
        self.ops = ops if ops is not None else KernelOps(device)
        # the groups of the grid's columns (polar) and rows (azimuth); every rank creates every
        # group, in the same order
        self.polar_group = self.azimuth_group = None
        for a in range(azimuth_size):
            g = dist.new_group([p * azimuth_size + a for p in range(polar_size)])
            if a == self.a:
                self.polar_group = g
        for p in range(polar_size):
            g = dist.new_group([p * azimuth_size + a for a in range(azimuth_size)])
            if p == self.p:
                self.azimuth_group = g
        geometry = (in_shape[0], in_shape[1], out_shape[0], out_shape[1], kernel_shape, theta_cutoff, grid_in,
                    grid_out)
        self.shards = AzimuthShards(in_shape[1], out_shape[1], in_channels, azimuth_size)
        if self.rs:
            self.bands = polar.InputBands(*geometry[:6], polar_size, grid_in, grid_out)
            self.psi = self.ops.psi(geometry, inputs=self.bands.in_rows[self.p])
        else:
            self.bands = polar.PolarBands(*geometry[:6], polar_size, grid_in, grid_out)
            self.psi = self.ops.psi(geometry, rows=self.bands.out_rows[self.p]) if self.halo else self.ops.psi(geometry)
        K = self.psi.K
        # where the channels of this rank's shard sit in w (fused=True)
        self._cols, self._mask = channel_shard(in_channels, out_channels, groups, self.shards.chans[self.a])
        cg = in_channels // groups
        # every rank joins one collective before the first point-to-point exchange
        if self.world > 1:
            dist.barrier()
        dev = getattr(self.psi, "device", None)
        scale = 1.0 / math.sqrt(cg * K)
        self.weight = torch.nn.Parameter(torch.randn(out_channels, cg, K, device=dev, dtype=dtype) * scale)
        self.bias = torch.nn.Parameter(torch.zeros(out_channels, device=dev, dtype=dtype)) if bias else None

    def shard_weight(self, w):
        return shard_weight(w, self._cols, self._mask)

    def unshard_weight_grad(self, dws):
        return unshard_weight_grad(dws, self._cols, self._mask, self.out_channels, self.in_channels // self.groups)

    def forward(self, x_own):
        return _DistributedFn.apply(x_own.contiguous(), self.weight, self.bias, self)
