"""Polar-band distribution of the DISCO layer: the "halo-exchange" polar mode.

Follows the polar_mode parameter on the page
"torch_harmonics.distributed.DistributedDiscreteContinuousConvS2": the data is split over
ranks in the polar (latitude) direction; a rank computes the output latitudes it owns outright,
borrowing the input rows those latitudes reach from its neighbours, so the K-expanded
intermediate shrinks with the number of ranks; a filter that reaches past the neighbouring
rank's rows is refused at construction.  Readings where the page is silent:

  * the latitudes are split into contiguous bands as evenly as possible, the first
    (n mod P) bands one row longer (input and output grids each split this way);
  * the backward pass is the adjoint of the forward one: each rank's input gradient on the
    borrowed rows is sent back to the rows' owners and summed there; dw and dbias are
    summed over ranks (all-reduce).

Every rank runs the same collective steps in the same order.  torch.distributed carries the
halo rows (NCCL over NVLink on GPUs, gloo on CPU); the contraction runs in libdisco's kernels
on each rank's band (disco_psi_build_band).
"""

from __future__ import annotations

import math

import torch
import torch.distributed as dist

from . import conv
from . import disco as D


def split_rows(n: int, parts: int):
    """[(begin, end)] of `parts` contiguous bands covering range(n), sizes differing by at most one."""
    if parts < 1 or n < parts:
        raise ValueError(f"cannot split {n} rows over {parts} ranks")
    q, r = divmod(n, parts)
    out, b = [], 0
    for p in range(parts):
        e = b + q + (1 if p < r else 0)
        out.append((b, e))
        b = e
    return out


class PolarBands:
    """Which rows each rank owns and borrows, for one layer geometry and `world` ranks.

    out_rows[r], in_rows[r]: the output / input latitudes rank r owns.  reach[r]: the input rows
    [i_begin, i_end) its output rows reach (from the band's Psi).  recv[r]: (src, lo, hi) input
    row ranges rank r borrows from rank src; send[r]: (dst, lo, hi) ranges it lends to dst.
    """

    def __init__(self, nlat_in, nlon_in, nlat_out, nlon_out, kernel_shape, theta_cutoff, world: int,
                 grid_in: str = "equiangular", grid_out: str = "equiangular"):
        self.world = world
        self.spec = D.make_spec(nlat_in, nlon_in, nlat_out, nlon_out, kernel_shape, theta_cutoff,
                                D.GRID_CODES[grid_in], D.GRID_CODES[grid_out])
        self.geometry = (nlat_in, nlon_in, nlat_out, nlon_out, kernel_shape, theta_cutoff, grid_in, grid_out)
        self.out_rows = split_rows(nlat_out, world)
        self.in_rows = split_rows(nlat_in, world)
        self.reach = []
        for jb, je in self.out_rows:
            h, ib, ie = D.disco_psi_build_band(self.spec, jb, je, -1)  # host-only: geometry only
            D.disco_psi_destroy(h)
            self.reach.append((ib, ie))
        self.recv = [[] for _ in range(world)]
        self.send = [[] for _ in range(world)]
        for r, (ib, ie) in enumerate(self.reach):
            lo_ok = self.in_rows[max(r - 1, 0)][0]
            hi_ok = self.in_rows[min(r + 1, world - 1)][1]
            if ib < lo_ok or ie > hi_ok:
                raise ValueError(
                    f"rank {r}'s output latitudes {self.out_rows[r]} reach input rows [{ib}, {ie}), beyond its "
                    f"neighbours' rows [{lo_ok}, {hi_ok}): the filter is too wide for {world} polar ranks")
            for s, (ob, oe) in enumerate(self.in_rows):
                lo, hi = max(ib, ob), min(ie, oe)
                if s != r and lo < hi:
                    self.recv[r].append((s, lo, hi))
                    self.send[s].append((r, lo, hi))


def _exchange(ops):
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()


def _peer(group, r: int) -> int:
    """Global rank of rank r of `group` (None: the default group)."""
    return r if group is None else dist.get_global_rank(group, r)


def halo_gather(bands: PolarBands, rank: int, x_own: torch.Tensor, group=None) -> torch.Tensor:
    """x on the rows rank `rank` reaches, [..., i_end - i_begin, nlon], from x on its own rows;
    ranks are those of `group` (None: the default group)."""
    ob, oe = bands.in_rows[rank]
    ib, ie = bands.reach[rank]
    if x_own.shape[-2] != oe - ob:
        raise ValueError(f"rank {rank} holds input rows [{ob}, {oe}); got {x_own.shape[-2]} rows")
    x_band = x_own.new_empty(x_own.shape[:-2] + (ie - ib, x_own.shape[-1]))
    lo, hi = max(ib, ob), min(ie, oe)
    if lo < hi:
        x_band[..., lo - ib:hi - ib, :] = x_own[..., lo - ob:hi - ob, :]
    ops, keep = [], []
    for dst, lo, hi in bands.send[rank]:
        buf = x_own[..., lo - ob:hi - ob, :].contiguous()
        keep.append(buf)
        ops.append(dist.P2POp(dist.isend, buf, _peer(group, dst), group))
    recvs = []
    for src, lo, hi in bands.recv[rank]:
        buf = x_own.new_empty(x_own.shape[:-2] + (hi - lo, x_own.shape[-1]))
        recvs.append((buf, lo))
        ops.append(dist.P2POp(dist.irecv, buf, _peer(group, src), group))
    _exchange(ops)
    for buf, lo in recvs:
        x_band[..., lo - ib:lo - ib + buf.shape[-2], :] = buf
    return x_band


def halo_reduce(bands: PolarBands, rank: int, g_band: torch.Tensor, group=None) -> torch.Tensor:
    """The adjoint of halo_gather: a gradient on the reached rows, summed onto each row's owner."""
    ob, oe = bands.in_rows[rank]
    ib, ie = bands.reach[rank]
    g_own = g_band.new_zeros(g_band.shape[:-2] + (oe - ob, g_band.shape[-1]))
    lo, hi = max(ib, ob), min(ie, oe)
    if lo < hi:
        g_own[..., lo - ob:hi - ob, :] += g_band[..., lo - ib:hi - ib, :]
    ops, keep, recvs = [], [], []
    for src, lo, hi in bands.recv[rank]:  # rows borrowed from src go back to src
        buf = g_band[..., lo - ib:hi - ib, :].contiguous()
        keep.append(buf)
        ops.append(dist.P2POp(dist.isend, buf, _peer(group, src), group))
    for dst, lo, hi in bands.send[rank]:  # rows lent to dst come back from dst
        buf = g_band.new_empty(g_band.shape[:-2] + (hi - lo, g_band.shape[-1]))
        recvs.append((buf, lo))
        ops.append(dist.P2POp(dist.irecv, buf, _peer(group, dst), group))
    _exchange(ops)
    for buf, lo in recvs:
        g_own[..., lo - ob:lo - ob + buf.shape[-2], :] += buf
    return g_own


class _PolarFn(torch.autograd.Function):
    """fused=False saves the band's K-expanded y; fused=True saves the halo-extended x and
    recomputes y in backward (the page's fused flag, orthogonal to the polar mode)."""

    @staticmethod
    def forward(ctx, x_own, w, bias, layer):
        x_band = halo_gather(layer.bands, layer.rank, x_own)
        out, y = conv.disco_forward(layer.psi, x_band, w, bias, layer.groups, fused=layer.fused)
        ctx.layer = layer
        ctx.has_bias = bias is not None
        ctx.C_in = x_own.shape[1]
        ctx.save_for_backward(x_band if layer.fused else y, w)
        return out

    @staticmethod
    def backward(ctx, dout):
        saved, w = ctx.saved_tensors
        layer = ctx.layer
        dout = dout.contiguous()
        dx_band = conv.disco_backward_input(layer.psi, dout, w, ctx.C_in, layer.groups)
        dx = halo_reduce(layer.bands, layer.rank, dx_band)
        if layer.fused:
            dw, db = conv.disco_backward_weight(layer.psi, dout, x=saved, groups=layer.groups,
                                                need_bias=ctx.has_bias)
        else:
            dw, db = conv.disco_backward_weight(layer.psi, dout, y=saved, groups=layer.groups,
                                                need_bias=ctx.has_bias)
        dist.all_reduce(dw)
        if db is not None:
            dist.all_reduce(db)
        return dx, dw, db, None


class PolarDiscoConvS2(torch.nn.Module):
    """DISCO convolution with its latitudes split over the ranks of the default process group.

    Each rank passes x on its own input latitudes (bands.in_rows[rank]) and gets out on its own
    output latitudes (bands.out_rows[rank]).  Weights and bias are replicated (same seed on every
    rank, or a broadcast, is the caller's business); their gradients are summed over ranks.
    """

    def __init__(self, in_channels, out_channels, in_shape, out_shape, kernel_shape, theta_cutoff, groups=1,
                 grid_in="equiangular", grid_out="equiangular", bias=True, fused=False, device=None,
                 dtype=torch.float32):
        super().__init__()
        if in_channels % groups or out_channels % groups:
            raise ValueError("groups must divide in_channels and out_channels")
        self.rank, world = dist.get_rank(), dist.get_world_size()
        self.groups, self.fused = groups, fused
        self.bands = PolarBands(in_shape[0], in_shape[1], out_shape[0], out_shape[1], kernel_shape, theta_cutoff,
                                world, grid_in, grid_out)
        jb, je = self.bands.out_rows[self.rank]
        self.psi = conv.Psi(in_shape[0], in_shape[1], out_shape[0], out_shape[1], kernel_shape, theta_cutoff, device,
                            grid_in, grid_out, rows=(jb, je))
        if self.psi.in_rows != self.bands.reach[self.rank]:
            raise RuntimeError("band Psi and band geometry disagree on the rows reached")
        # every rank joins one collective before the first point-to-point exchange (a rank
        # whose band borrows nothing issues no send or receive of its own)
        if world > 1:
            dist.barrier()
        K = self.psi.K
        scale = 1.0 / math.sqrt((in_channels // groups) * K)
        self.weight = torch.nn.Parameter(
            torch.randn(out_channels, in_channels // groups, K, device=self.psi.device, dtype=dtype) * scale)
        self.bias = torch.nn.Parameter(torch.zeros(out_channels, device=self.psi.device, dtype=dtype)) if bias \
            else None

    def forward(self, x_own):
        return _PolarFn.apply(x_own.contiguous(), self.weight, self.bias, self)


# ------------------------------------------------------------------ the "reduce-scatter" polar mode
#
# polar_mode="reduce-scatter" on the same page: every rank computes a partial sum over all output
# latitudes from the input latitudes it owns, and a reduce-scatter completes the sums and splits
# them by output band.  No bound on the angular reach; the partial sums stay at the full nlat_out.
# Readings where the page is silent:
#
#   * the reduce-scatter runs on out (C_out channels), after each rank's weight einsum of its
#     partial y, not on the K-expanded y: the einsum is linear, so the sums are the same with K
#     times less collective volume; rank 0's partial sum carries the bias, so it is added once;
#   * backward is the adjoint: dout on the rank's output rows is all-gathered to every output row,
#     each rank's dx is its input band's adjoint, dw is summed over ranks and dbias is the sum of
#     the gathered dout, the same on every rank.


class InputBands:
    """Input latitudes each rank owns (in_rows[r]) and output latitudes it receives the completed
    sums of (out_rows[r]), both split as evenly as possible into contiguous bands."""

    def __init__(self, nlat_in, nlon_in, nlat_out, nlon_out, kernel_shape, theta_cutoff, world: int,
                 grid_in: str = "equiangular", grid_out: str = "equiangular"):
        self.world = world
        self.spec = D.make_spec(nlat_in, nlon_in, nlat_out, nlon_out, kernel_shape, theta_cutoff,
                                D.GRID_CODES[grid_in], D.GRID_CODES[grid_out])
        self.geometry = (nlat_in, nlon_in, nlat_out, nlon_out, kernel_shape, theta_cutoff, grid_in, grid_out)
        self.in_rows = split_rows(nlat_in, world)
        self.out_rows = split_rows(nlat_out, world)
        self.nlat_out = nlat_out


def _padded(bands_rows):
    return max(e - b for b, e in bands_rows)


def reduce_scatter_dim(spans, rank: int, t: torch.Tensor, dim: int, group=None) -> torch.Tensor:
    """t partial over the ranks of `group` (None: the default group) -> the sum over them of
    t's slice spans[rank] = (begin, end) along dimension `dim`."""
    world = len(spans)
    dim = dim % t.dim()
    jb, je = spans[rank]
    if world == 1:
        return t.narrow(dim, jb, je - jb).contiguous()
    if dist.get_backend(group) == "nccl":
        # equal chunks of the longest span (padded with zeros), one reduce-scatter
        m = _padded(spans)
        tm = t.movedim(dim, -1)
        chunks = t.new_zeros((world,) + tm.shape[:-1] + (m,))
        for r, (b, e) in enumerate(spans):
            chunks[r, ..., : e - b] = tm[..., b:e]
        own = t.new_empty(tm.shape[:-1] + (m,))
        dist.reduce_scatter_tensor(own, chunks.reshape((world * chunks.shape[1],) + chunks.shape[2:]), group=group)
        return own[..., : je - jb].movedim(-1, dim).contiguous()
    # backends without reduce-scatter (gloo): the sum everywhere, then the rank's slice
    s = t.contiguous().clone()
    dist.all_reduce(s, group=group)
    return s.narrow(dim, jb, je - jb).contiguous()


def all_gather_dim(spans, rank: int, t_own: torch.Tensor, dim: int, group=None) -> torch.Tensor:
    """The adjoint of reduce_scatter_dim: every rank's slice, concatenated along `dim`."""
    world = len(spans)
    if world == 1:
        return t_own.contiguous()
    dim = dim % t_own.dim()
    m = _padded(spans)
    jb, je = spans[rank]
    tm = t_own.movedim(dim, -1)
    pad = t_own.new_zeros(tm.shape[:-1] + (m,))
    pad[..., : je - jb] = tm
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad.contiguous(), group=group)
    return torch.cat([parts[r][..., : e - b] for r, (b, e) in enumerate(spans)], dim=-1).movedim(-1, dim).contiguous()


def reduce_scatter_rows(out_rows, rank: int, t: torch.Tensor, group=None) -> torch.Tensor:
    """t[..., J, L] partial on every row -> the sum over the ranks of `group` (None: the default
    group) on rank's rows out_rows[rank]."""
    return reduce_scatter_dim(out_rows, rank, t, -2, group)


def all_gather_rows(out_rows, rank: int, t_own: torch.Tensor, group=None) -> torch.Tensor:
    """The adjoint of reduce_scatter_rows: every rank's rows, gathered onto every output row."""
    return all_gather_dim(out_rows, rank, t_own, -2, group)


class _ReduceScatterFn(torch.autograd.Function):
    """fused=False saves the band's partial y; fused=True runs the fused forward, saves x on the band
    and recomputes y in backward."""

    @staticmethod
    def forward(ctx, x_own, w, bias, layer):
        # rank 0's partial sum carries the bias, so the reduce-scatter adds it exactly once
        out_part, y = conv.disco_forward(layer.psi, x_own, w, bias if layer.rank == 0 else None, layer.groups,
                                         fused=layer.fused)
        out = reduce_scatter_rows(layer.bands.out_rows, layer.rank, out_part)
        ctx.layer = layer
        ctx.has_bias = bias is not None
        ctx.C_in = x_own.shape[1]
        ctx.save_for_backward(x_own if layer.fused else y, w)
        return out

    @staticmethod
    def backward(ctx, dout_own):
        saved, w = ctx.saved_tensors
        layer = ctx.layer
        dout_own = dout_own.contiguous()
        dout = all_gather_rows(layer.bands.out_rows, layer.rank, dout_own)
        dx = conv.disco_backward_input(layer.psi, dout, w, ctx.C_in, layer.groups)
        # dw is the band's part (summed over ranks); dbias comes from dout on every output row,
        # the same complete sum on every rank
        if layer.fused:
            dw, db = conv.disco_backward_weight(layer.psi, dout, x=saved, groups=layer.groups,
                                                need_bias=ctx.has_bias)
        else:
            dw, db = conv.disco_backward_weight(layer.psi, dout, y=saved, groups=layer.groups,
                                                need_bias=ctx.has_bias)
        dist.all_reduce(dw)
        return dx, dw, db, None


class PolarReduceScatterConvS2(torch.nn.Module):
    """DISCO convolution, latitudes split over the ranks of the default process group in the
    reduce-scatter polar mode: rank r passes x on its input latitudes (bands.in_rows[r]) and gets
    out on its output latitudes (bands.out_rows[r]).  Weights and bias are replicated; their
    gradients are summed over ranks."""

    def __init__(self, in_channels, out_channels, in_shape, out_shape, kernel_shape, theta_cutoff, groups=1,
                 grid_in="equiangular", grid_out="equiangular", bias=True, fused=False, device=None,
                 dtype=torch.float32):
        super().__init__()
        if in_channels % groups or out_channels % groups:
            raise ValueError("groups must divide in_channels and out_channels")
        self.rank, world = dist.get_rank(), dist.get_world_size()
        self.groups, self.fused = groups, fused
        self.bands = InputBands(in_shape[0], in_shape[1], out_shape[0], out_shape[1], kernel_shape, theta_cutoff,
                                world, grid_in, grid_out)
        self.psi = conv.Psi(in_shape[0], in_shape[1], out_shape[0], out_shape[1], kernel_shape, theta_cutoff, device,
                            grid_in, grid_out, inputs=self.bands.in_rows[self.rank])
        K = self.psi.K
        scale = 1.0 / math.sqrt((in_channels // groups) * K)
        self.weight = torch.nn.Parameter(
            torch.randn(out_channels, in_channels // groups, K, device=self.psi.device, dtype=dtype) * scale)
        self.bias = torch.nn.Parameter(torch.zeros(out_channels, device=self.psi.device, dtype=dtype)) if bias \
            else None

    def forward(self, x_own):
        return _ReduceScatterFn.apply(x_own.contiguous(), self.weight, self.bias, self)
