"""PyTorch-facing DISCO layer on top of the libdisco C ABI.

PyTorch supplies device memory, streams and autograd bookkeeping; every step
of the convolution runs in libdisco's CUDA kernels (there is no CPU path).
The layer mirrors the constructor of the page
"torch_harmonics.DiscreteContinuousConvS2": in/out channels and shapes,
kernel_shape, basis_type='piecewise linear', basis_norm_mode='nodal',
groups, grid_in / grid_out, bias, theta_cutoff and `fused`.  With
fused=False the K-expanded intermediate is saved for backward; with
fused=True only x is saved and the intermediate is recomputed in backward
(K times less activation memory, one extra contraction).
"""

from __future__ import annotations

import math

import torch

from . import disco as D

_DTYPES = {torch.float32: D.DISCO_F32, torch.bfloat16: D.DISCO_BF16}


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype not in _DTYPES:
        raise TypeError(f"unsupported dtype {t.dtype}; use float32 or bfloat16")
    return _DTYPES[t.dtype]


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("libdisco takes contiguous CUDA tensors")
    dts = {t.dtype for t in ts if t is not None}
    if len(dts) > 1:
        raise TypeError(f"libdisco takes tensors of one dtype; got {sorted(map(str, dts))}")


def _shape(t, want, what):
    """The C ABI sees only pointers: every tensor's shape is checked here, before a kernel reads it."""
    if t is not None and tuple(t.shape) != tuple(want):
        raise ValueError(f"{what} has shape {tuple(t.shape)}, expected {tuple(want)}")


def _weight(w, C_out, C_in, groups, K):
    if groups <= 0 or C_in % groups or C_out % groups:
        raise ValueError(f"groups={groups} must divide C_in={C_in} and C_out={C_out}")
    _shape(w, (C_out, C_in // groups, K), "w")


class Psi:
    """Precomputed sparse convolution tensor of one layer geometry, on one device."""

    def __init__(self, nlat_in: int, nlon_in: int, nlat_out: int, nlon_out: int, kernel_shape, theta_cutoff: float,
                 device=None, grid_in: str = "equiangular", grid_out: str = "equiangular", rows=None,
                 inputs=None):
        """rows=(j_begin, j_end) builds the Psi of those output latitudes only (a polar band): the
        handle then takes x on input rows self.in_rows = (i_begin, i_end) and gives out rows
        j_begin..j_end-1.  inputs=(i_begin, i_end) builds the Psi of those input latitudes over
        every output latitude (a band's partial sums, the reduce-scatter polar mode)."""
        dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.device = dev
        self.index = dev.index if dev.index is not None else torch.cuda.current_device()
        self.in_shape = (nlat_in, nlon_in)
        self.out_shape = (nlat_out, nlon_out)
        self.in_rows = (0, nlat_in)
        self.kernel_shape = kernel_shape
        self.theta_cutoff = float(theta_cutoff)
        if grid_in not in D.GRID_CODES or grid_out not in D.GRID_CODES:
            raise ValueError(f"grids are one of {sorted(D.GRID_CODES)}")
        self.grid_in, self.grid_out = grid_in, grid_out
        self.spec = D.make_spec(nlat_in, nlon_in, nlat_out, nlon_out, kernel_shape, theta_cutoff,
                                D.GRID_CODES[grid_in], D.GRID_CODES[grid_out])
        with torch.cuda.device(self.index):
            if inputs is not None:
                self.handle = D.disco_psi_build_inputs(self.spec, inputs[0], inputs[1], self.index)
                self.in_rows = (inputs[0], inputs[1])
                self.in_shape = (inputs[1] - inputs[0], nlon_in)
            elif rows is None:
                self.handle = D.disco_psi_build(self.spec, self.index)
            else:
                self.handle, ib, ie = D.disco_psi_build_band(self.spec, rows[0], rows[1], self.index)
                self.in_rows = (ib, ie)
                self.in_shape = (ie - ib, nlon_in)
                self.out_shape = (rows[1] - rows[0], nlon_out)
        self.K, self.nnz = D.disco_psi_info(self.handle)

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and D is not None:
            try:
                D.disco_psi_destroy(h)
            except Exception:
                pass
            self.handle = None

    def workspace(self, op: int, B: int, C_in: int, C_out: int, groups: int, dtype: int):
        n = D.disco_workspace_size(self.handle, op, B, C_in, C_out, groups, dtype)
        if n == 0:
            return None, 0
        return torch.empty(n, dtype=torch.uint8, device=self.device), n


def disco_contract(psi: Psi, x: torch.Tensor) -> torch.Tensor:
    """y = the K-expanded contraction of x with Psi, shape (B, C, K, nlat_out, nlon_out)."""
    _need_cuda(x)
    B, C = x.shape[:2]
    _shape(x, (B, C) + psi.in_shape, "x")
    y = torch.empty((B, C, psi.K) + psi.out_shape, dtype=x.dtype, device=x.device)
    D.disco_contract(psi.handle, B, C, _dtype_code(x), _ptr(x), _ptr(y), _stream(x.device))
    return y


def disco_forward(psi: Psi, x: torch.Tensor, w: torch.Tensor, bias=None, groups: int = 1, fused: bool = False):
    """Returns (out, y); y is None when fused."""
    _need_cuda(x, w, bias)
    B, C_in = x.shape[:2]
    C_out = w.shape[0]
    _shape(x, (B, C_in) + psi.in_shape, "x")
    _weight(w, C_out, C_in, groups, psi.K)
    _shape(bias, (C_out,), "bias")
    dt = _dtype_code(x)
    out = torch.empty((B, C_out) + psi.out_shape, dtype=x.dtype, device=x.device)
    st = _stream(x.device)
    if fused:
        ws, n = psi.workspace(D.DISCO_OP_FWD_FUSED, B, C_in, C_out, groups, dt)
        D.disco_fwd_fused(psi.handle, B, C_in, C_out, groups, dt, _ptr(x), _ptr(w), _ptr(bias), _ptr(out),
                          _ptr(ws), n, st)
        return out, None
    y = torch.empty((B, C_in, psi.K) + psi.out_shape, dtype=x.dtype, device=x.device)
    ws, n = psi.workspace(D.DISCO_OP_FWD, B, C_in, C_out, groups, dt)
    D.disco_fwd(psi.handle, B, C_in, C_out, groups, dt, _ptr(x), _ptr(w), _ptr(bias), _ptr(y), _ptr(out),
                _ptr(ws), n, st)
    return out, y


def disco_backward_input(psi: Psi, dout: torch.Tensor, w: torch.Tensor, C_in: int, groups: int = 1):
    _need_cuda(dout, w)
    B, C_out = dout.shape[:2]
    _shape(dout, (B, C_out) + psi.out_shape, "dout")
    _weight(w, C_out, C_in, groups, psi.K)
    dt = _dtype_code(dout)
    dx = torch.empty((B, C_in) + psi.in_shape, dtype=dout.dtype, device=dout.device)
    ws, n = psi.workspace(D.DISCO_OP_BWD_INPUT, B, C_in, C_out, groups, dt)
    D.disco_bwd_input(psi.handle, B, C_in, C_out, groups, dt, _ptr(dout), _ptr(w), _ptr(dx), _ptr(ws), n,
                      _stream(dout.device))
    return dx


def disco_backward_weight(psi: Psi, dout: torch.Tensor, y=None, x=None, groups: int = 1, C_in: int = None,
                          need_bias: bool = True):
    """(dw, dbias); y given, or x to recompute y."""
    _need_cuda(dout, y, x)
    if y is None and x is None:
        raise ValueError("give y, or x to recompute it")
    B, C_out = dout.shape[:2]
    C_in = y.shape[1] if y is not None else x.shape[1]
    _shape(dout, (B, C_out) + psi.out_shape, "dout")
    _shape(y, (B, C_in, psi.K) + psi.out_shape, "y")
    _shape(x, (B, C_in) + psi.in_shape, "x")
    _weight(None, C_out, C_in, groups, psi.K)
    dt = _dtype_code(dout)
    dw = torch.empty((C_out, C_in // groups, psi.K), dtype=dout.dtype, device=dout.device)
    db = torch.empty((C_out,), dtype=dout.dtype, device=dout.device) if need_bias else None
    op = D.DISCO_OP_BWD_WEIGHT if y is not None else D.DISCO_OP_BWD_WEIGHT_RECOMPUTE
    ws, n = psi.workspace(op, B, C_in, C_out, groups, dt)
    D.disco_bwd_weight(psi.handle, B, C_in, C_out, groups, dt, _ptr(dout), _ptr(y), _ptr(x), _ptr(dw), _ptr(db),
                       _ptr(ws), n, _stream(dout.device))
    return dw, db


def disco_contract_adjoint(psi: Psi, dy: torch.Tensor) -> torch.Tensor:
    """dx = the adjoint of the contraction applied to dy (B, C, K, nlat_out, nlon_out)."""
    _need_cuda(dy)
    B, C = dy.shape[:2]
    _shape(dy, (B, C, psi.K) + psi.out_shape, "dy")
    dx = torch.empty((B, C) + psi.in_shape, dtype=dy.dtype, device=dy.device)
    D.disco_contract_adjoint(psi.handle, B, C, _dtype_code(dy), _ptr(dy), _ptr(dx), _stream(dy.device))
    return dx


def mix(y: torch.Tensor, w: torch.Tensor, bias=None, groups: int = 1) -> torch.Tensor:
    """The weight einsum on any set of points: y (B, C_in, K, *pts) -> out (B, C_out, *pts)."""
    _need_cuda(y, w, bias)
    y = y.contiguous()
    if y.dim() < 4:
        raise ValueError(f"y has shape {tuple(y.shape)}, expected (B, C_in, K, *points)")
    B, C_in, K = y.shape[:3]
    pts = y.shape[3:]
    C_out = w.shape[0]
    _weight(w, C_out, C_in, groups, K)
    _shape(bias, (C_out,), "bias")
    out = torch.empty((B, C_out) + pts, dtype=y.dtype, device=y.device)
    D.disco_mix(B, C_in, C_out, groups, K, math.prod(pts), _dtype_code(y), _ptr(y), _ptr(w), _ptr(bias), _ptr(out),
                _stream(y.device))
    return out


def mix_adjoint(dout: torch.Tensor, w: torch.Tensor, C_in: int, groups: int = 1) -> torch.Tensor:
    """The transposed weight einsum: dout (B, C_out, *pts) -> dy (B, C_in, K, *pts)."""
    _need_cuda(dout, w)
    dout = dout.contiguous()
    if dout.dim() < 3 or w.dim() != 3:
        raise ValueError("dout is (B, C_out, *points) and w (C_out, C_in/groups, K)")
    B, C_out = dout.shape[:2]
    pts = dout.shape[2:]
    K = w.shape[2]
    _weight(w, C_out, C_in, groups, K)
    dt, n = _dtype_code(dout), math.prod(pts)
    dy = torch.empty((B, C_in, K) + pts, dtype=dout.dtype, device=dout.device)
    nb = D.disco_mix_workspace_size(D.DISCO_OP_EINSUM_ADJOINT, B, C_in, C_out, groups, K, n, dt)
    ws = torch.empty(nb, dtype=torch.uint8, device=dout.device)
    D.disco_mix_adjoint(B, C_in, C_out, groups, K, n, dt, _ptr(dout), _ptr(w), _ptr(dy), _ptr(ws), nb,
                        _stream(dout.device))
    return dy


def mix_weight(dout: torch.Tensor, y: torch.Tensor, groups: int = 1, need_bias: bool = True):
    """(dw, dbias) of the weight einsum on any set of points: dout (B, C_out, *pts), y (B, C_in, K, *pts)."""
    _need_cuda(dout, y)
    dout, y = dout.contiguous(), y.contiguous()
    B, C_out = dout.shape[:2]
    C_in, K = y.shape[1:3]
    _shape(y, (B, C_in, K) + tuple(dout.shape[2:]), "y")
    _weight(None, C_out, C_in, groups, K)
    dt, n = _dtype_code(dout), math.prod(dout.shape[2:])
    dw = torch.empty((C_out, C_in // groups, K), dtype=dout.dtype, device=dout.device)
    db = torch.empty((C_out,), dtype=dout.dtype, device=dout.device) if need_bias else None
    nb = D.disco_mix_workspace_size(D.DISCO_OP_BWD_WEIGHT, B, C_in, C_out, groups, K, n, dt)
    ws = torch.empty(nb, dtype=torch.uint8, device=dout.device)
    D.disco_mix_weight(B, C_in, C_out, groups, K, n, dt, _ptr(dout), _ptr(y), _ptr(dw), _ptr(db), _ptr(ws), nb,
                       _stream(dout.device))
    return dw, db


class _DiscoFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, w, bias, psi, groups):
        out, y = disco_forward(psi, x.contiguous(), w.contiguous(), None if bias is None else bias.contiguous(),
                               groups, fused=False)
        ctx.save_for_backward(y, w)
        ctx.psi, ctx.groups, ctx.C_in, ctx.has_bias = psi, groups, x.shape[1], bias is not None
        return out

    @staticmethod
    def backward(ctx, dout):
        y, w = ctx.saved_tensors
        dout = dout.contiguous()
        dx = disco_backward_input(ctx.psi, dout, w, ctx.C_in, ctx.groups) if ctx.needs_input_grad[0] else None
        dw, db = disco_backward_weight(ctx.psi, dout, y=y, groups=ctx.groups, need_bias=ctx.has_bias)
        return dx, dw, db, None, None


class _DiscoFusedFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, w, bias, psi, groups):
        x = x.contiguous()
        out, _ = disco_forward(psi, x, w.contiguous(), None if bias is None else bias.contiguous(), groups,
                               fused=True)
        ctx.save_for_backward(x, w)
        ctx.psi, ctx.groups, ctx.has_bias = psi, groups, bias is not None
        return out

    @staticmethod
    def backward(ctx, dout):
        x, w = ctx.saved_tensors
        dout = dout.contiguous()
        dx = disco_backward_input(ctx.psi, dout, w, x.shape[1], ctx.groups) if ctx.needs_input_grad[0] else None
        dw, db = disco_backward_weight(ctx.psi, dout, x=x, groups=ctx.groups, need_bias=ctx.has_bias)
        return dx, dw, db, None, None


class DiscreteContinuousConvS2(torch.nn.Module):
    """DISCO convolution on the 2-sphere (piecewise-linear basis, nodal norm; grid_in / grid_out one of
    "equiangular", "legendre-gauss", "lobatto", "equiangular-trapezoidal")."""

    def __init__(self, in_channels, out_channels, in_shape, out_shape, kernel_shape, basis_type="piecewise linear",
                 basis_norm_mode="nodal", groups=1, grid_in="equiangular", grid_out="equiangular", bias=True,
                 theta_cutoff=None, optimized_kernel=True, fused=False, device=None, dtype=torch.float32):
        super().__init__()
        if basis_type != "piecewise linear" or basis_norm_mode != "nodal":
            raise NotImplementedError("only basis_type='piecewise linear' with basis_norm_mode='nodal'")
        if theta_cutoff is None:
            raise ValueError("theta_cutoff is required (no default is defined for it)")
        if not optimized_kernel:
            raise NotImplementedError("only the CUDA kernels exist")
        if in_channels % groups or out_channels % groups:
            raise ValueError("groups must divide in_channels and out_channels")
        self.groups, self.fused = groups, fused
        self.psi = Psi(in_shape[0], in_shape[1], out_shape[0], out_shape[1], kernel_shape, theta_cutoff, device,
                       grid_in, grid_out)
        K = self.psi.K
        scale = 1.0 / math.sqrt((in_channels // groups) * K)
        self.weight = torch.nn.Parameter(
            torch.randn(out_channels, in_channels // groups, K, device=self.psi.device, dtype=dtype) * scale)
        self.bias = torch.nn.Parameter(torch.zeros(out_channels, device=self.psi.device, dtype=dtype)) if bias \
            else None

    def forward(self, x):
        fn = _DiscoFusedFn if self.fused else _DiscoFn
        return fn.apply(x, self.weight, self.bias, self.psi, self.groups)
