"""GPU parity: libdisco's CUDA path against the CPU oracle, element by element.

Tolerances (max-abs error relative to the oracle's L-infinity norm): 1e-4 for
fp32 layers, 2e-2 for bf16-storage layers.  Inputs are the seeded workloads;
bf16 layers take the same bf16-representable values on both sides.  All five
workloads run at full size; the K-expanded y of the two largest is compared
on a subset of channel planes (every element of those planes).
"""

import functools
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
from spherical_disco_convolution_b200 import conv  # noqa: E402
from spherical_disco_convolution_b200 import disco as D  # noqa: E402
from spherical_disco_convolution_b200.workloads import WORKLOADS, Workload, make_inputs  # noqa: E402

pytestmark = pytest.mark.gpu

ALL = ["tiny", "mid", "downsample", "weather", "grouped"]

# Small geometries with ragged tails (nlon_out not a multiple of the 8-output task or of the
# block), odd latitude counts, stride-2 downsampling, groups, no bias, and channel counts that
# leave a partial channel block.
EDGE = {
    "ragged_iso_f32": Workload("ragged_iso_f32", 3, 6, 9, 3, 13, 20, 13, 20, (3, 1), 0.61, "f32"),
    "ragged_down_bf16": Workload("ragged_down_bf16", 3, 6, 9, 3, 19, 24, 10, 12, (3, 4), 0.7, "bf16", bias=False),
    "wide_row_f32": Workload("wide_row_f32", 2, 5, 4, 1, 33, 264, 33, 132, (5, 1), 0.35, "f32"),
    "aniso_k9_f32": Workload("aniso_k9_f32", 1, 17, 17, 1, 21, 40, 21, 40, (3, 4), 0.5, "f32"),
    # bf16 layers small enough to debug that still take the tensor-core paths (TMA-aligned rows,
    # channel counts in multiples of 16/32) with partial 128-wide tiles
    "tc_small_bf16": Workload("tc_small_bf16", 2, 32, 64, 2, 33, 64, 33, 64, (3, 1), 0.3, "bf16"),
    "tc_down_bf16": Workload("tc_down_bf16", 1, 16, 32, 1, 33, 128, 17, 64, (3, 4), 0.5, "bf16"),
    # layers of the fused tensor-core forward (64 input channels per group): two groups with a
    # ragged last 128-output block, and K = 5 with one contraction accumulator buffer
    "tz_fused_k3": Workload("tz_fused_k3", 2, 128, 64, 2, 33, 192, 33, 192, (3, 1), 0.3, "bf16"),
    "tz_fused_k5": Workload("tz_fused_k5", 1, 64, 48, 1, 25, 64, 25, 64, (5, 1), 0.45, "bf16", bias=False),
    # cutoff of two grid spacings, as on the 721x1440 layer: full-ring polar windows; 70 channels
    # take the plane-pair form of the strip-staged contraction with a partial second group of 64
    "ring_k3": Workload("ring_k3", 1, 70, 64, 1, 65, 128, 65, 128, (3, 1), 2 * math.pi / 64, "bf16"),
    # fused tensor-core forward with K = 9: one-half tiles of 64 outputs (ragged last tile)
    "tz_fused_k9": Workload("tz_fused_k9", 1, 128, 96, 2, 21, 160, 21, 160, (3, 4), 0.5, "bf16"),
    # fused forward on the TMA-staged strip kernel (64 channels per batch element, mirror rows):
    # two batch elements, 48 output channels, a ragged last longitude tile and full-ring polar
    # windows; and 64 output channels without bias
    "ring_fused_k3": Workload("ring_fused_k3", 2, 64, 48, 1, 49, 160, 49, 160, (3, 1), 2 * math.pi / 48, "bf16"),
    "ring_fused_nb": Workload("ring_fused_nb", 1, 64, 64, 1, 33, 96, 33, 96, (3, 1), 0.3, "bf16", bias=False),
    # input gradient on the same kernel (64 output channels, 32 input channels, two batch elements)
    "ring_dx_k3": Workload("ring_dx_k3", 2, 32, 64, 1, 49, 160, 49, 160, (3, 1), 2 * math.pi / 48, "bf16"),
}


def tol(wl):
    return 1e-4 if wl.dtype == "f32" else 2e-2


def workload(name):
    return WORKLOADS[name] if name in WORKLOADS else EDGE[name]


def ospec(wl):
    return oracle.Spec(wl.nlat_in, wl.nlon_in, wl.nlat_out, wl.nlon_out, wl.kernel_shape[0], wl.kernel_shape[1],
                       wl.theta_cutoff)


@functools.lru_cache(maxsize=None)
def inputs(name):
    return make_inputs(workload(name), 0)


@functools.lru_cache(maxsize=None)
def oracle_psi(name):
    return oracle.Psi(ospec(workload(name)))


@functools.lru_cache(maxsize=None)
def oracle_out(name):
    wl, inp = workload(name), inputs(name)
    return oracle_psi(name).forward(inp["x"], inp["w"], inp["bias"], groups=wl.groups)


@functools.lru_cache(maxsize=None)
def oracle_dx(name):
    wl, inp = workload(name), inputs(name)
    return oracle_psi(name).backward_input(inp["dout"], inp["w"], wl.C_in, groups=wl.groups)


@functools.lru_cache(maxsize=None)
def oracle_dw(name):
    wl, inp = workload(name), inputs(name)
    return oracle_psi(name).backward_weight(inp["dout"], inp["x"], groups=wl.groups)


@functools.lru_cache(maxsize=None)
def gpu_psi(name):
    wl = workload(name)
    return conv.Psi(wl.nlat_in, wl.nlon_in, wl.nlat_out, wl.nlon_out, wl.kernel_shape, wl.theta_cutoff, "cuda:0")


def dev(a, wl):
    if a is None:
        return None
    dt = torch.float32 if wl.dtype == "f32" else torch.bfloat16
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda:0").to(dt)


def host(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def check(got, ref, rel, what):
    err = np.abs(got - ref).max()
    scale = np.abs(ref).max()
    assert np.isfinite(err) and err <= rel * scale, f"{what}: max err {err:.3e} > {rel:g} x {scale:.3e}"


@pytest.fixture(scope="module", autouse=True)
def need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def y_channels(wl):
    """Channel planes of y compared element by element."""
    if wl.B * wl.C_in * wl.K * wl.nlat_out * wl.nlon_out <= 64_000_000:
        return None  # all
    return [0, 1, wl.C_in // 2, wl.C_in - 1]


@pytest.mark.parametrize("name", ALL + list(EDGE))
def test_forward_matches_oracle(name):
    wl, inp = workload(name), inputs(name)
    out, y = conv.disco_forward(gpu_psi(name), dev(inp["x"], wl), dev(inp["w"], wl), dev(inp["bias"], wl),
                                wl.groups)
    torch.cuda.synchronize()
    check(host(out), oracle_out(name), tol(wl), "out")
    sel = y_channels(wl)
    if sel is None:
        y_ref = oracle_psi(name).contract(inp["x"])
        check(host(y), y_ref, tol(wl), "y")
    else:
        y_ref = oracle_psi(name).contract(inp["x"][:, sel])
        check(host(y[:, sel]), y_ref, tol(wl), "y (sampled channel planes)")


@pytest.mark.parametrize("name", ALL + list(EDGE))
def test_fused_forward_matches_oracle(name):
    wl, inp = workload(name), inputs(name)
    out, y = conv.disco_forward(gpu_psi(name), dev(inp["x"], wl), dev(inp["w"], wl), dev(inp["bias"], wl),
                                wl.groups, fused=True)
    torch.cuda.synchronize()
    assert y is None
    check(host(out), oracle_out(name), tol(wl), "fused out")


@pytest.mark.parametrize("name", ALL + list(EDGE))
def test_backward_input_matches_oracle(name):
    wl, inp = workload(name), inputs(name)
    dx = conv.disco_backward_input(gpu_psi(name), dev(inp["dout"], wl), dev(inp["w"], wl), wl.C_in, wl.groups)
    torch.cuda.synchronize()
    check(host(dx), oracle_dx(name), tol(wl), "dx")


@pytest.mark.parametrize("name", ALL + list(EDGE))
def test_backward_weight_matches_oracle(name):
    wl, inp = workload(name), inputs(name)
    psi = gpu_psi(name)
    x = dev(inp["x"], wl)
    _, y = conv.disco_forward(psi, x, dev(inp["w"], wl), dev(inp["bias"], wl), wl.groups)
    dout = dev(inp["dout"], wl)
    dw_ref, db_ref = oracle_dw(name)
    dw, db = conv.disco_backward_weight(psi, dout, y=y, groups=wl.groups)
    dw2, db2 = conv.disco_backward_weight(psi, dout, x=x, groups=wl.groups)
    torch.cuda.synchronize()
    check(host(dw), dw_ref, tol(wl), "dw")
    check(host(db), db_ref, tol(wl), "dbias")
    check(host(dw2), dw_ref, tol(wl), "dw (recomputed y)")
    # deterministic: the split-K reduction runs in a fixed order
    dw3, _ = conv.disco_backward_weight(psi, dout, y=y, groups=wl.groups)
    assert torch.equal(dw, dw3)


def test_autograd_layer_matches_oracle():
    name = "ragged_down_bf16"
    wl, inp = workload(name), inputs(name)
    for fused in (False, True):
        layer = conv.DiscreteContinuousConvS2(wl.C_in, wl.C_out, (wl.nlat_in, wl.nlon_in),
                                              (wl.nlat_out, wl.nlon_out), wl.kernel_shape, groups=wl.groups,
                                              bias=False, theta_cutoff=wl.theta_cutoff, fused=fused,
                                              device="cuda:0", dtype=torch.bfloat16)
        with torch.no_grad():
            layer.weight.copy_(dev(inp["w"], wl))
        x = dev(inp["x"], wl).requires_grad_(True)
        out = layer(x)
        out.backward(dev(inp["dout"], wl))
        torch.cuda.synchronize()
        check(host(out), oracle_out(name), tol(wl), "layer out")
        check(host(x.grad), oracle_dx(name), tol(wl), "layer dx")
        check(host(layer.weight.grad), oracle_dw(name)[0], tol(wl), "layer dw")


def test_invalid_calls_raise():
    wl = workload("ragged_iso_f32")
    psi = gpu_psi("ragged_iso_f32")
    x = torch.zeros((0, wl.C_in, wl.nlat_in, wl.nlon_in), device="cuda:0")
    w = torch.zeros((wl.C_out, wl.C_in // wl.groups, wl.K), device="cuda:0")
    with pytest.raises(D.DiscoError) as e:
        conv.disco_forward(psi, x, w, None, wl.groups)
    assert e.value.status == D.DISCO_ERR_INVALID_ARG
    x = torch.zeros((1, wl.C_in, wl.nlat_in, wl.nlon_in), device="cuda:0")
    y = torch.zeros((1, wl.C_in, wl.K, wl.nlat_out, wl.nlon_out), device="cuda:0")
    out = torch.zeros((1, wl.C_out, wl.nlat_out, wl.nlon_out), device="cuda:0")
    st = torch.cuda.current_stream().cuda_stream
    with pytest.raises(D.DiscoError) as e:  # the library's own check, under the Python layer's
        D.disco_fwd(psi.handle, 1, wl.C_in, wl.C_out, 4, D.DISCO_F32, x.data_ptr(), w.data_ptr(), None, y.data_ptr(),
                    out.data_ptr(), None, 0, st)  # 4 divides neither 6 nor 9
    assert e.value.status == D.DISCO_ERR_INVALID_ARG
    # the Python layer checks every shape before a kernel sees a pointer
    with pytest.raises(ValueError):
        conv.disco_forward(psi, x, w, None, 4)
    with pytest.raises(ValueError):  # x of another grid
        conv.disco_contract(psi, torch.zeros((1, wl.C_in, wl.nlat_in, wl.nlon_in + 1), device="cuda:0"))
    with pytest.raises(ValueError):  # dy without its K axis
        conv.disco_contract_adjoint(psi, torch.zeros((1, wl.C_in * wl.K, wl.nlat_out, wl.nlon_out), device="cuda:0"))
    with pytest.raises(ValueError):  # w of another K
        conv.mix(y, w[:, :, :1].contiguous(), None, wl.groups)
    with pytest.raises(ValueError):  # y on other points than dout
        conv.mix_weight(out, y[..., :-1].contiguous(), wl.groups)
    with pytest.raises(TypeError):  # mixed dtypes
        conv.disco_forward(psi, x, w.to(torch.bfloat16), None, wl.groups)


@pytest.mark.parametrize("name", ["tc_small_bf16", "ring_k3", "weather", "grouped"])
def test_contract_tensor_core_matches_gather(name, monkeypatch):
    """The Toeplitz tensor-core contraction (bf16, stride 1) against the gather kernels and the
    oracle: both paths round y to bf16 once, so they agree to a few bf16 units."""
    wl, inp = workload(name), inputs(name)
    sel = y_channels(wl)
    x = dev(inp["x"], wl)
    if sel is not None:
        x = x[:, sel].contiguous()
    y_tc = conv.disco_contract(gpu_psi(name), x)
    monkeypatch.setenv("DISCO_SIMT_CONTRACT", "1")
    psi_simt = conv.Psi(wl.nlat_in, wl.nlon_in, wl.nlat_out, wl.nlon_out, wl.kernel_shape, wl.theta_cutoff,
                        "cuda:0")
    y_g = conv.disco_contract(psi_simt, x)
    torch.cuda.synchronize()
    x_ref = inp["x"] if sel is None else inp["x"][:, sel]
    y_ref = oracle_psi(name).contract(x_ref)
    # The tensor-core blocks hold each Psi value rounded once to bf16 and y is rounded once to
    # bf16 (8 significant bits: relative error <= u = 2^-8 each): with Psi >= 0 and every (k, j)
    # row summing to one, the error is at most u (max|x| + max|y|), plus the same y rounding on the
    # gather side.
    u = 2.0 ** -8
    bound = u * (np.abs(x_ref).max() + np.abs(y_ref).max())
    err = np.abs(host(y_tc) - y_ref).max()
    assert err <= 1.05 * bound, f"y (tensor cores): max err {err:.3e} > bound {bound:.3e}"
    err_g = np.abs(host(y_tc) - host(y_g)).max()
    assert err_g <= 1.05 * (bound + u * np.abs(y_ref).max()), f"y (tensor cores vs gather): {err_g:.3e}"
    check(host(y_tc), y_ref, tol(wl), "y (tensor cores, bf16 tolerance)")


@pytest.mark.parametrize("name", ["tc_small_bf16", "ring_k3", "weather", "grouped"])
def test_adjoint_tensor_core_matches_gather(name, monkeypatch):
    """dx through the reversed-Psi Toeplitz blocks on tensor cores against the gather kernels and
    the oracle (bf16, stride 1)."""
    wl, inp = workload(name), inputs(name)
    dout, w = dev(inp["dout"], wl), dev(inp["w"], wl)
    dx_tc = conv.disco_backward_input(gpu_psi(name), dout, w, wl.C_in, wl.groups)
    monkeypatch.setenv("DISCO_SIMT_CONTRACT", "1")
    psi_simt = conv.Psi(wl.nlat_in, wl.nlon_in, wl.nlat_out, wl.nlon_out, wl.kernel_shape, wl.theta_cutoff,
                        "cuda:0")
    dx_g = conv.disco_backward_input(psi_simt, dout, w, wl.C_in, wl.groups)
    torch.cuda.synchronize()
    check(host(dx_tc), oracle_dx(name), 1e-2, "dx (tensor cores)")
    check(host(dx_tc), host(dx_g), 8e-3, "dx (tensor cores vs gather)")


@pytest.mark.parametrize("name", ["tz_fused_k3", "tz_fused_k5", "tz_fused_k9", "weather", "grouped"])
def test_fused_tensor_core_matches_unfused(name):
    """The fused forward (Toeplitz contraction and channel mix on tensor cores, y tile on chip)
    against the unfused path, which rounds the same y to bf16 before the same mix."""
    wl, inp = workload(name), inputs(name)
    args = (gpu_psi(name), dev(inp["x"], wl), dev(inp["w"], wl), dev(inp["bias"], wl), wl.groups)
    out_f, _ = conv.disco_forward(*args, fused=True)
    out_u, _ = conv.disco_forward(*args)
    torch.cuda.synchronize()
    check(host(out_f), host(out_u), 8e-3, "fused vs unfused out")
    check(host(out_f), oracle_out(name), tol(wl), "fused out")


@pytest.mark.parametrize("name", ["ragged_iso_f32", "tc_small_bf16", "ragged_down_bf16", "grouped"])
def test_input_gradient_halves_compose(name):
    """disco_einsum_adjoint followed by disco_contract_adjoint is disco_bwd_input, bit for bit
    (the same kernels in the same order), on layers that the one-launch input gradient (64 output
    channels, groups 1, mirror rows) does not serve; that one is checked against the oracle."""
    wl, inp = workload(name), inputs(name)
    psi = gpu_psi(name)
    dout, w = dev(inp["dout"], wl), dev(inp["w"], wl)
    dx_ref = conv.disco_backward_input(psi, dout, w, wl.C_in, wl.groups)
    dcode = D.DISCO_BF16 if wl.dtype == "bf16" else D.DISCO_F32
    ws, n = psi.workspace(D.DISCO_OP_EINSUM_ADJOINT, wl.B, wl.C_in, wl.C_out, wl.groups, dcode)
    dy = torch.empty(wl.shapes()["y"], dtype=dx_ref.dtype, device="cuda:0")
    dx = torch.empty_like(dx_ref)
    st = torch.cuda.current_stream().cuda_stream
    D.disco_einsum_adjoint(psi.handle, wl.B, wl.C_in, wl.C_out, wl.groups, dcode, dout.data_ptr(), w.data_ptr(),
                           dy.data_ptr(), ws.data_ptr(), n, st)
    D.disco_contract_adjoint(psi.handle, wl.B, wl.C_in, dcode, dy.data_ptr(), dx.data_ptr(), st)
    torch.cuda.synchronize()
    assert torch.equal(dx, dx_ref)
    check(host(dx), oracle_dx(name), tol(wl), "dx from the two halves")


# Layers on the other latitude grids of the constructor's grid_in / grid_out: only Psi changes, so
# the same kernels must reproduce the oracle.  One bf16 layer on the tensor-core paths (64
# channels, TMA-aligned rows), one fp32 stride-2 layer on the gather paths.
GRID_EDGE = {
    "gauss_to_lobatto_bf16": (Workload("gauss_to_lobatto_bf16", 2, 64, 64, 1, 33, 64, 33, 64, (3, 1), 0.3, "bf16"),
                              "legendre-gauss", "lobatto"),
    "trap_to_gauss_f32": (Workload("trap_to_gauss_f32", 2, 6, 9, 3, 19, 24, 10, 12, (3, 4), 0.7, "f32"),
                          "equiangular-trapezoidal", "legendre-gauss"),
}


@pytest.mark.parametrize("name", list(GRID_EDGE))
def test_other_grids_match_oracle(name):
    wl, gi, go = GRID_EDGE[name]
    inp = make_inputs(wl, 0)
    P = oracle.Psi(oracle.Spec(wl.nlat_in, wl.nlon_in, wl.nlat_out, wl.nlon_out, wl.kernel_shape[0],
                               wl.kernel_shape[1], wl.theta_cutoff, gi, go))
    psi = conv.Psi(wl.nlat_in, wl.nlon_in, wl.nlat_out, wl.nlon_out, wl.kernel_shape, wl.theta_cutoff, "cuda:0",
                   grid_in=gi, grid_out=go)
    x, w, b, dout = (dev(inp[k], wl) for k in ("x", "w", "bias", "dout"))
    out, y = conv.disco_forward(psi, x, w, b, wl.groups)
    out_f, _ = conv.disco_forward(psi, x, w, b, wl.groups, fused=True)
    dx = conv.disco_backward_input(psi, dout, w, wl.C_in, wl.groups)
    dw, db = conv.disco_backward_weight(psi, dout, x=x, groups=wl.groups)
    torch.cuda.synchronize()
    out_ref = P.forward(inp["x"], inp["w"], inp["bias"], groups=wl.groups)
    check(host(out), out_ref, tol(wl), "out")
    check(host(y), P.contract(inp["x"]), tol(wl), "y")
    check(host(out_f), out_ref, tol(wl), "fused out")
    check(host(dx), P.backward_input(inp["dout"], inp["w"], wl.C_in, groups=wl.groups), tol(wl), "dx")
    dw_ref, db_ref = P.backward_weight(inp["dout"], inp["x"], groups=wl.groups)
    check(host(dw), dw_ref, tol(wl), "dw")
    check(host(db), db_ref, tol(wl), "dbias")


@pytest.mark.parametrize("name", ["tz_fused_k3", "ragged_down_bf16", "aniso_k9_f32"])
def test_polar_bands_reassemble_the_full_layer(name):
    """Three polar bands (disco_psi_build_band), each through the kernels on its own rows, stitched
    together: out and y by row, dx summed over the rows the bands share, dw and dbias summed,
    against the oracle's full layer.  This is the per-rank computation of the halo-exchange mode
    without the transfers."""
    from spherical_disco_convolution_b200 import polar

    wl, inp = workload(name), inputs(name)
    w, b = dev(inp["w"], wl), dev(inp["bias"], wl)
    out = np.zeros(oracle_out(name).shape)
    out_f = np.zeros_like(out)
    dx = np.zeros(inp["x"].shape)
    dw, db = 0.0, 0.0
    for jb, je in polar.split_rows(wl.nlat_out, 3):
        psi = conv.Psi(wl.nlat_in, wl.nlon_in, wl.nlat_out, wl.nlon_out, wl.kernel_shape, wl.theta_cutoff, "cuda:0",
                       rows=(jb, je))
        ib, ie = psi.in_rows
        xb = dev(inp["x"][:, :, ib:ie], wl)
        db_ = dev(inp["dout"][:, :, jb:je], wl)
        o, y = conv.disco_forward(psi, xb, w, b, wl.groups)
        of, _ = conv.disco_forward(psi, xb, w, b, wl.groups, fused=True)
        dxb = conv.disco_backward_input(psi, db_, w, wl.C_in, wl.groups)
        dwb, dbb = conv.disco_backward_weight(psi, db_, y=y, groups=wl.groups)
        torch.cuda.synchronize()
        out[:, :, jb:je], out_f[:, :, jb:je] = host(o), host(of)
        dx[:, :, ib:ie] += host(dxb)
        dw, db = dw + host(dwb), db + host(dbb)
    check(out, oracle_out(name), tol(wl), "out from bands")
    check(out_f, oracle_out(name), tol(wl), "fused out from bands")
    check(dx, oracle_dx(name), tol(wl), "dx from bands")
    dw_ref, db_ref = oracle_dw(name)
    check(dw, dw_ref, tol(wl), "dw from bands")
    check(db, db_ref, tol(wl), "dbias from bands")


@pytest.mark.parametrize("name", ["tz_fused_k3", "ragged_down_bf16", "aniso_k9_f32", "ring_k3", "mid"])
def test_input_bands_reassemble_the_full_layer(name):
    """Three bands of input latitudes (disco_psi_build_inputs), each through the kernels: the
    partial y and out (unfused and fused) summed over the bands (+ the bias once), dx stitched by
    row, dw summed, against the oracle's full layer; every output row that a band does not reach
    comes out exactly zero (exactly the bias from the fused forward given one).  This is the per-rank computation of the reduce-scatter mode without the
    collectives."""
    from spherical_disco_convolution_b200 import polar

    wl, inp = workload(name), inputs(name)
    w, b = dev(inp["w"], wl), dev(inp["bias"], wl)
    dout = dev(inp["dout"], wl)
    y_sum = np.zeros((wl.B, wl.C_in, wl.K, wl.nlat_out, wl.nlon_out))
    out = np.zeros(oracle_out(name).shape)
    out_f = np.zeros_like(out)
    dx = np.zeros(inp["x"].shape)
    dw = 0.0
    entries = D.disco_psi_export(gpu_psi(name).handle)
    for ib, ie in polar.split_rows(wl.nlat_in, 3):
        psi = conv.Psi(wl.nlat_in, wl.nlon_in, wl.nlat_out, wl.nlon_out, wl.kernel_shape, wl.theta_cutoff, "cuda:0",
                       inputs=(ib, ie))
        xb = dev(inp["x"][:, :, ib:ie], wl)
        o, y = conv.disco_forward(psi, xb, w, None, wl.groups)
        of, _ = conv.disco_forward(psi, xb, w, None, wl.groups, fused=True)
        ofb = conv.disco_forward(psi, xb, w, b, wl.groups, fused=True)[0] if b is not None else None
        dxb = conv.disco_backward_input(psi, dout, w, wl.C_in, wl.groups)
        dwb, _ = conv.disco_backward_weight(psi, dout, y=y, groups=wl.groups, need_bias=False)
        torch.cuda.synchronize()
        yh = host(y)
        reached = np.zeros(wl.nlat_out, dtype=bool)
        reached[entries[1][(entries[2] >= ib) & (entries[2] < ie)]] = True
        assert not np.any(yh[:, :, :, ~reached]), "an output row the band does not reach is not zero"
        assert not np.any(host(of)[:, :, ~reached]), "fused: an output row the band does not reach is not zero"
        if ofb is not None:  # the bias exactly, on the rows the band does not reach
            hb = host(ofb)[:, :, ~reached]
            assert np.array_equal(hb, np.broadcast_to(host(b)[None, :, None, None], hb.shape)), \
                "fused: unreached rows are not the bias"
        y_sum += yh
        out += host(o)
        out_f += host(of)
        dx[:, :, ib:ie] = host(dxb)
        dw = dw + host(dwb)
    if inp["bias"] is not None:
        out += host(b)[None, :, None, None]
        out_f += host(b)[None, :, None, None]
    check(out, oracle_out(name), tol(wl), "out from input bands")
    check(out_f, oracle_out(name), tol(wl), "fused out from input bands")
    check(dx, oracle_dx(name), tol(wl), "dx from input bands")
    check(dw, oracle_dw(name)[0], tol(wl), "dw from input bands")
    if wl.B * wl.C_in <= 512:
        check(y_sum, oracle_psi(name).contract(inp["x"]), tol(wl), "y from input bands")


@pytest.mark.parametrize("name,A", [("tz_fused_k3", 2), ("ragged_down_bf16", 3), ("aniso_k9_f32", 2), ("mid", 3)])
def test_azimuth_shards_reassemble_the_full_layer(name, A):
    """The per-rank kernels of the azimuth all-to-all on A emulated ranks, without the transfers.
    Standard mode: the contraction on each channel shard, y cut into longitude shards, the weight
    einsum, its transpose and the weight gradient on each shard's points (disco_mix*), the
    adjoint contraction on each channel shard.  Reordered mode: the fused forward of each channel
    shard with its dense block weight (partial out over full rows, summed), the one-call input
    gradient and the recomputing weight gradient per shard.  Against the oracle's full layer."""
    from spherical_disco_convolution_b200 import distributed

    wl, inp = workload(name), inputs(name)
    sh = distributed.AzimuthShards(wl.nlon_in, wl.nlon_out, wl.C_in, A)
    psi = gpu_psi(name)
    x, w, b, dout = dev(inp["x"], wl), dev(inp["w"], wl), dev(inp["bias"], wl), dev(inp["dout"], wl)
    has_b, G = b is not None, wl.groups
    # standard
    y = torch.cat([conv.disco_contract(psi, x[:, cb:ce].contiguous()) for cb, ce in sh.chans], dim=1)
    out = np.zeros(oracle_out(name).shape)
    dy = torch.empty_like(y)
    dw, db = 0.0, 0.0
    for qb, qe in sh.lon_out:
        y_a, d_a = y[..., qb:qe].contiguous(), dout[..., qb:qe].contiguous()
        out[..., qb:qe] = host(conv.mix(y_a, w, b, G))
        dy[..., qb:qe] = conv.mix_adjoint(d_a, w, wl.C_in, G)
        dw_a, db_a = conv.mix_weight(d_a, y_a, G, need_bias=has_b)
        dw = dw + host(dw_a)
        db = db + (host(db_a) if has_b else 0.0)
    dx = torch.cat([conv.disco_contract_adjoint(psi, dy[:, cb:ce].contiguous()) for cb, ce in sh.chans], dim=1)
    torch.cuda.synchronize()
    check(out, oracle_out(name), tol(wl), "out from azimuth shards")
    check(host(dx), oracle_dx(name), tol(wl), "dx from azimuth shards")
    dw_ref, db_ref = oracle_dw(name)
    check(dw, dw_ref, tol(wl), "dw from azimuth shards")
    if has_b:
        check(db, db_ref, tol(wl), "dbias from azimuth shards")
    # reordered (fused)
    out_f = np.zeros_like(out)
    dx_f = np.zeros(inp["x"].shape)
    dw_f = 0.0
    for a, (cb, ce) in enumerate(sh.chans):
        cols, mask = distributed.channel_shard(wl.C_in, wl.C_out, G, (cb, ce))
        ws = distributed.shard_weight(w, cols, mask)
        xc = x[:, cb:ce].contiguous()
        out_f += host(conv.disco_forward(psi, xc, ws, b if a == 0 else None, 1, fused=True)[0])
        dx_f[:, cb:ce] = host(conv.disco_backward_input(psi, dout, ws, ce - cb, 1))
        dws, _ = conv.disco_backward_weight(psi, dout, x=xc, groups=1, need_bias=False)
        dw_f = dw_f + host(distributed.unshard_weight_grad(dws, cols, mask, wl.C_out, wl.C_in // G))
    torch.cuda.synchronize()
    check(out_f, oracle_out(name), tol(wl), "fused out from channel shards")
    check(dx_f, oracle_dx(name), tol(wl), "fused dx from channel shards")
    check(dw_f, dw_ref, tol(wl), "fused dw from channel shards")


@pytest.mark.parametrize("B,C_in,C_out,G,K,npts,bias", [
    (1, 64, 128, 1, 3, 4104, True),     # 128 outputs per tile, 256-point tiles (all 512 TMEM columns)
    (2, 64, 64, 2, 3, 1000, False),     # 32 outputs per group, ragged last tile, no bias
    (1, 32, 16, 1, 5, 776, True),       # 16 outputs, K = 5 (K-chunks past the rows read as zeros)
    (1, 64, 256, 1, 3, 2056, True),     # 256 outputs: the one-tile kernel
    (1, 64, 128, 1, 9, 1032, True),     # 128 outputs, K = 9: the persistent kernel with 128-point tiles
    (1, 64, 64, 1, 3, 1001, True),      # a point count TMA cannot address: the SIMT kernel
])
def test_weight_einsum_on_points_matches_fp64(B, C_in, C_out, G, K, npts, bias):
    """disco_mix, disco_mix_adjoint and disco_mix_weight on bf16 inputs against the same sums in
    fp64 on the host (the einsum of the forward equation and its two adjoints), over the tile
    shapes the launcher picks: every output tile size, both point-tile widths, groups, a ragged
    last tile and no bias."""
    rng = np.random.default_rng(B * 1000 + C_out + npts)
    bf = lambda a: torch.from_numpy(a).to(torch.bfloat16)  # noqa: E731
    y = bf(rng.standard_normal((B, C_in, K, npts)))
    w = bf(rng.standard_normal((C_out, C_in // G, K)) / math.sqrt(C_in // G * K))
    b = bf(rng.standard_normal(C_out)) if bias else None
    dout = bf(rng.standard_normal((B, C_out, npts)))
    yh, wh, dh = (t.double().numpy() for t in (y, w, dout))
    Og, Cg = C_out // G, C_in // G
    ref = np.einsum("gock,bgckn->bgon", wh.reshape(G, Og, Cg, K), yh.reshape(B, G, Cg, K, npts)).reshape(B, C_out, npts)
    if bias:
        ref = ref + b.double().numpy()[None, :, None]
    dy_ref = np.einsum("gock,bgon->bgckn", wh.reshape(G, Og, Cg, K), dh.reshape(B, G, Og, npts)).reshape(yh.shape)
    dw_ref = np.einsum("bgon,bgckn->gock", dh.reshape(B, G, Og, npts), yh.reshape(B, G, Cg, K, npts)).reshape(wh.shape)
    dev0 = "cuda:0"
    out = conv.mix(y.to(dev0), w.to(dev0), None if b is None else b.to(dev0), G)
    dy = conv.mix_adjoint(dout.to(dev0), w.to(dev0), C_in, G)
    dw, db = conv.mix_weight(dout.to(dev0), y.to(dev0), G, need_bias=True)
    torch.cuda.synchronize()
    check(host(out), ref, 2e-2, "mix")
    check(host(dy), dy_ref, 2e-2, "mix_adjoint")
    check(host(dw), dw_ref, 2e-2, "mix_weight dw")
    check(host(db), dh.sum(axis=(0, 2)), 2e-2, "mix_weight dbias")


def test_polar_layer_on_one_rank_matches_oracle():
    """PolarDiscoConvS2, PolarReduceScatterConvS2 and DistributedDiscoConvS2 (both polar modes)
    through autograd on a one-rank NCCL group (the whole layer is one band and one longitude
    shard; the collectives move nothing), unfused and fused, against the oracle."""
    import datetime
    import socket

    import torch.distributed as dist

    from spherical_disco_convolution_b200 import distributed, polar

    name = "ragged_down_bf16"
    wl, inp = workload(name), inputs(name)
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda:0"))
    try:
        for fused in (False, True):
            layer = polar.PolarDiscoConvS2(wl.C_in, wl.C_out, (wl.nlat_in, wl.nlon_in), (wl.nlat_out, wl.nlon_out),
                                           wl.kernel_shape, wl.theta_cutoff, groups=wl.groups, bias=False,
                                           fused=fused, device="cuda:0", dtype=torch.bfloat16)
            with torch.no_grad():
                layer.weight.copy_(dev(inp["w"], wl))
            x = dev(inp["x"], wl).requires_grad_(True)
            out = layer(x)
            out.backward(dev(inp["dout"], wl))
            torch.cuda.synchronize()
            check(host(out), oracle_out(name), tol(wl), "polar layer out")
            check(host(x.grad), oracle_dx(name), tol(wl), "polar layer dx")
            check(host(layer.weight.grad), oracle_dw(name)[0], tol(wl), "polar layer dw")
        # the reduce-scatter polar mode and the polar x azimuth layer, each on the 1 x 1 grid
        layers = [("reduce-scatter", fused, polar.PolarReduceScatterConvS2) for fused in (False, True)]
        layers += [(mode, fused, distributed.DistributedDiscoConvS2) for mode in distributed.POLAR_MODES
                   for fused in (False, True)]
        for mode, fused, cls in layers:
            kw = dict(polar_mode=mode) if cls is distributed.DistributedDiscoConvS2 else {}
            layer = cls(wl.C_in, wl.C_out, (wl.nlat_in, wl.nlon_in), (wl.nlat_out, wl.nlon_out), wl.kernel_shape,
                        wl.theta_cutoff, groups=wl.groups, bias=True, fused=fused, device="cuda:0",
                        dtype=torch.bfloat16, **kw)
            bias = np.linspace(-1.0, 1.0, wl.C_out)
            with torch.no_grad():
                layer.weight.copy_(dev(inp["w"], wl))
                layer.bias.copy_(dev(bias, wl))
            x = dev(inp["x"], wl).requires_grad_(True)
            out = layer(x)
            out.backward(dev(inp["dout"], wl))
            torch.cuda.synchronize()
            what = f"{cls.__name__} {mode} fused={fused}"
            ref = oracle_psi(name).forward(inp["x"], inp["w"], host(dev(bias, wl)), groups=wl.groups)
            check(host(out), ref, tol(wl), what + " out")
            check(host(x.grad), oracle_dx(name), tol(wl), what + " dx")
            check(host(layer.weight.grad), oracle_dw(name)[0], tol(wl), what + " dw")
            check(host(layer.bias.grad), inp["dout"].sum(axis=(0, 2, 3)), tol(wl), what + " dbias")
    finally:
        dist.destroy_process_group()
