"""GPU checks beyond the element-by-element parity tests.

* The failure path of the bounded device-side waits: a wait that nothing satisfies returns the
  timeout status quickly and leaves the context usable (no GPU fault, no hang).
* The strip-staged contraction (ring plans) against the per-pair tensor-core kernel on layers
  that take its mirror-row and plane-pair forms.
* Equivariance under a roll of the longitude ring (page "torch_harmonics.DiscreteContinuousConvS2",
  class description: Psi is shifted along the longitude for every output longitude): rolling x
  by s*m longitudes rolls out by m, within the tolerance of the layer's precision.
"""

import time

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from spherical_disco_convolution_b200 import conv  # noqa: E402
from spherical_disco_convolution_b200 import disco as D  # noqa: E402
from tests.test_gpu_parity import (GRID_EDGE, check, dev, host, inputs, oracle_out, tol,  # noqa: E402
                                   workload)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_bounded_wait_expires_and_the_context_stays_usable():
    st = torch.cuda.current_stream().cuda_stream
    t0 = time.perf_counter()
    D.disco_wait_selftest(2000, st)  # 2 ms
    with pytest.raises(D.DiscoError) as e:
        D.disco_sync_status(st)
    assert e.value.status == D.DISCO_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 1.0
    D.disco_sync_status(st)  # the status was cleared by the report
    with pytest.raises(D.DiscoError) as e:
        D.disco_wait_selftest(0, st)
    assert e.value.status == D.DISCO_ERR_INVALID_ARG
    # the same process still computes a correct forward
    name = "tc_small_bf16"
    wl, inp = workload(name), inputs(name)
    psi = conv.Psi(wl.nlat_in, wl.nlon_in, wl.nlat_out, wl.nlon_out, wl.kernel_shape, wl.theta_cutoff, "cuda:0")
    out, _ = conv.disco_forward(psi, dev(inp["x"], wl), dev(inp["w"], wl), dev(inp["bias"], wl), wl.groups)
    D.disco_sync_status(st)
    check(host(out), oracle_out(name), tol(wl), "out after the timeout")


def _grid_workload(name):
    return GRID_EDGE[name] if name in GRID_EDGE else (workload(name), "equiangular", "equiangular")


@pytest.mark.parametrize("name", ["tc_small_bf16", "ring_k3", "gauss_to_lobatto_bf16", "weather"])
def test_ring_kernel_matches_per_pair_kernel(name, monkeypatch):
    """y from the strip-staged kernel (default for these layers) against the per-pair kernel
    (DISCO_RING=0): the first holds Psi in bf16, the second as a bf16 hi + lo pair, and both round
    y to bf16, so they differ by at most u (max|x| + 2 max|y|) with u = 2^-8."""
    wl, gi, go = _grid_workload(name)
    inp = inputs(name) if name not in GRID_EDGE else None
    if inp is None:
        from spherical_disco_convolution_b200.workloads import make_inputs
        inp = make_inputs(wl, 0)
    x = dev(inp["x"], wl)
    if wl.B * wl.C_in > 8 and name == "weather":
        x = x[:, :8].contiguous()
    args = (wl.nlat_in, wl.nlon_in, wl.nlat_out, wl.nlon_out, wl.kernel_shape, wl.theta_cutoff, "cuda:0", gi, go)
    psi_r = conv.Psi(*args)
    assert D.disco_ring_info(psi_r.handle, 0 if x.shape[0] * x.shape[1] <= 64 else 1)["n_items"] > 0
    y_r = conv.disco_contract(psi_r, x)
    monkeypatch.setenv("DISCO_RING", "0")
    psi_p = conv.Psi(*args)
    y_p = conv.disco_contract(psi_p, x)
    torch.cuda.synchronize()
    yr, yp = host(y_r), host(y_p)
    u = 2.0 ** -8
    bound = u * (np.abs(host(x)).max() + 2 * np.abs(yp).max())
    err = np.abs(yr - yp).max()
    assert err <= 1.05 * bound, f"{name}: ring vs per-pair max err {err:.3e} > {bound:.3e}"


@pytest.mark.parametrize("name", ["mid", "tc_small_bf16", "ring_k3", "downsample"])
@pytest.mark.parametrize("m", [1, 7, 64])
def test_roll_equivariance(name, m):
    wl, inp = workload(name), inputs(name)
    s = wl.nlon_in // wl.nlon_out
    psi = conv.Psi(wl.nlat_in, wl.nlon_in, wl.nlat_out, wl.nlon_out, wl.kernel_shape, wl.theta_cutoff, "cuda:0")
    x, w, b = dev(inp["x"], wl), dev(inp["w"], wl), dev(inp["bias"], wl)
    out, _ = conv.disco_forward(psi, x, w, b, wl.groups)
    out_r, _ = conv.disco_forward(psi, torch.roll(x, s * m, dims=-1).contiguous(), w, b, wl.groups)
    out_f, _ = conv.disco_forward(psi, torch.roll(x, s * m, dims=-1).contiguous(), w, b, wl.groups, fused=True)
    torch.cuda.synchronize()
    ref = np.roll(host(out), m, axis=-1)
    check(host(out_r), ref, tol(wl), f"out(roll(x, {s * m})) vs roll(out, {m})")
    check(host(out_f), ref, tol(wl), f"fused out(roll(x, {s * m})) vs roll(out, {m})")
