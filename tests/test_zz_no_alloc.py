"""disco_bwd_weight_noalloc: the weight gradient for callers that cannot allocate.

Code that runs inside an application which owns all device memory through its own
allocator, or that must not allocate once it is running, cannot call cudaMalloc or
hand the library a workspace.  The no-allocation variant keeps its split-K partial sums
in a fixed array inside the library instead.  These checks call it through the C ABI
and compare it with disco_bwd_weight (the workspace version) on two calls in a row, so a
stale or missing scratch address, or partial sums left over from an earlier call, would
show up as a mismatch.  This file is collected last on purpose.
"""

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from spherical_disco_convolution_b200 import conv  # noqa: E402
from spherical_disco_convolution_b200 import disco as D  # noqa: E402
from spherical_disco_convolution_b200.workloads import WORKLOADS, make_inputs  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _layer(name):
    wl = WORKLOADS[name]
    dt = torch.float32 if wl.dtype == "f32" else torch.bfloat16
    code = D.DISCO_F32 if wl.dtype == "f32" else D.DISCO_BF16
    psi = conv.Psi(wl.nlat_in, wl.nlon_in, wl.nlat_out, wl.nlon_out, wl.kernel_shape, wl.theta_cutoff, "cuda:0")
    inp = make_inputs(wl, 0)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to("cuda:0").to(dt)  # noqa: E731
    return wl, dt, code, psi, dev(inp["x"]), dev(inp["w"]), dev(inp["bias"]), dev(inp["dout"])


@pytest.mark.parametrize("name", ["mid", "downsample", "weather"])
def test_noalloc_weight_gradient_matches_workspace_version(name):
    wl, dt, code, psi, x, w, b, dout = _layer(name)
    _, y = conv.disco_forward(psi, x, w, b, wl.groups)
    dw_ref, db_ref = conv.disco_backward_weight(psi, dout, y=y, groups=wl.groups)
    torch.cuda.synchronize()
    tol = 1e-4 if wl.dtype == "f32" else 2e-2
    stream = torch.cuda.current_stream().cuda_stream
    results = []
    for _ in range(2):
        dw = torch.full_like(dw_ref, float("nan"))
        db = torch.full_like(db_ref, float("nan"))
        D.disco_bwd_weight_noalloc(psi.handle, wl.B, wl.C_in, wl.C_out, wl.groups, code, dout.data_ptr(),
                                   y.data_ptr(), dw.data_ptr(), db.data_ptr(), stream)
        torch.cuda.synchronize()
        for got, ref in ((dw, dw_ref), (db, db_ref)):
            g, r = got.float().cpu().numpy(), ref.float().cpu().numpy()
            assert np.isfinite(g).all()
            assert np.abs(g - r).max() <= tol * np.abs(r).max()
        results.append(dw.clone())
    assert torch.equal(results[0], results[1])


def test_noalloc_rejects_layers_beyond_its_scratch():
    wl, dt, code, psi, x, w, b, dout = _layer("tiny")
    stream = torch.cuda.current_stream().cuda_stream
    big = 4096  # 4096 * 4096 * 3 partial weights per split: far beyond 2^21 floats
    with pytest.raises(D.DiscoError) as e:
        D.disco_bwd_weight_noalloc(psi.handle, 1, big, big, 1, code, dout.data_ptr(), x.data_ptr(), w.data_ptr(),
                                   b.data_ptr(), stream)
    assert e.value.status == D.DISCO_ERR_UNSUPPORTED and "scratch" in str(e.value)
