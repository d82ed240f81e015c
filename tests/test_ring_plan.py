"""Ring plans of the strip-staged tensor-core kernel, checked on the CPU.

A NumPy re-enactment of the kernel's script (tests/plan_emulator.py: ring) runs the exported
plans of host-only handles: it fills the ring slots the way the producer does, applies every
item's Toeplitz K-steps the way the MMA issuer does and writes rows the way the epilogue does,
asserting on the way that every shared-memory octet and B K-step read lies inside its load and
slot and that slots and accumulator buffers are reused only when the kernel's barriers allow
it.  Its result must equal the contraction (and its adjoint) with the library's own Psi rounded
once to bf16, the precision of the blocks, to 1e-12: so a wrong window, offset, wrap, mirror
row or block layout fails here before any kernel runs.
"""

import math

import numpy as np
import pytest

from spherical_disco_convolution_b200 import disco
from tests import plan_emulator


def _bf16(v):
    f = np.asarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    f = (f + 0x7FFF + ((f >> 16) & 1)) >> 16
    return (f.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _host(nlat_in, nlon, nlat_out, kshape, theta, grid_in=0, grid_out=0):
    spec = disco.make_spec(nlat_in, nlon, nlat_out, nlon, kshape, theta, grid_in=grid_in, grid_out=grid_out)
    return disco.disco_psi_build(spec, -1)


def _reference(psi, x, adjoint, K, nlat_in, nlat_out, nlon, mirror):
    k, j, i, p, v = disco.disco_psi_export(psi)
    if mirror:
        # mirror plans apply the northern row's blocks to its southern mirror: use its values
        north = {(a, b, c, d): w for a, b, c, d, w in zip(k, j, i, p, v) if b <= nlat_out - 1 - b}
        v = np.array([north[(a, min(b, nlat_out - 1 - b), c if b <= nlat_out - 1 - b else nlat_in - 1 - c, d)]
                      for a, b, c, d in zip(k, j, i, p)])
    vb = _bf16(v)
    BC = x.shape[0]
    q = np.arange(nlon)
    if not adjoint:
        y = np.zeros((BC, K, nlat_out, nlon))
        for t in range(len(k)):
            y[:, k[t], j[t], :] += vb[t] * x[:, i[t], (q + p[t]) % nlon]
        return y
    dx = np.zeros((BC, 1, nlat_in, nlon))
    for t in range(len(k)):
        dx[:, 0, i[t], :] += vb[t] * x[:, k[t] * nlat_out + j[t], (q - p[t]) % nlon]
    return dx


LAYERS = [
    ("tiny", (17, 32, 17, (3,), 2 * math.pi / 16, 0, 0)),
    ("mid", (91, 176, 91, (3,), 2 * math.pi / 90, 0, 0)),
    ("gauss", (24, 48, 24, (3,), 2 * math.pi / 24, 1, 1)),
    ("aniso", (17, 32, 17, (3, 4), 3 * math.pi / 16, 0, 0)),
    ("k5", (33, 64, 33, (5,), 4 * math.pi / 32, 0, 0)),
    # cutoff of two grid spacings as on the 721x1440 layer: full-ring windows near the poles,
    # loaded in chunks, and wrapping around the ring
    ("two_spacings", (65, 128, 65, (3,), 2 * math.pi / 64, 0, 0)),
]


@pytest.mark.parametrize("name,layer", LAYERS, ids=[n for n, _ in LAYERS])
@pytest.mark.parametrize("which", [0, 1, 2, 3])
def test_ring_plan_reenactment_matches_contraction(name, layer, which):
    nlat_in, nlon, nlat_out, kshape, theta, gi, go = layer
    psi = _host(nlat_in, nlon, nlat_out, kshape, theta, gi, go)
    try:
        iso = len(kshape) == 1
        Kf = kshape[0] if iso else 1 + (kshape[0] - 1) * kshape[1]
        expect = (which in (1, 3) or iso) and (which >= 2 or Kf in (3, 5))
        if not expect:
            with pytest.raises(disco.DiscoError):
                disco.disco_ring_info(psi, which)
            return
        plan = disco.disco_ring_export(psi, which)
        adjoint = which >= 2
        rng = np.random.default_rng(3)
        BC = 3 if which in (0, 2) else 70  # plane pairs: a second, partial group of 64 planes
        Kb = len(np.unique(disco.disco_psi_export(psi)[0]))
        n_src = Kb * nlat_out if adjoint else nlat_in
        n_out = nlat_in if adjoint else nlat_out
        x = rng.standard_normal((BC, n_src, nlon))
        got = plan_emulator.ring(plan, x, n_out)
        ref = _reference(psi, x, adjoint, plan["K"], nlat_in, nlat_out, nlon, plan["mirror"] == 1)
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    finally:
        disco.disco_psi_destroy(psi)


def test_ring_plan_of_the_weather_layer_shares_sources():
    # the 721x1440 layer: mirror rows, and almost every source row loaded once per strip
    psi = _host(721, 1440, 721, (3,), 2 * math.pi / 720)
    try:
        d = disco.disco_ring_info(psi, 0)
        assert d["mirror"] == 1 and d["K"] == 3 and d["N"] == 48
        plan = disco.disco_ring_export(psi, 0)
        assert d["n_rows"] == 361
        # loads per tile column: a shared source once per strip, long windows in chunks
        assert d["n_loads"] < 2 * 721
    finally:
        disco.disco_psi_destroy(psi)
