"""Tile-script plans of the TMA-staged strip kernel, checked on the CPU.

A NumPy re-enactment of the kernel (tests/plan_emulator.py: tile) runs the exported plans of
host-only handles: it stages each load's chunks the way the TMA boxes do (zeros outside the
ring), fills the B batches from the copies, replays the four issuers' command streams and writes
rows the way the epilogue does, asserting on the way that every operand lies inside a staged
chunk or its batch and that slots, batches and row buffers are waited for and released in the
order the kernel's barriers need.  Its result must equal the contraction (and its adjoint) with
the library's own Psi rounded once to bf16 to 1e-12: a wrong window, seam split, chunk address,
mirror row or block layout fails here before any kernel runs.
"""

import math

import numpy as np
import pytest

from spherical_disco_convolution_b200 import disco
from tests import plan_emulator
from tests.test_ring_plan import _host, _reference

LAYERS = [
    ("mid", (91, 176, 91, (3,), 2 * math.pi / 90, 0, 0)),
    ("gauss", (32, 64, 32, (3,), 2 * math.pi / 32, 1, 1)),
    ("aniso", (33, 64, 33, (3, 4), 3 * math.pi / 32, 0, 0)),
    ("k5", (33, 64, 33, (5,), 4 * math.pi / 32, 0, 0)),
    ("lon96", (33, 96, 33, (3,), 2 * math.pi / 32, 0, 0)),
    # cutoff of two grid spacings as on the 721x1440 layer: full-ring windows near the poles,
    # staged in pieces, and windows across the seam
    ("two_spacings", (65, 128, 65, (3,), 2 * math.pi / 64, 0, 0)),
    ("ragged", (49, 200, 49, (3,), 2 * math.pi / 48, 0, 0)),
]


@pytest.mark.parametrize("name,layer", LAYERS, ids=[n for n, _ in LAYERS])
@pytest.mark.parametrize("which", [0, 1, 2, 3])
def test_tile_plan_reenactment_matches_contraction(name, layer, which):
    nlat_in, nlon, nlat_out, kshape, theta, gi, go = layer
    psi = _host(nlat_in, nlon, nlat_out, kshape, theta, gi, go)
    try:
        iso = len(kshape) == 1
        Kf = kshape[0] if iso else 1 + (kshape[0] - 1) * kshape[1]
        expect = (which in (1, 3) or iso) and (which >= 2 or Kf in (1, 3, 5))
        if not expect:
            with pytest.raises(disco.DiscoError):
                disco.disco_tile_info(psi, which)
            return
        plan = disco.disco_tile_export(psi, which)
        adjoint = which >= 2
        rng = np.random.default_rng(5)
        BC = 3 if which in (0, 2) else 70  # plane pairs: a second, partial group of 64 planes
        Kb = len(np.unique(disco.disco_psi_export(psi)[0]))
        n_src = Kb * nlat_out if adjoint else nlat_in
        n_out = nlat_in if adjoint else nlat_out
        x = rng.standard_normal((BC, n_src, nlon))
        got = plan_emulator.tile(plan, x, n_out)
        ref = _reference(psi, x, adjoint, plan["K"], nlat_in, nlat_out, nlon, plan["mirror"] == 1)
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    finally:
        disco.disco_psi_destroy(psi)


def test_tile_plans_need_64_longitudes():
    psi = _host(17, 32, 17, (3,), 2 * math.pi / 16)
    try:
        for which in range(4):
            with pytest.raises(disco.DiscoError):
                disco.disco_tile_info(psi, which)
    finally:
        disco.disco_psi_destroy(psi)


def test_tile_plan_of_the_weather_layer():
    # the 721x1440 layer: mirror rows, shared sources, scripts balanced over 148 CTAs
    psi = _host(721, 1440, 721, (3,), 2 * math.pi / 720)
    try:
        d = disco.disco_tile_info(psi, 0)
        assert d["mirror"] == 1 and d["K"] == 3 and d["N"] == 48 and d["n_qt"] == 23
        assert d["n_ctas"] == 148 and d["n_rows"] == 361 * 23
        plan = disco.disco_tile_export(psi, 0)
        cta = plan["cta_tiles"]
        assert sorted(cta[149:].tolist()) == list(range(d["n_strips"] * 23))
        cost = plan["tiles"][:, 12].astype(np.int64)
        per = np.array([cost[cta[149 + cta[c]: 149 + cta[c + 1]]].sum() for c in range(148)])
        assert per.max() <= 1.25 * per.mean()
    finally:
        disco.disco_psi_destroy(psi)
