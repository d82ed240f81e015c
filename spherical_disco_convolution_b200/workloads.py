"""Seeded synthetic workloads for the DISCO convolution.

This module holds only the layer shapes and the random input recipes; it
contains none of the convolution's arithmetic.  Both the CUDA path and the
CPU oracle take their inputs from here, so the two sides see identical
numbers.  Draw order from ``numpy.random.default_rng(seed)``: x, w, bias,
dout.  Inputs of bf16 layers are rounded once (nearest-even) to values that
bf16 represents exactly and are handed out as float32 arrays.

The five shapes cover what the DISCO layer is documented to take
(page "torch_harmonics.DiscreteContinuousConvS2": input (batch, in_channels,
nlat_in, nlon_in), output (batch, out_channels, nlat_out, nlon_out),
kernel_shape, groups, theta_cutoff, equiangular grids):

* ``tiny``       17x32 -> 17x32, C 4->4, isotropic K=3, fp32
* ``mid``        91x180 -> 91x180, B4, C 32->32, isotropic K=3, fp32, with a
                 smooth spherical-harmonic component added to the noise
* ``downsample`` 181x360 -> 91x180, B2, C 64->128, anisotropic (3,4) K=9, bf16
* ``weather``    721x1440 -> 721x1440, B1, C 64->64, isotropic K=3, bf16,
                 per-channel mean and spread (ERA5-like shape, synthetic)
* ``grouped``    361x720 -> 361x720, B2, C 256->256, groups 4, (3,4) K=9, bf16
"""

from __future__ import annotations

import math
from dataclasses import dataclass, replace

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    C_in: int
    C_out: int
    groups: int
    nlat_in: int
    nlon_in: int
    nlat_out: int
    nlon_out: int
    kernel_shape: tuple  # (n_r, n_alpha); n_alpha == 1 is isotropic
    theta_cutoff: float
    dtype: str  # "f32" or "bf16"
    x_kind: str = "normal"  # normal | sh | channel_stats
    bias: bool = True

    @property
    def K(self) -> int:
        n_r, n_a = self.kernel_shape
        return n_r if n_a == 1 else 1 + (n_r - 1) * n_a

    @property
    def stride(self) -> int:
        return self.nlon_in // self.nlon_out

    def shapes(self):
        return dict(
            x=(self.B, self.C_in, self.nlat_in, self.nlon_in),
            w=(self.C_out, self.C_in // self.groups, self.K),
            bias=(self.C_out,),
            y=(self.B, self.C_in, self.K, self.nlat_out, self.nlon_out),
            out=(self.B, self.C_out, self.nlat_out, self.nlon_out),
        )

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 4, 4, 1, 17, 32, 17, 32, (3, 1), 2 * math.pi / 16, "f32"),
    "mid": Workload("mid", 4, 32, 32, 1, 91, 180, 91, 180, (3, 1), 2 * math.pi / 90, "f32", x_kind="sh"),
    "downsample": Workload("downsample", 2, 64, 128, 1, 181, 360, 91, 180, (3, 4), 3 * math.pi / 90, "bf16"),
    "weather": Workload("weather", 1, 64, 64, 1, 721, 1440, 721, 1440, (3, 1), 2 * math.pi / 720, "bf16",
                        x_kind="channel_stats"),
    "grouped": Workload("grouped", 2, 256, 256, 4, 361, 720, 361, 720, (3, 4), 3 * math.pi / 360, "bf16"),
}


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def _storage(a: np.ndarray, dtype: str) -> np.ndarray:
    a = np.asarray(a, dtype=np.float32)
    return round_bf16(a) if dtype == "bf16" else np.ascontiguousarray(a)


def _real_sh(l: int, m: int, theta: np.ndarray, lam: np.ndarray) -> np.ndarray:
    from scipy.special import sph_harm_y

    y = sph_harm_y(l, abs(m), theta, lam)
    if m > 0:
        return np.sqrt(2.0) * y.real
    if m < 0:
        return np.sqrt(2.0) * y.imag
    return y.real


def make_inputs(wl: Workload, seed: int = 0, need=("x", "w", "bias", "dout")) -> dict:
    """Seeded inputs as float32 arrays (bf16-representable for bf16 layers)."""
    rng = np.random.default_rng(seed)
    sh = wl.shapes()
    out = {}
    if wl.x_kind == "channel_stats":
        mu = rng.normal(0.0, 0.5, size=(wl.B, wl.C_in, 1, 1)).astype(np.float32)
        sd = rng.uniform(0.5, 2.0, size=(wl.B, wl.C_in, 1, 1)).astype(np.float32)
        x = mu + sd * rng.standard_normal(sh["x"], dtype=np.float32)
    else:
        x = rng.standard_normal(sh["x"], dtype=np.float32)
    if wl.x_kind == "sh":
        theta = np.pi * np.arange(wl.nlat_in) / (wl.nlat_in - 1)
        lam = 2 * np.pi * np.arange(wl.nlon_in) / wl.nlon_in
        TH, LA = np.meshgrid(theta, lam, indexing="ij")
        for b in range(wl.B):
            for c in range(wl.C_in):
                for _ in range(8):
                    l = int(rng.integers(0, 11))
                    m = int(rng.integers(-l, l + 1))
                    f = _real_sh(l, m, TH, LA)
                    x[b, c] += (f / np.abs(f).max()).astype(np.float32)
    out["x"] = _storage(x, wl.dtype)
    fan_in = (wl.C_in // wl.groups) * wl.K
    out["w"] = _storage(rng.normal(0.0, 1.0 / math.sqrt(fan_in), size=sh["w"]), wl.dtype)
    out["bias"] = _storage(rng.uniform(-0.1, 0.1, size=sh["bias"]), wl.dtype) if wl.bias else None
    if "dout" in need:
        out["dout"] = _storage(rng.standard_normal(sh["out"], dtype=np.float32), wl.dtype)
    return {k: v for k, v in out.items() if k in need or k == "bias"}
