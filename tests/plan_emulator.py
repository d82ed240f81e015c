"""NumPy re-enactment of the gather kernels' index arithmetic (test helper).

The CUDA gather kernels read, for output m of a row, the staged element
t0 + m*step + u of a chunk's source row, where staged element t holds source
longitude (start + t) mod n_src (block offset zero), and add value x (sum of
the source row) for every ring term.  This module applies
exactly that rule to the plan records exported by libdisco, in fp64, so a
wrong offset, wrap, residue class or value layout in the host plans shows up
against the oracle on the CPU, before any kernel runs.
"""

import numpy as np


def forward(plan, x, nlat_out, nlon_out, K):
    """y (B*C, K, nlat_out, nlon_out) from x (B*C, nlat_in, nlon_in) via the forward plan."""
    BC, _, n_src = x.shape
    y = np.zeros((BC, K, nlat_out, nlon_out))
    m = np.arange(nlon_out)
    step = plan["step"]
    for r in plan["rows"]:
        row, sb = r[0], r[1]
        for t in range(r[11], r[12]):
            srow, k = plan["rings"][t][:2]
            y[:, k, row, :] += float(plan["ring_v"][t]) * x[:, srow, :].sum(axis=-1)[:, None]
        for ch in range(r[3], r[7]):
            src, t0, voff, wk = plan["chunks"][ch]
            srow, start = plan["srcs"][sb + src][:2]
            w, kmask = wk & 0xFF, wk >> 8
            for k in range(K):
                if not (kmask >> k) & 1:
                    continue
                for u in range(w):
                    v = float(plan["vals"][voff + k * 8 + u])
                    y[:, k, row, :] += v * x[:, srow, (start + t0 + m * step + u) % n_src]
    return y


def adjoint(plan, dy, nlat_in, nlon_in, stride):
    """dx (B*C, nlat_in, nlon_in) from dy (B*C, K*nlat_out, nlon_out) via the adjoint plan."""
    BC, _, n_src = dy.shape
    dx = np.zeros((BC, nlat_in, nlon_in))
    m = np.arange(n_src)
    for r in plan["rows"]:
        row, sb = r[0], r[1]
        for t in range(r[11], r[12]):
            srow = plan["rings"][t][0]
            dx[:, row, :] += float(plan["ring_v"][t]) * dy[:, srow, :].sum(axis=-1)[:, None]
        for rho in range(stride):
            for ch in range(r[3 + rho], r[7 + rho]):
                src, t0, voff, wk = plan["chunks"][ch]
                srow, start = plan["srcs"][sb + src][:2]
                for u in range(wk & 0xFF):
                    v = float(plan["vals"][voff + u])
                    dx[:, row, stride * m + rho] += v * dy[:, srow, (start + t0 + m + u) % n_src]
    return dx
