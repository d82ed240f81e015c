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


def _bf16_values(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def toeplitz(plan, src, n_out_rows):
    """Re-enacts the tensor-core kernel on a Toeplitz plan, in fp64.

    src (B*C, source rows, nlon) -> out (B*C, K, n_out_rows, nlon).  For output q the kernel
    takes the group of 8 outputs q8 = q - q % 8 and, per slab (i, lon_off, nk, offset), the
    window of source longitudes (q8 + lon_off + p') mod nlon, p' < 16*nk, against column
    (k, u = q % 8) of the slab's block, summing the hi and lo parts."""
    K, parts, N = plan["K"], plan["parts"], plan["N"]
    BC, _, nlon = src.shape
    out = np.zeros((BC, K, n_out_rows, nlon))
    vals = _bf16_values(plan["b"])
    q = np.arange(nlon)
    u = q % 8
    q8 = q - u
    for row, s0, s1, _ in plan["slots"]:
        for i, lon_off, nk, boff in plan["slabs"][s0:s1]:
            n = 16 * nk
            blk = vals[8 * boff: 8 * boff + parts * 2 * nk * N * 8].reshape(parts, 2 * nk, N, 8)
            bm = blk.transpose(0, 1, 3, 2).reshape(parts, n, N)  # [part][p' = 8*octet + e][column]
            wsum = bm[0][:, : 8 * K] + (bm[0][:, 8 * K: 16 * K] if parts == 1 else bm[1][:, : 8 * K])
            wsum = wsum.reshape(n, K, 8)  # [p', k, u]
            idx = (q8[:, None] + lon_off + np.arange(n)[None, :]) % nlon  # [q, p']
            coef = wsum[np.arange(n)[None, :], :, u[:, None]]  # [q, p', k]
            out[:, :, row, :] += np.einsum("cqp,qpk->ckq", src[:, i, :][:, idx], coef)
    return out


def packed(plan, src, n_out_rows):
    """Re-enacts the packed tensor-core kernel on a packed plan, in fp64, and checks its slot
    protocol: every strip row starts once and completes once, after its last entry, and the
    rows live at any entry sit in distinct slots (row mod NR).

    src (B*C, source rows, nlon) -> out (B*C, K, n_out_rows, nlon), zero on the rows the plan
    leaves to the per-pair kernel."""
    K, Nr, NR = plan["K"], plan["Nr"], plan["NR"]
    BC, _, nlon = src.shape
    out = np.zeros((BC, K, n_out_rows, nlon))
    vals = _bf16_values(plan["b"])
    q = np.arange(nlon)
    u = q % 8
    q8 = q - u
    for e0, e1, o0, nrows in plan["strips"]:
        started, finished = set(), set()
        for s_row, lon_start, w2, boff, new_mask, done, _, _ in plan["entries"][e0:e1]:
            ks, n_rows, o_a = w2 & 0xFF, (w2 >> 8) & 0xFF, w2 >> 16
            for r in range(n_rows):
                o = o_a + r
                if (new_mask >> r) & 1:
                    assert o not in started
                    started.add(o)
                assert o in started and o not in finished, "contribution outside the row's life"
            live = started - finished
            assert len({o % NR for o in live}) == len(live), "two live rows share a slot"
            n = 16 * ks
            NC = n_rows * Nr
            blk = vals[8 * boff: 8 * boff + 2 * ks * NC * 8].reshape(2 * ks, NC, 8)
            bm = blk.transpose(0, 2, 1).reshape(n, n_rows, Nr)  # [p'][row][column]
            idx = (q8[:, None] + lon_start + np.arange(n)[None, :]) % nlon
            xs = src[:, s_row, :][:, idx]  # [c, q, p']
            for r in range(n_rows):
                wsum = (bm[:, r, : 8 * K] + bm[:, r, 8 * K: 16 * K]).reshape(n, K, 8)
                coef = wsum[np.arange(n)[None, :], :, u[:, None]]  # [q, p', k]
                out[:, :, o0 + o_a + r, :] += np.einsum("cqp,qpk->ckq", xs, coef)
            base, mask = done & 0xFFFF, (done >> 16) & 0xFFFF
            for bit in range(16):
                if (mask >> bit) & 1:
                    assert base + bit in started and base + bit not in finished
                    finished.add(base + bit)
        assert started == finished == set(range(nrows)), "a strip row never starts or never completes"
    return out
