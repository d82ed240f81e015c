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


def _s16(v):
    v = int(v) & 0xFFFF
    return v - 0x10000 if v & 0x8000 else v


def ring(plan, src, n_out_rows):
    """Re-enacts the strip-staged kernel on a ring plan, in fp64, and checks its protocol.

    src (B*C, source rows, nlon) -> out (B*C, K, n_out_rows, nlon).  For every tile (strip,
    q-tile, plane tile) the producer's loads fill ring slots octet by octet, (q0/8 + first octet
    + o) mod (nlon/8), group 0 from the source row and group 1 from the mirror source row (or the
    next 64 planes); every item then runs, for each block b and each of its K-steps k inside the
    load, the MMA D[(group, plane), (k', u)] += sum over 16 longitudes of A * B with A = octets
    a_off + 2b + 2k, +1 of the slot and B = K-step k - kb0 of the item's Toeplitz copy; finished
    rows are written like the epilogue's TMA stores (clipped at nlon and at the last plane).
    Asserted on the way: every octet read lies inside its load and its slot, every B K-step
    inside the item's copy (at most bk), a slot is refilled only after its previous load had
    its last use, a row buffer is reused only after the rows started before have completed, and
    every load and row of a strip ends within the strip."""
    K, N, nb, wmax, ns, nrb, bk = (plan[k] for k in ("K", "N", "nb", "wmax", "ns", "nrb", "bk"))
    mirror = plan["mirror"]
    BC, n_src, nlon = src.shape
    PT = 64 if mirror else 128
    n_pt = -(-BC // PT)
    n_qt = -(-nlon // (16 * nb))
    ring_oct = nlon // 8
    vals = _bf16_values(plan["b"])
    out = np.zeros((BC, K, n_out_rows, nlon))
    srcp = np.zeros((n_pt * PT + 64, n_src, nlon))
    srcp[:BC] = src
    for st in plan["strips"]:
        item0, item1, load0, load1, row0, row1 = (int(v) for v in st[:6])
        for qt in range(n_qt):
            for pt in range(n_pt):
                q0, plane0 = qt * 16 * nb, pt * PT
                slots = np.zeros((ns, wmax, 2, 64, 8))
                owner = [-1] * ns
                released = set()
                issued = 0
                acc, buf_row = {}, {}
                started_rows, done_rows = [], set()
                buf_prev = {}
                for n in range(item0, item1):
                    w0, w1, w2, boff = (int(v) for v in plan["items"][n])
                    L, row = w0 & 0xFFFF, w0 >> 16
                    a_off, ks, flags = _s16(w1), (w1 >> 16) & 0xFF, (w1 >> 24) & 0xFF
                    kb0, nkb, n_oct_it = w2 & 0xFF, (w2 >> 8) & 0xFF, (w2 >> 16) & 0xFF
                    rb, slot = (w2 >> 24) & 0xF, (w2 >> 28) & 0xF
                    while issued <= L:
                        l0, l1 = (int(v) for v in plan["loads"][load0 + issued])
                        s, sbar = l0 & 0xFFFF, (l0 >> 16) & 0xFFFF
                        o0, n_oct, sl = _s16(l1), (l1 >> 16) & 0xFF, (l1 >> 24) & 0xF
                        assert 0 < n_oct <= wmax and sl < ns, "load larger than a slot"
                        assert owner[sl] < 0 or owner[sl] in released, "slot refilled before its last use"
                        for o in range(n_oct):
                            oc = (q0 // 8 + o0 + o) % ring_oct
                            lon = slice(8 * oc, 8 * oc + 8)
                            slots[sl, o, 0] = srcp[plane0: plane0 + 64, s, lon]
                            slots[sl, o, 1] = (srcp[plane0: plane0 + 64, sbar, lon] if mirror
                                               else srcp[plane0 + 64: plane0 + 128, s, lon])
                        owner[sl] = issued
                        issued += 1
                    assert load0 + L < load1 and owner[slot] == L, "item reads a slot its load is not in"
                    n_oct = (int(plan["loads"][load0 + L][1]) >> 16) & 0xFF
                    assert n_oct_it == n_oct, "item and load disagree on the load's size"
                    if flags & 4:
                        prev = buf_prev.get(rb)
                        if prev is not None:
                            # drained in start order: every row started up to prev is complete
                            upto = started_rows.index(prev)
                            assert all(r in done_rows for r in started_rows[: upto + 1]), "row buffer reused early"
                        acc[rb] = np.zeros((nb, 128, N))
                        buf_row[rb] = row
                        buf_prev[rb] = row
                        started_rows.append(row)
                    assert buf_row.get(rb) == row, "item outside its row's buffer"
                    assert 0 < nkb <= bk, "B copy larger than a slot"
                    blk = vals[8 * boff: 8 * boff + nkb * 2 * N * 8].reshape(nkb, 2, N, 8)
                    Bm = blk.transpose(0, 1, 3, 2).reshape(nkb, 16, N)  # [K-step][8*octet + e][n]
                    for b in range(nb):
                        base = a_off + 2 * b
                        for k in range(kb0, min(kb0 + nkb, ks)):
                            o = base + 2 * k
                            if o < 0 or o + 2 > n_oct:
                                continue
                            assert o + 2 <= wmax
                            A = slots[slot, o: o + 2].transpose(1, 2, 0, 3).reshape(128, 16)
                            acc[rb][b] += A @ Bm[k - kb0]
                    if flags & 1:
                        released.add(L)
                    if flags & 2:
                        r0, _ = (int(v) for v in plan["rows"][row0 + row])
                        r, rbar = r0 & 0xFFFF, (r0 >> 16) & 0xFFFF
                        for b in range(nb):
                            q = q0 + 16 * b
                            if q >= nlon:
                                continue
                            w = min(16, nlon - q)
                            d = acc[rb][b].reshape(2, 64, K, 16)
                            p1 = min(BC, plane0 + 64)
                            out[plane0:p1, :, r, q: q + w] = d[0, : p1 - plane0, :, :w]
                            if mirror:
                                if rbar != r and rbar != 0xFFFF:
                                    out[plane0:p1, :, rbar, q: q + w] = d[1, : p1 - plane0, :, :w]
                            elif plane0 + 64 < BC:
                                p2 = min(BC, plane0 + 128)
                                out[plane0 + 64: p2, :, r, q: q + w] = d[1, : p2 - plane0 - 64, :, :w]
                        done_rows.add(row)
                assert issued == load1 - load0 and released == set(range(issued)), "a load never issued or released"
                assert set(started_rows) == done_rows, "a row never completed"
    return out
