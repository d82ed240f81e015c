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


def tile(plan, src, n_out_rows):
    """Re-enacts the TMA-staged strip kernel on a tile-script plan, in fp64, and checks its protocol.

    src (B*C, source rows, nlon) -> out (B*C, K, n_out_rows, nlon).  For every script (strip,
    longitude tile) and plane tile: each load fills its ring slot's chunks, chunk c holding the
    64 longitudes from x0 + 56c (zeros outside [0, nlon)) of the source row (M rows 0..63) and of
    the mirror source row or the next 64 planes (M rows 64..127); the copies of each batch fill a
    B slot with the batch record and the Toeplitz K-steps.  Per batch, each issuer takes the
    loads and rows that the record says start in it, then runs its MMA list: an MMA word adds A
    (128 x 16: the 16 longitudes from octet `pos` of the addressed chunk) times B (16 x N: the
    addressed K-step of the slot) into its block's columns of the row buffer, the first one of a
    (row, block) replacing it.  Finished rows are written like the epilogue's stores (clipped at
    nlon and at the last plane).
    Asserted on the way: the record and K-steps lie inside the B slot and the record is complete;
    every A operand lies inside a staged chunk of the slot's current load and in a batch no later
    than that load's release batch; a slot takes its next load, and a row buffer its next row,
    only in a batch after the release of the previous one (for a row buffer: of every row started
    up to the previous one); every B operand lies inside its slot's K-steps; the accumulate bit is
    clear exactly on the first MMA of a (row, block); every row's MMAs lie in batches up to its
    recorded last one; every load, copy and row of a script is used; every (row, tile) is written
    once."""
    K, N, nb, ns, nrb, nbs, bslot = (plan[k] for k in ("K", "N", "nb", "ns", "nrb", "nbs", "bslot_bytes"))
    assert nb == 4
    META = 1024
    mirror = plan["mirror"]
    BC, n_src, nlon = src.shape
    PT = 64 if mirror else 128
    n_pt = -(-BC // PT)
    n_qt = plan["n_qt"]
    assert n_qt == -(-nlon // 64)
    kstep = 32 * N
    bbytes = plan["b"].astype(np.uint16).tobytes()
    rbytes = plan["cmds"].astype(np.uint32).tobytes()
    out = np.zeros((BC, K, n_out_rows, nlon))
    written = np.zeros((n_out_rows, n_qt), dtype=np.int64)
    srcp = np.zeros((n_pt * PT + 64, n_src, nlon))
    srcp[:BC] = src
    cta = plan["cta_tiles"]
    n_ctas = plan["n_ctas"]
    assert sorted(cta[n_ctas + 1:].tolist()) == list(range(plan["n_strips"] * n_qt)), "a script not run exactly once"
    for si, rec in enumerate(plan["tiles"]):
        load0, load1, copy0, copy1, row0, row1 = (int(v) for v in rec[:6])
        nbatch = int(rec[11])
        q0 = (si % n_qt) * 64
        loads = plan["loads"][load0:load1]
        copies = plan["copies"][copy0:copy1]
        rows = plan["rows"][row0:row1]
        # batch slots from the copies
        batches, cur = [], None
        for c in copies:
            off16, nbytes, dst, fl = (int(v) for v in c)
            flags, total = fl & 0xFF, (fl >> 8) & 0xFFFF
            if flags & 1:
                assert cur is None and flags & 4, "a batch does not start with its record"
                cur = {"total": total, "data": bytearray(bslot), "filled": 0, "kend": META,
                       "ncopies": (fl >> 24) & 0xFF, "seen": 0}
            assert cur is not None and dst % 16 == 0 and dst + nbytes <= bslot and nbytes % 16 == 0
            srcb = rbytes if flags & 4 else bbytes
            assert 16 * off16 + nbytes <= len(srcb), "copy outside its source array"
            cur["data"][dst: dst + nbytes] = srcb[16 * off16: 16 * off16 + nbytes]
            cur["filled"] += nbytes
            cur["seen"] += 1
            if flags & 4:
                assert dst == 0 and nbytes <= META
            else:
                assert dst >= META and nbytes % kstep == 0
                cur["kend"] = max(cur["kend"], dst + nbytes)
            if flags & 2:
                assert cur["filled"] == cur["total"] <= bslot, "batch bytes disagree with its copies"
                assert cur["seen"] == cur["ncopies"] <= 32, "batch copy count disagrees with its copies"
                batches.append(cur)
                cur = None
        assert cur is None and len(batches) == nbatch, "batch count disagrees with the script"
        for bt in batches:
            w = np.frombuffer(bytes(bt["data"][:META]), dtype=np.uint32)
            bt["words"] = w
            bt["vals"] = _bf16_values(np.frombuffer(bytes(bt["data"]), dtype=np.uint16))
        # loads by slot, in order
        by_slot = {}
        for L, ld in enumerate(loads):
            slot, mask = int(ld[1]) & 0xFF, (int(ld[1]) >> 8) & 0xFF
            assert slot < ns and 0 < mask < 4 and 0 <= (int(ld[3]) & 0xFFFF) < nbatch
            by_slot.setdefault(slot, []).append(L)
        # rows by buffer, in start order
        by_buf, start_order = {}, []
        for R, rw in enumerate(rows):
            if not int(rw[1]) & 1:
                by_buf.setdefault((int(rw[1]) >> 8) & 0xF, []).append(R)
                start_order.append(R)
        row_done_batch = {R: int(rows[R][1]) >> 12 for R in start_order}
        for pt in range(n_pt):
            plane0 = pt * PT

            def chunk(ld, c):
                s, sbar = int(ld[0]) & 0xFFFF, (int(ld[0]) >> 16) & 0xFFFF
                x0 = int(ld[2]) + 56 * c
                ch = np.zeros((2, 64, 64))
                lo, hi = max(0, x0), min(nlon, x0 + 64)
                if hi > lo:
                    ch[0, :, lo - x0: hi - x0] = srcp[plane0: plane0 + 64, s, lo:hi]
                    ch[1, :, lo - x0: hi - x0] = (srcp[plane0: plane0 + 64, sbar, lo:hi] if mirror
                                                  else srcp[plane0 + 64: plane0 + 128, s, lo:hi])
                return ch.reshape(128, 64)

            def store(R, iw, Dblk):
                r, rbar = int(rows[R][0]) & 0xFFFF, (int(rows[R][0]) >> 16) & 0xFFFF
                q = q0 + 16 * iw
                if q >= nlon:
                    return
                wd = min(16, nlon - q)
                d = Dblk.reshape(2, 64, K, 16)
                p1 = min(BC, plane0 + 64)
                out[plane0:p1, :, r, q: q + wd] = d[0, : p1 - plane0, :, :wd]
                if mirror:
                    if rbar != r and rbar != 0xFFFF:
                        out[plane0:p1, :, rbar, q: q + wd] = d[1, : p1 - plane0, :, :wd]
                elif plane0 + 64 < BC:
                    p2 = min(BC, plane0 + 128)
                    out[plane0 + 64: p2, :, r, q: q + wd] = d[1, : p2 - plane0 - 64, :, :wd]

            D = np.zeros((nrb, 128, nb * N))
            row_stored = {}
            for iw in range(nb):
                slot_load, slot_use = {}, {s: 0 for s in range(ns)}
                buf_row, buf_use = {}, {r: 0 for r in range(nrb)}
                started = set()
                cols = slice(iw * N, (iw + 1) * N)
                for bcur, bt in enumerate(batches):
                    h = bt["words"]
                    n = int(h[0] >> (8 * iw)) & 0xFF
                    off = 4 if iw == 0 else int(h[1] >> (10 * (iw - 1))) & 0x3FF
                    offs = [4] + [int(h[1] >> (10 * j)) & 0x3FF for j in range(3)]
                    cnts = [int(h[0] >> (8 * j)) & 0xFF for j in range(4)]
                    assert all(offs[j] + cnts[j] == offs[j + 1] for j in range(3)), "record lists overlap"
                    assert 4 * (offs[3] + cnts[3]) <= META
                    for j in range(int(h[2]) & 7):
                        slot = int(h[2] >> (3 + 4 * j)) & 0xF
                        seq = by_slot.get(slot, [])
                        assert slot_use[slot] < len(seq), "slot started more often than loaded"
                        if slot in slot_load:
                            assert bcur > (int(loads[slot_load[slot]][3]) & 0xFFFF), \
                                "slot refilled before its release batch"
                        assert int(loads[seq[slot_use[slot]]][3]) >> 16 == bcur, "load's first batch field wrong"
                        slot_load[slot] = seq[slot_use[slot]]
                        slot_use[slot] += 1
                    for j in range(int(h[3]) & 7):
                        rb = int(h[3] >> (3 + 3 * j)) & 7
                        seq = by_buf.get(rb, [])
                        assert buf_use[rb] < len(seq), "row buffer started more often than rows use it"
                        if rb in buf_row:
                            prev = buf_row[rb]
                            upto = start_order.index(prev)
                            assert all(bcur > row_done_batch[R] for R in start_order[: upto + 1]), \
                                "row buffer reused before the rows started earlier are complete"
                            store(prev, iw, D[rb][:, cols])
                            row_stored.setdefault(prev, set()).add(iw)
                        buf_row[rb] = seq[buf_use[rb]]
                        buf_use[rb] += 1
                    for w in (int(v) for v in h[off: off + n]):
                        a = (w & 0x3FFF) * 16
                        boff = ((w >> 14) & 0x3FF) * 16
                        rb, accb = (w >> 24) & 7, (w >> 27) & 1
                        slot, c, pos = a // 32768, (a % 32768) // 16384, (a % 16384) // 16
                        assert pos <= 6 and slot in slot_load, "A outside a started slot or its chunk"
                        ld = loads[slot_load[slot]]
                        assert (int(ld[1]) >> 8) & (1 << c), "A in a chunk that was not staged"
                        assert bcur <= (int(ld[3]) & 0xFFFF), "A read after its load's release batch"
                        assert META <= boff and boff + kstep <= bt["kend"], "B outside the slot's K-steps"
                        assert rb in buf_row, "MMA into a row buffer not started"
                        R = buf_row[rb]
                        assert bcur <= row_done_batch[R], "MMA after the row's last batch"
                        assert accb == (1 if (R, iw) in started else 0), "accumulate bit wrong"
                        started.add((R, iw))
                        A = chunk(ld, c)[:, 8 * pos: 8 * pos + 16]
                        blk = bt["vals"][boff // 2: boff // 2 + kstep // 2].reshape(2, N, 8)
                        Bm = blk.transpose(0, 2, 1).reshape(16, N)
                        D[rb][:, cols] = (D[rb][:, cols] if accb else 0) + A @ Bm
                for rb, R in buf_row.items():
                    store(R, iw, D[rb][:, cols])
                    row_stored.setdefault(R, set()).add(iw)
                assert all(slot_use[s] == len(by_slot.get(s, [])) for s in range(ns)), "a load never used"
                assert all(buf_use[r] == len(by_buf.get(r, [])) for r in range(nrb)), "a row never started"
            for R, rw in enumerate(rows):
                r, rbar = int(rw[0]) & 0xFFFF, (int(rw[0]) >> 16) & 0xFFFF
                if int(rw[1]) & 1:
                    assert R not in row_stored
                else:
                    assert row_stored.get(R) == set(range(nb)), "a row not finished by every issuer"
                if pt == 0:
                    written[r, si % n_qt] += 1
                    if mirror and rbar != r and rbar != 0xFFFF:
                        written[rbar, si % n_qt] += 1
    assert (written == 1).all(), "a (row, tile) written other than once"
    return out
