"""CPU check of the engine's launch geometry: every bulk copy the producer issues and every
shared-memory read a consumer makes stays inside its buffer, its stage and the rows that were
actually copied, for many shapes. Restates the address arithmetic of engine.cu on the host so
that no out-of-range access is ever tried on a GPU first."""
import itertools

import pytest

fmoe = pytest.importorskip("bit_dequant_expert_gemv_b200")

MAX_SMEM = 232448
KMAXW = 8

SHAPES = [
    # H, I, E, K, bits
    (4096, 1024, 512, 4, 4), (4096, 1024, 512, 4, 2), (256, 128, 16, 2, 4), (256, 128, 16, 2, 2),
    (64, 64, 1, 1, 4), (64, 64, 3, 3, 2), (192, 320, 7, 3, 4), (8192, 1024, 64, 8, 4),
    (7168, 2048, 256, 4, 4), (4160, 576, 33, 5, 2), (1024, 8192, 8, 1, 4), (2048, 704, 128, 6, 4),
    (128, 64, 4096, 8, 2),
]
FLAGS = [15, 7, 5, 1, 2]  # full layer+gate, no gate, no shared, router only, expert only


def chunks(G):
    for c in range(G["off5"]):
        p = max(i for i in range(5) if G[f"off{i}"] <= c and G[f"n{i}"] > 0)
        j = c - G[f"off{p}"]
        k = 0
        if p == 0:
            r0, n = j * G["rr"], min(G["rr"], G["nr"] - j * G["rr"])
        elif p == 1:
            r0, n = j * G["rcg"], min(G["rcg"], G["I"] - j * G["rcg"])
        elif p == 2:
            r0, n = j * G["rsd"], min(G["rsd"], G["H"] - j * G["rsd"])
        elif p == 3:
            k, jj = divmod(j, G["nb"])
            r0, n = jj * G["rcg"], min(G["rcg"], G["I"] - jj * G["rcg"])
        else:
            r0, n = j * G["rrd"], min(G["rrd"], G["H"] - j * G["rrd"])
        assert n > 0
        yield c, p, j, k, r0, n


def producer_copies(G, p, k, r0, n):
    """(buffer, src_off, dst_off, bytes) per copy, as the producer issues them."""
    H, I, E, K = G["H"], G["I"], G["E"], G["K"]
    out = []
    if p == 0:
        rowb = 4 * H
        a, b = r0, min(r0 + n, E)
        if b > a:
            out.append(("router", a * rowb, 0, (b - a) * rowb))
        if r0 + n > E:
            out.append(("gate", 0, (E - r0) * rowb, rowb))
    elif p in (1, 3):
        buf = "shared" if p == 1 else "expert"
        cb, sbb = n * G["rc_h"], n * G["rs_h"]
        sbo = I * G["rc_h"]
        out += [(buf, r0 * G["rc_h"], 0, cb),
                (buf, G["q_gu"] + r0 * G["rc_h"], G["rcg"] * G["rc_h"], cb),
                (buf, sbo + r0 * G["rs_h"], 2 * G["rcg"] * G["rc_h"], sbb),
                (buf, G["q_gu"] + sbo + r0 * G["rs_h"], 2 * G["rcg"] * G["rc_h"] + G["rcg"] * G["rs_h"], sbb)]
    elif p == 2:
        base = 2 * G["q_gu"]
        cb, sbb = n * G["rc_i"], n * G["rs_i"]
        out += [("shared", base + r0 * G["rc_i"], 0, cb),
                ("shared", base + H * G["rc_i"] + r0 * G["rs_i"], G["rsd"] * G["rc_i"], sbb)]
    else:
        cb, sbb = n * G["rc_i"], n * G["rs_i"]
        dsb = K * G["rrd"] * G["rc_i"]
        base = 2 * G["q_gu"]
        for kk in range(K):
            out += [("expert", base + r0 * G["rc_i"], kk * G["rrd"] * G["rc_i"], cb),
                    ("expert", base + H * G["rc_i"] + r0 * G["rs_i"], dsb + kk * G["rrd"] * G["rs_i"], sbb)]
    return out


def consumer_reads(G, p, n):
    """Yield (kind, stage_off, bytes, x_buf, x_index) for every valid read of every thread."""
    bits = G["bits"]
    sbytes = 16 if bits == 4 else 8
    K = G["K"]
    if p in (1, 3):
        sp, P, sl, W = G["sp_h"], G["p_h"], G["sl_h"], G["w_gu"]
        half = G["rcg"]
    elif p == 2:
        sp, P, sl, W, half = G["sp_i"], G["p_i"], G["sl_i"], 4, 0
    else:
        sp, P, sl, W, half = G["sp_d"], G["p_d"], G["sl_d"], 4, 0
    for t in range(256):
        pp, s = divmod(t, sp)
        if not (pp < P and s < sl):
            continue
        if p in (1, 3):
            a_row, a_slice = G["rc_h"], s * sbytes
            b_base, b_row, b_slice = 2 * G["rcg"] * G["rc_h"], G["rs_h"], (s >> 1) * 4
            xbuf, xlen, sxlen = "XG", G["H"], G["sl_h"]
        elif p == 2:
            a_row, a_slice = G["rc_i"], s * sbytes
            b_base, b_row, b_slice = G["rsd"] * G["rc_i"], G["rs_i"], (s >> 1) * 4
            xbuf, xlen, sxlen = "XS", G["I"], G["sl_i"]
        else:
            kk, si = divmod(s, G["sl_i"])
            a_row, a_slice = G["rc_i"], kk * G["rrd"] * G["rc_i"] + si * sbytes
            b_base, b_row, b_slice = K * G["rrd"] * G["rc_i"], G["rs_i"], kk * G["rrd"] * G["rs_i"] + (si >> 1) * 4
            xbuf, xlen, sxlen = "XD", K * G["I"], G["sl_d"]
        assert s * 32 + 32 <= xlen and s < sxlen, (xbuf, s)
        for w in range(W):
            vr = pp + w * P
            if half:
                ok = vr < 2 * half and ((vr < half and vr < n) or (vr >= half and vr - half < n))
            else:
                ok = vr < n
            if ok:
                yield "code", a_slice + vr * a_row, sbytes, vr, s
                yield "sb", b_base + b_slice + vr * b_row, 4, vr, s


def clamped_reads(G, p):
    """Every thread reads a clamped, in-stage address even for rows or slices it then zeroes."""
    bits = G["bits"]
    sbytes = 16 if bits == 4 else 8
    K = G["K"]
    if p in (1, 3):
        sp, P, sl, W, vmax = G["sp_h"], G["p_h"], G["sl_h"], G["w_gu"], 2 * G["rcg"] - 1
    elif p == 2:
        sp, P, sl, W, vmax = G["sp_i"], G["p_i"], G["sl_i"], 4, G["rsd"] - 1
    else:
        sp, P, sl, W, vmax = G["sp_d"], G["p_d"], G["sl_d"], 4, G["rrd"] - 1
    for t in range(256):
        pp, s = divmod(t, sp)
        sc = min(s, sl - 1)
        for w in range(W):
            vc = min(pp + w * P, vmax)
            if p in (1, 3):
                a = sc * sbytes + vc * G["rc_h"]
                b = 2 * G["rcg"] * G["rc_h"] + (sc >> 1) * 4 + vc * G["rs_h"]
            elif p == 2:
                a = sc * sbytes + vc * G["rc_i"]
                b = G["rsd"] * G["rc_i"] + (sc >> 1) * 4 + vc * G["rs_i"]
            else:
                kk, si = divmod(sc, G["sl_i"])
                a = kk * G["rrd"] * G["rc_i"] + si * sbytes + vc * G["rc_i"]
                b = K * G["rrd"] * G["rc_i"] + kk * G["rrd"] * G["rs_i"] + (si >> 1) * 4 + vc * G["rs_i"]
            yield a, sbytes, b


def reduce_red_extent(G, p):
    sp = {1: G["sp_h"], 3: G["sp_h"], 2: G["sp_i"], 4: G["sp_d"]}[p]
    W = G["w_gu"] if p in (1, 3) else 4
    width = min(sp, 32)
    if sp >= 32:
        return (8 - 1) * KMAXW + W
    return (256 // sp - 1) * KMAXW + W if W <= width else (256 // sp - 1) * KMAXW + W


@pytest.mark.parametrize("shape,flags", list(itertools.product(SHAPES, FLAGS)))
def test_geometry_in_bounds(shape, flags):
    H, I, E, K, bits = shape
    try:
        G = fmoe.describe_geometry(H, I, E, K, bits, flags, MAX_SMEM)
    except fmoe.FmoeError as e:
        assert e.code == fmoe.FMOE_ERR_UNSUPPORTED
        pytest.skip(str(e))
    assert G["smem_bytes"] <= MAX_SMEM
    ns, sb = G["nstage"], G["stage_bytes"]
    assert ns >= 2 and sb % 128 == 0
    # carve-up: ring | x areas | barriers | meta, non-overlapping and in order
    areas = [("ring", 0, ns * sb), ("xr", G["o_xr"], 4 * H), ("xg", G["o_xg"], 4 * H),
             ("sxg", G["o_sxg"], 4 * (H // 32)), ("xs", G["o_xs"], 4 * I), ("sxs", G["o_sxs"], 4 * (I // 32)),
             ("xd", G["o_xd"], 4 * K * I), ("sxd", G["o_sxd"], 4 * K * (I // 32)), ("red", G["o_red"], 16),
             ("box", G["o_box"], 4 * 4 * G["box_floats"]), ("misc", G["o_misc"], 512), ("full", G["o_full"], 8 * ns), ("empty", G["o_empty"], 8 * ns),
             ("meta", G["o_meta"], 4 * ns)]
    for (n1, a1, l1), (n2, a2, l2) in zip(areas, areas[1:]):
        assert a1 + l1 <= a2, (n1, n2)
    assert areas[-1][1] + areas[-1][2] <= G["smem_bytes"]
    assert G["o_full"] % 8 == 0 and G["o_empty"] % 8 == 0 and G["o_xr"] % 16 == 0
    sizes = {"router": E * H * 4, "gate": H * 4, "shared": fmoe.expert_bytes(H, I, bits),
             "expert": fmoe.expert_bytes(H, I, bits)}
    assert G["q_gu"] * 2 + G["q_dn"] == sizes["expert"]
    seen = set()
    for c, p, j, k, r0, n in chunks(G):
        copies = producer_copies(G, p, k, r0, n)
        assert len(copies) <= 16
        covered = []
        for buf, so, do, nb in copies:
            assert nb > 0 and nb % 16 == 0 and so % 16 == 0 and do % 16 == 0, (p, buf, so, do, nb)
            assert so + nb <= sizes[buf], (p, buf, so, nb, sizes[buf])
            assert do + nb <= sb, (p, do, nb, sb)
            covered.append((do, do + nb))
        covered.sort()
        for (a, b), (c2, d) in zip(covered, covered[1:]):
            assert b <= c2, "copies overlap in the stage"
        if p == 0:
            assert n <= 32 and n * 4 * H <= sb and 2 * 8 * n <= G["red_part"]
            continue
        jn = G[f"n{p}"]
        if p == 3:
            j = j % G["nb"]
            jn = G["nb"]
        if j not in (0, 1, jn - 1):  # thread reads: first, second and last (ragged) chunk
            continue
        for kind, off, nbytes, vr, s in consumer_reads(G, p, n):
            assert any(a <= off and off + nbytes <= b for a, b in covered), (p, kind, off, nbytes, vr, s, covered)
        assert reduce_red_extent(G, p) <= G["red_part"]
        for a, nb, b in clamped_reads(G, p):
            assert 0 <= a and a + nb <= sb and 0 <= b and b + 4 <= sb, (p, a, b, sb)
        # reduction slot: partials of every segment, then one base per output row
        nseg = lambda sp: 8 if sp >= 32 else 256 // sp
        spp = {1: G["sp_h"], 3: G["sp_h"], 2: G["sp_i"], 4: G["sp_d"]}.get(p)
        if spp:
            assert nseg(spp) * KMAXW <= G["red_part"]
        assert G["red_part"] + n <= G["box_floats"]
        if p in (1, 3):
            assert r0 + n <= I and n <= G["rcg"] and k < K
        else:
            assert r0 + n <= H
        seen.add(p)
    # every output row and every h entry is produced exactly once per unit
    if G["routed_on"]:
        rows = [(r0, n) for c, p, j, k, r0, n in chunks(G) if p == 4]
        assert sum(n for _, n in rows) == H
        hk = sorted((k, r0, n) for c, p, j, k, r0, n in chunks(G) if p == 3)
        assert sum(n for _, _, n in hk) == K * I
    if G["shared_on"]:
        assert sum(n for c, p, j, k, r0, n in chunks(G) if p == 1) == I
        assert sum(n for c, p, j, k, r0, n in chunks(G) if p == 2) == H
    if G["route_on"]:
        assert sum(n for c, p, j, k, r0, n in chunks(G) if p == 0) == G["nr"]


def test_unsupported_shapes_are_refused():
    for shape in [(16384, 1024, 8, 2, 4), (4096, 4096, 8, 4, 4), (4096, 1024, 16, 9, 4)]:
        with pytest.raises(fmoe.FmoeError) as ei:
            fmoe.describe_geometry(*shape)
        assert ei.value.code == fmoe.FMOE_ERR_UNSUPPORTED
    with pytest.raises(fmoe.FmoeError) as ei:
        fmoe.describe_geometry(100, 128, 8, 2, 4)
    assert ei.value.code == fmoe.FMOE_ERR_INVALID
