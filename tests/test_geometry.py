"""CPU check of the engine's launch geometry: every bulk copy the producer and the stager issue
and every shared-memory read a consumer warp makes stays inside its buffer, its stage and the
rows that were actually copied, for many shapes. Restates the address arithmetic of engine.cu
on the host so that no out-of-range access is ever tried on a GPU first."""
import itertools

import pytest

fmoe = pytest.importorskip("bit_dequant_expert_gemv_b200")

MAX_SMEM = 232448
ROWS_PER_LANE = 8
CONSUMER_WARPS = 8

SHAPES = [
    # H, I, E, K, bits
    (4096, 1024, 512, 4, 4), (4096, 1024, 512, 4, 2), (256, 128, 16, 2, 4), (256, 128, 16, 2, 2),
    (64, 64, 1, 1, 4), (64, 64, 3, 3, 2), (192, 320, 7, 3, 4), (8192, 1024, 64, 8, 4),
    (7168, 2048, 256, 4, 4), (4160, 576, 33, 5, 2), (1024, 8192, 8, 1, 4), (2048, 704, 128, 6, 4),
    (128, 64, 4096, 8, 2), (8128, 192, 16, 2, 4),
]
FLAGS = [15, 7, 5, 1, 2]  # full layer+gate, no gate, no shared, router only, expert only
K_ROUTER, K_SGU, K_RGU, K_DN = range(4)


def chunks(G):
    """(c, kind, j, k, seg, r0, n) for every chunk of one unit, as the kernel decodes them."""
    for c in range(G["off4"]):
        kind = max(i for i in range(4) if G[f"off{i}"] <= c and G[f"n{i}"] > 0)
        j = c - G[f"off{kind}"]
        k = seg = 0
        if kind == K_ROUTER:
            rb, seg = divmod(j, G["rseg"])
            r0 = rb * G["rrows"]
            n = min(G["rrows"], G["nr"] - r0)
        elif kind == K_SGU:
            r0, n = j * G["R"], min(G["R"], G["I"] - j * G["R"])
        elif kind == K_RGU:
            k, jj = divmod(j, G["nb"])
            r0, n = jj * G["R"], min(G["R"], G["I"] - jj * G["R"])
        else:
            r0, n = j * G["Rd"], min(G["Rd"], G["H"] - j * G["Rd"])
        assert n > 0
        yield c, kind, j, k, seg, r0, n


def producer_copies(G, kind, k, seg, r0, n):
    """(buffer, src_off, dst_off, bytes) per copy, as the producer issues them."""
    H, I, E = G["H"], G["I"], G["E"]
    out = []
    if kind == K_ROUTER:
        if G["rseg"] == 1:
            rowb = 4 * H
            a, b = r0, min(r0 + n, E)
            if b > a:
                out.append(("router", a * rowb, 0, (b - a) * rowb))
            if r0 + n > E:
                out.append(("gate", 0, (E - r0) * rowb, rowb))
        else:
            buf, base = ("router", r0 * 4 * H) if r0 < E else ("gate", 0)
            out.append((buf, base + seg * G["rcols"] * 4, 0, 4 * G["rcols"]))
    elif kind in (K_SGU, K_RGU):
        buf = "shared" if kind == K_SGU else "expert"
        cb, sbb = n * G["rc_h"], n * G["rs_h"]
        sbo = I * G["rc_h"]
        R = G["R"]
        out += [(buf, r0 * G["rc_h"], 0, cb),
                (buf, G["q_gu"] + r0 * G["rc_h"], R * G["rc_h"], cb),
                (buf, sbo + r0 * G["rs_h"], 2 * R * G["rc_h"], sbb),
                (buf, G["q_gu"] + sbo + r0 * G["rs_h"], 2 * R * G["rc_h"] + R * G["rs_h"], sbb)]
    else:
        cb, sbb = n * G["rc_i"], n * G["rs_i"]
        Rd, nseg = G["Rd"], G["nseg"]
        dsb = nseg * Rd * G["rc_i"]
        dn = 2 * G["q_gu"]
        for s in range(nseg):
            buf = "shared" if (G["shared_on"] and s == 0) else "expert"
            out += [(buf, dn + r0 * G["rc_i"], s * Rd * G["rc_i"], cb),
                    (buf, dn + H * G["rc_i"] + r0 * G["rs_i"], dsb + s * Rd * G["rs_i"], sbb)]
    return out


def lane_reads(G, kind, n):
    """Every shared-memory read of every lane of the consumer warp for a dot-product chunk:
    yields (valid, code_off, code_bytes, sb_off, row, slice), including the clamped reads that
    rows or slices outside the chunk make (valid False)."""
    cbytes = 16 if G["bits"] == 4 else 8
    if kind in (K_SGU, K_RGU):
        pre = "gu"
        nrows, R = 2 * G["R"], G["R"]
        valid = lambda rho: rho < 2 * R and (rho if rho < R else rho - R) < n
        rc, rs, seg_c, seg_s = G["rc_h"], G["rs_h"], 0, 0
        sb0, spseg = 2 * R * G["rc_h"], G["H"] // 32
    else:
        pre = "dn"
        nrows = n
        valid = lambda rho: rho < n
        rc, rs = G["rc_i"], G["rs_i"]
        seg_c, seg_s = G["Rd"] * G["rc_i"], G["Rd"] * G["rs_i"]
        sb0, spseg = G["nseg"] * G["Rd"] * G["rc_i"], G["I"] // 32
    nsl, S, P, nrl = (G[f"{pre}_{f}"] for f in ("nsl", "S", "P", "nrl"))
    NRL = 3 if nrl <= 3 else 4 if nrl == 4 else 6 if nrl <= 6 else 8
    GW = 4 if NRL % 4 == 0 else 3
    nj = (nsl + S - 1) // S
    for lane in range(32):
        ls, lp = lane % S, lane // S
        for j in range(nj):
            t = ls + S * j
            tok = t < nsl
            tc = t if tok else nsl - 1
            seg, loc = divmod(tc, spseg)
            cbase = seg * seg_c + loc * cbytes
            sbase = sb0 + seg * seg_s + (loc >> 1) * 4
            for g in range(0, NRL, GW):
                if g and not P * g < nrows:
                    continue
                for w in range(GW):
                    rho = lp + P * (g + w)
                    ok = tok and valid(rho)
                    rr = rho if ok else 0
                    yield ok, cbase + rr * rc, cbytes, sbase + rr * rs, rho, tc


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
    assert 2 <= ns <= 32 and sb % 128 == 0
    nseg = G["nseg"]
    xa_len = 4 * max(H, nseg * I)
    # carve-up: ring | fixed areas | barriers, non-overlapping and in order
    # x areas: 128 bytes per 32-column slice (raw floats, or six digit chunks + {scale, sum})
    areas = [("ring", 0, ns * sb), ("xa", G["o_xa"], xa_len), ("xg", G["o_xg"], 4 * H),
             ("red", G["o_red"], 4 * CONSUMER_WARPS * 16 * ROWS_PER_LANE),
             ("misc", G["o_misc"], 512), ("full", G["o_full"], 8 * ns), ("empty", G["o_empty"], 8 * ns)]
    for (n1, a1, l1), (n2, a2, l2) in zip(areas, areas[1:]):
        assert a1 + l1 <= a2, (n1, n2)
    assert areas[-1][1] + areas[-1][2] <= G["smem_bytes"]
    assert G["o_full"] % 8 == 0 and G["o_misc"] % 16 == 0
    for name in ("o_xa", "o_xg", "o_red"):
        assert G[name] % 16 == 0, name
    # stager bulk copies into XA: x, then h_s | h_k
    assert 4 * H <= xa_len and 4 * (nseg * I) <= xa_len
    assert (4 * I) % 16 == 0 and (4 * K * I) % 16 == 0 and (4 * H) % 16 == 0
    sizes = {"router": E * H * 4, "gate": H * 4, "shared": fmoe.expert_bytes(H, I, bits),
             "expert": fmoe.expert_bytes(H, I, bits)}
    assert G["q_gu"] * 2 + H * (G["rc_i"] + G["rs_i"]) == sizes["expert"]
    seen = set()
    for c, kind, j, k, seg, r0, n in chunks(G):
        copies = producer_copies(G, kind, k, seg, r0, n)
        assert len(copies) <= 2 * 9
        covered = []
        for buf, so, do, nb in copies:
            assert nb > 0 and nb % 16 == 0 and so % 16 == 0 and do % 16 == 0, (kind, buf, so, do, nb)
            assert so + nb <= sizes[buf], (kind, buf, so, nb, sizes[buf])
            assert do + nb <= sb, (kind, do, nb, sb)
            covered.append((do, do + nb))
        covered.sort()
        for (a, b), (c2, d) in zip(covered, covered[1:]):
            assert b <= c2, "copies overlap in the stage"
        if kind == K_ROUTER:
            # rows r0..r0+n-1 of rcols floats each, read as float4 by 32 lanes
            assert n * 4 * G["rcols"] <= sb and G["rcols"] % 4 == 0
            assert (seg + 1) * G["rcols"] <= H
            assert sum(b - a for a, b in covered) == n * 4 * G["rcols"]
            continue
        if kind in (K_SGU, K_RGU):
            assert r0 + n <= I and n <= G["R"] and k < K
        else:
            assert r0 + n <= H and n <= G["Rd"]
        # lane reads: first, second and last (ragged) chunk of each kind
        last = {K_SGU: G["nb"] - 1, K_RGU: G["nb"] - 1, K_DN: G["n3"] - 1}[kind]
        jj = j % G["nb"] if kind == K_RGU else j
        if jj not in (0, 1, last) or (kind, jj) in seen:
            continue
        seen.add((kind, jj))
        pre = "gu" if kind in (K_SGU, K_RGU) else "dn"
        x_len = H if pre == "gu" else nseg * I
        assert G[f"{pre}_nrl"] <= ROWS_PER_LANE and G[f"{pre}_P"] <= 16
        for ok, co, cbn, so, rho, t in lane_reads(G, kind, n):
            assert 0 <= co and co + cbn <= sb and 0 <= so and so + 4 <= sb, (kind, co, so, sb)
            assert 32 * t + 32 <= x_len, (kind, t, x_len)   # x' slice (the swizzle stays in it)
            if ok:
                assert any(a <= co and co + cbn <= b for a, b in covered), (kind, co, rho, t)
                assert any(a <= so and so + 4 <= b for a, b in covered), (kind, so, rho, t)
    # every output row and every h entry is produced exactly once per unit
    ch = list(chunks(G))
    if G["routed_on"] or G["shared_on"]:
        assert sum(n for c, kd, j, k, s, r0, n in ch if kd == K_DN) == H
        assert nseg == G["shared_on"] + (K if G["routed_on"] else 0)
    if G["routed_on"]:
        assert sum(n for c, kd, j, k, s, r0, n in ch if kd == K_RGU) == K * I
    if G["shared_on"]:
        assert sum(n for c, kd, j, k, s, r0, n in ch if kd == K_SGU) == I
    if G["route_on"]:
        assert sum(n for c, kd, j, k, s, r0, n in ch if kd == K_ROUTER) == G["nr"] * G["rseg"]
    assert G["ncl0"] == G["n0"] and G["ncl1"] == G["n1"] + G["n2"] and G["ncl2"] == G["n3"]


def test_unsupported_shapes_are_refused():
    for shape in [(16384, 1024, 8, 2, 4), (4096, 4096, 8, 4, 4), (4096, 1024, 16, 9, 4)]:
        with pytest.raises(fmoe.FmoeError) as ei:
            fmoe.describe_geometry(*shape)
        assert ei.value.code == fmoe.FMOE_ERR_UNSUPPORTED
    with pytest.raises(fmoe.FmoeError) as ei:
        fmoe.describe_geometry(100, 128, 8, 2, 4)
    assert ei.value.code == fmoe.FMOE_ERR_INVALID


def test_full_shape_chunking():
    """The 4-bit full-shape layer: 11.25 KB stages, gate/up chunks of 2+2 rows, down chunks of
    4 virtual rows of 5 segments (so both run the same 4-row dot-product code), router rows
    split in two column halves."""
    G = fmoe.describe_geometry(4096, 1024, 512, 4, 4, 15, MAX_SMEM)
    assert (G["rseg"], G["rcols"], G["R"], G["Rd"], G["nseg"]) == (2, 2048, 2, 4, 5)
    assert G["stage_bytes"] == 11520 and G["nstage"] >= 16
    assert (G["gu_S"], G["gu_P"], G["gu_nrl"]) == (32, 1, 4)
    assert (G["dn_S"], G["dn_P"], G["dn_nrl"]) == (32, 1, 4)
