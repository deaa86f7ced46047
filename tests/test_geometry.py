"""CPU check of the engine's launch geometry: every bulk copy the producers and the controller
issue and every shared-memory access the consumer warps make stays inside its buffer, its stage
and the rows that were actually copied, for many shapes and grid sizes; every router row,
h-row and output row is owned by exactly one CTA. Restates the address arithmetic of
engine.cu on the host, so that no out-of-range access is ever tried on a GPU first."""
import itertools

import pytest

fmoe = pytest.importorskip("bit_dequant_expert_gemv_b200")

MAX_SMEM = 232448
MISC_BYTES = 4096

SHAPES = [
    # H, I, E, K, bits
    (4096, 1024, 512, 4, 4), (4096, 1024, 512, 4, 2), (256, 128, 16, 2, 4), (256, 128, 16, 2, 2),
    (64, 64, 1, 1, 4), (64, 64, 3, 3, 2), (192, 320, 7, 3, 4), (8192, 1024, 64, 8, 4),
    (7168, 2048, 256, 4, 4), (4160, 576, 33, 5, 2), (1024, 8192, 8, 1, 4), (2048, 704, 128, 6, 4),
    (128, 64, 4096, 8, 2), (8128, 192, 16, 2, 4), (128, 64, 1100, 8, 4), (1024, 576, 33, 5, 2),
    (256, 128, 600, 4, 4), (8192, 8192, 2, 1, 2), (4608, 1024, 512, 4, 4),
]
FLAGS = [15, 7, 5, 1, 2]  # full layer+gate, no gate, no shared, router only, expert only
GRIDS = [148, 132, 7, 1]
CK_ROUTER, CK_GU, CK_DN = range(3)


def share(n, unit, c, nc):
    nu = n // unit
    return (nu * c // nc) * unit, (nu * (c + 1) // nc) * unit


def make_share(G, c, nc):
    S = {}
    S["r0"], S["r1"] = share(G["nr"], 1, c, nc)
    S["h0"], S["h1"] = share(G["I"], G["au"], c, nc)
    S["d0"], S["d1"] = share(G["H"], G["ad"], c, nc)
    nrr = S["r1"] - S["r0"]
    if not G["route_on"]:
        S["nrc"] = 0
    elif G["rseg"] > 1:
        S["nrc"] = nrr * G["rseg"]
    else:
        S["nrc"] = -(-nrr // G["rrows"])
    gu = G["shared_on"] or G["routed_on"]
    S["ngc"] = -(-(S["h1"] - S["h0"]) // G["hr"]) if gu else 0
    S["ndc"] = -(-(S["d1"] - S["d0"]) // G["dr"]) if G["nseg"] > 0 else 0
    S["na"] = S["nrc"] + (S["ngc"] + S["ndc"] if G["shared_on"] else 0)
    S["nb"] = G["K"] * (S["ngc"] + S["ndc"]) if G["routed_on"] else 0
    return S


def chunk_a(G, S, i):
    if i < S["nrc"]:
        if G["rseg"] > 1:
            rr, seg = divmod(i, G["rseg"])
            return CK_ROUTER, -1, S["r0"] + rr, 1, seg
        r0 = S["r0"] + i * G["rrows"]
        return CK_ROUTER, -1, r0, min(G["rrows"], S["r1"] - r0), 0
    i -= S["nrc"]
    if i < S["ngc"]:
        r0 = S["h0"] + i * G["hr"]
        return CK_GU, -1, r0, min(G["hr"], S["h1"] - r0), 0
    i -= S["ngc"]
    r0 = S["d0"] + i * G["dr"]
    return CK_DN, -1, r0, min(G["dr"], S["d1"] - r0), 0


def chunk_b(G, S, i):
    gu = G["K"] * S["ngc"]
    if i < gu:
        e, j = divmod(i, S["ngc"])
        r0 = S["h0"] + j * G["hr"]
        return CK_GU, e, r0, min(G["hr"], S["h1"] - r0), 0
    i -= gu
    e, j = divmod(i, S["ndc"])
    r0 = S["d0"] + j * G["dr"]
    return CK_DN, e, r0, min(G["dr"], S["d1"] - r0), 0


def copies(G, kind, r0, n, seg):
    """(buffer, src_off, dst_off, bytes) of each bulk copy, as copy_desc issues them."""
    H, I, E = G["H"], G["I"], G["E"]
    out = []
    if kind == CK_ROUTER:
        rowb = 4 * H
        if G["rseg"] > 1:
            buf, base = ("router", r0 * rowb) if r0 < E else ("gate", 0)
            out.append((buf, base + seg * G["rcols"] * 4, 0, 4 * G["rcols"]))
        else:
            a, b = r0, min(r0 + n, E)
            if b > a:
                out.append(("router", a * rowb, 0, (b - a) * rowb))
            if r0 + n > E:
                out.append(("gate", 0, (E - r0) * rowb, rowb))
    elif kind == CK_GU:
        hr, rc, rs, q = G["hr"], G["rc_h"], G["rs_h"], G["q_gu"]
        out += [("expert", r0 * rc, 0, n * rc), ("expert", q + r0 * rc, hr * rc, n * rc),
                ("expert", I * rc + r0 * rs, 2 * hr * rc, n * rs),
                ("expert", q + I * rc + r0 * rs, 2 * hr * rc + hr * rs, n * rs)]
    else:
        dn, rc, rs = 2 * G["q_gu"], G["rc_i"], G["rs_i"]
        out += [("expert", dn + r0 * rc, 0, n * rc),
                ("expert", dn + H * rc + r0 * rs, G["dr"] * rc, n * rs)]
    return out


def chunk_bytes(G, kind, n):
    if kind == CK_ROUTER:
        return 4 * G["rcols"] if G["rseg"] > 1 else 4 * G["H"] * n
    if kind == CK_GU:
        return 2 * n * (G["rc_h"] + G["rs_h"])
    return n * (G["rc_i"] + G["rs_i"])


def inside(cov, a, nb):
    return any(lo <= a and a + nb <= hi for lo, hi in cov)


def check_reads(G, kind, r0, n, seg, cov, d0):
    """The consumer reads of one chunk; gate/up chunks are checked as chunk 0 or chunk 1 of a
    pass (both positions), with the pass partner holding the same rows."""
    WARPS = G["consumer_warps"]
    THREADS = 32 * WARPS
    sb = G["stage_bytes"]
    cb = 16 if G["bits"] == 4 else 8
    if kind == CK_ROUTER:
        cols = G["rcols"]
        nf = cols // 4
        assert nf <= 4 * THREADS  # the x columns a thread holds (4 float4)
        for r in range(n):
            for f in range(nf):
                assert inside(cov, (r * nf + f) * 16, 16), (r, f)
            assert (seg * cols + 4 * (nf - 1) + 4) <= G["H"]
        assert (n * WARPS) * 8 <= G["red_slot"]
        if G["rseg"] == 1 and G["rrows"] <= 4:  # batches of up to 4 rows across chunks
            assert (4 * WARPS) * 8 <= G["red_slot"]
        return
    if kind == CK_GU:
        NR = G["max_rows_thread"]
        hr, gh, wh, sh = G["hr"], G["gh"], G["wh"], G["sh"]
        wn = wh // 32 if wh > 32 else 1
        sb0 = 2 * hr * G["rc_h"]
        for np_, pos in [(1, 0)] + ([(2, 0), (2, 1)] if G["gpass"] == 2 else []):
            seen = set()
            for t in range(THREADS):
                g, s = divmod(t, wh)
                act = g < gh and s < sh
                om = s >> 5 if wh > 32 else 0
                for i in range(NR):
                    q = g + gh * i
                    c = 1 if q >= 2 * hr else 0
                    rho = q - 2 * hr * c
                    rr = rho if rho < hr else rho - hr
                    if act and c < np_ and rr < n:
                        if c == pos:  # a slot of this chunk reads its stage
                            assert inside(cov, rho * G["rc_h"] + s * cb, cb), (t, rho, s)
                            assert inside(cov, sb0 + rho * G["rs_h"] + (s >> 1) * 4, 4), (t, rho, s)
                            seen.add(rho)
                    if act and q < 2 * hr * np_:
                        assert (q * wn + om) * 4 + 4 <= G["red_slot"]
            # every valid row of the chunk is some thread's row
            assert all(r in seen for r in range(n)) and all(hr + r in seen for r in range(n))
        return
    NR = G["max_rows_warp"]
    wi, pi, ji, si = G["wi"], G["pi"], G["ji"], G["si"]
    sbb = G["dr"] * G["rc_i"]
    seen = set()
    for w in range(WARPS):
        for lane in range(32):
            ls, lp = lane % wi, lane // wi
            for j in range(ji):
                s = ls + wi * j
                assert 32 * min(s, si - 1) + 32 <= G["I"]  # the slice's digit form
                for i in range(NR):
                    rho = w * pi + lp + WARPS * pi * i
                    if s < si and rho < n:
                        assert inside(cov, rho * G["rc_i"] + s * cb, cb), (w, lane, rho, s)
                        assert inside(cov, sbb + rho * G["rs_i"] + (s >> 1) * 4, 4)
                        seen.add(rho)
                        assert r0 - d0 + rho < G["oacc_n"]
    assert seen == set(range(n))


@pytest.mark.parametrize("shape,flags", list(itertools.product(SHAPES, FLAGS)))
def test_geometry_in_bounds(shape, flags):
    H, I, E, K, bits = shape
    for nc in GRIDS:
        try:
            G = fmoe.describe_geometry(H, I, E, K, bits, flags, MAX_SMEM, nc)
        except fmoe.FmoeError as e:
            assert e.code == fmoe.FMOE_ERR_UNSUPPORTED
            continue
        check_geometry(G, nc)


def check_geometry(G, nc):
    H, I, E, K = G["H"], G["I"], G["E"], G["K"]
    sb = G["stage_bytes"]
    nA, nB = G["nA"], G["nB"]
    assert G["smem_bytes"] <= MAX_SMEM and sb % 128 == 0
    assert 1 <= nA <= 16 and 1 <= nB <= 16
    nseg = G["nseg"]
    areas = [("ringA", G["o_ringA"], nA * sb), ("ringB", G["o_ringB"], nB * sb),
             ("x", G["o_x"], 4 * H), ("h", G["o_h"], max(4 * nseg * I, 4 * H, 128)),
             ("red", G["o_red"], G["red_slot"] * (nA + nB)), ("oacc", G["o_oacc"], 4 * max(G["oacc_n"], 1)),
             ("misc", G["o_misc"], MISC_BYTES), ("bar", G["o_bar"], 16 * (nA + nB))]
    for (n1, a1, l1), (n2, a2, l2) in zip(areas, areas[1:]):
        assert a1 + l1 <= a2, (n1, n2)
    assert areas[-1][1] + areas[-1][2] <= G["smem_bytes"]
    for name, off, _ in areas[:-1]:
        assert off % 128 == 0, name
    assert G["o_bar"] % 8 == 0
    # the controller's bulk copies: x (4H bytes), each h segment (4I bytes at 4I k)
    assert (4 * H) % 16 == 0 and (4 * I) % 16 == 0
    # consumer layouts
    THREADS = 32 * G["consumer_warps"]
    assert G["sh"] == H // 32 and G["gh"] * G["wh"] <= THREADS and G["gh"] >= 1
    assert G["wh"] >= G["sh"] and (G["wh"] <= 32 or G["wh"] % 32 == 0)
    if G["wh"] <= 32:
        assert G["wh"] & (G["wh"] - 1) == 0
    assert G["wi"] * G["pi"] == 32 and G["wi"] * G["ji"] >= G["si"]
    nrg = -(-2 * G["gpass"] * G["hr"] // G["gh"])
    nrd = -(-G["dr"] // (G["consumer_warps"] * G["pi"]))
    assert nrg <= G["max_rows_thread"] and nrd <= G["max_rows_warp"]
    # transform work items stay inside their vectors
    for bits_ts, nsl, length in [(4 if G["bits"] == 4 else 2, H // 32, H),
                                 (4 if G["bits"] == 4 else 2, I // 32, I)]:
        nv = 32 // bits_ts
        assert nsl * 32 <= length and nv * bits_ts == 32
    sizes = {"router": E * H * 4, "gate": H * 4,
             "expert": fmoe.expert_bytes(H, I, G["bits"])}
    assert G["q_gu"] * 2 + H * (G["rc_i"] + G["rs_i"]) == sizes["expert"]
    own = {"r": [], "h": [], "d": []}
    checked = set()  # the consumer reads depend only on (kind, valid rows, segment, row offset)
    for c in range(nc):
        S = make_share(G, c, nc)
        own["r"].append((S["r0"], S["r1"]))
        own["h"].append((S["h0"], S["h1"]))
        own["d"].append((S["d0"], S["d1"]))
        assert S["d1"] - S["d0"] <= max(G["oacc_n"], 0) or G["nseg"] == 0
        lists = [chunk_a(G, S, i) for i in range(S["na"])] + [chunk_b(G, S, i) for i in range(S["nb"])]
        covered_rows = {CK_ROUTER: [], CK_GU: {}, CK_DN: {}}
        for kind, e, r0, n, seg in lists:
            assert n > 0
            cps = copies(G, kind, r0, n, seg)
            cov = []
            for buf, so, do, nb in cps:
                assert nb > 0 and nb % 16 == 0 and so % 16 == 0 and do % 16 == 0, (kind, so, do, nb)
                assert so + nb <= sizes[buf], (kind, buf, so, nb)
                assert do + nb <= sb, (kind, do, nb, sb)
                cov.append((do, do + nb))
            cov.sort()
            for (a, b), (c2, d) in zip(cov, cov[1:]):
                assert b <= c2, "copies overlap in the stage"
            assert sum(b - a for a, b in cov) == chunk_bytes(G, kind, n)
            key = (kind, n, seg, r0 - S["d0"] if kind == CK_DN else 0)
            if key not in checked:
                checked.add(key)
                check_reads(G, kind, r0, n, seg, cov, S["d0"])
            if kind == CK_ROUTER:
                covered_rows[CK_ROUTER] += [(r, seg) for r in range(r0, r0 + n)]
            else:
                covered_rows[kind].setdefault(e, []).extend(range(r0, r0 + n))
        if G["route_on"]:
            assert sorted(covered_rows[CK_ROUTER]) == sorted(
                (r, s) for r in range(S["r0"], S["r1"]) for s in range(G["rseg"]))
        for kind, lo, hi in [(CK_GU, S["h0"], S["h1"]), (CK_DN, S["d0"], S["d1"])]:
            for e, rows in covered_rows[kind].items():
                assert sorted(rows) == list(range(lo, hi)), (kind, e)
    # ownership: each phase's rows are split into disjoint contiguous shares covering all rows
    for key, total in (("r", G["nr"]), ("h", I), ("d", H)):
        spans = own[key]
        assert spans[0][0] == 0 and spans[-1][1] == total
        for (a, b), (c2, d) in zip(spans, spans[1:]):
            assert b == c2 and a <= b


def test_main_shape_layout():
    G = fmoe.describe_geometry(4096, 1024, 512, 4, 4, 15, MAX_SMEM, 148)
    # a CTA's whole gate/up share of one expert (7 of 1024 h-rows, 8 with the largest share)
    # fits one 36 KB stage; two stages in ring B, three in ring A
    assert G["hr"] == 8 and G["nA"] >= 3 and G["nB"] >= 2 and G["oacc_n"] == 28
    assert G["smem_bytes"] <= MAX_SMEM
