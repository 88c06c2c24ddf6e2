"""The work plan of the tensor-core single-token kernel (decode_tc.cu), checked on the CPU
before any launch.  Each phase's units (128-row block x 256-wide K chunk of one expert)
are split over the CTAs as in decode.cu (shared expert first); a CTA's units of one
(expert, row block) form a segment (a "piece" of that row block), accumulated in one of
seven TMEM buffers by both MMA issuers.  This mirrors the kernel's index arithmetic
(TcPlan, tc_unit, tc_segments, tc_segment_of, tc_stage) and checks: every unit of every
expert is covered exactly once; the pieces of a row block, walked from K chunk 0 by their
lengths, cover its K chunks (the finisher's and the combine's walk); every row block has
exactly one finisher, the CTA holding its first K chunk, and a finisher only waits on
pieces that other CTAs hold as their first segment of the part (so the waits cannot form
a cycle); a CTA meets at most three experts in phase 2; the stages of a segment are
contiguous and its K chunks fit the two 8-column groups of a 16-column region; the
combine's output rows lie in at most two row blocks; and the shared-memory layout fits at
the decode sizes."""
import pytest

KS = 256          # K elements per stage
ISSUERS = 2
BUFS = 7          # segment accumulator buffers
STAGES = 5
STAGE_BYTES = 2 * 128 * 128 + 1024
P2_LOCAL = 3
SMEM_LIMIT = 232448


def split(upe, n_routed, G, b):
    s_lo = b * upe // G
    ns = (b + 1) * upe // G - s_lo
    M = (n_routed + 1) * upe
    t_lo, t_hi = b * M // G, (b + 1) * M // G
    return dict(s_lo=s_lo, ns=ns, r_lo=t_lo - s_lo, nr=(t_hi - t_lo) - ns, upe=upe)


def units(r):
    return r["ns"] + r["nr"]


def tc_unit(r, NK, ul):
    if ul < r["ns"]:
        slot, u, lo, hi = -1, r["s_lo"] + ul, 0, r["ns"] - 1
    else:
        ru = r["r_lo"] + ul - r["ns"]
        slot, u, lo, hi = ru // r["upe"], ru % r["upe"], r["ns"], units(r) - 1
    rb, kc = u // NK, u % NK
    return dict(slot=slot, rb=rb, kc=kc, ua=max(ul - kc, lo), ub=min(ul + NK - 1 - kc, hi))


def tc_segments(r, NK):
    a = (r["s_lo"] + r["ns"] - 1) // NK - r["s_lo"] // NK + 1 if r["ns"] > 0 else 0
    b = (r["r_lo"] + r["nr"] - 1) // NK - r["r_lo"] // NK + 1 if r["nr"] > 0 else 0
    return a + b


def tc_segment_of(r, NK, ul):
    if ul < r["ns"]:
        return (r["s_lo"] + ul) // NK - r["s_lo"] // NK
    a = (r["s_lo"] + r["ns"] - 1) // NK - r["s_lo"] // NK + 1 if r["ns"] > 0 else 0
    return a + (r["r_lo"] + ul - r["ns"]) // NK - r["r_lo"] // NK


class Plan:
    def __init__(self, k, d, f, G, b):
        self.r1 = split((f // 128) * (d // KS), k, G, b)
        self.r2 = split((d // 128) * (f // KS), k, G, b)
        self.NK1, self.NK2 = d // KS, f // KS
        self.n1, self.n2 = 2 * units(self.r1), units(self.r2)

    def stage(self, q):
        if q < self.n1:
            u = tc_unit(self.r1, self.NK1, q >> 1)
            return dict(u=u, ph=1, mat=q & 1, seg=tc_segment_of(self.r1, self.NK1, q >> 1),
                        qa=2 * u["ua"], qb=2 * u["ub"] + 1)
        u = tc_unit(self.r2, self.NK2, q - self.n1)
        return dict(u=u, ph=2, mat=0,
                    seg=tc_segments(self.r1, self.NK1) + tc_segment_of(self.r2, self.NK2, q - self.n1),
                    qa=self.n1 + u["ua"], qb=self.n1 + u["ub"])


def smem_bytes(d, f):
    b_tiles = max(d // 128, P2_LOCAL * (f // 128))
    bars = 3 * STAGES + 2 * BUFS + 2 + ISSUERS + 1
    base = STAGES * STAGE_BYTES + b_tiles * 1024 + 512 + 8 * bars
    info = 4 * (8 + 33 + 64 + 16)
    return base + info + 4 * (d // 128) + 4 * P2_LOCAL * (f // 128) + 16 + 1024


def tc_fits(k, d, f, G):
    if k < 1 or k > 32 or G < 1 or d % KS or f % KS or d > 4096 or f > 4096:
        return False
    if smem_bytes(d, f) > SMEM_LIMIT:
        return False
    for b in range(G):
        p = Plan(k, d, f, G, b)
        if p.r1["nr"] < 0 or p.r2["nr"] < 0 or p.r2["nr"] > p.r2["upe"] + 1:
            return False
        m0, m1 = b * d // G, (b + 1) * d // G
        nrb = (m1 - 1) // 128 - m0 // 128 + 1 if m1 > m0 else 0
        b_tiles = max(d // 128, P2_LOCAL * (f // 128))
        if nrb > 2 or (k + 1) * (nrb * 17 + (m1 - m0)) * 4 > b_tiles * 1024:
            return False
    return True


SHAPES = [(6, 4096, 2048, 148), (2, 512, 512, 148), (1, 1024, 512, 148), (8, 1024, 1536, 148),
          (4, 4096, 1024, 148), (32, 512, 512, 148), (6, 2048, 1024, 148), (6, 4096, 2048, 16),
          (3, 1024, 1024, 12), (6, 4096, 2048, 132)]


@pytest.mark.parametrize("k,d,f,G", SHAPES)
def test_units_pieces_and_local_experts(k, d, f, G):
    assert tc_fits(k, d, f, G)
    RB1, RB2 = f // 128, d // 128
    NK1, NK2 = d // KS, f // KS
    cover1, cover2 = {}, {}
    pieces1, pieces2 = {}, {}
    for b in range(G):
        p = Plan(k, d, f, G, b)
        for ph, r, NK, cover, pieces in ((1, p.r1, NK1, cover1, pieces1), (2, p.r2, NK2, cover2, pieces2)):
            ul = 0
            seen_slots = set()
            while ul < units(r):
                u = tc_unit(r, NK, ul)
                assert u["ua"] == ul
                sidx = k if u["slot"] < 0 else u["slot"]
                assert 0 <= sidx <= k
                for v in range(u["ua"], u["ub"] + 1):
                    w = tc_unit(r, NK, v)
                    assert (w["slot"], w["rb"]) == (u["slot"], u["rb"])
                    key = (sidx, w["rb"], w["kc"])
                    assert key not in cover, key
                    cover[key] = b
                pieces.setdefault((sidx, u["rb"]), []).append((u["kc"], u["ub"] - u["ua"] + 1))
                seen_slots.add(sidx)
                ul = u["ub"] + 1
            if ph == 2:
                assert len(seen_slots) <= P2_LOCAL
                routed = [s for s in seen_slots if s < k]
                if routed:  # the kernel's local index ls = 1 + slot - first routed slot
                    assert max(routed) - p.r2["r_lo"] // p.r2["upe"] <= 1
    assert len(cover1) == (k + 1) * RB1 * NK1
    assert len(cover2) == (k + 1) * RB2 * NK2
    for pieces, NK in ((pieces1, NK1), (pieces2, NK2)):
        for key, ps in pieces.items():
            # the finisher's walk: from K chunk 0, each piece's length leads to the next
            start = {kc: n for kc, n in ps}
            kc, total = 0, 0
            while kc < NK:
                assert kc in start, (key, ps)
                total += start[kc]
                kc += start[kc]
            assert kc == NK and total == NK == sum(n for _, n in ps)


@pytest.mark.parametrize("k,d,f,G", SHAPES)
def test_segments_finishers_and_waits(k, d, f, G):
    finisher = {}   # (sidx, rb) of phase 1 -> CTA
    owner = {}      # (phase, sidx, rb, first K chunk) -> (CTA, index of the segment in its part)
    for b in range(G):
        p = Plan(k, d, f, G, b)
        nq = p.n1 + p.n2
        # the stages of each segment are contiguous and in segment order
        prev_seg, first = -1, {}
        for q in range(nq):
            s = p.stage(q)
            assert s["seg"] in (prev_seg, prev_seg + 1)
            if s["seg"] != prev_seg:
                assert q == s["qa"]
                first[s["seg"]] = q
                prev_seg = s["seg"]
            assert s["qa"] <= q <= s["qb"]
            assert s["u"]["kc"] < 16  # one 16-column region per matrix holds the K chunks
        for ph, r, NK in ((1, p.r1, p.NK1), (2, p.r2, p.NK2)):
            ul, idx_in_part = 0, 0
            while ul < units(r):
                u = tc_unit(r, NK, ul)
                if ul == r["ns"]:
                    idx_in_part = 0  # the routed part starts
                sidx = k if u["slot"] < 0 else u["slot"]
                owner[(ph, sidx, u["rb"], u["kc"])] = (b, idx_in_part)
                if ph == 1 and u["kc"] == 0:
                    assert (sidx, u["rb"]) not in finisher
                    finisher[(sidx, u["rb"])] = b
                idx_in_part += 1
                ul = u["ub"] + 1
    RB1 = f // 128
    assert sorted(finisher) == [(s, rb) for s in range(k + 1) for rb in range(RB1)]
    for (ph, sidx, rb, kc), (b, i) in owner.items():
        if ph != 1 or kc == 0:
            continue
        fb = finisher[(sidx, rb)]
        # the finisher waits on this piece: it lies in a later CTA, as that CTA's first
        # segment of the part
        assert b > fb and i == 0, (sidx, rb, kc, b, fb, i)


@pytest.mark.parametrize("k,d,f,G", SHAPES)
def test_combine_rows(k, d, f, G):
    rows = []
    for b in range(G):
        m0, m1 = b * d // G, (b + 1) * d // G
        rows += list(range(m0, m1))
        assert m1 <= m0 or (m1 - 1) // 128 - m0 // 128 <= 1
    assert rows == list(range(d))


def test_smem_fits_at_decode_sizes():
    assert smem_bytes(4096, 2048) <= SMEM_LIMIT
    assert smem_bytes(4096, 2560) > SMEM_LIMIT   # the CUDA-core form takes this shape
    assert not tc_fits(6, 8192, 2048, 148)        # K above 4096: four column groups at most
