"""The single-token layer kernel (decode.cu) splits each phase's units over its CTAs: CTA b
takes [b*M/G, (b+1)*M/G) of all M = (active routed experts + 1) * U units (U the units per
expert: f/8 in phase 1, d/16 in phase 2), of which the first are its share of the shared
expert's units [b*U/G, (b+1)*U/G) (streamed before routing is known) and the rest a
contiguous range of the routed experts' units.  A CTA keeps at most 16 units' partial sums
and, in phase 2, the hidden state of the shared expert and of at most two routed experts
in shared memory.  This checks on the CPU, before any launch, that the host's condition
(decode_fits in decode.cu) implies those limits for every shape it accepts and every
number of active experts, that the ranges cover every unit exactly once, that every TMA
box the kernel addresses lies inside its tensor, and that the shared-memory layout fits
the 227 KB a B200 CTA may use at the decode workload's sizes."""
import itertools

import pytest

MAX_UNITS = 16    # kDcMaxUnits
P2_SLOTS = 3      # kDcP2Slots: shared + two routed
WARPS = 16
STAGE_BYTES = 16 * 256 + 16 * 16
STAGES = 3
SMEM_LIMIT = 232448   # bytes of shared memory a CTA may opt into on sm_100


def split(upe, n_routed, G, b, wsh=1):
    """Mirror of the kernel's Range: (s_lo, ns, r_lo, nr); a shared unit weighs wsh."""
    s_lo = b * upe // G
    ns = (b + 1) * upe // G - s_lo
    M = (n_routed + wsh) * upe
    t_lo, t_hi = b * M // G, (b + 1) * M // G
    return s_lo, ns, t_lo - wsh * s_lo, (t_hi - t_lo) - wsh * ns


def decode_fits(k, d, f, ctas, q2=False):
    """Mirror of decode_fits() in decode.cu: every CTA's ranges, for every count of active
    experts, within the per-CTA limits."""
    if k < 1 or k > 32 or d % 512 or f % 512 or ctas < 1:
        return False
    if q2 and (d % 2048 or f % 2048):
        return False
    wsh = 2 if q2 else 1
    upe1, upe2 = f // 8, d // 16
    for n in range(1, k + 1):
        for b in range(ctas):
            for upe in (upe1, upe2):
                _, ns, _, nr = split(upe, n, ctas, b, wsh)
                if nr < 0 or ns + nr > MAX_UNITS:
                    return False
            if split(upe2, n, ctas, b, wsh)[3] > upe2 + 1:
                return False
    return True


def smem_bytes(d, f, q2=False):
    """Mirror of DcSmem::bytes()."""
    area = WARPS * STAGES * STAGE_BYTES
    p1_end = area + (3 if q2 else 2) * d + d // 32 + MAX_UNITS * (d // 512) * 64
    p2_end = area + (4 if q2 else 2 * P2_SLOTS) * f + P2_SLOTS * (f // 32) + \
        MAX_UNITS * (f // 512) * 64
    bars = (max(p1_end, p2_end) + 7) // 8 * 8
    info = bars + (WARPS * STAGES + 1) * 8
    return info + 4 * (4 + 3 * 33 + 64) + 1024


@pytest.mark.parametrize("ctas", [148, 132, 100])
def test_accepted_shapes_fit_every_range(ctas):
    checked = 0
    for k, d, f in itertools.product(range(1, 33), (512, 1024, 2048, 4096, 7168, 8192),
                                     (512, 1024, 1536, 2048, 4096)):
        if not decode_fits(k, d, f, ctas):
            continue
        for n_act in range(1, k + 1):   # a caller's dispatch may repeat experts
            for upe in (f // 8, d // 16):
                shared, routed = [], []
                for b in range(ctas):
                    s_lo, ns, r_lo, nr = split(upe, n_act, ctas, b)
                    assert nr >= 0 and ns + nr <= MAX_UNITS
                    shared.extend(range(s_lo, s_lo + ns))
                    routed.extend(range(r_lo, r_lo + nr))
                    if upe == d // 16 and nr:
                        slots = (r_lo + nr - 1) // upe - r_lo // upe + 1
                        assert slots <= P2_SLOTS - 1
                assert shared == list(range(upe))
                assert routed == list(range(n_act * upe))
                checked += 1
    assert checked > 500


def test_decode_workload_is_accepted_and_fits_shared_memory():
    assert decode_fits(6, 4096, 2048, 148)
    assert smem_bytes(4096, 2048) <= SMEM_LIMIT
    # every CTA holds one or two shared units to stream before routing is known
    for b in range(148):
        s_lo, ns, r_lo, nr = split(2048 // 8, 6, 148, b)
        assert 1 <= ns <= 2 and ns + nr in (12, 13)


def test_tma_boxes_stay_inside_their_tensors():
    """Phase 1 boxes: rows e*f + u*8 .. +8 of [(E+1)*f] rows, code pieces 2c, 2c+1 of d/256,
    scale bytes 16c .. 16c+16 of d/32; phase 2 likewise with 16 rows, d and f swapped."""
    for E, k, d, f in ((256, 6, 4096, 2048), (8, 2, 512, 512), (1024, 8, 1024, 512),
                       (64, 32, 512, 512)):
        assert decode_fits(k, d, f, 148)
        for rows_box, upe, K, rows_per in ((8, f // 8, d, f), (16, d // 16, f, d)):
            for e in (0, E):
                last_row = e * rows_per + (upe - 1) * rows_box + rows_box
                assert last_row <= (E + 1) * rows_per
            for c in range(K // 512):
                assert 2 * c + 1 < K // 256
                assert 16 * c + 16 <= K // 32


def test_every_warp_takes_its_tasks_once():
    """Tasks go round-robin (task = warp + 16 q); the first ones of each warp (as many as its
    ring holds) are issued before routing only when they belong to the shared expert."""
    S1 = 4096 // 512
    for b in (0, 73, 147):
        s_lo, ns, r_lo, nr = split(2048 // 8, 6, 148, b)
        n_tasks = (ns + nr) * S1
        seen = []
        for w in range(WARPS):
            q1 = -(-(n_tasks - w) // WARPS) if n_tasks > w else 0
            seen.extend(w + WARPS * q for q in range(q1))
            shared_q = -(-(ns * S1 - w) // WARPS) if ns * S1 > w else 0
            for q in range(min(shared_q, STAGES)):
                assert (w + WARPS * q) // S1 < ns
        assert sorted(seen) == list(range(n_tasks))


@pytest.mark.parametrize("ctas", [148, 132])
def test_q2_form_ranges_cover_every_unit_once(ctas):
    """The Q2 form (2-bit routed experts, a shared unit weighing 2): for every accepted
    shape and count of active experts, the ranges cover the shared and the routed units
    once each, with at most 16 units per CTA and a phase-2 routed range over at most two
    experts; the decode workload is accepted and fits shared memory."""
    checked = 0
    for k, d, f in itertools.product(range(1, 12), (2048, 4096, 8192), (2048, 4096)):
        if not decode_fits(k, d, f, ctas, q2=True):
            continue
        for n_act in range(1, k + 1):
            for upe in (f // 8, d // 16):
                shared, routed = [], []
                for b in range(ctas):
                    s_lo, ns, r_lo, nr = split(upe, n_act, ctas, b, 2)
                    assert nr >= 0 and ns + nr <= MAX_UNITS
                    shared.extend(range(s_lo, s_lo + ns))
                    routed.extend(range(r_lo, r_lo + nr))
                assert shared == list(range(upe))
                assert routed == list(range(n_act * upe))
                checked += 1
    assert checked > 50
    assert decode_fits(6, 4096, 2048, 148, q2=True)
    assert smem_bytes(4096, 2048, q2=True) <= SMEM_LIMIT
    assert not decode_fits(6, 1024, 2048, 148, q2=True)
