"""The single-token GEMV kernels cut the units (8 h-rows per unit in phase 1, 16 down rows
in phase 2, of every active expert, in plan order) into one contiguous range per CTA:
CTA b takes units [b*N/G, (b+1)*N/G).  A CTA keeps at most two experts' activations and
16 units' partial sums in shared memory, so the host sends a shape to these kernels only
when every range fits.  This checks, on the CPU, that the host's conditions imply the
kernel's limits for every shape the host accepts, and that the ranges cover every unit
exactly once."""
import itertools

import pytest

MAX_UNITS = 16   # units per CTA range (kGvMaxUnits)
MAX_SLOTS = 2    # experts per CTA range (kGvMaxSlots)
MAX_CTAS = 148


def host_accepts(T, k, d, f, ctas):
    """The shape conditions of use_gemv() in abi.cu (alignment and shared memory aside)."""
    if T != 1 or d % 512 or f % 512:
        return False
    experts = T * k + 1
    if experts > ctas:
        return False
    cap = MAX_UNITS * ctas
    return experts * (f // 8) <= cap and experts * (d // 16) <= cap


def ranges(n_act, upe, G):
    N = n_act * upe
    return [(b * N // G, (b + 1) * N // G) for b in range(G)]


@pytest.mark.parametrize("ctas", [148, 132, 100])
def test_accepted_shapes_fit_every_range(ctas):
    checked = 0
    for k, d, f in itertools.product(range(1, 40), (512, 1024, 2048, 4096, 7168, 8192),
                                     (512, 1024, 1536, 2048, 4096)):
        if not host_accepts(1, k, d, f, ctas):
            continue
        for n_act in range(1, k + 2):          # distinct experts hit, plus the shared one
            for upe in (f // 8, d // 16):        # phase 1, phase 2
                covered = []
                for lo, hi in ranges(n_act, upe, ctas):
                    assert hi - lo <= MAX_UNITS
                    if hi > lo:
                        assert (hi - 1) // upe - lo // upe + 1 <= MAX_SLOTS
                    covered.extend(range(lo, hi))
                assert covered == list(range(n_act * upe))
                checked += 1
    assert checked > 1000


def test_decode_workload_is_accepted():
    # 256 routed experts + 1 shared, top-6, d = 4096, f = 2048 on 148 SMs: 12-13 units each
    assert host_accepts(1, 6, 4096, 2048, MAX_CTAS)
    r = ranges(7, 2048 // 8, MAX_CTAS)
    assert {hi - lo for lo, hi in r} == {12, 13}
