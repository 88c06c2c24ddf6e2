"""The FFN kernels' work split, checked on CPU with the same integer formulas the kernel
uses (whole tiles in rounds of G, then an even stream-K split of the remaining tiles'
chunks): every chunk of every tile is processed exactly once, the CTAs' shares differ by
at most one chunk, the partial-slot ids of split tiles are unique, and the finisher's
walk over a split tile meets its segments' owners in chunk order."""
import pytest


def begin(W, G, b):
    return b * W // G


def owner(W, G, c):
    return ((c + 1) * G - 1) // W


def schedule(T, nk, G):
    Q = T // G
    base = Q * G
    W = (T - base) * nk
    segs = {}
    for b in range(G):
        out = [(b + j * G, 0, nk) for j in range(Q)]
        c, tend = begin(W, G, b), begin(W, G, b + 1)
        while c < tend:
            k0 = c % nk
            k1 = min(nk, k0 + (tend - c))
            out.append((base + c // nk, k0, k1))
            c += k1 - k0
        segs[b] = out
    return base, W, segs


CASES = [(T, nk, G) for T in list(range(1, 24)) + [56, 112, 147, 148, 149, 295, 4688]
         for nk in (1, 16, 32) for G in (1, 3, 7, 148)]


@pytest.mark.parametrize("T,nk,G", CASES)
def test_split(T, nk, G):
    base, W, segs = schedule(T, nk, G)
    cover, slots = {}, {}
    for b, lst in segs.items():
        tbeg = begin(W, G, b)
        for tile, k0, k1 in lst:
            for kc in range(k0, k1):
                assert (tile, kc) not in cover
                cover[(tile, kc)] = b
            tt = tile - base
            if tt < 0:
                continue
            nseg, cc = 0, tt * nk
            while cc < tt * nk + nk:
                nseg += 1
                cc = begin(W, G, owner(W, G, cc) + 1)
            if nseg > 1:
                slot = 2 * b + (0 if tbeg // nk == tt else 1)
                assert slots.setdefault(slot, (b, tt)) == (b, tt)
    assert len(cover) == T * nk
    work = [sum(k1 - k0 for _, k0, k1 in segs[b]) for b in range(G)]
    assert max(work) - min(work) <= 1
    for tt in range(T - base):
        cc, walk = tt * nk, []
        while cc < tt * nk + nk:
            s = owner(W, G, cc)
            walk.append(s)
            cc = begin(W, G, s + 1)
        real = []
        for kc in range(nk):
            o = cover[(base + tt, kc)]
            if not real or real[-1] != o:
                real.append(o)
        assert walk == real
        if len(walk) > 1:
            for s in walk:
                slot = 2 * s + (0 if begin(W, G, s) // nk == tt else 1)
                assert slots[slot] == (s, tt)
