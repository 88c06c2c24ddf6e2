"""CPU checks of the facts the single-token GEMV kernels rely on (gemv.cu).

- Every e2m1 value and every finite e4m3 value is exact in f16, and the product of one
  of each is exact in fp32, so the f16 MMA with fp32 accumulation adds exact products.
- The ue8m0 -> fp32 bit construction gives 2^(e-127) for every byte e < 255 (2^-127 as
  a subnormal).
- The stage layout: the byte offsets of (row, block, lane) cover each code byte of a
  stage once, and the eight rows that one 4-byte shared-memory read touches fall on
  distinct banks (the 128-byte swizzle of the TMA boxes).
- The K order: lane t of a quad feeds elements 8t..8t+7 of a block to both operands of
  the two m16n8k16 MMAs, so each block's 32 products are summed once each.
"""
import numpy as np

import oracle

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def e2m1_values():
    return [s * m for s in (1.0, -1.0) for m in E2M1]


def e4m3_finite_values():
    return [oracle.e4m3_value(c) for c in range(256) if c not in (0x7F, 0xFF)]


def test_operands_exact_in_f16_and_products_exact_in_fp32():
    a = np.array(e2m1_values())
    b = np.array(e4m3_finite_values())
    assert np.array_equal(a.astype(np.float16).astype(np.float64), a)
    assert np.array_equal(b.astype(np.float16).astype(np.float64), b)
    prod64 = np.outer(a, b)
    prod32 = np.outer(a.astype(np.float32), b.astype(np.float32))
    assert np.array_equal(prod32.astype(np.float64), prod64)


def ue8m0_f32(e):
    bits = max((e << 23) & 0x7F800000, 0x00400000)
    return np.array([bits], dtype=np.uint32).view(np.float32)[0]


def test_ue8m0_bit_construction():
    for e in range(255):
        assert float(ue8m0_f32(e)) == 2.0 ** (e - 127), e


def code_offset(phase, r, b, t):
    half, chunk = b >> 3, b & 7
    if phase == 1:
        box, rb = ((r >> 3) * 2 + half) * 1024, r & 7
    else:
        box, rb = half * 2048, r
    return box + rb * 128 + ((chunk ^ (r & 7)) << 4) + 4 * t


def logical_offset(phase, r, b, t):
    """Where TMA puts byte 4t of block b of stage row r, before the swizzle: box
    [matrix][piece][row][128 bytes] (phase 1, 8-row boxes) or [piece][row][128 bytes]
    (phase 2), piece = b / 8, 16 bytes per block."""
    half, chunk = b >> 3, b & 7
    if phase == 1:
        return ((r >> 3) * 2 + half) * 1024 + (r & 7) * 128 + chunk * 16 + 4 * t
    return half * 2048 + r * 128 + chunk * 16 + 4 * t


def swizzle128(addr):
    # the 128-byte TMA swizzle: 16-byte chunk index (bits 4-6) XOR the 128-byte line
    # index within a 1024-byte span (bits 7-9)
    return addr ^ (((addr >> 7) & 7) << 4)


def test_stage_offsets_are_the_swizzled_layout_and_a_bijection():
    for phase in (1, 2):
        seen = set()
        for r in range(16):
            for b in range(16):
                for t in range(4):
                    off = code_offset(phase, r, b, t)
                    assert off == swizzle128(logical_offset(phase, r, b, t))
                    assert off % 4 == 0 and 0 <= off < 4096
                    seen.add(off)
        assert len(seen) == 16 * 16 * 4  # every 4-byte word of the 4 KB stage once


def test_one_read_of_eight_rows_hits_32_banks():
    # lanes (g, t), g = 0..7, t = 0..3 read row g (or g + 8) of the same block b
    for phase in (1, 2):
        for b in range(16):
            for row_base in (0, 8):
                banks = {(code_offset(phase, row_base + g, b, t) // 4) % 32
                         for g in range(8) for t in range(4)}
                assert len(banks) == 32, (phase, b, row_base)


def test_mma_k_order_covers_each_block_element_once():
    # m16n8k16: lane (g, t) holds A k-pairs {2t, 2t+1} (a0, a1 rows g, g+8) and
    # {2t+8, 2t+9} (a2, a3); B k-pairs {2t, 2t+1} (b0) and {2t+8, 2t+9} (b1).  The kernel
    # feeds lane t's block elements 8t..8t+7 as: MMA 1 a0/b0 <- 8t, 8t+1; a2/b1 <- 8t+2,
    # 8t+3; MMA 2 a0/b0 <- 8t+4, 8t+5; a2/b1 <- 8t+6, 8t+7.
    used = []
    for mma in range(2):
        for t in range(4):
            for slot in range(2):  # (a0, b0) then (a2, b1)
                for e in range(2):
                    k_logical = 2 * t + 8 * slot + e
                    element = 8 * t + 4 * mma + 2 * slot + e
                    used.append((mma, k_logical, element))
    assert sorted(u[2] for u in used) == list(range(32))
    for mma in range(2):
        assert sorted(u[1] for u in used if u[0] == mma) == list(range(16))
