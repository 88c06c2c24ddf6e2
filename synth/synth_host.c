/*
 * Seeded synthetic FP4 expert weights, host side.
 *
 * Input generator only: this file holds none of the MoE method's arithmetic.
 * It fills byte arrays with pseudo-random FP4 code bytes and UE8M0 scale bytes
 * so that the oracle (CPU) and the CUDA path see the same weights.  The device
 * side (synth_dev.cu) implements the same generator independently from the
 * same published definition.
 *
 * Generator: SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014; constants as published by
 * S. Vigna).  Its state after n steps is s0 + n * 0x9E3779B97F4A7C15 and each
 * output is a fixed bijective mix of that state, so output n can be computed
 * directly from n: it is counter-based.
 *
 * Streams: one stream per (layer, expert, matrix, kind), with initial state
 *   s0 = seed XOR (stream_id << 40),
 *   stream_id = ((layer * 1024 + expert) * 4 + matrix) * 2 + kind,
 * matrix 0 = gate, 1 = up, 2 = down; kind 0 = codes, 1 = scales.
 * Byte i of a matrix's array is byte (i mod 8) (little-endian) of output
 * number floor(i / 8) + 1 of its stream.
 *   code byte  = that byte (two uniform 4-bit codes, low nibble first),
 *   scale byte = 121 + (that byte AND 3), i.e. 2^e with e uniform in {-6..-3}.
 */
#include <stdint.h>
#include <stddef.h>

#define SM64_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t sm64_mix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t synth_stream_id(int layer, int expert, int matrix, int kind) {
    return ((((uint64_t)layer * 1024u + (uint64_t)expert) * 4u + (uint64_t)matrix) * 2u +
            (uint64_t)kind);
}

/* Output number n (n >= 1) of the stream. */
uint64_t synth_word(uint64_t seed, uint64_t stream_id, uint64_t n) {
    uint64_t s0 = seed ^ (stream_id << 40);
    return sm64_mix(s0 + n * SM64_GAMMA);
}

/* Fill `nbytes` bytes of one matrix's codes (kind 0) or scales (kind 1),
 * starting at byte `first` of the stream. */
void synth_fill(uint64_t seed, int layer, int expert, int matrix, int kind,
                uint8_t* out, size_t first, size_t nbytes) {
    uint64_t sid = synth_stream_id(layer, expert, matrix, kind);
    size_t i = 0;
    while (i < nbytes) {
        size_t b = first + i;
        uint64_t w = synth_word(seed, sid, (uint64_t)(b >> 3) + 1u);
        for (unsigned k = (unsigned)(b & 7u); k < 8u && i < nbytes; ++k, ++i) {
            uint8_t v = (uint8_t)(w >> (8u * k));
            out[i] = kind == 0 ? v : (uint8_t)(121u + (v & 3u));
        }
    }
}
