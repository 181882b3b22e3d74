/*
 * Seeded synthetic inputs for the Q4_0 GEMV path: GGUF-layout Q4_0 weight
 * rows and f16 activation vectors.
 *
 * This module only draws random numbers and encodes them; it holds none of
 * the dequantise-and-multiply arithmetic.  Both the fp64 oracle (tests) and
 * the CUDA path (tests, bench) consume what it writes.
 *
 * Random numbers: splitmix64 (Steele, Lea & Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014), used counter-style so any
 * element can be regenerated alone:
 *     at(s, i)  = mix64(s + (i + 1) * GAMMA)      (output #i of the sequence
 *                                                   whose state starts at s)
 *     key(seed, tensor_id) = at(seed, tensor_id)
 *     draw(seed, tensor_id, i) = at(key(seed, tensor_id), i)
 *
 * Q4_0 block (GGUF layout, 18 bytes: f16 scale d little-endian, then 16 bytes
 * of nibbles): block index bi = row * (K/32) + b uses draws 3bi, 3bi+1, 3bi+2.
 *   d    = f16_rne(sign * (0.002 + 0.048 * u)),  u = low 53 bits of draw 3bi
 *          times 2^-53, sign from its top bit (1 -> negative);
 *   qs[0..7] = bytes of draw 3bi+1 (little-endian), qs[8..15] = draw 3bi+2.
 * f16 activation element i: Box-Muller on draws 2i and 2i+1,
 *   z = sqrt(-2 ln u1) cos(2 pi u2), u1 in (0,1], u2 in [0,1), then f16_rne.
 *
 * Compile with -ffp-contract=off so the double arithmetic is not fused.
 */
#include <stdint.h>
#include <string.h>
#include <math.h>

#define SYNTH_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t synth_splitmix64_at(uint64_t state, uint64_t i) {
    return mix64(state + (i + 1) * SYNTH_GAMMA);
}

uint64_t synth_stream_key(uint64_t seed, uint64_t tensor_id) {
    return synth_splitmix64_at(seed, tensor_id);
}

/* IEEE-754 binary64 -> binary16, round to nearest, ties to even.
 * binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits;
 * subnormals have unit 2^-24; exponent 31 encodes Inf/NaN. */
uint16_t synth_f64_to_f16(double v) {
    uint64_t b;
    memcpy(&b, &v, sizeof b);
    uint16_t sign = (uint16_t)((b >> 48) & 0x8000u);
    int exp = (int)((b >> 52) & 0x7FF);
    uint64_t frac = b & ((1ULL << 52) - 1);
    if (exp == 0x7FF) return sign | (frac ? 0x7E00 : 0x7C00);
    if (exp == 0) return sign;                 /* |v| < 2^-1022: rounds to 0 */
    int e = exp - 1023;                        /* v = sig * 2^(e-52) */
    uint64_t sig = frac | (1ULL << 52);
    int shift;                                 /* bits of sig dropped */
    if (e >= -14) shift = 42;                  /* keep 11 significant bits */
    else shift = 28 - e;                       /* subnormal: unit 2^-24 */
    uint64_t q;
    if (shift >= 64) {
        q = 0;                                 /* sig < 2^53 <= half unit */
    } else {
        q = sig >> shift;
        uint64_t rem = sig & ((1ULL << shift) - 1);
        uint64_t half = 1ULL << (shift - 1);
        if (rem > half || (rem == half && (q & 1))) q++;
    }
    if (e >= -14) {
        if (q == (1ULL << 11)) { q = 1ULL << 10; e++; }
        if (e > 15) return sign | 0x7C00;      /* overflow to infinity */
        return sign | (uint16_t)((e + 15) << 10) | (uint16_t)(q & 0x3FF);
    }
    return sign | (uint16_t)q;                 /* q == 1024 encodes 2^-14 */
}

void synth_f64_to_f16_array(const double* v, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = synth_f64_to_f16(v[i]);
}

/* Rows [row0, row0 + nrows) of a Q4_0 matrix with K columns (K % 32 == 0),
 * written as GGUF blocks: out holds nrows * (K/32) * 18 bytes. */
void synth_q4_0_rows(uint64_t seed, uint64_t tensor_id, int64_t K,
                     int64_t row0, int64_t nrows, uint8_t* out) {
    const uint64_t key = synth_stream_key(seed, tensor_id);
    const int64_t nb = K / 32;
    for (int64_t r = 0; r < nrows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const uint64_t bi = (uint64_t)(row0 + r) * (uint64_t)nb + (uint64_t)b;
            const uint64_t r0 = synth_splitmix64_at(key, 3 * bi);
            const uint64_t r1 = synth_splitmix64_at(key, 3 * bi + 1);
            const uint64_t r2 = synth_splitmix64_at(key, 3 * bi + 2);
            const double u = (double)(r0 & ((1ULL << 53) - 1)) * 0x1p-53;
            double mag = 0.002 + 0.048 * u;
            if (r0 >> 63) mag = -mag;
            const uint16_t d = synth_f64_to_f16(mag);
            uint8_t* blk = out + (r * nb + b) * 18;
            blk[0] = (uint8_t)(d & 0xFF);
            blk[1] = (uint8_t)(d >> 8);
            for (int j = 0; j < 8; ++j) {
                blk[2 + j] = (uint8_t)(r1 >> (8 * j));
                blk[10 + j] = (uint8_t)(r2 >> (8 * j));
            }
        }
    }
}

/* Rows [row0, row0 + nrows) of a Q8_0 matrix with K columns (K % 32 == 0),
 * written as GGUF blocks of 34 bytes: f16 d (little-endian), then 32 int8
 * codes.  d = f16(+-(0.002 + 0.048 u) / 16) (u, sign: draw 5bi) keeps the
 * weights in the range of the Q4_0 matrices; the codes are the raw bytes of
 * draws 5bi+1 .. 5bi+4 (uniform over -128..127). */
void synth_q8_0_rows(uint64_t seed, uint64_t tensor_id, int64_t K,
                     int64_t row0, int64_t nrows, uint8_t* out) {
    const uint64_t key = synth_stream_key(seed, tensor_id);
    const int64_t nb = K / 32;
    for (int64_t r = 0; r < nrows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const uint64_t bi = (uint64_t)(row0 + r) * (uint64_t)nb + (uint64_t)b;
            const uint64_t r0 = synth_splitmix64_at(key, 5 * bi);
            const double u = (double)(r0 & ((1ULL << 53) - 1)) * 0x1p-53;
            double mag = (0.002 + 0.048 * u) / 16.0;
            if (r0 >> 63) mag = -mag;
            const uint16_t d = synth_f64_to_f16(mag);
            uint8_t* blk = out + (r * nb + b) * 34;
            blk[0] = (uint8_t)(d & 0xFF);
            blk[1] = (uint8_t)(d >> 8);
            for (int w = 0; w < 4; ++w) {
                const uint64_t rw = synth_splitmix64_at(key, 5 * bi + 1 + (uint64_t)w);
                for (int j = 0; j < 8; ++j) blk[2 + 8 * w + j] = (uint8_t)(rw >> (8 * j));
            }
        }
    }
}

/* Elements [i0, i0 + n) of an f16 N(0,1) vector. */
void synth_normal_f16(uint64_t seed, uint64_t tensor_id, int64_t i0, int64_t n,
                      uint16_t* out) {
    const uint64_t key = synth_stream_key(seed, tensor_id);
    const double two_pi = 6.283185307179586476925286766559;
    for (int64_t t = 0; t < n; ++t) {
        const uint64_t i = (uint64_t)(i0 + t);
        const uint64_t a = synth_splitmix64_at(key, 2 * i);
        const uint64_t c = synth_splitmix64_at(key, 2 * i + 1);
        const double u1 = (double)((a >> 11) + 1) * 0x1p-53;   /* (0, 1] */
        const double u2 = (double)(c >> 11) * 0x1p-53;         /* [0, 1) */
        const double z = sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
        out[t] = synth_f64_to_f16(z);
    }
}
