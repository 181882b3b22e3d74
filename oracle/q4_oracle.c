/*
 * ORACLE -- test infrastructure only.  A plain, slow CPU restatement of the
 * Q4_0 dequantise-and-multiply matrix-vector product, in fp64.  Only the
 * tests, the smoke check and the benchmark's CPU-baseline leg may load it;
 * the product path never does.  It shares no code, header or table with the
 * CUDA library.
 *
 * What it follows:
 *  - "SwarmLLM" press page on originshq.com, section "The Engine: ~50 WGSL
 *    Kernels Written From Scratch": decode reads every weight once,
 *    dequantises the 4-bit values and accumulates the matrix-vector product.
 *  - The Q4_0 format the pages name (taozi.news page, section "支持模型与限制";
 *    originshq.com page, "Key Takeaways") but never lay out.  The plainest
 *    reading, GGUF's Q4_0 block, is used: 18 bytes per 32 weights, an f16
 *    scale d (little-endian) followed by 16 bytes qs; weight j of the block
 *    has code q_j = qs[j] & 15 for j < 16 and qs[j-16] >> 4 for j >= 16, and
 *    value (q_j - 8) * d.
 *  - y[m][n] = sum_k W[n][k] * x[m][k], x and y row-major, W row n holding
 *    the K/32 blocks of output n.
 *
 * Parity pins live in tests/test_oracle_pins.py (closed forms, unit vectors,
 * brute force in exact rationals, scale linearity, codec tables).
 */
#include <stdint.h>
#include <stddef.h>
#include <math.h>

/* IEEE-754 binary16 -> binary64: sign, 5-bit exponent (bias 15), 10-bit
 * fraction; exponent 0 is subnormal (f * 2^-24); exponent 31 is Inf/NaN. */
double oracle_f16_to_f64(uint16_t h) {
    const int s = (h >> 15) & 1;
    const int e = (h >> 10) & 0x1F;
    const int f = h & 0x3FF;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25);
    return s ? -v : v;
}

/* binary64 -> binary16, round to nearest, ties to even (used where the path
 * defines an f16 result: renormalised vectors).  Works on the value: finds
 * the f16 quantum for |v| and rounds |v| / quantum to an integer. */
uint16_t oracle_f64_to_f16(double v) {
    if (isnan(v)) return 0x7E00;
    const uint16_t sign = signbit(v) ? 0x8000 : 0;
    if (isinf(v)) return sign | 0x7C00;
    double a = fabs(v);
    if (a == 0.0) return sign;
    int ex;
    frexp(a, &ex);                   /* a = m * 2^ex, m in [0.5, 1) */
    int E = ex - 1;                  /* a in [2^E, 2^(E+1)) */
    if (E < -14) E = -14;            /* subnormal range shares quantum 2^-24 */
    const double quantum = ldexp(1.0, E - 10);
    double n = a / quantum;          /* exact: power-of-two division */
    double r = floor(n);
    const double frac = n - r;
    if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
    /* r * quantum is the rounded magnitude; re-encode it */
    const double rounded = r * quantum;
    if (rounded > 65504.0) return sign | 0x7C00;   /* beyond the f16 max */
    if (rounded < ldexp(1.0, -14))   /* subnormal: r counts 2^-24 units */
        return sign | (uint16_t)r;
    int ex2;
    const double m2 = frexp(rounded, &ex2);          /* [0.5, 1) */
    const int E2 = ex2 - 1;
    const uint16_t frac10 = (uint16_t)((m2 * 2.0 - 1.0) * 1024.0);
    return sign | (uint16_t)((E2 + 15) << 10) | frac10;
}

/* One Q4_0 weight: row bytes `row`, column k. */
static double q4_0_weight(const uint8_t* row, int64_t k) {
    const uint8_t* blk = row + (k / 32) * 18;
    const uint16_t dbits = (uint16_t)(blk[0] | (blk[1] << 8));
    const double d = oracle_f16_to_f64(dbits);
    const int j = (int)(k % 32);
    const int q = (j < 16) ? (blk[2 + j] & 0x0F) : (blk[2 + j - 16] >> 4);
    return (double)(q - 8) * d;
}

/* y[m * nrows + r] = sum_k W[r][k] * x[m * K + k] for the nrows GGUF rows at
 * `rows` (each K/32*18 bytes), m in [0, M).  x holds f16 bit patterns. */
void oracle_q4_gemv(const uint8_t* rows, int64_t nrows, int64_t K,
                    const uint16_t* x, int64_t M, double* y) {
    const int64_t rb = (K / 32) * 18;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t r = 0; r < nrows; ++r) {
            const uint8_t* row = rows + r * rb;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += q4_0_weight(row, k) * oracle_f16_to_f64(x[m * K + k]);
            y[m * nrows + r] = acc;
        }
    }
}

/* The packed layout the repack step must produce, restated from the library's
 * documented contract.  Rows are padded to Np = ceil(N/32)*32 (padding rows
 * hold qs bytes 0x88, i.e. q = 8, and d = +0) and grouped into tiles of 32.
 * With KB = K/32, segment s = t*KB + b holds block b of the 32 rows of tile
 * t in the 576 bytes from 576*s.  Row n = 32t + r is written as r = g + 8i
 * (g in [0,8), i in [0,4)).
 *   byte 576*s + 16*(4g + c) + 4i + e      <-  qs[4c + e]     (c, e in [0,4))
 *   bytes 576*s + 512 + 8g + 2i + {0,1}    <-  d (little-endian f16)        */
void oracle_repack(const uint8_t* gguf, int64_t N, int64_t K, uint8_t* packed) {
    const int64_t KB = K / 32;
    const int64_t Np = (N + 31) / 32 * 32;
    for (int64_t n = 0; n < Np; ++n) {
        const int64_t t = n / 32, r = n % 32;
        const int64_t g = r % 8, i = r / 8;
        for (int64_t b = 0; b < KB; ++b) {
            uint8_t* seg = packed + 576 * (t * KB + b);
            uint8_t blk[18];
            for (int h = 0; h < 18; ++h)
                blk[h] = (n < N) ? gguf[(n * KB + b) * 18 + h] : (h < 2 ? 0x00 : 0x88);
            for (int64_t j = 0; j < 16; ++j) {
                const int64_t c = j / 4, e = j % 4;
                seg[16 * (4 * g + c) + 4 * i + e] = blk[2 + j];
            }
            for (int64_t h = 0; h < 2; ++h)
                seg[512 + 8 * g + 2 * i + h] = blk[h];
        }
    }
}

/* ---- Q8_0: GGUF's other block format, named by the pages (taozi.news page,
 * section "支持模型与限制") without a layout.  The plainest reading, GGUF's
 * Q8_0 block: 34 bytes per 32 weights, an f16 scale d (little-endian) then
 * 32 signed 8-bit codes; weight j is qs[j] * d. */
static double q8_0_weight(const uint8_t* row, int64_t k) {
    const uint8_t* blk = row + (k / 32) * 34;
    const uint16_t dbits = (uint16_t)(blk[0] | (blk[1] << 8));
    const double d = oracle_f16_to_f64(dbits);
    const int q = (int)(int8_t)blk[2 + k % 32];
    return (double)q * d;
}

/* As oracle_q4_gemv, for Q8_0 rows of K/32*34 bytes. */
void oracle_q8_gemv(const uint8_t* rows, int64_t nrows, int64_t K,
                    const uint16_t* x, int64_t M, double* y) {
    const int64_t rb = (K / 32) * 34;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t r = 0; r < nrows; ++r) {
            const uint8_t* row = rows + r * rb;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += q8_0_weight(row, k) * oracle_f16_to_f64(x[m * K + k]);
            y[m * nrows + r] = acc;
        }
    }
}

/* The packed Q8_0 layout, restated from the library's documented contract:
 * rows padded to Np = ceil(N/32)*32 (padding rows: codes 0, d = +0), tiles of
 * 32 rows, segment s = t*KB + b in the 1088 bytes from 1088*s; row
 * n = 32t + g + 8i (g in [0,8), i in [0,4)):
 *   byte 1088*s + 32*(4g + c) + 8i + e      <-  qs[4c + e]        (c, e in [0,4))
 *   byte 1088*s + 32*(4g + c) + 8i + 4 + e  <-  qs[16 + 4c + e]
 *   bytes 1088*s + 1024 + 8g + 2i + {0,1}   <-  d (little-endian f16)       */
void oracle_repack_q8(const uint8_t* gguf, int64_t N, int64_t K, uint8_t* packed) {
    const int64_t KB = K / 32;
    const int64_t Np = (N + 31) / 32 * 32;
    for (int64_t n = 0; n < Np; ++n) {
        const int64_t t = n / 32, r = n % 32;
        const int64_t g = r % 8, i = r / 8;
        for (int64_t b = 0; b < KB; ++b) {
            uint8_t* seg = packed + 1088 * (t * KB + b);
            uint8_t blk[34];
            for (int h = 0; h < 34; ++h) blk[h] = (n < N) ? gguf[(n * KB + b) * 34 + h] : 0x00;
            for (int64_t c = 0; c < 4; ++c)
                for (int64_t e = 0; e < 4; ++e) {
                    seg[32 * (4 * g + c) + 8 * i + e] = blk[2 + 4 * c + e];
                    seg[32 * (4 * g + c) + 8 * i + 4 + e] = blk[2 + 16 + 4 * c + e];
                }
            for (int64_t h = 0; h < 2; ++h) seg[1024 + 8 * g + 2 * i + h] = blk[h];
        }
    }
}

/* Unit-RMS scale of an f16 vector: s = sum v_i^2 (fp64), 1 / sqrt(s / len);
 * 0 for an all-zero vector (which then stays zero). */
double oracle_unit_rms_scale(const uint16_t* v, int64_t len) {
    double s = 0.0;
    for (int64_t i = 0; i < len; ++i) {
        const double a = oracle_f16_to_f64(v[i]);
        s += a * a;
    }
    if (s == 0.0) return 0.0;
    return 1.0 / sqrt(s / (double)len);
}

/* Renormalise an f16 vector to unit RMS as an f16 vector: out_i =
 * f16(v_i * scale). */
void oracle_renorm(const uint16_t* v, int64_t len, uint16_t* out) {
    const double scale = oracle_unit_rms_scale(v, len);
    for (int64_t i = 0; i < len; ++i)
        out[i] = oracle_f64_to_f16(oracle_f16_to_f64(v[i]) * scale);
}

/* Round an fp64 vector to f16 (the boundary's output type). */
void oracle_round_f16(const double* v, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f64_to_f16(v[i]);
}

/* SiLU(gate) * up for a 2K-entry f16 vector [gate | up] (the gate+up GEMV's
 * output), in fp64: u_k = g_k / (1 + exp(-g_k)) * up_k.  The pages name the
 * model family (Qwen 3.8 27B: taozi.news page, section "支持模型与限制";
 * originshq.com page, "Limitations and Open Questions") but not its FFN
 * activation; the reading used is that family's gated unit: SiLU of the gate
 * half times the up half, fed to the down GEMV unrounded. */
void oracle_swiglu(const uint16_t* gate_up, int64_t K, int64_t M, double* u) {
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t* v = gate_up + m * 2 * K;
        for (int64_t k = 0; k < K; ++k) {
            const double g = oracle_f16_to_f64(v[k]);
            const double p = oracle_f16_to_f64(v[K + k]);
            u[m * K + k] = g / (1.0 + exp(-g)) * p;
        }
    }
}

/* As oracle_q4_gemv with an fp64 input x[M][K] (not f16 bit patterns). */
void oracle_q4_gemv_f64(const uint8_t* rows, int64_t nrows, int64_t K,
                        const double* x, int64_t M, double* y) {
    const int64_t rb = (K / 32) * 18;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t r = 0; r < nrows; ++r) {
            const uint8_t* row = rows + r * rb;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += q4_0_weight(row, k) * x[m * K + k];
            y[m * nrows + r] = acc;
        }
    }
}
