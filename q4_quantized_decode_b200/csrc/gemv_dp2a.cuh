// Q4_0 GEMV for M = 1..2 on CUDA cores with exact integer block dot products.
//
// The pages' engine sweeps each weight row with a 64-thread group,
// dequantises in registers and reduces in shared memory (originshq.com page,
// section "The Engine: ~50 WGSL Kernels Written From Scratch").  On sm_100a
// the row sweep is replaced by a flat, perfectly balanced split of all
// (tile of 32 rows, 32-column block) segments over every warp of the grid:
//   * each warp streams its contiguous run of 576-byte segments (512 bytes of
//     codes, 64 of scales) through a private ring of shared-memory stages,
//     each filled by one bulk asynchronous copy (TMA); a few warps per SM
//     keep ~150 KB per SM in flight, which register-staged loads cannot;
//   * lane (g, c) reads qs word c of rows g, g+8, g+16, g+24 (16 bytes) and
//     the four row scales (8 bytes) of a segment from the stage;
//   * the activations are loaded once per CTA with plain 16-byte loads and
//     converted in registers, per 32-column block, to 16-bit integers with a
//     power-of-two scale (the block maximum held exactly); they are stored in
//     shared memory in the lane order of the weight words.  Each weight word
//     is split into two byte vectors of codes with one shift and two masks and
//     multiplied with dp2a (16-bit x 8-bit dot products), so the block sum of
//     (q - 8) * X is an exact integer;
//   * the block sum is scaled by d * 2^e in fp32 and accumulated per row;
//   * a warp's accumulators are combined across its four column lanes with
//     two shuffles.  A tile split between warps is combined in two levels,
//     each a sum in a fixed order, so results are deterministic: the warps of
//     one CTA park their partials in shared memory and the CTA's first
//     contributing warp sums them in warp order; a tile shared by several
//     CTAs then leaves one partial per CTA in global memory, summed in CTA
//     order by the last CTA to arrive (per-tile counter).
#pragma once

#include "device_common.cuh"
#include "partition.cuh"

namespace q4 {

constexpr int kSegBytes = 576;       // one Q4_0 segment: 512 bytes of codes, then 64 of scales
constexpr int kSegSclOff = 512;
// Q8_0 segments (32 rows x one block of 32 signed 8-bit codes): 1024 bytes
// of codes, then the same 64 bytes of scales.  Lane (g, c) finds, for row
// g + 8i, codes 4c..4c+3 and 16+4c..16+4c+3 in the 8 bytes at 32*(4g+c) + 8i.
constexpr int kSegBytesQ8 = 1088;
constexpr int kSegSclOffQ8 = 1024;
template <bool Q8>
struct SegFmt {
    static constexpr int kBytes = Q8 ? kSegBytesQ8 : kSegBytes;
    static constexpr int kScl = Q8 ? kSegSclOffQ8 : kSegSclOff;
};
constexpr int kXChunksPerThread = 9; // activation staging: M*K <= 9 * 8 * threads

// Row-sharded decode step over peer memory (M = 1).  Every entry of a
// gathered vector is one 32-bit word: the binary16 value in the low half and
// the stamp of the GEMV that wrote it in the high half.  A GEMV stores its
// rows as such words straight into every rank's gather buffer; the next GEMV
// polls the words it stages until each carries the stamp it expects.  A word
// is written and read whole (single-copy atomic), so no fence, flag or
// arrival count orders the exchange.  Stamps are (steps run x GEMVs per step
// + GEMV index) mod 2^16: the word a reader finds is the one it expects or
// the one written four GEMVs earlier into the same buffer, never equal.
struct PeerArgs {
    uint32_t* const* y;           // [n]: this rank's slice in rank p's gather buffer (rank p's memory)
    const uint32_t* xw;           // wait: the gathered input words (this rank's memory)
    const unsigned* seq;          // [0]: steps run including this one, [1]: steps since the arrival
                                  //      counts were zeroed
    int n;                        // ranks; 0: a plain GEMV
    int g;                        // this GEMV's index in the step
    int per_step;                 // GEMVs per step
    int wait;                     // 1: the input is xw, stamped by GEMV g - 1
    unsigned poll_limit;          // polls of one chunk before giving up
    unsigned unreachable;         // test knob: 1 waits for a stamp no GEMV writes yet
    // Filled in by the kernel from seq at its start (peer_prepare):
    uint32_t stamp_out;           // this GEMV's stamp, bits 16-31 of its words
    uint32_t stamp_in;            // the stamp its input words must carry
    unsigned rounds;              // earlier rounds of its split tiles' arrival counts
};

__device__ __forceinline__ uint32_t peer_stamp(const unsigned* seq, int per_step, int g) {
    return (seq[0] * (unsigned)per_step + (unsigned)g) & 0xFFFFu;
}

// The step-dependent values of a GEMV, read once at its start.  The arrival
// counts of GEMV g are shared with the same matrix of every layer (the same
// split, so the same arrivals per tile) and run on across steps: this
// GEMV's arrivals follow (steps since they were zeroed - 1) * layers + layer
// earlier rounds of them.
__device__ __forceinline__ void peer_prepare(PeerArgs& p) {
    const unsigned s0 = p.seq[0], s1 = p.seq[1];
    p.stamp_out = (s0 * (unsigned)p.per_step + (unsigned)p.g) & 0xFFFFu;
    p.stamp_in = (s0 * (unsigned)p.per_step + (unsigned)(p.g - 1) + p.unreachable) & 0xFFFFu;
    p.rounds = (s1 - 1u) * (unsigned)(p.per_step / 4) + (unsigned)(p.g / 4);
}

__device__ __forceinline__ void st_relaxed_sys_u32(uint32_t* p, uint32_t v) {
    asm volatile("st.relaxed.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint4 ld_relaxed_sys_v4(const uint32_t* p) {
    uint4 v;
    asm volatile("ld.relaxed.sys.global.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p)
                 : "memory");
    return v;
}

// The eight binary16 entries of two loaded word quads, and whether all
// eight words carry `stamp`.
__device__ __forceinline__ bool peer_words_ok(uint4 lo, uint4 hi, uint32_t stamp) {
    const uint32_t s = stamp << 16;
    return (((lo.x ^ s) | (lo.y ^ s) | (lo.z ^ s) | (lo.w ^ s) | (hi.x ^ s) | (hi.y ^ s) | (hi.z ^ s) |
             (hi.w ^ s)) >> 16) == 0u;
}
__device__ __forceinline__ uint4 peer_words_f16(uint4 lo, uint4 hi) {
    return make_uint4(__byte_perm(lo.x, lo.y, 0x5410), __byte_perm(lo.z, lo.w, 0x5410),
                      __byte_perm(hi.x, hi.y, 0x5410), __byte_perm(hi.z, hi.w, 0x5410));
}

// Polls the chunk of eight words at w (first read: lo, hi) until all carry
// `stamp`; bounded by poll_limit, and given up at once when an earlier wait
// has already run out (the error word is set), so a lost peer costs one
// time-out per step.  Returns the chunk's eight values.
static __device__ __noinline__ uint4 peer_poll_chunk(const uint32_t* w, uint4 lo, uint4 hi, uint32_t stamp,
                                                     unsigned poll_limit, int* err) {
    uint32_t it = 0;
    while (!peer_words_ok(lo, hi, stamp)) {
        if (++it > poll_limit || (!(it & 1023u) && *reinterpret_cast<volatile int*>(err) != 0)) {
            set_device_error(err, kDevTimeout);
            break;
        }
        lo = ld_relaxed_sys_v4(w);
        hi = ld_relaxed_sys_v4(w + 4);
    }
    return peer_words_f16(lo, hi);
}

// Chunks q0 + stride * i (i < QN; 0 past nq) of eight stamped words each:
// all loads issued together, then each chunk still stale polled on its own
// until it carries `stamp`.  (Reloading every stale chunk each round was
// measured slower: more L2 traffic while the input is still being written.)
template <int QN>
__device__ __forceinline__ void peer_load_chunks(const uint32_t* words, int nq, int q0, int stride,
                                                 uint32_t stamp, unsigned poll_limit, int* err,
                                                 uint4 (&xr)[QN]) {
    uint4 hi[QN];             // xr holds a chunk's first four words until it converts
#pragma unroll
    for (int i = 0; i < QN; ++i) {
        const int q = q0 + stride * i;
        if (q < nq) {
            xr[i] = ld_relaxed_sys_v4(words + (size_t)q * 8);
            hi[i] = ld_relaxed_sys_v4(words + (size_t)q * 8 + 4);
        }
    }
#pragma unroll
    for (int i = 0; i < QN; ++i) {
        const int q = q0 + stride * i;
        if (q >= nq)
            xr[i] = make_uint4(0, 0, 0, 0);
        else if (peer_words_ok(xr[i], hi[i], stamp))
            xr[i] = peer_words_f16(xr[i], hi[i]);
        else
            xr[i] = peer_poll_chunk(words + (size_t)q * 8, xr[i], hi[i], stamp, poll_limit, err);
    }
}

struct GemvArgs {
    const uint8_t* W;       // packed matrix (segments of 576 bytes)
    const __half* x;        // [M][K] activations (renorm: the previous f16 output, unscaled)
    __half* y;              // [M][N]
    float* ws;              // CTA partials of tiles shared by CTAs [CTAs][2][M][32]
    int* cnt;               // per-tile arrival counters [T], zero between calls
    int* err;               // device error word
    __half* trace_x;        // nullable: CTA 0 writes the f16 input vector it used
    int64_t N;
    int K, KB, T;
    int S;                  // segments = T * KB
    int G;                  // warps that own segments (G <= S)
    int renorm;             // 1 (M == 1): the input is s * x[0:K], s its unit-RMS scale, applied
                            // to the outputs; 0: the input is x
    SplitConsts sc;         // make_split(S, G)
    PeerArgs peer = {};     // n > 0: outputs stored into every rank's gather buffer (M = 1)
};

// One finished output: y, or with peers this rank's slice in every rank's
// gather buffer as a stamped word (NVLink stores to the other GPUs).
__device__ __forceinline__ void store_out(const GemvArgs& a, int m, int64_t row, __half v) {
    if (a.peer.n > 0) {
        const uint32_t w = (a.peer.stamp_out << 16) |
                           (uint32_t)__half_as_ushort(v);
        for (int p = 0; p < a.peer.n; ++p) st_relaxed_sys_u32(a.peer.y[p] + row, w);
    } else {
        a.y[(size_t)m * a.N + row] = v;
    }
}

// Step bookkeeping of the peer exchange (one thread): a new step -- the
// stamps' step count and the arrival counts' epoch advance.
static __global__ void peer_step_kernel(unsigned* seq) {
    seq[0] = seq[0] + 1u;
    seq[1] = seq[1] + 1u;
}

// Per-warp ring of R stages of C segments.
__host__ __device__ constexpr size_t ring_bytes(int warps, int R, int C, int seg = kSegBytes) {
    return (size_t)warps * R * C * seg;
}

// Per warp, two parked tile partials (the first and the last tile of its
// run), M vectors of 32 fp32 each.
__host__ __device__ constexpr size_t warp_partial_bytes(int M, int warps) {
    return (size_t)warps * 2 * M * 32 * sizeof(float);
}

// Per-block sums of squares of an activation vector of K entries (fp32,
// padded to 16 bytes).
__host__ __device__ constexpr size_t tile_sum_bytes(int K) {
    return ((size_t)(K / 32) * 4 + 15) / 16 * 16;
}

// Shared-memory footprint of the M <= 2 kernel: the ring, the int16
// activations (2 bytes per element), per block and lane group the pair
// {-8 * sum X, block scale} (8 bytes, 32 per block), the warp partials, then
// the block sums of squares of vector 0.
__host__ __device__ constexpr size_t gemv_dp2a_smem_bytes(int M, int K, int warps, int R, int C,
                                                        int seg = kSegBytes) {
    return ring_bytes(warps, R, C, seg) + (size_t)M * K * 2 + (size_t)M * (K / 32) * 32 +
           warp_partial_bytes(M, warps) + tile_sum_bytes(K);
}

// Position of element j of a 32-column block in the permuted X layout: the
// eight entries lane group c needs ([4c..4c+3] and [4c+16..4c+19]) are
// contiguous.
__host__ __device__ __forceinline__ int xperm_pos(int j) {
    return ((j & 15) >> 2) * 8 + ((j >> 4) << 2) + (j & 3);
}

// A warp's private ring: stage k holds C consecutive segments of the warp's
// run [s0, s1), filled by one elected lane with one bulk copy.
template <int R, int C, int SEG = kSegBytes>
struct WarpRing {
    uint32_t stage0;        // shared address of this warp's first stage
    uint64_t* bars;         // R full-barriers
    const uint8_t* src;     // segment s0 in global memory
    int nseg;               // s1 - s0
    int nch;                // ceil(nseg / C)

    __device__ void init(uint32_t ring_base, uint64_t* bar_base, int warp, const uint8_t* W, int s0,
                         int s1) {
        stage0 = ring_base + (uint32_t)warp * R * C * SEG;
        bars = bar_base + warp * R;
        src = W + (size_t)s0 * SEG;
        nseg = s1 - s0;
        nch = (nseg + C - 1) / C;
    }
    __device__ uint32_t stage(int k) const { return stage0 + (uint32_t)k * C * SEG; }
    // Lane 0 only.
    __device__ void issue(int ch) const {
        const int k = ch % R;
        const uint32_t bytes = (uint32_t)min(C, nseg - ch * C) * SEG;
        mbar_arrive_expect_tx(bars + k, bytes);
        bulk_g2s_addr(stage(k), src + (size_t)ch * C * SEG, bytes, bars + k);
    }
    __device__ bool wait(int ch) const {
        return mbar_wait_bounded(bars + (ch % R), (uint32_t)((ch / R) & 1), 1u << 22);
    }
};

// ---- Activation blocks: exact int16 codes and sums of squares.
//
// A 32-entry block v of an f16 activation vector becomes X = rint(v *
// 2^(14-E)) (E: exponent of the block maximum, so |X| <= 32752 and the
// maximum is exact), stored in lane order (xperm_pos), and lane group c gets
// the record {0x4B400000 - 8 * sum of its eight X, 2^(E-14)}: started from
// that word, the dp2a sum of a lane's four rows ends as the bit pattern of
// the float 1.5 * 2^23 + sum (q - 8) X (exact: the sum is below 2^22 in
// magnitude), so one subtraction makes it a float.  X is read from the low
// mantissa bits of v * 2^(14-E) + 1.5 * 2^23: the product is exact and
// |X| < 2^22, so the one rounding of the addition is the round to the nearest
// integer (ties to even) and the bits hold 0x4B400000 + X.  All-zero block:
// X = 0, scale 0; non-finite block: scale NaN (its products are NaN whatever
// X holds).
//
// The block's sum of squares (for the unit-RMS scale of the next input) is
// taken in one fixed binary tree: squares rounded to fp32, then pairs of
// entries whose indices differ in bit 0, then bit 1, ... bit 4, every sum
// rounded to fp32 (no fused operations).  Two layouts compute the same tree:
// a chunk layout (four lanes per block, lane u holding entries 8u..8u+7) and
// a lane layout (one entry per lane, lane 4g + c holding entry g + 8c).

__device__ __forceinline__ void block_exponent(uint32_t mx, float& inv, float& sc) {
    const int E = (int)(mx >> 23) - 127;                                   // max in [2^E, 2^(E+1))
    const bool live = mx != 0u && mx < 0x7F800000u;
    inv = live ? __uint_as_float((uint32_t)(141 - E) << 23) : 0.f;          // 2^(14-E)
    sc = live ? __uint_as_float((uint32_t)(113 + E) << 23)                  // 2^(E-14)
              : (mx == 0u ? 0.f : __uint_as_float(0x7FC00000u));
}
constexpr float kRoundMagic = 12582912.0f;    // 1.5 * 2^23
constexpr uint32_t kRoundMagicBits = 0x4B400000u;

// Chunk layout: this lane holds entries 8u..8u+7 (u = lane & 3) of a block
// in v[]; the four lanes of the block call together (all 32 lanes of the
// warp execute it).  Outputs: the two 8-byte X words of the lane order
// positions of its entries, the record sums h0 (group 2(u&1)) and h1 (group
// 2(u&1)+1), the block scale and the block's sum of squares (all 4 lanes).
struct ChunkQ {
    uint2 x0, x1;        // X of entries 8u..8u+3 and 8u+4..8u+7 (int16 pairs)
    int h0, h1;
    float sc, sq;
};
__device__ __forceinline__ ChunkQ quant_chunk(const float v[8]) {
    ChunkQ o;
    uint32_t mx = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) mx = max(mx, __float_as_uint(fabsf(v[e])));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    float inv;
    block_exponent(mx, inv, o.sc);
    uint32_t xb[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) xb[e] = __float_as_uint(fmaf(v[e], inv, kRoundMagic));
    o.h0 = (int)(xb[0] + xb[1] + xb[2] + xb[3] - 4u * kRoundMagicBits);
    o.h1 = (int)(xb[4] + xb[5] + xb[6] + xb[7] - 4u * kRoundMagicBits);
    o.h0 += __shfl_xor_sync(0xffffffffu, o.h0, 2);      // quarters u and u^2 share lane groups
    o.h1 += __shfl_xor_sync(0xffffffffu, o.h1, 2);
    // The low 16 bits of xb[e] are X[e] in two's complement.
    o.x0 = make_uint2(__byte_perm(xb[0], xb[1], 0x5410), __byte_perm(xb[2], xb[3], 0x5410));
    o.x1 = make_uint2(__byte_perm(xb[4], xb[5], 0x5410), __byte_perm(xb[6], xb[7], 0x5410));
    float q[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) q[e] = __fmul_rn(v[e], v[e]);
    const float a0 = __fadd_rn(q[0], q[1]), a1 = __fadd_rn(q[2], q[3]);
    const float a2 = __fadd_rn(q[4], q[5]), a3 = __fadd_rn(q[6], q[7]);
    float t = __fadd_rn(__fadd_rn(a0, a1), __fadd_rn(a2, a3));
    t = __fadd_rn(t, __shfl_xor_sync(0xffffffffu, t, 1));   // entry bit 3 = u bit 0
    t = __fadd_rn(t, __shfl_xor_sync(0xffffffffu, t, 2));   // entry bit 4 = u bit 1
    o.sq = t;
    return o;
}
// Store a chunk's X words and records: block b, quarter u, at X base xb_addr
// (64 bytes per block) and record base rb_addr (32 bytes per block), shared
// memory.
__device__ __forceinline__ void store_chunk_smem(const ChunkQ& o, uint32_t x_base, uint32_t r_base,
                                                 int b, int u) {
    const int pos0 = (u & 1) * 16 + (u >> 1) * 4;   // lane order of entries 8u..8u+3 (+8 for the rest)
    const uint32_t xa = x_base + (uint32_t)b * 64 + pos0 * 2;
    sts64(xa, o.x0);
    sts64(xa + 16, o.x1);
    if (u < 2) {
        const uint32_t ra = r_base + (uint32_t)b * 32 + (u & 1) * 16;
        sts64(ra, make_uint2(kRoundMagicBits - 8u * (uint32_t)o.h0, __float_as_uint(o.sc)));
        sts64(ra + 8, make_uint2(kRoundMagicBits - 8u * (uint32_t)o.h1, __float_as_uint(o.sc)));
    }
}

// Lane layout (all 32 lanes): this lane holds entry j = (lane >> 2) + 8 *
// (lane & 3) of block b.  Writes X, the records and the sum of squares of
// the block to global memory (the persistent step's pre-quantised input).
__device__ __forceinline__ void quant_lane_store(float v, int b, int16_t* xq, uint2* xrec, float* xsq) {
    const int lane = threadIdx.x & 31;
    const int j = (lane >> 2) + 8 * (lane & 3);
    uint32_t mx = __float_as_uint(fabsf(v));
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float inv, sc;
    block_exponent(mx, inv, sc);
    const uint32_t xb = __float_as_uint(fmaf(v, inv, kRoundMagic));
    int h = (int)(xb - kRoundMagicBits);
    xq[(size_t)b * 32 + xperm_pos(j)] = (int16_t)(xb & 0xFFFFu);
    // lane group (j & 15) >> 2: entry bits 0, 1 and 4 vary = lane bits 2, 3, 1
    h += __shfl_xor_sync(0xffffffffu, h, 4);
    h += __shfl_xor_sync(0xffffffffu, h, 8);
    h += __shfl_xor_sync(0xffffffffu, h, 2);
    if ((lane & 0xE) == 0) {
        const int grp = (j & 15) >> 2;
        xrec[(size_t)b * 4 + grp] = make_uint2(kRoundMagicBits - 8u * (uint32_t)h, __float_as_uint(sc));
    }
    // entry bits 0, 1, 2, 3, 4 = lane bits 2, 3, 4, 0, 1
    float t = __fmul_rn(v, v);
    t = __fadd_rn(t, __shfl_xor_sync(0xffffffffu, t, 4));
    t = __fadd_rn(t, __shfl_xor_sync(0xffffffffu, t, 8));
    t = __fadd_rn(t, __shfl_xor_sync(0xffffffffu, t, 16));
    t = __fadd_rn(t, __shfl_xor_sync(0xffffffffu, t, 1));
    t = __fadd_rn(t, __shfl_xor_sync(0xffffffffu, t, 2));
    if (lane == 0) xsq[b] = t;
}

// Unit-RMS scale from the nb block sums of squares (shared or global
// memory, any warp; every lane returns it).  Lane l takes blocks l + 32j in
// rounds of eight j (loads issued together, zeros past nb), each round summed
// in a fixed three-level tree and added to the lane's sum in round order;
// then the lanes in an xor tree.
__device__ __forceinline__ float unit_rms_scale(const float* sq, int nb, int K) {
    const int lane = threadIdx.x & 31;
    float acc = 0.f;
    for (int j0 = 0; j0 * 32 < nb; j0 += 8) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int t = lane + 32 * (j0 + u);
            v[u] = t < nb ? sq[t] : 0.f;
        }
        const float a0 = __fadd_rn(v[0], v[1]), a1 = __fadd_rn(v[2], v[3]);
        const float a2 = __fadd_rn(v[4], v[5]), a3 = __fadd_rn(v[6], v[7]);
        acc = __fadd_rn(acc, __fadd_rn(__fadd_rn(a0, a1), __fadd_rn(a2, a3)));
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, o));
    return renorm_scale(acc, K);
}

// Activation staging for the M <= 2 kernel, all threads of the CTA.  Thread
// t holds the 16-byte chunks q = t, t + NT, ... of x (8 entries each; four
// chunks make a 32-entry block, held by four consecutive lanes) and writes
// the blocks' codes and records to shared memory, and (vector 0) the block
// sums of squares to sq[].  CTA 0 writes the input it read to trace_x.
// QN: chunks held per thread (M * K <= QN * 8 * NT); all QN rounds run
// (chunks past the end are zeros), so callers pick the smallest QN that
// covers the vector: the rounds then overlap instead of running one by one.
template <int M, int NT, int QN>
__device__ __forceinline__ void stage_activations(const GemvArgs& a, uint32_t xs, uint32_t rec,
                                                  float* sq) {
    const int tid = threadIdx.x;
    const int nq = M * a.K / 8;
    uint4 xr[QN];
    if (M == 1 && a.peer.n > 0 && a.peer.wait) {
        // stamped words of the previous GEMV, every rank's rows
        peer_load_chunks<QN>(a.peer.xw, nq, tid, NT, a.peer.stamp_in, a.peer.poll_limit, a.err, xr);
    } else {
#pragma unroll
        for (int i = 0; i < QN; ++i) {
            const int q = tid + NT * i;
            xr[i] = q < nq ? *reinterpret_cast<const uint4*>(a.x + (size_t)q * 8) : make_uint4(0, 0, 0, 0);
        }
    }
#pragma unroll
    for (int i = 0; i < QN; ++i) {
        const int q = tid + NT * i;
        if (M == 1 && a.trace_x != nullptr && blockIdx.x == 0 && q < nq)
            *reinterpret_cast<uint4*>(a.trace_x + (size_t)q * 8) = xr[i];
        // The four chunks of a block sit in lanes 4j..4j+3 (NT*i is a multiple
        // of 4), so every lane takes part in the shuffles.
        const __half2* h = reinterpret_cast<const __half2*>(&xr[i]);
        float v[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(h[e]);
            v[2 * e] = f.x;
            v[2 * e + 1] = f.y;
        }
        const ChunkQ o = quant_chunk(v);
        if (q < nq) {
            store_chunk_smem(o, xs, rec, q >> 2, q & 3);
            if ((q & 3) == 0 && q < a.K / 8) sq[q >> 2] = o.sq;
        }
    }
    __syncthreads();
}

// One warp's share of one GEMV on the dp2a path: accumulators, position in
// its run of segments, and the split-tile bookkeeping.
// Where a GEMV of the persistent step also writes its finished output
// blocks pre-quantised for the next GEMV (lane-order X, records, sums of
// squares; lane layout); nb: blocks the next GEMV reads (0: none).
struct QuantOut {
    int16_t* x;
    uint2* rec;
    float* sq;
    int nb;
};

template <int M, bool Q8 = false>
struct Dp2aConsumer {
    static constexpr int SEG = SegFmt<Q8>::kBytes;
    float acc[M][4];
    WarpSplit sp;
    int gw, lane, g, c, r;   // r: the tile row this lane emits
    int KB, t_cur, b;        // b: block of the next segment
    uint32_t x_lane0, r_lane0, xp, rp;   // running shared addresses of block b's X words and record
    uint32_t xstride, rstride;           // per activation vector
    float* park;             // this warp's two parked partials [2][M][32] (shared memory)
    float oscale;            // outputs are f16(oscale * sum): the input's unit-RMS scale, or 1
    QuantOut qo;

    __device__ __forceinline__ void init(const GemvArgs& a, int gw_, uint32_t xs, uint32_t rec,
                                         float* park_) {
        gw = gw_;
        park = park_;
        oscale = 1.f;
        qo.nb = 0;
        lane = threadIdx.x & 31;
        g = lane >> 2;
        c = lane & 3;
        r = g + 8 * c;
        KB = a.KB;
        sp.init(gw, a.sc, KB);
        t_cur = sp.t_first;
        b = sp.s0 - sp.t_first * KB;
        x_lane0 = xs + (uint32_t)c * 16;
        r_lane0 = rec + (uint32_t)c * 8;
        xp = x_lane0 + (uint32_t)b * 64;
        rp = r_lane0 + (uint32_t)b * 32;
        xstride = (uint32_t)a.K * 2;
        rstride = (uint32_t)KB * 32;
#pragma unroll
        for (int m = 0; m < M; ++m)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[m][i] = 0.f;
    }

    // Combine a finished tile: reduce over the four column lanes, then either
    // write y (this warp owns the whole tile) or park the partial.
    __device__ __forceinline__ void flush(const GemvArgs& a, int t) {
#pragma unroll
        for (int m = 0; m < M; ++m)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float v = acc[m][i];
                v += __shfl_xor_sync(0xffffffffu, v, 1);
                v += __shfl_xor_sync(0xffffffffu, v, 2);
                acc[m][i] = v;
            }
        const bool whole = sp.whole(t);
        const int64_t row = (int64_t)t * 32 + r;
#pragma unroll
        for (int m = 0; m < M; ++m) {
            const float val = (c == 0) ? acc[m][0] : (c == 1) ? acc[m][1] : (c == 2) ? acc[m][2] : acc[m][3];
            if (whole) {
                const __half yh = __float2half_rn(__fmul_rn(oscale, val));
                if (row < a.N) store_out(a, m, row, yh);
                if (M == 1 && t < qo.nb) quant_lane_store(__half2float(yh), t, qo.x, qo.rec, qo.sq);
            } else {
                park[(sp.slot(t) * M + m) * 32 + r] = val;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[m][i] = 0.f;
        }
    }

    // One segment at shared address `seg`, whose block's X words and record
    // are at xb and rb: codes and scales from a ring stage, X from the staged
    // activations.  Rows are handled in pairs on the packed fp32x2 pipes.
    __device__ __forceinline__ void segment(uint32_t seg, uint32_t xb, uint32_t rb) {
        if constexpr (Q8) {
            segment_q8(seg, xb, rb);
            return;
        }
        const uint4 w = lds128(seg + lane * 16);
        const uint2 dd = lds64(seg + kSegSclOff + g * 8);
        const float2 d01 = __half22float2(*reinterpret_cast<const __half2*>(&dd.x));
        const float2 d23 = __half22float2(*reinterpret_cast<const __half2*>(&dd.y));
        const uint32_t words[4] = {w.x, w.y, w.z, w.w};
        uint4 xq[M];
        uint2 rc[M];
#pragma unroll
        for (int m = 0; m < M; ++m) {
            xq[m] = lds128(xb + (uint32_t)m * xstride);
            rc[m] = lds64(rb + (uint32_t)m * rstride);
        }
        int v[M][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t lo = words[i] & 0x0F0F0F0Fu;          // codes 4c..4c+3
            const uint32_t hi = (words[i] >> 4) & 0x0F0F0F0Fu;   // codes 4c+16..4c+19
#pragma unroll
            for (int m = 0; m < M; ++m) {
                int t = dp2a_lo(xq[m].x, lo, (int)rc[m].x);
                t = dp2a_hi(xq[m].y, lo, t);
                t = dp2a_lo(xq[m].z, hi, t);
                v[m][i] = dp2a_hi(xq[m].w, hi, t);
            }
        }
        const float2 mm = make_float2(-kRoundMagic, -kRoundMagic);
#pragma unroll
        for (int m = 0; m < M; ++m) {
            const float sbm = __uint_as_float(rc[m].y);
            const float2 s2 = make_float2(sbm, sbm);
            const float2 ds01 = fmul2(d01, s2), ds23 = fmul2(d23, s2);
            float2 a01 = make_float2(acc[m][0], acc[m][1]), a23 = make_float2(acc[m][2], acc[m][3]);
            const float2 f01 = fadd2(make_float2(__int_as_float(v[m][0]), __int_as_float(v[m][1])), mm);
            const float2 f23 = fadd2(make_float2(__int_as_float(v[m][2]), __int_as_float(v[m][3])), mm);
            a01 = ffma2(f01, ds01, a01);
            a23 = ffma2(f23, ds23, a23);
            acc[m][0] = a01.x;
            acc[m][1] = a01.y;
            acc[m][2] = a23.x;
            acc[m][3] = a23.y;
        }
    }

    // Q8_0 segment: per row, two words of four signed codes (columns 4c.. and
    // 16+4c..) against the same int16 activation words; the block sum is an
    // exact integer (|sum| < 2^26) converted to fp32 once.
    __device__ __forceinline__ void segment_q8(uint32_t seg, uint32_t xb, uint32_t rb) {
        const uint4 w01 = lds128(seg + lane * 32), w23 = lds128(seg + lane * 32 + 16);
        const uint2 dd = lds64(seg + kSegSclOffQ8 + g * 8);
        const float2 d01 = __half22float2(*reinterpret_cast<const __half2*>(&dd.x));
        const float2 d23 = __half22float2(*reinterpret_cast<const __half2*>(&dd.y));
        const uint32_t wa[4] = {w01.x, w01.z, w23.x, w23.z};   // codes 4c..4c+3 of rows g + 8i
        const uint32_t wb[4] = {w01.y, w01.w, w23.y, w23.w};   // codes 16+4c..
        const float dr[4] = {d01.x, d01.y, d23.x, d23.y};
#pragma unroll
        for (int m = 0; m < M; ++m) {
            const uint4 xq = lds128(xb + (uint32_t)m * xstride);
            const float sbm = __uint_as_float(lds64(rb + (uint32_t)m * rstride).y);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                int t = dp2a_lo_s8(xq.x, wa[i], 0);
                t = dp2a_hi_s8(xq.y, wa[i], t);
                t = dp2a_lo_s8(xq.z, wb[i], t);
                t = dp2a_hi_s8(xq.w, wb[i], t);
                acc[m][i] = fmaf((float)t, __fmul_rn(dr[i], sbm), acc[m][i]);
            }
        }
    }

    // Next segment of the run (flushing a finished tile first).
    __device__ __forceinline__ void step(const GemvArgs& a, uint32_t seg) {
        if (b == KB) {
            flush(a, t_cur);
            ++t_cur;
            b = 0;
            xp = x_lane0;
            rp = r_lane0;
        }
        segment(seg, xp, rp);
        ++b;
        xp += 64;
        rp += 32;
    }

    // A whole ring stage of C segments.  When no tile ends inside it the
    // segments are addressed with constant offsets and no per-segment checks.
    template <int C>
    __device__ __forceinline__ void stage_full(const GemvArgs& a, uint32_t st) {
        if (b + C <= KB) {
#pragma unroll
            for (int j = 0; j < C; ++j)
                segment(st + j * SEG, xp + j * 64, rp + j * 32);
            b += C;
            xp += C * 64;
            rp += C * 32;
        } else {
#pragma unroll
            for (int j = 0; j < C; ++j) step(a, st + j * SEG);
        }
    }

    // End of the run: the last tile.
    __device__ __forceinline__ void flush_last(const GemvArgs& a) {
        if (sp.s1 > sp.s0) flush(a, t_cur);
    }

    // First level of the split-tile combine, after a CTA-wide barrier that
    // follows every warp's flush_last.  Of each tile split between warps, the
    // CTA's first contributing warp sums the parked partials of the CTA's
    // contributors in warp order (lane = row).  A tile inside the CTA is then
    // finished (y written); for a tile shared with other CTAs the CTA's
    // partial goes to ws[cta][slot], slot 0 if the CTA's run starts in the
    // tile, else 1, and the tile is returned in xt[] (at most two, -1: none)
    // with its contributing CTAs [xcf, xcl].  Lane 4g + c handles row g + 8c.
    template <int WARPS>
    __device__ __forceinline__ void combine_cta(const GemvArgs& a, const float* park_base, float* ws,
                                                int xt[2], int xcf[2], int xcl[2]) {
        xt[0] = xt[1] = -1;
        if (sp.s1 <= sp.s0) return;
        const int cta_lo = blockIdx.x * WARPS, cta_hi = cta_lo + WARPS - 1;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int t = e == 0 ? sp.t_first : sp.t_last;
            const int gf = e == 0 ? sp.gf0 : sp.gf1, gl = e == 0 ? sp.gl0 : sp.gl1;
            if (!cta_combiner(sp, e, gw, cta_lo)) continue;
            const int w_to = min(gl, cta_hi);
            float sum[M];
#pragma unroll
            for (int m = 0; m < M; ++m) sum[m] = 0.f;
            for (int w = gw; w <= w_to; ++w) {
                const int sl = park_slot_read(sp, gw, w, t);
                const float* p = park_base + ((size_t)(w - cta_lo) * 2 + sl) * M * 32;
#pragma unroll
                for (int m = 0; m < M; ++m) sum[m] += p[m * 32 + r];
            }
            if (gf >= cta_lo && gl <= cta_hi) {
                const int64_t row = (int64_t)t * 32 + r;
#pragma unroll
                for (int m = 0; m < M; ++m) {
                    const __half yh = __float2half_rn(__fmul_rn(oscale, sum[m]));
                    if (row < a.N) store_out(a, m, row, yh);
                    if (M == 1 && t < qo.nb) quant_lane_store(__half2float(yh), t, qo.x, qo.rec, qo.sq);
                }
            } else {
                const int slc = cta_slot_write(blockIdx.x, t, KB, a.sc, WARPS);
#pragma unroll
                for (int m = 0; m < M; ++m)
                    ws[(((size_t)blockIdx.x * 2 + slc) * M + m) * 32 + r] = sum[m];
                xt[e] = t;
                xcf[e] = gf / WARPS;
                xcl[e] = gl / WARPS;
            }
        }
    }
};

// Second level, q4gemv_run's kernel: CTAs that left a partial of tile t count
// their arrival; the last to arrive sums the CTA partials in CTA order,
// writes y and re-arms the counter.  One warp, lane = row.
template <int M, int WARPS>
__device__ __forceinline__ void combine_ctas_arrive(const GemvArgs& a, int t, int cf, int cl,
                                                    float oscale) {
    const int lane = threadIdx.x & 31;
    __syncwarp();
    int old = 0;
    if (lane == 0) old = atom_add_acq_rel_gpu(a.cnt + t, 1);
    old = __shfl_sync(0xffffffffu, old, 0);
    __syncwarp();                       // order the lanes' reads after lane 0's acquire
    const int need = cl - cf + 1;
    // With peers the counts run on (nothing resets them): this arrival
    // follows a.peer.rounds earlier rounds.
    if (a.peer.n > 0) old = (int)((unsigned)old - (unsigned)need * a.peer.rounds);
    if (old == need - 1) {
        float sum[M];
#pragma unroll
        for (int m = 0; m < M; ++m) sum[m] = 0.f;
        // Eight contributors per round: their loads are issued together, the
        // sum is still taken in CTA order.
        for (int c0 = cf; c0 <= cl; c0 += 8) {
            float pv[8][M];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int c = c0 + u;
                const int sl = cta_slot_read(c, cf, t, a.KB, a.sc, WARPS);
#pragma unroll
                for (int m = 0; m < M; ++m)
                    pv[u][m] = c <= cl ? ld_relaxed_gpu(a.ws + (((size_t)c * 2 + sl) * M + m) * 32 + lane)
                                       : 0.f;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (c0 + u <= cl)
#pragma unroll
                    for (int m = 0; m < M; ++m) sum[m] += pv[u][m];
        }
        const int64_t row = (int64_t)t * 32 + lane;
#pragma unroll
        for (int m = 0; m < M; ++m)
            if (row < a.N) store_out(a, m, row, __float2half_rn(__fmul_rn(oscale, sum[m])));
        if (lane == 0 && a.peer.n == 0) a.cnt[t] = 0;
    } else if (old >= need || old < 0) {
        if (lane == 0) set_device_error(a.err, kDevConcurrent);
    }
}

template <int M, int WARPS, int R, int C, bool Q8 = false>
__global__ void __launch_bounds__(WARPS * 32, 1) gemv_dp2a_kernel(const GemvArgs a_in) {
    GemvArgs a = a_in;
    if (a.peer.n > 0) peer_prepare(a.peer);
    constexpr int SEG = SegFmt<Q8>::kBytes;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t bars[WARPS * R];

    const uint32_t smem_base = smem_addr(smem);
    const uint32_t xs = smem_base + (uint32_t)ring_bytes(WARPS, R, C, SEG);   // int16 X, lane order
    const uint32_t rec = xs + (uint32_t)(M * a.K * 2);                  // {-8 sum X, scale}
    float* park = reinterpret_cast<float*>(smem + ring_bytes(WARPS, R, C, SEG) + (size_t)M * a.K * 2 +
                                           (size_t)M * a.KB * 32);      // [WARPS][2][M][32]
    float* sq = park + WARPS * 2 * M * 32;                              // block sums of squares

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gw = blockIdx.x * WARPS + warp;
    // G <= S, so every warp below G owns at least one segment; warps of the
    // last CTA beyond G only help stage the activations.
    Dp2aConsumer<M, Q8> cons;
    WarpRing<R, C, SEG> ring;
    {
        WarpSplit sp;
        sp.init(gw, a.sc, a.KB);
        ring.init(smem_base, bars, warp, a.W, sp.s0, sp.s1);
    }
    if (lane == 0) {
        for (int k = 0; k < R; ++k) mbar_init(bars + warp * R + k, 1);
        fence_barrier_init();
    }
    __syncwarp();
    // Weights do not depend on the previous kernel: start the stream before
    // the dependency wait.
    if (lane == 0)
        for (int ch = 0; ch < R && ch < ring.nch; ++ch) ring.issue(ch);
    cons.init(a, gw, xs, rec, park + (size_t)warp * 2 * M * 32);
    pdl_launch_dependents();
    // With peers a waiting GEMV's input is the stamped words, its arrival
    // counts and split workspace are its own: it runs beside the previous
    // kernel's tail instead of after it.
    if (a.peer.n == 0 || !a.peer.wait) pdl_wait();

    {
        constexpr int NT = WARPS * 32;
        const int nq = M * a.K / 8;
        if (nq <= 2 * NT) stage_activations<M, NT, 2>(a, xs, rec, sq);
        else if (nq <= 5 * NT) stage_activations<M, NT, 5>(a, xs, rec, sq);
        else stage_activations<M, NT, kXChunksPerThread>(a, xs, rec, sq);
    }
    // A renormalised input (M = 1) is the loaded vector times its unit-RMS
    // scale, applied to the outputs.
    if (M == 1 && a.renorm) cons.oscale = unit_rms_scale(sq, a.KB, a.K);

    for (int ch = 0; ch < ring.nch; ++ch) {
        if (!ring.wait(ch)) set_device_error(a.err, kDevTimeout);   // data then unreliable
        const uint32_t st = ring.stage(ch % R);
        const int n = min(C, ring.nseg - ch * C);
        if (n == C) {
            cons.template stage_full<C>(a, st);
        } else {
            for (int j = 0; j < n; ++j) cons.step(a, st + j * SEG);
        }
        // Stage fully read: hand it back to the async proxy for the refill.
        __syncwarp();
        fence_proxy_async_smem();
        if (lane == 0 && ch + R < ring.nch) ring.issue(ch + R);
    }
    cons.flush_last(a);
    __syncthreads();
    int xt[2], xcf[2], xcl[2];
    cons.template combine_cta<WARPS>(a, park, a.ws, xt, xcf, xcl);
    if (xt[0] >= 0) combine_ctas_arrive<M, WARPS>(a, xt[0], xcf[0], xcl[0], cons.oscale);
    if (xt[1] >= 0) combine_ctas_arrive<M, WARPS>(a, xt[1], xcf[1], xcl[1], cons.oscale);
}

// Unit-RMS renorm of in[0:len) into out: out_i = f16(s * in_i), s from the
// block sums of squares in the fixed tree and order above (the same s the
// GEMVs apply), all NT threads of one CTA.  Fix completes chunks that exist
// only as partial sums (the persistent step); sq: scratch for len/32 floats.
template <int NT, int QN, bool kCoherent, class Fix>
__device__ __forceinline__ void renorm_block(const __half* in, __half* out, int len, float* sq,
                                             const Fix& fix, uint32_t patch) {
    const int tid = threadIdx.x;
    const int nq = len / 8;
    uint4 xr[QN];
#pragma unroll
    for (int i = 0; i < QN; ++i) {
        const int q = tid + NT * i;
        const uint4* src = reinterpret_cast<const uint4*>(in + (size_t)q * 8);
        xr[i] = q < nq ? (kCoherent ? __ldcg(src) : *src) : make_uint4(0, 0, 0, 0);
    }
    if constexpr (Fix::kActive) {
        fix.template prepare<NT>(nq, patch);
        __syncthreads();
#pragma unroll
        for (int i = 0; i < QN; ++i) {
            const int q = tid + NT * i;
            if (q < nq) xr[i] = fix.apply(q, xr[i], patch);
        }
    }
#pragma unroll
    for (int i = 0; i < QN; ++i) {
        const int q = tid + NT * i;
        const __half2* h = reinterpret_cast<const __half2*>(&xr[i]);
        float v[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(h[e]);
            v[2 * e] = f.x;
            v[2 * e + 1] = f.y;
        }
        const ChunkQ o = quant_chunk(v);     // only the sum of squares is used
        if (q < nq && (q & 3) == 0) sq[q >> 2] = o.sq;
    }
    __syncthreads();
    const float scale = unit_rms_scale(sq, len / 32, len);
#pragma unroll
    for (int i = 0; i < QN; ++i) {
        const int q = tid + NT * i;
        __half2* h = reinterpret_cast<__half2*>(&xr[i]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(h[e]);
            h[e] = __floats2half2_rn(__fmul_rn(scale, f.x), __fmul_rn(scale, f.y));
        }
        if (q < nq) *reinterpret_cast<uint4*>(out + (size_t)q * 8) = xr[i];
    }
}

struct NoFix {
    static constexpr bool kActive = false;
    template <int NT>
    __device__ __forceinline__ void prepare(int, uint32_t) const {}
    __device__ __forceinline__ uint4 apply(int, uint4 v, uint32_t) const { return v; }
};

// Final renorm of the decode step: out = f16(s * in[0:len)).
template <int WARPS>
__global__ void __launch_bounds__(WARPS * 32, 1) renorm_kernel(const __half* in, __half* out, int len) {
    __shared__ float sq[(kXChunksPerThread * 8 * WARPS * 32) / 32];
    pdl_wait();
    renorm_block<WARPS * 32, kXChunksPerThread, false>(in, out, len, sq, NoFix(), 0u);
}

// Final renorm of the peer-exchange step: waits for the last GEMV's stamped
// words (every rank's rows), unpacks them into out, then out = f16(s * out)
// in place (each thread reads back the chunks it wrote).
template <int WARPS>
__global__ void __launch_bounds__(WARPS * 32, 1) peer_renorm_kernel(const uint32_t* words, __half* out,
                                                                  int len, PeerArgs pa, int* err) {
    __shared__ float sq[(kXChunksPerThread * 8 * WARPS * 32) / 32];
    constexpr int NT = WARPS * 32;
    const uint32_t stamp = (peer_stamp(pa.seq, pa.per_step, pa.g - 1) + pa.unreachable) & 0xFFFFu;
    uint4 xr[kXChunksPerThread];
    peer_load_chunks<kXChunksPerThread>(words, len / 8, threadIdx.x, NT, stamp, pa.poll_limit, err, xr);
#pragma unroll
    for (int i = 0; i < kXChunksPerThread; ++i) {
        const int q = threadIdx.x + NT * i;
        if (q < len / 8) *reinterpret_cast<uint4*>(out + (size_t)q * 8) = xr[i];
    }
    __syncthreads();
    renorm_block<NT, kXChunksPerThread, false>(out, out, len, sq, NoFix(), 0u);
}

// GGUF Q8_0 -> packed layout, one warp per segment (grid-stride): lane
// (g, c) writes the 32 code bytes of its four rows and lane group 0 the
// scales.
static __global__ void __launch_bounds__(256) repack_q8_kernel(const uint8_t* __restrict__ gguf,
                                                          uint8_t* __restrict__ packed, int64_t N,
                                                          int KB, int64_t S) {
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t s = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); s < S; s += nwarps) {
        const int64_t t = s / KB, b = s - t * KB;
        uint32_t words[8];
        uint16_t dv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t row = t * 32 + g + 8 * i;
            if (row < N) {
                const uint8_t* blk = gguf + (row * KB + b) * 34;
                // codes start at byte 2 of the block: 2-byte aligned only
                const uint16_t* h = reinterpret_cast<const uint16_t*>(blk);
                words[2 * i] = (uint32_t)h[1 + 2 * c] | ((uint32_t)h[2 + 2 * c] << 16);
                words[2 * i + 1] = (uint32_t)h[9 + 2 * c] | ((uint32_t)h[10 + 2 * c] << 16);
                dv[i] = h[0];
            } else {
                words[2 * i] = words[2 * i + 1] = 0u;
                dv[i] = 0;
            }
        }
        uint8_t* seg = packed + s * kSegBytesQ8;
        *reinterpret_cast<uint4*>(seg + lane * 32) = make_uint4(words[0], words[1], words[2], words[3]);
        *reinterpret_cast<uint4*>(seg + lane * 32 + 16) = make_uint4(words[4], words[5], words[6], words[7]);
        if (c == 0) {
            *reinterpret_cast<uint2*>(seg + kSegSclOffQ8 + g * 8) =
                make_uint2((uint32_t)dv[0] | ((uint32_t)dv[1] << 16),
                           (uint32_t)dv[2] | ((uint32_t)dv[3] << 16));
        }
    }
}

// GGUF Q4_0 -> packed layout, one warp per segment (grid-stride).
static __global__ void __launch_bounds__(256) repack_kernel(const uint8_t* __restrict__ gguf,
                                                     uint8_t* __restrict__ packed, int64_t N,
                                                     int KB, int64_t S) {
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t s = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); s < S; s += nwarps) {
        const int64_t t = s / KB, b = s - t * KB;
        uint32_t words[4];
        uint16_t dv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t row = t * 32 + g + 8 * i;
            if (row < N) {
                const uint16_t* blk = reinterpret_cast<const uint16_t*>(gguf + (row * KB + b) * 18);
                words[i] = (uint32_t)blk[1 + 2 * c] | ((uint32_t)blk[2 + 2 * c] << 16);
                dv[i] = blk[0];
            } else {
                words[i] = 0x88888888u;
                dv[i] = 0;
            }
        }
        uint8_t* seg = packed + s * kSegBytes;
        *reinterpret_cast<uint4*>(seg + lane * 16) = make_uint4(words[0], words[1], words[2], words[3]);
        if (c == 0) {
            *reinterpret_cast<uint2*>(seg + kSegSclOff + g * 8) =
                make_uint2((uint32_t)dv[0] | ((uint32_t)dv[1] << 16),
                           (uint32_t)dv[2] | ((uint32_t)dv[3] << 16));
        }
    }
}

}  // namespace q4
