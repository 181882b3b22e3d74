// Q4_0 GEMV for M = 3..16 activation vectors (speculative verify, prefill
// chunks): each dequantised weight tile is applied to all M vectors with
// tensor-core mma.sync.m16n8k16 (f16 inputs, f32 accumulate).
//
// Speculative verification runs a batch of draft tokens through the trunk in
// one pass and prefill batches 16 tokens per round trip (aipolix en-US page,
// section "Speculation is used to amortize network round trips";
// originshq.com page, section "Multi-Device Performance and the Network
// Penalty"); the weight stream is the same as decode, the arithmetic grows
// with M.  With M >= 4 the CUDA-core dp2a path needs more issue slots per
// weight than the HBM rate allows on B200, so the block products move to the
// tensor cores while the rest of the design is shared with the M <= 2 kernel
// (segment-tiled layout, per-warp TMA ring, flat warp split, deterministic
// split-tile combine).
//
// Per segment (32 rows x one 32-column block) and lane (g, c): the four
// 32-bit code words of rows g, g+8, g+16, g+24 give, with one shift and four
// masks, exact (q - 8) as f16 pairs (magic exponent 2^10 in the mantissa,
// then one subtract or fused multiply-add); they are the A fragments of two
// 16-row MMA tiles in the fragment order of m16n8k16 after a fixed
// permutation of k inside the block, matched by the order in which the
// activations are staged in shared memory.  Two MMAs (low and high nibbles)
// give the exact block dot products in fp32; the per-row scale d is applied
// with one FFMA per output, so no rounding of d * (q - 8) is ever made.
#pragma once

#include "gemv_dp2a.cuh"

namespace q4 {

// The launch is a grid of P column panels (blockIdx.y) × CTAs (blockIdx.x).
// Panel p covers blocks [p0, p0 + KBv) of every row (p0 = p * KBv; the last
// panel takes what is left); its segments are numbered in panel order,
// v = t * KBv + j for block p0 + j of tile t, and split flat over the panel's
// warps.  With one panel the outputs are written as f16; with several, each
// panel writes its fp32 sums to ypart[p] and panel_reduce_kernel adds them in
// panel order.  Narrow panels let a CTA stage a short activation slice for
// many rows, and make matrices wider than one CTA's staging possible.
struct MmaArgs {
    const uint8_t* W;    // packed matrix (segments of 576 bytes)
    const __half* x;     // [M][K]
    __half* y;           // [M][N]
    float* ws;           // per panel: [G][2][16][32] warp partials, [CTAs][2][16][32] CTA partials
    int* cnt;            // per panel: [T] arrival counters, zero between calls
    int* err;
    float* ypart;        // [P][M][N] fp32 panel sums (P > 1)
    int64_t N;
    int K, KB, T, S, G;  // S = T * KBv; G: the panel's warps that own segments
    int KBv, p0;         // panel: blocks per tile, first block
    int M;               // 1..16 (columns >= M are zero-padded)
    SplitConsts sc;      // make_split(S, G)
    int P;               // panels
    int S_last, G_last;  // the last panel's segments, warps and split
    SplitConsts sc_last;
    int64_t ws_panel;    // floats of ws per panel
};

// This CTA's view of the launch: its panel's geometry, split and slices of
// the scratch.
__device__ __forceinline__ MmaArgs panel_view(const MmaArgs& in) {
    MmaArgs a = in;
    const int p = blockIdx.y;
    if (in.P > 1) {
        const bool last = p == in.P - 1;
        a.p0 = p * in.KBv;
        if (last) {
            a.KBv = in.KB - a.p0;
            a.S = in.S_last;
            a.G = in.G_last;
            a.sc = in.sc_last;
        }
        a.ws = in.ws + (size_t)p * in.ws_panel;
        a.cnt = in.cnt + (size_t)p * in.T;
        a.ypart = in.ypart + (size_t)p * in.M * in.N;
    }
    return a;
}

// y = f16(sum of the panels' fp32 sums, in panel order).
static __global__ void __launch_bounds__(256) panel_reduce_kernel(const float* __restrict__ part,
                                                                __half* __restrict__ y, int P,
                                                                int64_t MN) {
    pdl_wait();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < MN; i += stride) {
        float sum = 0.f;
        for (int p = 0; p < P; ++p) sum += part[(size_t)p * MN + i];
        y[i] = __float2half_rn(sum);
    }
}

// A warp's ring over a panel: stage k holds C consecutive panel segments of
// the warp's run [s0, s1), filled by one bulk copy per contiguous piece (a
// stage that crosses a tile boundary of a narrower panel takes two or more).
template <int R, int C, int SEG = kSegBytes>
struct PanelRing {
    uint32_t stage0;
    uint64_t* bars;
    const uint8_t* W;
    int s0, nseg, nch, KBv, KB, p0;
    int it, ij;           // issue cursor: tile and block (in the panel) of the next chunk

    __device__ void init(uint32_t ring_base, uint64_t* bar_base, int warp, const MmaArgs& a, int s0_,
                         int s1_) {
        stage0 = ring_base + (uint32_t)warp * R * C * SEG;
        bars = bar_base + warp * R;
        W = a.W;
        s0 = s0_;
        nseg = s1_ - s0_;
        nch = (nseg + C - 1) / C;
        KBv = a.KBv;
        KB = a.KB;
        p0 = a.p0;
        it = s0_ / KBv;
        ij = s0_ - it * KBv;
    }
    __device__ uint32_t stage(int k) const { return stage0 + (uint32_t)k * C * SEG; }
    // Lane 0 only, chunks in order.
    __device__ void issue(int ch) {
        const int k = ch % R;
        int n = min(C, nseg - ch * C);
        mbar_arrive_expect_tx(bars + k, (uint32_t)n * SEG);
        uint32_t dst = stage(k);
        while (n > 0) {
            const int len = min(n, KBv - ij);
            bulk_g2s_addr(dst, W + ((size_t)it * KB + p0 + ij) * SEG, (uint32_t)len * SEG, bars + k);
            dst += (uint32_t)len * SEG;
            n -= len;
            ij += len;
            if (ij == KBv) {
                ij = 0;
                ++it;
            }
        }
    }
    __device__ bool wait(int ch) const {
        return mbar_wait_bounded(bars + (ch % R), (uint32_t)((ch / R) & 1), 1u << 22);
    }
};

// Bytes per staged activation vector for `nblk` blocks: 64 per block, padded
// so consecutive vectors start 64 bytes apart modulo 128 (conflict-free
// 16-byte loads by the eight lane groups).
__host__ __device__ constexpr int mma_vstride(int nblk) {
    return nblk * 64 + ((nblk & 1) ? 0 : 64);
}
// Only the M real vectors are staged: MMA columns past M read vector M - 1
// (their outputs are never used).
__host__ __device__ constexpr size_t gemv_mma_smem_bytes(int M, int nblk) {
    return (size_t)M * mma_vstride(nblk);
}

// Position of element e of a 32-column block in the staged order: lane group
// c reads [x4c, x4c+2, x4c+1, x4c+3 | x4c+16, x4c+18, x4c+17, x4c+19].
__host__ __device__ __forceinline__ int mma_xpos(int e) {
    const int r = e & 3;
    return ((e & 15) >> 2) * 8 + (e >> 4) * 4 + (((r & 1) << 1) | (r >> 1));
}

__device__ __forceinline__ void mma_16816(float& d0, float& d1, float& d2, float& d3, uint32_t a0,
                                          uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                          uint32_t b1, float c0, float c1, float c2, float c3) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%11,%12,%13};"
        : "=f"(d0), "=f"(d1), "=f"(d2), "=f"(d3)
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c0), "f"(c1), "f"(c2),
          "f"(c3));
}

// Exact (q - 8) f16 pairs from one code word: lo/hi nibbles of bytes (0, 2)
// and (1, 3).
struct CodePairs {
    uint32_t p, q, r, s;   // p: k(4c, 4c+2)  q: k(4c+1, 4c+3)  r: k(4c+16, 4c+18)  s: k(4c+17, 4c+19)
};
__device__ __forceinline__ CodePairs unpack_pairs(uint32_t w) {
    // Codes into the mantissa of f16 1024 (0x6400): 1024 + q (low nibbles)
    // or 1024 + 16q (high nibbles); then - 1032, or * 1/16 - 72: exact q - 8.
    CodePairs o;
    asm("{\n\t.reg .b32 w8, t0, t1, t2, t3;\n\t"
        "shr.b32 w8, %4, 8;\n\t"
        "lop3.b32 t0, %4, 0x000F000F, 0x64006400, 0xEA;\n\t"
        "lop3.b32 t1, w8, 0x000F000F, 0x64006400, 0xEA;\n\t"
        "lop3.b32 t2, %4, 0x00F000F0, 0x64006400, 0xEA;\n\t"
        "lop3.b32 t3, w8, 0x00F000F0, 0x64006400, 0xEA;\n\t"
        "sub.rn.f16x2 %0, t0, %5;\n\t"
        "sub.rn.f16x2 %1, t1, %5;\n\t"
        "fma.rn.f16x2 %2, t2, %6, %7;\n\t"
        "fma.rn.f16x2 %3, t3, %6, %7;\n\t}"
        : "=r"(o.p), "=r"(o.q), "=r"(o.r), "=r"(o.s)
        : "r"(w), "r"(0x64086408u), "r"(0x2C002C00u), "r"(0xD480D480u));
    return o;
}

// Exact f16 pairs from two Q8_0 code words (signed bytes; lo: codes 4c..4c+3,
// hi: codes 16+4c..): a byte with its sign bit flipped, placed in the
// mantissa of f16 1024, is 1024 + q + 128; minus 1152 it is exactly q.  The
// same k order as unpack_pairs.
__device__ __forceinline__ CodePairs unpack_pairs_q8(uint32_t lo, uint32_t hi) {
    CodePairs o;
    asm("{\n\t.reg .b32 xl, xh, t0, t1, t2, t3;\n\t"
        "xor.b32 xl, %4, 0x80808080;\n\t"
        "xor.b32 xh, %5, 0x80808080;\n\t"
        "prmt.b32 t0, xl, 0x64646464, 0x4240;\n\t"
        "prmt.b32 t1, xl, 0x64646464, 0x4341;\n\t"
        "prmt.b32 t2, xh, 0x64646464, 0x4240;\n\t"
        "prmt.b32 t3, xh, 0x64646464, 0x4341;\n\t"
        "sub.rn.f16x2 %0, t0, %6;\n\t"
        "sub.rn.f16x2 %1, t1, %6;\n\t"
        "sub.rn.f16x2 %2, t2, %6;\n\t"
        "sub.rn.f16x2 %3, t3, %6;\n\t}"
        : "=r"(o.p), "=r"(o.q), "=r"(o.r), "=r"(o.s)
        : "r"(lo), "r"(hi), "r"(0x64806480u));
    return o;
}

template <int NT8, int WARPS, int R, int C, bool Q8 = false>
__global__ void __launch_bounds__(WARPS * 32, 1) gemv_mma_kernel(const MmaArgs a_in) {
    constexpr int SEG = SegFmt<Q8>::kBytes;
    const MmaArgs a = panel_view(a_in);
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t bars[WARPS * R];
    constexpr int NT = WARPS * 32;
    const uint32_t smem_base = smem_addr(smem);
    const uint32_t xsm = smem_base + (uint32_t)ring_bytes(WARPS, R, C, SEG);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int gw = blockIdx.x * WARPS + warp;
    WarpSplit sp;
    sp.init(gw, a.sc, a.KBv);
    const int s0 = sp.s0, s1 = sp.s1;
    const int KB = a.KBv;                       // blocks per tile of this panel

    // The CTA's blocks: its warps own one contiguous run of segments.
    const int w_lo = blockIdx.x * WARPS;
    const int w_hi = min(w_lo + WARPS, a.G);
    const int cs0 = w_lo < a.G ? seg_begin(w_lo, a.sc) : a.S;
    const int cs1 = w_hi > w_lo ? (w_hi < a.G ? seg_begin(w_hi, a.sc) : a.S) : cs0;
    const int nblk = (cs1 - cs0 >= KB) ? KB : (cs1 - cs0);
    const int b0 = (cs1 - cs0 >= KB) ? 0 : (cs0 % KB);
    const int vstride = mma_vstride(nblk);

    PanelRing<R, C, SEG> ring;
    ring.init(smem_base, bars, warp, a, s0, s1);
    if (lane == 0) {
        for (int k = 0; k < R; ++k) mbar_init(bars + warp * R + k, 1);
        fence_barrier_init();
    }
    __syncwarp();
    if (lane == 0)
        for (int ch = 0; ch < R && ch < ring.nch; ++ch) ring.issue(ch);
    pdl_launch_dependents();
    pdl_wait();

    // Stage the CTA's activation blocks with plain 16-byte loads (eight per
    // round per thread), reordered into lane order (the M real vectors only).
    {
        const int nchunk = a.M * nblk * 4;
        for (int p0 = threadIdx.x; p0 < nchunk; p0 += 8 * NT) {
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int p = p0 + u * NT;
                if (p < nchunk) {
                    const int vv = p / (nblk * 4), rem = p - vv * nblk * 4;
                    int b = b0 + (rem >> 2);
                    if (b >= KB) b -= KB;
                    v[u] = *reinterpret_cast<const uint4*>(a.x + (size_t)vv * a.K + (a.p0 + b) * 32 +
                                                           (rem & 3) * 8);
                }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int p = p0 + u * NT;
                if (p < nchunk) {
                    const int vv = p / (nblk * 4), rem = p - vv * nblk * 4;
                    const int jb = rem >> 2, qt = rem & 3;
                    const int pos0 = (qt & 1) * 16 + (qt >> 1) * 4;
                    const uint32_t dst = xsm + (uint32_t)vv * vstride + (uint32_t)jb * 64 + pos0 * 2;
                    sts64(dst, make_uint2(__byte_perm(v[u].x, v[u].y, 0x5410),
                                          __byte_perm(v[u].x, v[u].y, 0x7632)));
                    sts64(dst + 16, make_uint2(__byte_perm(v[u].z, v[u].w, 0x5410),
                                               __byte_perm(v[u].z, v[u].w, 0x7632)));
                }
            }
        }
        __syncthreads();
    }

    float acc[2][NT8][4];
#pragma unroll
    for (int tt = 0; tt < 2; ++tt)
#pragma unroll
        for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[tt][nt][i] = 0.f;

    const int t_first = sp.t_first;
    int t_cur = t_first;

    // A finished output (all blocks of this panel summed).
    auto emit = [&](int col, int64_t row, float v) {
        const size_t o = (size_t)col * a.N + row;
        if (a.P == 1) a.y[o] = __float2half_rn(v);
        else a.ypart[o] = v;
    };

    // Output (row, column) held by acc[tt][nt][i]:
    //   row = 16*tt + g + 8*(i >> 1), column = 8*nt + 2c + (i & 1).
    auto flush = [&](int t) {
        const bool whole = sp.whole(t);
        const int slot = sp.slot(t);
#pragma unroll
        for (int tt = 0; tt < 2; ++tt)
#pragma unroll
            for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int r = 16 * tt + g + 8 * (i >> 1);
                    const int col = 8 * nt + 2 * c + (i & 1);
                    const int64_t row = (int64_t)t * 32 + r;
                    if (whole) {
                        if (col < a.M && row < a.N) emit(col, row, acc[tt][nt][i]);
                    } else {
                        a.ws[(((size_t)gw * 2 + slot) * 16 + col) * 32 + r] = acc[tt][nt][i];
                    }
                    acc[tt][nt][i] = 0.f;
                }
    };

    int b = s0 - t_first * KB;                 // block of the next segment
    int jb = b - b0;                           // its staged slot
    if (jb < 0) jb += KB;
    // MMA column 8 nt + g reads vector min(8 nt + g, M - 1).
    uint32_t x_lane[NT8];
#pragma unroll
    for (int nt = 0; nt < NT8; ++nt)
        x_lane[nt] = xsm + (uint32_t)min(8 * nt + g, a.M - 1) * vstride + (uint32_t)c * 16;

    auto segment = [&](uint32_t seg, int jbs) {
        uint4 w, w2;
        if constexpr (Q8) {
            w = lds128(seg + lane * 32);        // rows g (lo, hi words), g+8 (lo, hi)
            w2 = lds128(seg + lane * 32 + 16);  // rows g+16, g+24
        } else {
            w = lds128(seg + lane * 16);        // rows g, g+8, g+16, g+24
            w2 = w;
        }
        const uint2 dd = lds64(seg + SegFmt<Q8>::kScl + g * 8);
        uint4 xv[NT8];
#pragma unroll
        for (int nt = 0; nt < NT8; ++nt)
            xv[nt] = lds128(x_lane[nt] + (uint32_t)jbs * 64);
        const float2 d01 = __half22float2(*reinterpret_cast<const __half2*>(&dd.x));
        const float2 d23 = __half22float2(*reinterpret_cast<const __half2*>(&dd.y));
        const float dA[2] = {d01.x, d23.x};   // rows g, g+16
        const float dB[2] = {d01.y, d23.y};   // rows g+8, g+24
        const uint32_t w0s[2] = {w.x, w.z};
        const uint32_t w1s[2] = {w.y, w.w};
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
            CodePairs u0, u1;
            if constexpr (Q8) {
                u0 = tt == 0 ? unpack_pairs_q8(w.x, w.y) : unpack_pairs_q8(w2.x, w2.y);    // row g (+16)
                u1 = tt == 0 ? unpack_pairs_q8(w.z, w.w) : unpack_pairs_q8(w2.z, w2.w);    // row g+8 (+16)
            } else {
                u0 = unpack_pairs(w0s[tt]);   // row g (+16)
                u1 = unpack_pairs(w1s[tt]);   // row g+8 (+16)
            }
#pragma unroll
            for (int nt = 0; nt < NT8; ++nt) {
                float e0, e1, e2, e3;
                mma_16816(e0, e1, e2, e3, u0.p, u1.p, u0.q, u1.q, xv[nt].x, xv[nt].y, 0.f, 0.f,
                          0.f, 0.f);
                mma_16816(e0, e1, e2, e3, u0.r, u1.r, u0.s, u1.s, xv[nt].z, xv[nt].w, e0, e1, e2,
                          e3);
                const float2 r01 = ffma2(make_float2(e0, e1), make_float2(dA[tt], dA[tt]),
                                         make_float2(acc[tt][nt][0], acc[tt][nt][1]));
                const float2 r23 = ffma2(make_float2(e2, e3), make_float2(dB[tt], dB[tt]),
                                         make_float2(acc[tt][nt][2], acc[tt][nt][3]));
                acc[tt][nt][0] = r01.x;
                acc[tt][nt][1] = r01.y;
                acc[tt][nt][2] = r23.x;
                acc[tt][nt][3] = r23.y;
            }
        }
    };

    for (int ch = 0; ch < ring.nch; ++ch) {
        if (!ring.wait(ch)) set_device_error(a.err, kDevTimeout);   // data then unreliable
        const uint32_t st = ring.stage(ch % R);
        const int n = min(C, ring.nseg - ch * C);
        if (n == C && b + C <= KB && jb + C <= KB) {
            // No tile ends inside this stage: its segments at constant
            // offsets, free to interleave.
#pragma unroll
            for (int j = 0; j < C; ++j) segment(st + j * SEG, jb + j);
            b += C;
            jb += C;
            if (jb == KB) jb = 0;
        } else {
            for (int j = 0; j < n; ++j) {
                if (b == KB) {
                    flush(t_cur);
                    ++t_cur;
                    b = 0;
                    jb = KB - b0;
                    if (jb >= KB) jb -= KB;
                }
                segment(st + j * SEG, jb);
                ++b;
                if (++jb == KB) jb = 0;
            }
        }
        __syncwarp();
        fence_proxy_async_smem();
        if (lane == 0 && ch + R < ring.nch) ring.issue(ch + R);
    }
    if (s1 > s0) flush(t_cur);

    // Split tiles, two levels, each summed in a fixed order.  Level 1: all
    // threads of the CTA sum, per output, the parked partials of the CTA's
    // contributing warps in warp order (loads of many outputs in flight at
    // once); a tile inside the CTA is then finished.  Level 2: a tile shared
    // with other CTAs leaves the CTA's partial (slot 0 if the CTA's run starts
    // in it, else 1) and the last CTA to arrive (per-tile counter) sums the
    // CTA partials in CTA order.
    __shared__ int tl_t[2 * WARPS], tl_gf[2 * WARPS], tl_gl[2 * WARPS], tl_s0[2 * WARPS];
    __shared__ int tl_n, tl_k2[2], tl_old[2];
    if (threadIdx.x == 0) tl_n = 0;
    __syncthreads();
    const int cta_lo = w_lo, cta_hi = w_hi - 1;
    if (s1 > s0 && lane == 0) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            if (!cta_combiner(sp, e, gw, cta_lo)) continue;
            const int k = atomicAdd(&tl_n, 1);
            tl_t[k] = e == 0 ? sp.t_first : sp.t_last;
            tl_gf[k] = e == 0 ? sp.gf0 : sp.gf1;
            tl_gl[k] = e == 0 ? sp.gl0 : sp.gl1;
            tl_s0[k] = park_slot_read(sp, gw, gw, tl_t[k]);   // this (first) warp's slot
        }
    }
    __syncthreads();
    const int ntl = tl_n;
    float* ws_cta = a.ws + (size_t)a.G * 2 * 16 * 32;       // [CTAs][2][16][32]
    const int per_tile = 32 * a.M;
    for (int idx = threadIdx.x; idx < ntl * per_tile; idx += NT) {
        const int k = idx / per_tile, rem = idx - k * per_tile;
        const int col = rem >> 5, r = rem & 31;
        const int t = tl_t[k], gf = tl_gf[k], gl = tl_gl[k];
        const int wf = max(gf, cta_lo), wl = min(gl, cta_hi);
        float sum = 0.f;
        // Eight contributors per round: their loads are issued together, the
        // sum still runs in warp order.
        for (int w0 = wf; w0 <= wl; w0 += 8) {
            float pv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int w = w0 + u;
                const int sl = w == wf ? tl_s0[k] : 0;
                pv[u] = w <= wl ? ld_relaxed_gpu(a.ws + (((size_t)w * 2 + sl) * 16 + col) * 32 + r) : 0.f;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (w0 + u <= wl) sum += pv[u];
        }
        if (gf >= cta_lo && gl <= cta_hi) {
            const int64_t row = (int64_t)t * 32 + r;
            if (row < a.N) emit(col, row, sum);
        } else {
            const int slc = cta_slot_write(blockIdx.x, t, KB, a.sc, WARPS);
            ws_cta[(((size_t)blockIdx.x * 2 + slc) * 16 + col) * 32 + r] = sum;
        }
    }
    __syncthreads();
    // Level 2: the listed tiles this CTA shares with others (at most two: its
    // first tile, j = 0, and its last, j = 1).
    if (threadIdx.x == 0) {
        tl_k2[0] = tl_k2[1] = -1;
        for (int k = 0; k < ntl; ++k) {
            if (tl_gf[k] >= cta_lo && tl_gl[k] <= cta_hi) continue;
            const int j = (tl_gf[k] < cta_lo) ? 0 : 1;
            tl_k2[j] = k;
            tl_old[j] = atom_add_acq_rel_gpu(a.cnt + tl_t[k], 1);
        }
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int k = tl_k2[j];
        if (k < 0) continue;
        const int old = tl_old[j];
        const int t = tl_t[k];
        const int cf = tl_gf[k] / WARPS, cl = tl_gl[k] / WARPS;
        const int need = cl - cf + 1;
        if (old == need - 1) {
            for (int idx = threadIdx.x; idx < per_tile; idx += NT) {
                const int col = idx >> 5, r = idx & 31;
                float sum = 0.f;
                for (int cc = cf; cc <= cl; ++cc) {
                    const int sl = cta_slot_read(cc, cf, t, KB, a.sc, WARPS);
                    sum += ld_relaxed_gpu(ws_cta + (((size_t)cc * 2 + sl) * 16 + col) * 32 + r);
                }
                const int64_t row = (int64_t)t * 32 + r;
                if (row < a.N) emit(col, row, sum);
            }
            if (threadIdx.x == 0) a.cnt[t] = 0;
        } else if (old >= need) {
            if (threadIdx.x == 0) set_device_error(a.err, kDevConcurrent);
        }
    }
}

}  // namespace q4
