// Flat, balanced split of the S segments of a packed matrix over G warps,
// and the bookkeeping of tiles that straddle two or more warps.
//
// Warp g owns segments [seg_begin(g), seg_begin(g + 1)), seg_begin(g) =
// floor(g*S/G); with G <= S every warp owns at least one.  A tile (KB
// consecutive segments) is either owned whole by one warp or split; a split
// tile's contributors are the consecutive warps warp_of_seg(t*KB) ..
// warp_of_seg(t*KB + KB - 1), each of which parks one partial (slot 0 when
// the tile is where its run starts, else slot 1) and the last to arrive sums
// them in warp order.
//
// All arithmetic is 32-bit: with S = Q*G + Rm, floor(g*S/G) = g*Q +
// floor(g*Rm/G) and g*Rm < G^2 < 2^32 for G < 65536.
#pragma once

#include <cstdint>

namespace q4 {

constexpr int kMaxSplitWarps = 65535;

__host__ __device__ __forceinline__ int seg_begin(int g, int S, int G) {
    const uint32_t Q = (uint32_t)S / (uint32_t)G, Rm = (uint32_t)S - Q * (uint32_t)G;
    return (int)((uint32_t)g * Q + ((uint32_t)g * Rm) / (uint32_t)G);
}

// Largest g < G with seg_begin(g) <= s, for 0 <= s < S: a single-precision
// estimate of floor((s+1)*G/S) corrected against seg_begin.
__host__ __device__ __forceinline__ int warp_of_seg(int s, int S, int G) {
    int g = (int)((float)(s + 1) * ((float)G / (float)S));
    if (g > G - 1) g = G - 1;
    if (g < 0) g = 0;
    while (g > 0 && seg_begin(g, S, G) > s) --g;
    while (g + 1 < G && seg_begin(g + 1, S, G) <= s) ++g;
    return g;
}

// Per-warp view of the split, computed once at kernel start.
struct WarpSplit {
    int s0, s1;             // owned segments
    int t_first, t_last;    // first and last tile touched (t_last < t_first if none)
    int gf0, gl0, gf1, gl1; // contributors of t_first and t_last

    __host__ __device__ __forceinline__ void init(int gw, int S, int G, int KB) {
        s0 = gw < G ? seg_begin(gw, S, G) : S;
        s1 = gw < G ? seg_begin(gw + 1, S, G) : S;
        t_first = s0 / KB;
        t_last = (s1 > s0) ? (s1 - 1) / KB : t_first - 1;
        if (s1 > s0) {
            gf0 = warp_of_seg(t_first * KB, S, G);
            gl0 = warp_of_seg(t_first * KB + KB - 1, S, G);
            gf1 = warp_of_seg(t_last * KB, S, G);
            gl1 = warp_of_seg(t_last * KB + KB - 1, S, G);
        } else {
            gf0 = gl0 = gf1 = gl1 = 0;
        }
    }
    // Tiles strictly inside the run are always owned whole.
    __host__ __device__ __forceinline__ bool whole(int t) const {
        if (t == t_first) return gf0 == gl0;
        if (t == t_last) return gf1 == gl1;
        return true;
    }
    __host__ __device__ __forceinline__ int slot(int t) const { return t == t_first ? 0 : 1; }
};

// Walks seg_begin(g) for g = g_start, g_start + 1, ... with additions only.
struct SegWalker {
    int sb, r, Q, Rm, G;
    __host__ __device__ __forceinline__ void init(int g_start, int S, int G_) {
        G = G_;
        Q = S / G;
        Rm = S - Q * G;
        sb = seg_begin(g_start, S, G);
        r = (int)(((uint32_t)g_start * (uint32_t)Rm) % (uint32_t)G);
    }
    __host__ __device__ __forceinline__ void next() {
        sb += Q;
        r += Rm;
        if (r >= G) {
            r -= G;
            ++sb;
        }
    }
};

}  // namespace q4
