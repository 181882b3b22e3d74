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
// The divisions by G and S are done by multiplication with host-computed
// reciprocals (SplitConsts): for n < 2^32 and M = ceil(2^64 / d),
// floor(n * M / 2^64) == floor(n / d) exactly, because the error n*(M/2^64 -
// 1/d) < 2^-32 is smaller than the gap 1/d between n/d and the next integer.
#pragma once

#include <cstdint>

namespace q4 {

constexpr int kMaxSplitWarps = 65535;

struct SplitConsts {
    int S, G;             // segments, warps (1 <= G <= S, G <= kMaxSplitWarps)
    uint32_t Q, Rm;       // S = Q*G + Rm
    uint64_t MG;          // ceil(2^64 / G) (0 when G == 1: then Rm == 0)
    uint64_t MS;          // ceil(2^64 / S) (0 when S == 1)
    int fast;             // S * G < 2^32: warp_of_seg numerators fit 32 bits
};

__host__ __device__ inline uint64_t recip64(uint32_t d) {
    return d <= 1 ? 0 : (~(uint64_t)0) / d + 1;   // ceil(2^64 / d) for d >= 2
}

__host__ __device__ inline SplitConsts make_split(int S, int G) {
    SplitConsts k;
    k.S = S;
    k.G = G;
    k.Q = (uint32_t)S / (uint32_t)G;
    k.Rm = (uint32_t)S - k.Q * (uint32_t)G;
    k.MG = recip64((uint32_t)G);
    k.MS = recip64((uint32_t)S);
    k.fast = ((uint64_t)S * (uint64_t)G < ((uint64_t)1 << 32)) ? 1 : 0;
    return k;
}

__host__ __device__ __forceinline__ uint32_t mulhi64(uint32_t n, uint64_t m) {
#ifdef __CUDA_ARCH__
    return (uint32_t)__umul64hi((uint64_t)n, m);
#else
    return (uint32_t)(((unsigned __int128)n * m) >> 64);
#endif
}

// floor(g * S / G)
__host__ __device__ __forceinline__ int seg_begin(int g, const SplitConsts& k) {
    const uint32_t n = (uint32_t)g * k.Rm;        // < G^2 < 2^32
    const uint32_t f = k.G == 1 ? 0u : mulhi64(n, k.MG);
    return (int)((uint32_t)g * k.Q + f);
}

// Largest g < G with seg_begin(g) <= s (0 <= s < S): floor(((s+1)*G - 1) / S).
__host__ __device__ __forceinline__ int warp_of_seg(int s, const SplitConsts& k) {
    if (k.S == 1) return k.G - 1;
    if (k.fast) return (int)mulhi64((uint32_t)(s + 1) * (uint32_t)k.G - 1u, k.MS);
    return (int)((((uint64_t)s + 1) * (uint64_t)k.G - 1) / (uint64_t)k.S);
}

// Per-warp view of the split, computed once per GEMV.
struct WarpSplit {
    int s0, s1;             // owned segments
    int t_first, t_last;    // first and last tile touched (t_last < t_first if none)
    int gf0, gl0, gf1, gl1; // contributors of t_first and t_last

    __host__ __device__ __forceinline__ void init(int gw, const SplitConsts& k, int KB) {
        s0 = gw < k.G ? seg_begin(gw, k) : k.S;
        s1 = gw < k.G ? seg_begin(gw + 1, k) : k.S;
        t_first = s0 / KB;
        t_last = (s1 > s0) ? (s1 - 1) / KB : t_first - 1;
        if (s1 > s0) {
            gf0 = warp_of_seg(t_first * KB, k);
            gl0 = warp_of_seg(t_first * KB + KB - 1, k);
            gf1 = warp_of_seg(t_last * KB, k);
            gl1 = warp_of_seg(t_last * KB + KB - 1, k);
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

// Two-level combine of split tiles, CTAs of `warps` consecutive warps.
//
// Level 1 (inside a CTA): every warp parks its partial of a split tile in
// its slot sp.slot(t); of each split tile the CTA's first contributing warp
// sums the parked partials of the CTA's contributors.  Warp gw is that warp
// for end e of its run (0: t_first, 1: t_last) when:
__host__ __device__ __forceinline__ bool cta_combiner(const WarpSplit& sp, int e, int gw,
                                                      int cta_lo) {
    if (e == 0) return sp.gf0 != sp.gl0 && (sp.gf0 == gw || gw == cta_lo);
    return sp.t_last != sp.t_first && sp.gf1 != sp.gl1;
}
// ... and the parked slot it reads of contributor w (gw <= w) for tile t:
// only its own run may end in t; every later warp's run starts in t.
__host__ __device__ __forceinline__ int park_slot_read(const WarpSplit& sp, int gw, int w, int t) {
    return (w == gw && t != sp.t_first) ? 1 : 0;
}
// Level 2 (tiles shared by CTAs): CTA c leaves its partial in slot
// cta_slot_write(c) = 0 if its run starts in t, else 1; the reader finds it
// from the tile's first contributing CTA cf alone.
__host__ __device__ __forceinline__ int cta_slot_write(int c, int t, int KB, const SplitConsts& k,
                                                       int warps) {
    return seg_begin(c * warps, k) >= t * KB ? 0 : 1;
}
__host__ __device__ __forceinline__ int cta_slot_read(int c, int cf, int t, int KB,
                                                      const SplitConsts& k, int warps) {
    return (c == cf && seg_begin(c * warps, k) < t * KB) ? 1 : 0;
}

// Tiles shared by CTAs, enumerated by CTA boundary: boundary b (1 <= b <
// CTAs owning segments) names the tile its CTA's run starts in when that run
// starts strictly inside the tile and CTA b-1's run starts at or before the
// tile's start (b is the tile's first interior boundary); else -1.  Every
// tile shared by CTAs is named by exactly one boundary.
__host__ __device__ __forceinline__ int shared_tile_of_boundary(int b, int KB, const SplitConsts& k,
                                                                int warps) {
    const int sb = seg_begin(b * warps, k);
    const int t = sb / KB;
    if (sb == t * KB) return -1;
    if (seg_begin((b - 1) * warps, k) > t * KB) return -1;
    return t;
}

// Walks seg_begin(g) for g = g_start, g_start + 1, ... with additions only.
struct SegWalker {
    int sb, r, Q, Rm, G;
    __host__ __device__ __forceinline__ void init(int g_start, const SplitConsts& k) {
        G = k.G;
        Q = (int)k.Q;
        Rm = (int)k.Rm;
        sb = seg_begin(g_start, k);
        r = (int)(((uint32_t)g_start * k.Rm) - (uint32_t)(sb - g_start * Q) * (uint32_t)G);
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
