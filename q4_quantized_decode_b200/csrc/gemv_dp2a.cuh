// Q4_0 GEMV for M = 1..2 on CUDA cores with exact integer block dot products.
//
// The pages' engine sweeps each weight row with a 64-thread group,
// dequantises in registers and reduces in shared memory (originshq.com page,
// section "The Engine: ~50 WGSL Kernels Written From Scratch").  On sm_100a
// the row sweep is replaced by a flat, perfectly balanced split of all
// (tile of 32 rows, 32-column block) segments over every warp of the grid:
//   * lane (g, c) of a warp loads, with one 16-byte streaming load, qs word c
//     of rows g, g+8, g+16, g+24 of a segment, so a warp reads 512 contiguous
//     bytes per segment, and the 64-byte scale chunk alongside;
//   * the activations of a 32-column block are converted once per CTA to
//     16-bit integers with a power-of-two scale (the block maximum held
//     exactly), staged in shared memory in the lane order of the weight
//     words; each weight word is split into two byte vectors of codes with
//     one shift and two masks and multiplied with dp2a (16-bit x 8-bit dot
//     products), so the block sum of (q - 8) * X is an exact integer;
//   * the block sum is scaled by d * 2^e in fp32 and accumulated per row;
//   * a warp's accumulators are combined across its four column lanes with
//     two shuffles; tiles split between warps are combined by the last warp
//     to arrive (per-tile counter), summing the partials in warp order, so
//     results are deterministic.
#pragma once

#include "device_common.cuh"

namespace q4 {

constexpr int kSegNibBytes = 512;   // 32 rows x 16 bytes of codes
constexpr int kSegSclBytes = 64;    // 32 rows x f16 scale

struct GemvArgs {
    const uint8_t* nib;     // packed nibble plane
    const uint8_t* scl;     // packed scale plane
    const __half* x;        // [M][K] activations, or the renorm source (M == 1)
    __half* y;              // [M][N]
    float* ws;              // split-tile partials [G][2][M][32]
    int* cnt;               // per-tile arrival counters [T], zero between calls
    int* err;               // device error word
    __half* trace_x;        // nullable: CTA 0 writes the f16 input vector it used
    int64_t N;
    int K, KB, T;
    int S;                  // segments = T * KB
    int G;                  // warps that own segments (G <= S)
    int renorm;             // 1: the input is renorm(x[0:K]) (M == 1 only)
};

// Shared-memory footprint of the kernel for M vectors of K columns.
__host__ __device__ constexpr size_t gemv_dp2a_smem_bytes(int M, int K) {
    // raw f16 x | int16 X (permuted) | -8*sum X per lane group | block scale
    return (size_t)M * K * 2 + (size_t)M * K * 2 + (size_t)M * (K / 32) * 16 +
           (size_t)M * (K / 32) * 4;
}

// First segment of warp g under the flat balanced split of S segments over
// G warps, and the warp that owns segment s.
__host__ __device__ __forceinline__ int seg_begin(int g, int S, int G) {
    return (int)(((int64_t)g * S) / G);
}
__host__ __device__ __forceinline__ int warp_of_seg(int s, int S, int G) {
    return (int)((((int64_t)s + 1) * G - 1) / S);
}

// Position of element j of a 32-column block in the permuted X layout: the
// eight entries lane group c needs ([4c..4c+3] and [4c+16..4c+19]) are
// contiguous.
__host__ __device__ __forceinline__ int xperm_pos(int j) {
    return ((j & 15) >> 2) * 8 + ((j >> 4) << 2) + (j & 3);
}

// Renormalise buf[0:len) (f16, shared memory) in place to unit RMS:
// s = sum v^2 in fp32 (fixed order: thread-strided partials, warp xor tree,
// then warps in order), scale = 1/sqrt(s/len), v <- f16(v * scale); an
// all-zero vector stays zero.  Must be called by all NT threads of the CTA.
template <int NT>
__device__ __forceinline__ void block_renorm_inplace(__half* buf, int len, float* red) {
    const int tid = threadIdx.x;
    float part = 0.f;
    for (int i = tid; i < len; i += NT) {
        const float v = __half2float(buf[i]);
        part = fmaf(v, v, part);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if ((tid & 31) == 0) red[tid >> 5] = part;
    __syncthreads();
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) s += red[w];
    const float scale = (s > 0.f) ? __fdiv_rn(1.0f, __fsqrt_rn(__fdiv_rn(s, (float)len))) : 0.f;
    for (int i = tid; i < len; i += NT)
        buf[i] = __float2half_rn(__half2float(buf[i]) * scale);
    __syncthreads();
}

// Stage x: bulk copy into shared memory (after the dependency wait),
// optional renorm, conversion to per-block 16-bit integers.
template <int M, int WARPS>
__device__ __forceinline__ bool stage_activations(const GemvArgs& a, __half* raw, int16_t* Xs,
                                                  int* negC, float* sb, uint64_t* bar,
                                                  float* red) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t bytes = (uint32_t)M * a.K * 2;
    if (tid == 0) {
        mbar_arrive_expect_tx(bar, bytes);
        bulk_g2s(raw, a.x, bytes, bar);
    }
    // ~1e6 polls: far beyond any real completion time, short of a hang.  The
    // CTA agrees on the outcome so that every thread leaves together.
    const bool arrived = mbar_wait_bounded(bar, 0, 1u << 20);
    if (!__syncthreads_and(arrived)) {
        if (tid == 0) set_device_error(a.err, kDevTimeout);
        return false;
    }
    if (M == 1 && a.renorm) block_renorm_inplace<WARPS * 32>(raw, a.K, red);
    if (a.trace_x != nullptr && blockIdx.x == 0) {
        for (int i = tid; i < a.K; i += WARPS * 32) a.trace_x[i] = raw[i];
    }
    const int nblk = M * a.KB;
    for (int bb = warp; bb < nblk; bb += WARPS) {
        const int m = bb / a.KB, b = bb - m * a.KB;
        const float v = __half2float(raw[(size_t)m * a.K + b * 32 + lane]);
        const uint32_t mx = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(v)));
        int X = 0;
        float s = 0.f;
        if (mx >= 0x7F800000u) {
            s = __uint_as_float(0x7FC00000u);          // non-finite block -> NaN outputs
        } else if (mx != 0u) {
            const int E = (int)(mx >> 23) - 127;        // block max in [2^E, 2^(E+1))
            const float inv = __uint_as_float((uint32_t)(141 - E) << 23);   // 2^(14-E)
            X = __float2int_rn(v * inv);                // |X| <= 32752, exact for the max
            s = __uint_as_float((uint32_t)(113 + E) << 23);                 // 2^(E-14)
        }
        Xs[(size_t)m * a.K + b * 32 + xperm_pos(lane)] = (int16_t)X;
        int gs = X;
        gs += __shfl_xor_sync(0xffffffffu, gs, 1);
        gs += __shfl_xor_sync(0xffffffffu, gs, 2);
        gs += __shfl_xor_sync(0xffffffffu, gs, 16);
        if (lane < 16 && (lane & 3) == 0) negC[((size_t)m * a.KB + b) * 4 + (lane >> 2)] = -8 * gs;
        if (lane == 0) sb[(size_t)m * a.KB + b] = s;
    }
    __syncthreads();
    return true;
}

template <int M, int WARPS, int U>
__global__ void __launch_bounds__(WARPS * 32, 1) gemv_dp2a_kernel(const GemvArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t bar;
    __shared__ float red[WARPS];

    __half* raw = reinterpret_cast<__half*>(smem);
    int16_t* Xs = reinterpret_cast<int16_t*>(smem + (size_t)M * a.K * 2);
    int* negC = reinterpret_cast<int*>(smem + (size_t)M * a.K * 4);
    float* sb = reinterpret_cast<float*>(smem + (size_t)M * a.K * 4 + (size_t)M * a.KB * 16);

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int gw = blockIdx.x * WARPS + warp;
    // G <= S, so every warp below G owns at least one segment; warps of the
    // last CTA beyond G only help stage the activations.
    const int s0 = gw < a.G ? seg_begin(gw, a.S, a.G) : a.S;
    const int s1 = gw < a.G ? seg_begin(gw + 1, a.S, a.G) : a.S;

    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }

    // Weight prefetch: independent of the previous kernel, so it is issued
    // before the dependency wait.
    uint4 wq[U];
    uint2 wd[U];
#pragma unroll
    for (int j = 0; j < U; ++j) {
        const int s = s0 + j;
        if (s < s1) {
            wq[j] = ldg_stream_v4(a.nib + (size_t)s * kSegNibBytes + lane * 16);
            wd[j] = ldg_stream_v2(a.scl + (size_t)s * kSegSclBytes + g * 8);
        }
    }
    pdl_launch_dependents();
    __syncthreads();   // barrier init visible to all threads
    pdl_wait();

    if (!stage_activations<M, WARPS>(a, raw, Xs, negC, sb, &bar, red)) return;

    float acc[M][4];
#pragma unroll
    for (int m = 0; m < M; ++m)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[m][i] = 0.f;

    const int KB = a.KB;
    const int t_first = s0 / KB;
    int t_cur = t_first;
    int tile_end = (t_cur + 1) * KB;
    const int r = g + 8 * c;                  // row of the tile this lane emits

    // Combine a finished tile: reduce over the four column lanes, then either
    // write y (this warp owns the whole tile) or park the partial.
    auto flush = [&](int t) {
#pragma unroll
        for (int m = 0; m < M; ++m)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float v = acc[m][i];
                v += __shfl_xor_sync(0xffffffffu, v, 1);
                v += __shfl_xor_sync(0xffffffffu, v, 2);
                acc[m][i] = v;
            }
        const bool whole = warp_of_seg(t * KB, a.S, a.G) == warp_of_seg(t * KB + KB - 1, a.S, a.G);
        const int64_t row = (int64_t)t * 32 + r;
#pragma unroll
        for (int m = 0; m < M; ++m) {
            const float val = (c == 0) ? acc[m][0] : (c == 1) ? acc[m][1] : (c == 2) ? acc[m][2] : acc[m][3];
            if (whole) {
                if (row < a.N) a.y[(size_t)m * a.N + row] = __float2half_rn(val);
            } else {
                const int slot = (t == t_first) ? 0 : 1;
                a.ws[(((size_t)gw * 2 + slot) * M + m) * 32 + r] = val;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[m][i] = 0.f;
        }
    };

    for (int base = s0; base < s1; base += U) {
#pragma unroll
        for (int j = 0; j < U; ++j) {
            const int s = base + j;
            if (s < s1) {
                if (s == tile_end) {
                    flush(t_cur);
                    ++t_cur;
                    tile_end += KB;
                }
                const int b = s - t_cur * KB;
                const uint4 w = wq[j];
                const uint2 dd = wd[j];
                const int sn = s + U;
                if (sn < s1) {
                    wq[j] = ldg_stream_v4(a.nib + (size_t)sn * kSegNibBytes + lane * 16);
                    wd[j] = ldg_stream_v2(a.scl + (size_t)sn * kSegSclBytes + g * 8);
                }
                const float2 d01 = __half22float2(*reinterpret_cast<const __half2*>(&dd.x));
                const float2 d23 = __half22float2(*reinterpret_cast<const __half2*>(&dd.y));
                const float d[4] = {d01.x, d01.y, d23.x, d23.y};
                const uint32_t words[4] = {w.x, w.y, w.z, w.w};
                uint4 xq[M];
                int nc[M];
                float sbm[M];
#pragma unroll
                for (int m = 0; m < M; ++m) {
                    xq[m] = *reinterpret_cast<const uint4*>(Xs + (size_t)m * a.K + b * 32 + c * 8);
                    nc[m] = negC[((size_t)m * KB + b) * 4 + c];
                    sbm[m] = sb[(size_t)m * KB + b];
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t lo = words[i] & 0x0F0F0F0Fu;          // codes 4c..4c+3
                    const uint32_t hi = (words[i] >> 4) & 0x0F0F0F0Fu;   // codes 4c+16..4c+19
#pragma unroll
                    for (int m = 0; m < M; ++m) {
                        int v = dp2a_lo(xq[m].x, lo, nc[m]);
                        v = dp2a_hi(xq[m].y, lo, v);
                        v = dp2a_lo(xq[m].z, hi, v);
                        v = dp2a_hi(xq[m].w, hi, v);
                        acc[m][i] = fmaf((float)v, d[i] * sbm[m], acc[m][i]);
                    }
                }
            }
        }
    }
    if (s1 > s0) flush(t_cur);

    // Tiles shared with other warps (at most the first and the last one of
    // this warp's range): count arrivals; the last warp to arrive sums the
    // partials in warp order, writes y and re-arms the counter.
    auto arrive = [&](int t) {
        const int gf = warp_of_seg(t * KB, a.S, a.G), gl = warp_of_seg(t * KB + KB - 1, a.S, a.G);
        if (gf == gl) return;
        __threadfence();
        __syncwarp();
        int old = 0;
        if (lane == 0) old = atomicAdd(a.cnt + t, 1);
        old = __shfl_sync(0xffffffffu, old, 0);
        const int need = gl - gf + 1;
        if (old == need - 1) {
            __threadfence();
            const int64_t row = (int64_t)t * 32 + r;
#pragma unroll
            for (int m = 0; m < M; ++m) {
                float sum = 0.f;
                for (int gg = gf; gg <= gl; ++gg) {
                    const int sl = (seg_begin(gg, a.S, a.G) / KB == t) ? 0 : 1;
                    sum += __ldcg(a.ws + (((size_t)gg * 2 + sl) * M + m) * 32 + r);
                }
                if (row < a.N) a.y[(size_t)m * a.N + row] = __float2half_rn(sum);
            }
            if (lane == 0) a.cnt[t] = 0;
        } else if (old >= need) {
            if (lane == 0) set_device_error(a.err, kDevConcurrent);
        }
    };
    if (s1 > s0) {
        const int t_last = (s1 - 1) / KB;
        arrive(t_first);
        if (t_last != t_first) arrive(t_last);
    }
}

// Final renorm of the decode step: out = renorm(in[0:len)).
template <int WARPS>
__global__ void __launch_bounds__(WARPS * 32, 1) renorm_kernel(const __half* in, __half* out, int len,
                                                             int* err) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t bar;
    __shared__ float red[WARPS];
    __half* buf = reinterpret_cast<__half*>(smem);
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    pdl_wait();
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(&bar, (uint32_t)len * 2);
        bulk_g2s(buf, in, (uint32_t)len * 2, &bar);
    }
    const bool arrived = mbar_wait_bounded(&bar, 0, 1u << 20);
    if (!__syncthreads_and(arrived)) {
        if (threadIdx.x == 0) set_device_error(err, kDevTimeout);
        return;
    }
    block_renorm_inplace<WARPS * 32>(buf, len, red);
    for (int i = threadIdx.x; i < len; i += WARPS * 32) out[i] = buf[i];
}

// GGUF Q4_0 -> packed layout, one warp per segment (grid-stride).
__global__ void __launch_bounds__(256) repack_kernel(const uint8_t* __restrict__ gguf,
                                                     uint8_t* __restrict__ packed, int64_t N,
                                                     int KB, int64_t S, int64_t Np) {
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    uint8_t* nib = packed;
    uint8_t* scl = packed + Np * KB * 16;
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
        *reinterpret_cast<uint4*>(nib + s * kSegNibBytes + lane * 16) =
            make_uint4(words[0], words[1], words[2], words[3]);
        if (c == 0) {
            *reinterpret_cast<uint2*>(scl + s * kSegSclBytes + g * 8) =
                make_uint2((uint32_t)dv[0] | ((uint32_t)dv[1] << 16),
                           (uint32_t)dv[2] | ((uint32_t)dv[3] << 16));
        }
    }
}

}  // namespace q4
