// The down GEMV fed directly by the gate+up GEMV's output: y = W u with
// u_k = SiLU(g_k) * up_k, where [g | up] is the 2K-entry f16 vector the
// gate+up GEMV wrote (gate half first).  The gated input is never written to
// memory: the staging computes it in fp32 from the two halves and converts it
// per 32-entry block exactly as any M = 1 input (block exponent, int16 codes
// in lane order, records, block sums of squares), so the weight stream and
// the exact integer block sums are those of gemv_dp2a_kernel<1>.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

#include "gemv_dp2a.cuh"

namespace q4 {

// SiLU(g) = g / (1 + e^-g) in fp32 with the hardware exponential and the
// fast quotient (reciprocal approximation times g, within 2 ulp): every CTA
// of the down GEMV converts all K entries, so the per-entry cost is on the
// critical path.  +-0 for very negative g, whose exponential overflows.
__device__ __forceinline__ float silu_f32(float g) { return __fdividef(g, 1.f + __expf(-g)); }

// Gated staging for the M = 1 kernel, all threads of the CTA: thread t takes
// the 16-byte chunks q = t, t + NT, ... of the gate half and the same chunks
// of the up half; QN chunks per thread (K <= QN * 8 * NT), all rounds run.
template <int NT, int QN>
__device__ __forceinline__ void stage_swiglu(const GemvArgs& a, uint32_t xs, uint32_t rec,
                                             float* sq) {
    const int tid = threadIdx.x;
    const int nq = a.K / 8;
    uint4 gr[QN], ur[QN];
#pragma unroll
    for (int i = 0; i < QN; ++i) {
        const int q = tid + NT * i;
        gr[i] = q < nq ? *reinterpret_cast<const uint4*>(a.x + (size_t)q * 8) : make_uint4(0, 0, 0, 0);
        ur[i] = q < nq ? *reinterpret_cast<const uint4*>(a.x + (size_t)a.K + (size_t)q * 8)
                       : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < QN; ++i) {
        const int q = tid + NT * i;
        const __half2* gh = reinterpret_cast<const __half2*>(&gr[i]);
        const __half2* uh = reinterpret_cast<const __half2*>(&ur[i]);
        float v[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 g2 = __half22float2(gh[e]);
            const float2 u2 = __half22float2(uh[e]);
            v[2 * e] = silu_f32(g2.x) * u2.x;
            v[2 * e + 1] = silu_f32(g2.y) * u2.y;
        }
        // All lanes convert (the four chunks of a block share shuffles).
        const ChunkQ o = quant_chunk(v);
        if (q < nq) {
            store_chunk_smem(o, xs, rec, q >> 2, q & 3);
            if ((q & 3) == 0) sq[q >> 2] = o.sq;
        }
    }
    __syncthreads();
}

// gemv_dp2a_kernel<1> with the gated staging; with a.renorm the outputs are
// scaled by the unit-RMS scale of u (the gated step's down GEMV), else not
// (q4gemv_run_swiglu).
template <int WARPS, int R, int C>
__global__ void __launch_bounds__(WARPS * 32, 1) gemv_swiglu_kernel(const GemvArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t bars[WARPS * R];

    const uint32_t smem_base = smem_addr(smem);
    const uint32_t xs = smem_base + (uint32_t)ring_bytes(WARPS, R, C);    // int16 X, lane order
    const uint32_t rec = xs + (uint32_t)(a.K * 2);                        // {-8 sum X, scale}
    float* park = reinterpret_cast<float*>(smem + ring_bytes(WARPS, R, C) + (size_t)a.K * 2 +
                                           (size_t)a.KB * 32);             // [WARPS][2][1][32]
    float* sq = park + WARPS * 2 * 32;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gw = blockIdx.x * WARPS + warp;
    Dp2aConsumer<1> cons;
    WarpRing<R, C> ring;
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
    if (lane == 0)
        for (int ch = 0; ch < R && ch < ring.nch; ++ch) ring.issue(ch);
    cons.init(a, gw, xs, rec, park + (size_t)warp * 2 * 32);
    pdl_launch_dependents();
    pdl_wait();

    {
        constexpr int NT = WARPS * 32;
        const int nq = a.K / 8;
        if (nq <= 2 * NT) stage_swiglu<NT, 2>(a, xs, rec, sq);
        else if (nq <= 5 * NT) stage_swiglu<NT, 5>(a, xs, rec, sq);
        else stage_swiglu<NT, kXChunksPerThread>(a, xs, rec, sq);
    }
    if (a.renorm) cons.oscale = unit_rms_scale(sq, a.KB, a.K);

    for (int ch = 0; ch < ring.nch; ++ch) {
        if (!ring.wait(ch)) set_device_error(a.err, kDevTimeout);   // data then unreliable
        const uint32_t st = ring.stage(ch % R);
        const int n = min(C, ring.nseg - ch * C);
        if (n == C) {
            cons.template stage_full<C>(a, st);
        } else {
            for (int j = 0; j < n; ++j) cons.step(a, st + j * kSegBytes);
        }
        __syncwarp();
        fence_proxy_async_smem();
        if (lane == 0 && ch + R < ring.nch) ring.issue(ch + R);
    }
    cons.flush_last(a);
    __syncthreads();
    int xt[2], xcf[2], xcl[2];
    cons.template combine_cta<WARPS>(a, park, a.ws, xt, xcf, xcl);
    if (xt[0] >= 0) combine_ctas_arrive<1, WARPS>(a, xt[0], xcf[0], xcl[0], cons.oscale);
    if (xt[1] >= 0) combine_ctas_arrive<1, WARPS>(a, xt[1], xcf[1], xcl[1], cons.oscale);
}

}  // namespace q4
