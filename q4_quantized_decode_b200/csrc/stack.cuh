// The whole synthetic decode step (4 * n_layers renormalised M = 1 GEMVs) as
// one persistent kernel: one CTA per SM, a grid-wide barrier between
// consecutive GEMVs, and each warp's weight stream running ahead across GEMV
// boundaries.
//
// The pages keep the GPU fed with one command submission per token
// (originshq.com page, section "The Engine: ~50 WGSL Kernels Written From
// Scratch").  Here one launch covers the step, and the dependency between
// GEMVs (the next input is the renormalised previous output) no longer
// drains the memory pipe: weights do not depend on activations, so while a
// CTA waits at the barrier and restages x, its warps' rings already hold the
// next GEMV's first segments (up to ~150 KB per SM).  Each GEMV is computed by
// the same per-warp consumer as q4gemv_run's M = 1 kernel, over the same
// balanced segment split, so results are identical to chaining that kernel.
#pragma once

#include "gemv_dp2a.cuh"

namespace q4 {

// One GEMV of the step (device array built by the host).
struct StackGemv {
    const uint8_t* W;     // packed matrix
    __half* y;            // output, N entries
    __half* trace_x;      // nullable: the input vector used
    int N, K;
    int renorm;           // 1: input = renorm(previous output[0:K]); 0: input = x_in
    int pad;
    SplitConsts sc;       // split of its segments over the grid's warps
};

struct StackArgs {
    const StackGemv* gemv;
    int n_gemv;
    const __half* x_in;   // input of GEMV 0
    __half* x_out;        // renorm(last output[0:hidden])
    int hidden;
    float* ws;            // split-tile partials (as q4gemv_run)
    int* cnt;             // per-tile arrival counters
    int* err;             // device error word
    int* sync;            // [0] grid arrivals, [1] abort flag; zero at launch
};

// Unit-RMS renorm of in[0:len) into out, same arithmetic and order as the
// renorm fused into the GEMV prologue (coherent loads: `in` may have been
// written by other CTAs of the running kernel).  All NT threads of one CTA.
template <int NT, bool kCoherent, int QN>
__device__ __forceinline__ void renorm_block(const __half* in, __half* out, int len, float* red) {
    const int tid = threadIdx.x, lane = tid & 31;
    const int nq = len / 8;
    uint4 xr[QN];
#pragma unroll
    for (int i = 0; i < QN; ++i) {
        const int q = tid + NT * i;
        const uint4* src = reinterpret_cast<const uint4*>(in + (size_t)q * 8);
        xr[i] = q < nq ? (kCoherent ? __ldcg(src) : *src) : make_uint4(0, 0, 0, 0);
    }
    float part = 0.f;
#pragma unroll
    for (int i = 0; i < QN; ++i) {
        const __half2* h = reinterpret_cast<const __half2*>(&xr[i]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(h[e]);
            part = fmaf(f.x, f.x, part);
            part = fmaf(f.y, f.y, part);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (lane == 0) red[tid >> 5] = part;
    __syncthreads();
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) s += red[w];
    const float scale = (s > 0.f) ? __fdiv_rn(1.0f, __fsqrt_rn(__fdiv_rn(s, (float)len))) : 0.f;
#pragma unroll
    for (int i = 0; i < QN; ++i) {
        const int q = tid + NT * i;
        __half2* h = reinterpret_cast<__half2*>(&xr[i]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(h[e]);
            h[e] = __floats2half2_rn(f.x * scale, f.y * scale);
        }
        if (q < nq) *reinterpret_cast<uint4*>(out + (size_t)q * 8) = xr[i];
    }
}

// The view of GEMV i that the per-warp consumer and the staging work on.
__device__ __forceinline__ GemvArgs stack_view(const StackArgs& sa, int i) {
    const StackGemv d = sa.gemv[i];
    GemvArgs a;
    a.W = d.W;
    a.x = (i == 0) ? sa.x_in : sa.gemv[i - 1].y;
    a.y = d.y;
    a.ws = sa.ws;
    a.cnt = sa.cnt;
    a.err = sa.err;
    a.trace_x = d.trace_x;
    a.N = d.N;
    a.K = d.K;
    a.KB = d.K / 32;
    a.T = (d.N + 31) / 32;
    a.S = d.sc.S;
    a.G = d.sc.G;
    a.renorm = d.renorm;
    a.sc = d.sc;
    return a;
}

// Activation chunks per thread in the persistent step: K <= 5 * 8 * threads.
constexpr int kStackXChunks = 5;

// Issues a warp's chunks (C segments, one bulk copy each) GEMV after GEMV,
// at most R ahead of consumption.  Every lane tracks the state; lane 0 issues.
// The descriptor of the GEMV after the current one is loaded a whole GEMV
// ahead, so advancing never waits on memory.
template <int R, int C>
struct StreamProducer {
    int gi;               // GEMV being issued
    int ch, nch, nseg;    // chunk within it, chunk count, segment count
    const uint8_t* src;   // first segment of this warp's run in GEMV gi
    int issued;           // chunks issued so far (all GEMVs)
    const uint8_t* nW;    // GEMV gi + 1: matrix and split (prefetched)
    SplitConsts nsc;

    __device__ __forceinline__ void load_next(const StackArgs& sa) {
        if (gi + 1 < sa.n_gemv) {
            const StackGemv* d = sa.gemv + gi + 1;
            nW = d->W;
            nsc = d->sc;
        }
    }
    // Position on GEMV gi or, if this warp owns nothing there, on the next
    // GEMV where it does.
    __device__ __forceinline__ void enter(const StackArgs& sa, int gw, const uint8_t* W,
                                          SplitConsts k) {
        while (true) {
            if (gw < k.G) {
                const int s0 = seg_begin(gw, k), s1 = seg_begin(gw + 1, k);
                nseg = s1 - s0;
                nch = (nseg + C - 1) / C;
                src = W + (size_t)s0 * kSegBytes;
                ch = 0;
                load_next(sa);
                return;
            }
            if (++gi >= sa.n_gemv) return;
            const StackGemv* d = sa.gemv + gi;
            W = d->W;
            k = d->sc;
        }
    }
    __device__ __forceinline__ void start(const StackArgs& sa, int gw) {
        gi = 0;
        issued = 0;
        enter(sa, gw, sa.gemv[0].W, sa.gemv[0].sc);
    }
    __device__ __forceinline__ void fill(const StackArgs& sa, int gw, int consumed, uint32_t stage0,
                                         uint64_t* bars, int lane) {
        while (gi < sa.n_gemv && issued - consumed < R) {
            const int k = issued % R;
            const uint32_t bytes = (uint32_t)min(C, nseg - ch * C) * kSegBytes;
            if (lane == 0) {
                mbar_arrive_expect_tx(bars + k, bytes);
                bulk_g2s_addr(stage0 + (uint32_t)k * C * kSegBytes, src + (size_t)ch * C * kSegBytes,
                              bytes, bars + k);
            }
            ++issued;
            if (++ch == nch) {
                if (++gi < sa.n_gemv) enter(sa, gw, nW, nsc);
            }
        }
    }
};

// Grid barrier: CTA-wide arrival already made; thread 0 waits (bounded) until
// `target` arrivals or an abort.  Returns false on timeout or abort.
__device__ __forceinline__ bool grid_wait(int* sync, int target, int* err, int* flag_smem) {
    if (threadIdx.x == 0) {
        int ok = 0;
        for (uint32_t it = 0; it < (1u << 26); ++it) {
            if (ld_acquire_gpu(sync) >= target) {
                ok = 1;
                break;
            }
            if ((it & 63) == 63 && ld_relaxed_gpu_int(sync + 1) != 0) break;
        }
        if (!ok) {
            set_device_error(err, kDevTimeout);
            atomicExch(sync + 1, 1);
        }
        *flag_smem = ok;
    }
    __syncthreads();
    const bool ok = *flag_smem != 0;
    __syncthreads();
    return ok;
}

template <int WARPS, int R, int C>
__global__ void __launch_bounds__(WARPS * 32, 1) stack_kernel(const StackArgs sa, int kmax) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t bars[WARPS * R];
    __shared__ float red[WARPS];
    __shared__ int flag;
    constexpr int NT = WARPS * 32;

    const uint32_t smem_base = smem_addr(smem);
    const uint32_t stage0_base = smem_base;
    const uint32_t xs = smem_base + (uint32_t)ring_bytes(WARPS, R, C);
    const uint32_t rec = xs + (uint32_t)kmax * 2;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gw = blockIdx.x * WARPS + warp;
    const uint32_t stage0 = stage0_base + (uint32_t)warp * R * C * kSegBytes;
    uint64_t* wbars = bars + warp * R;

    if (lane == 0) {
        for (int k = 0; k < R; ++k) mbar_init(wbars + k, 1);
        fence_barrier_init();
    }
    __syncwarp();

    StreamProducer<R, C> prod;
    prod.start(sa, gw);
    int consumed = 0;
    prod.fill(sa, gw, consumed, stage0, wbars, lane);

    bool ok = true;
    for (int i = 0; i < sa.n_gemv && ok; ++i) {
        const GemvArgs a = stack_view(sa, i);
        if (i > 0) ok = grid_wait(sa.sync, i * (int)gridDim.x, sa.err, &flag);
        if (!ok) break;
        stage_activations<1, NT, true, kStackXChunks>(a, xs, rec, red);
        Dp2aConsumer<1> cons;
        cons.init(a, gw, xs, rec);
        const int nseg = cons.sp.s1 - cons.sp.s0;
        for (int j = 0; j < nseg; j += C) {
            const int k = consumed % R;
            if (!mbar_wait_bounded(wbars + k, (uint32_t)((consumed / R) & 1), 1u << 22))
                set_device_error(sa.err, kDevTimeout);   // data then unreliable
            const uint32_t st = stage0 + (uint32_t)k * C * kSegBytes;
            const int n = min(C, nseg - j);
            if (n == C) {
                cons.template stage_full<C>(a, st);
            } else {
                for (int jj = 0; jj < n; ++jj) cons.step(a, st + jj * kSegBytes);
            }
            ++consumed;
            __syncwarp();
            fence_proxy_async_smem();
            prod.fill(sa, gw, consumed, stage0, wbars, lane);
        }
        cons.finish(a);
        // This CTA is done with GEMV i (outputs and partial combines written).
        __syncthreads();
        if (threadIdx.x == 0) red_add_release_gpu(sa.sync, 1);
    }
    if (ok) ok = grid_wait(sa.sync, sa.n_gemv * (int)gridDim.x, sa.err, &flag);
    if (ok) {
        if (blockIdx.x == 0)
            renorm_block<NT, true, kStackXChunks>(sa.gemv[sa.n_gemv - 1].y, sa.x_out, sa.hidden, red);
        return;
    }
    // Abort: let this warp's copies in flight land (bounded) before leaving.
    for (; consumed < prod.issued; ++consumed)
        mbar_wait_bounded(wbars + consumed % R, (uint32_t)((consumed / R) & 1), 1u << 22);
}

}  // namespace q4
