// The whole synthetic decode step (4 * n_layers M = 1 GEMVs, each input the
// previous f16 output scaled to unit RMS) as one persistent kernel: one CTA
// per SM, a grid-wide barrier between consecutive GEMVs, and each warp's
// weight stream running ahead across GEMV boundaries.
//
// The pages keep the GPU fed with one command submission per token
// (originshq.com page, section "The Engine: ~50 WGSL Kernels Written From
// Scratch").  Here one launch covers the step, and the dependency between
// GEMVs (the next input is the previous output) no longer drains the memory
// pipe: weights do not depend on activations, so while a CTA waits at the
// barrier and stages its input, its warps' rings already hold the next
// GEMV's first segments (~166 KB per SM).  Each GEMV's finished output blocks
// are also written converted for the next GEMV, which stages them with bulk
// copies.  Each GEMV is computed by the same per-warp consumer as
// q4gemv_run's M = 1 kernel, over the same balanced segment split and with
// the same combine order, so results are identical to chaining that kernel.
#pragma once

#include "gemv_dp2a.cuh"
#include "gemv_swiglu.cuh"

namespace q4 {

// One GEMV of the step (device array built by the host).
struct StackGemv {
    const uint8_t* W;     // packed matrix
    __half* y;            // output, N entries
    __half* trace_x;      // nullable: the input vector before its scale (filled at the end)
    int N, K;
    int renorm;           // 1: input = unit-RMS scale * previous output[0:K]; 0: input = x_in
    int fill_y;           // 1: also write y of tiles shared by CTAs (y is traced)
    int gated;            // 1: input = SiLU(gate) * up of the previous 2K outputs, scaled to unit RMS
    SplitConsts sc;       // split of its segments over the grid's warps
};

struct StackArgs {
    const StackGemv* gemv;
    int n_gemv;
    const __half* x_in;   // input of GEMV 0
    __half* x_out;        // f16(s * last output[0:hidden])
    int hidden;
    float* ws;            // CTA partials, two GEMV-parity halves of [CTAs][2][32]
    int ws_half;          // floats per half
    uint8_t* xq;          // pre-quantised inputs, two GEMV-parity halves of xq_half bytes:
    int xq_half;          //   X [kmax] int16 (lane order), records [kmax / 32][4] {-8 sum X, scale},
    int kmax;             //   block sums of squares [kmax / 32] fp32
    int* err;             // device error word
    int* sync;            // [0] grid arrivals, [1] abort flag; zero at launch
    uint32_t poll_limit;  // polls of a grid wait before it gives up
    int unreachable;      // test knob: the first grid wait asks for one arrival too many
    uint4* gscr;          // gated steps: per CTA, the combined shared tiles [kStackMaxCtas][4] (16 B each)
};

// Outputs of the previous GEMV in tiles shared by several CTAs exist only as
// per-CTA partials until they are read: every reader sums them in CTA order
// (the same sum q4gemv_run's kernel takes), scales by the previous GEMV's
// output scale and rounds to f16.  combine() gives one 8-row chunk of such a
// tile.  For the step's final output, prepare() combines, with all threads
// of the CTA, the shared tiles' chunks in the staged range into `patch`
// (shared memory, 16 bytes per chunk), so their loads overlap those of the
// rest of the vector, and apply() takes chunk q from the patch when its tile
// is shared.  ws == nullptr: no-op.  A traced step also completes y (fill_y)
// for those tiles: boundary b's tile is written by CTA b, or every one by
// the calling CTA (fill_all).
template <int WARPS>
struct SplitFix {
    static constexpr bool kActive = true;
    const float* ws;      // the previous GEMV's CTA partials [CTAs][2][32]
    SplitConsts sc;       // its split
    int KB;               // its blocks per row
    float oscale;         // its output scale
    __half* fill_y;       // nullable: its output, to complete
    int fill_n;           // its rows
    bool fill_all;

    // Chunk u (rows 8u..8u+7) of shared tile t, whose first contributing
    // CTA is cf; two contributors are loaded together (the usual case), any
    // further ones after them; the sum runs from +0.
    __device__ __forceinline__ uint4 combine(int t, int cf, int u) const {
        const int cl = warp_of_seg(t * KB + KB - 1, sc) / WARPS;
        const float4* p0 = reinterpret_cast<const float4*>(
            ws + ((size_t)cf * 2 + cta_slot_read(cf, cf, t, KB, sc, WARPS)) * 32 + u * 8);
        const float4* p1 = reinterpret_cast<const float4*>(ws + ((size_t)(cf + 1) * 2) * 32 + u * 8);
        const float4 a0 = __ldcg(p0), a1 = __ldcg(p0 + 1), b0 = __ldcg(p1), b1 = __ldcg(p1 + 1);
        float s[8] = {0.f + a0.x, 0.f + a0.y, 0.f + a0.z, 0.f + a0.w,
                      0.f + a1.x, 0.f + a1.y, 0.f + a1.z, 0.f + a1.w};
        s[0] += b0.x; s[1] += b0.y; s[2] += b0.z; s[3] += b0.w;
        s[4] += b1.x; s[5] += b1.y; s[6] += b1.z; s[7] += b1.w;
        for (int c = cf + 2; c <= cl; ++c) {
            const float4* pc = reinterpret_cast<const float4*>(ws + ((size_t)c * 2) * 32 + u * 8);
            const float4 c0 = __ldcg(pc), c1 = __ldcg(pc + 1);
            s[0] += c0.x; s[1] += c0.y; s[2] += c0.z; s[3] += c0.w;
            s[4] += c1.x; s[5] += c1.y; s[6] += c1.z; s[7] += c1.w;
        }
        uint4 o;
        __half2* h = reinterpret_cast<__half2*>(&o);
#pragma unroll
        for (int e = 0; e < 4; ++e)
            h[e] = __floats2half2_rn(__fmul_rn(oscale, s[2 * e]), __fmul_rn(oscale, s[2 * e + 1]));
        return o;
    }
    __device__ __forceinline__ void fill(int t, int u, uint4 v) const {
        const __half* h = reinterpret_cast<const __half*>(&v);
        for (int e = 0; e < 8; ++e)
            if (t * 32 + u * 8 + e < fill_n) fill_y[(size_t)t * 32 + u * 8 + e] = h[e];
    }

    template <int NT>
    __device__ __forceinline__ void prepare(int nq, uint32_t patch) const {
        if (ws == nullptr) return;
        const int nb = (sc.G + WARPS - 1) / WARPS;      // CTAs owning segments
        const int total = (nb - 1) * 4;                 // (boundary, chunk) pairs
        for (int p0 = threadIdx.x; p0 < total; p0 += 2 * NT) {
            // Two pairs per thread per round, so their loads overlap.
            int tt[2], qq[2];
            bool fl[2];
            uint4 v[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int p = p0 + k * NT;
                const int b = (p >> 2) + 1;
                tt[k] = p < total ? shared_tile_of_boundary(b, KB, sc, WARPS) : -1;
                qq[k] = tt[k] * 4 + (p & 3);
                fl[k] = fill_y != nullptr && (fill_all || b == (int)blockIdx.x);
                if (tt[k] >= 0 && (qq[k] < nq || fl[k])) v[k] = combine(tt[k], b - 1, p & 3);
                else tt[k] = -1;
            }
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                if (tt[k] < 0) continue;
                if (qq[k] < nq) sts128(patch + (uint32_t)qq[k] * 16, v[k]);
                if (fl[k]) fill(tt[k], qq[k] & 3, v[k]);
            }
        }
    }

    __device__ __forceinline__ uint4 apply(int q, uint4 v, uint32_t patch) const {
        if (ws == nullptr) return v;
        const int t = q >> 2;
        const int cf = warp_of_seg(t * KB, sc) / WARPS, cl = warp_of_seg(t * KB + KB - 1, sc) / WARPS;
        return cf == cl ? v : lds128(patch + (uint32_t)q * 16);
    }
};

// Staging of GEMV i >= 1 of the step from the pre-quantised input that GEMV
// i-1's CTAs wrote for their finished tiles: one bulk copy each of the codes,
// records and block sums of squares into shared memory, while all threads
// combine, scale, round and quantise the tiles shared by CTAs (the copy holds
// no valid data for those) and write them over the copy once it has landed.
// K: entries of GEMV i's input; xbar: this CTA's copy barrier, phase parity.
template <int WARPS, int NT>
__device__ __forceinline__ void stage_prequant(const StackArgs& sa, int i, int K,
                                               const SplitFix<WARPS>& fx, uint32_t xs, uint32_t rec,
                                               float* sq, uint64_t* xbar, uint32_t parity) {
    const int KB = K / 32;
    const uint8_t* base = sa.xq + (size_t)(i & 1) * sa.xq_half;
    if (threadIdx.x == 0) {
        // Other CTAs wrote these bytes with ordinary stores before the grid
        // barrier, and this CTA last read the destination with ordinary
        // loads: order both before the bulk copies.
        fence_proxy_async_global();
        fence_proxy_async_smem();
        const uint32_t bx = (uint32_t)K * 2, br = (uint32_t)K, bs = (uint32_t)tile_sum_bytes(K);
        mbar_arrive_expect_tx(xbar, bx + br + bs);
        bulk_g2s_addr(xs, base, bx, xbar);
        bulk_g2s_addr(rec, base + (size_t)sa.kmax * 2, br, xbar);
        bulk_g2s_addr(smem_addr(sq), base + (size_t)sa.kmax * 3, bs, xbar);
    }
    // Shared tiles of GEMV i-1, enumerated by CTA boundary and chunk (four
    // consecutive threads per tile, so the quantiser's shuffles stay inside
    // one tile); every lane runs the quantiser, idle ones on zeros.
    const int nb = (fx.sc.G + WARPS - 1) / WARPS;
    const int total = (nb - 1) * 4;
    constexpr int kRounds = 2;                          // total <= 2 * NT: up to 257 CTAs
    ChunkQ o[kRounds];
    int tq[kRounds];
#pragma unroll
    for (int k = 0; k < kRounds; ++k) {
        const int p = (int)threadIdx.x + k * NT;
        const int b = (p >> 2) + 1, u = p & 3;
        const int t = p < total ? shared_tile_of_boundary(b, fx.KB, fx.sc, WARPS) : -1;
        const bool fl = t >= 0 && fx.fill_y != nullptr && b == (int)blockIdx.x;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (t >= 0 && (t < KB || fl)) v = fx.combine(t, b - 1, u);
        if (fl) fx.fill(t, u, v);
        float f[8];
        const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 g = __half22float2(h[e]);
            f[2 * e] = g.x;
            f[2 * e + 1] = g.y;
        }
        o[k] = quant_chunk(f);
        tq[k] = (t >= 0 && t < KB) ? t * 4 + u : -1;
    }
    if (!mbar_wait_bounded(xbar, parity, 1u << 22)) set_device_error(sa.err, kDevTimeout);
#pragma unroll
    for (int k = 0; k < kRounds; ++k) {
        if (tq[k] < 0) continue;
        store_chunk_smem(o[k], xs, rec, tq[k] >> 2, tq[k] & 3);
        if ((tq[k] & 3) == 0) sq[tq[k] >> 2] = o[k].sq;
    }
    __syncthreads();
}

// Largest grid of the gated step (its per-CTA scratch holds one combined
// chunk per CTA boundary and chunk).
constexpr int kStackMaxCtas = 256;

// Staging of a gated GEMV i (the down GEMV of the FFN with its activation):
// its K-entry input is u = SiLU(gate) * up of GEMV i-1's 2K outputs (gate
// half first), computed in fp32 and converted per block as any input; the
// step's pre-converted hand-off is not used (u needs both halves, which
// different CTAs finish).  Two passes: the tiles of GEMV i-1 shared by CTAs
// are combined (CTA partials in CTA order, scaled, rounded: the values the
// plain staging would use) into this CTA's scratch, one 16-byte chunk per
// CTA boundary and chunk; then every thread loads its chunks of both halves
// -- from y for tiles one CTA finished, from the scratch for shared ones --
// and converts SiLU(g) * up.  QN: chunks of u per thread (K <= QN * 8 * NT).
template <int WARPS, int NT, int QN>
__device__ __forceinline__ void stage_gated(const StackArgs& sa, int K, const SplitFix<WARPS>& fx,
                                            const __half* y_prev, uint32_t xs, uint32_t rec, float* sq) {
    uint4* scr = sa.gscr + (size_t)blockIdx.x * kStackMaxCtas * 4;
    const int nb = (fx.sc.G + WARPS - 1) / WARPS;
    const int total = (nb - 1) * 4;
    for (int p = threadIdx.x; p < total; p += NT) {
        const int t = shared_tile_of_boundary((p >> 2) + 1, fx.KB, fx.sc, WARPS);
        if (t >= 0) scr[p] = fx.combine(t, p >> 2, p & 3);   // slot: first contributor, chunk
    }
    __syncthreads();
    const int nq = K / 8;
    auto chunk = [&](int c) -> uint4 {                       // chunk c of GEMV i-1's output
        const int t = c >> 2;
        const int cf = warp_of_seg(t * fx.KB, fx.sc) / WARPS;
        const int cl = warp_of_seg(t * fx.KB + fx.KB - 1, fx.sc) / WARPS;
        return cf == cl ? __ldcg(reinterpret_cast<const uint4*>(y_prev) + c) : scr[cf * 4 + (c & 3)];
    };
    uint4 gr[QN], ur[QN];
#pragma unroll
    for (int r = 0; r < QN; ++r) {
        const int q = (int)threadIdx.x + NT * r;
        gr[r] = q < nq ? chunk(q) : make_uint4(0, 0, 0, 0);
        ur[r] = q < nq ? chunk(q + nq) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int r = 0; r < QN; ++r) {
        const int q = (int)threadIdx.x + NT * r;
        const __half2* gh = reinterpret_cast<const __half2*>(&gr[r]);
        const __half2* uh = reinterpret_cast<const __half2*>(&ur[r]);
        float v[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 g2 = __half22float2(gh[e]);
            const float2 u2 = __half22float2(uh[e]);
            v[2 * e] = silu_f32(g2.x) * u2.x;
            v[2 * e + 1] = silu_f32(g2.y) * u2.y;
        }
        const ChunkQ o = quant_chunk(v);                    // all lanes (shuffles inside a block)
        if (q < nq) {
            store_chunk_smem(o, xs, rec, q >> 2, q & 3);
            if ((q & 3) == 0) sq[q >> 2] = o.sq;
        }
    }
    __syncthreads();
}

// The view of GEMV i that the per-warp consumer and the staging work on.
__device__ __forceinline__ GemvArgs stack_view(const StackArgs& sa, int i) {
    const StackGemv d = sa.gemv[i];
    GemvArgs a;
    a.W = d.W;
    a.x = (i == 0) ? sa.x_in : sa.gemv[i - 1].y;
    a.y = d.y;
    a.ws = sa.ws;
    a.cnt = nullptr;      // no arrival counters: shared tiles are combined by the next reader
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

// Shared memory of the persistent step for inputs of up to kmax elements:
// ring, int16 activations (2 bytes each), block records (1 byte per
// element), one tile partial pair per warp, block sums of squares.
__host__ __device__ constexpr size_t stack_smem_bytes(int kmax, int warps, int R, int C) {
    return ring_bytes(warps, R, C) + (size_t)kmax * 3 + warp_partial_bytes(1, warps) +
           tile_sum_bytes(kmax);
}

// Bytes of one parity half of the pre-quantised input buffer.
__host__ __device__ constexpr size_t stack_xq_half_bytes(int kmax) {
    return ((size_t)kmax * 3 + tile_sum_bytes(kmax) + 255) / 256 * 256;
}

// A warp's position in its stream of chunks (C segments each) across the
// GEMVs of the step: chunk ch of its run in GEMV gi.  Descriptors are read
// through L1 (they are prefetched there at kernel start).
template <int C>
struct StreamCursor {
    int gi;               // GEMV (n_gemv: past the end)
    int ch, nch, nseg;    // chunk of the run, chunks, segments
    const uint8_t* src;   // first segment of the run

    // Position on chunk 0 of GEMV gi or, if warp gw owns nothing there, of
    // the next GEMV where it does.
    __device__ __forceinline__ void enter(const StackArgs& sa, int gw) {
        for (; gi < sa.n_gemv; ++gi) {
            const StackGemv* d = sa.gemv + gi;
            SplitConsts k;
            k.G = __ldg(&d->sc.G);
            if (gw >= k.G) continue;
            k.Q = __ldg(&d->sc.Q);
            k.Rm = __ldg(&d->sc.Rm);
            k.MG = __ldg(reinterpret_cast<const unsigned long long*>(&d->sc.MG));
            const uint8_t* W = reinterpret_cast<const uint8_t*>(
                __ldg(reinterpret_cast<const unsigned long long*>(&d->W)));
            const int s0 = seg_begin(gw, k), s1 = seg_begin(gw + 1, k);
            nseg = s1 - s0;
            nch = (nseg + C - 1) / C;
            src = W + (size_t)s0 * kSegBytes;
            ch = 0;
            return;
        }
    }
    __device__ __forceinline__ void start(const StackArgs& sa, int gw) {
        gi = 0;
        enter(sa, gw);
    }
    __device__ __forceinline__ bool valid(const StackArgs& sa) const { return gi < sa.n_gemv; }
    __device__ __forceinline__ const uint8_t* addr() const { return src + (size_t)ch * C * kSegBytes; }
    __device__ __forceinline__ uint32_t bytes() const {
        return (uint32_t)min(C, nseg - ch * C) * kSegBytes;
    }
    __device__ __forceinline__ void advance(const StackArgs& sa, int gw) {
        if (++ch == nch) {
            ++gi;
            enter(sa, gw);
        }
    }
};

// Issues a warp's chunks into its ring of R stages, GEMV after GEMV, at most
// R ahead of consumption.  Every lane tracks the state; lane 0 issues.
template <int R, int C>
struct StreamProducer {
    StreamCursor<C> cur;
    int issued;           // chunks issued into the ring so far (all GEMVs)

    __device__ __forceinline__ void start(const StackArgs& sa, int gw) {
        cur.start(sa, gw);
        issued = 0;
    }
    __device__ __forceinline__ void fill(const StackArgs& sa, int gw, int consumed, uint32_t stage0,
                                         uint64_t* bars, int lane) {
        while (cur.valid(sa) && issued - consumed < R) {
            const int k = issued % R;
            if (lane == 0) {
                const uint32_t bytes = cur.bytes();
                mbar_arrive_expect_tx(bars + k, bytes);
                bulk_g2s_addr(stage0 + (uint32_t)k * C * kSegBytes, cur.addr(), bytes, bars + k);
            }
            ++issued;
            cur.advance(sa, gw);
        }
    }
};

// Grid barrier: CTA-wide arrival already made; thread 0 waits (bounded) until
// `target` arrivals or an abort.  Returns false on timeout or abort.
__device__ __forceinline__ bool grid_wait(int* sync, int target, int* err, int* flag_smem,
                                          uint32_t poll_limit) {
    if (threadIdx.x == 0) {
        int ok = 0;
        for (uint32_t it = 0; it < poll_limit; ++it) {
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
    // flag_smem is written again only after the CTA's next barriers.
    return *flag_smem != 0;
}

template <int WARPS, int R, int C, bool GATED = false>
__global__ void __launch_bounds__(WARPS * 32, 1) stack_kernel(const StackArgs sa, int kmax) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t bars[WARPS * R];
    __shared__ __align__(8) uint64_t xbar;
    __shared__ int flag;
    constexpr int NT = WARPS * 32;

    const uint32_t smem_base = smem_addr(smem);
    const uint32_t stage0_base = smem_base;
    const uint32_t xs = smem_base + (uint32_t)ring_bytes(WARPS, R, C);
    const uint32_t rec = xs + (uint32_t)kmax * 2;
    float* park = reinterpret_cast<float*>(smem + ring_bytes(WARPS, R, C) + (size_t)kmax * 3);
    float* sq = park + WARPS * 2 * 32;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gw = blockIdx.x * WARPS + warp;
    const uint32_t stage0 = stage0_base + (uint32_t)warp * R * C * kSegBytes;
    uint64_t* wbars = bars + warp * R;

    if (lane == 0) {
        for (int k = 0; k < R; ++k) mbar_init(wbars + k, 1);
        if (warp == 0) mbar_init(&xbar, 1);
        fence_barrier_init();
    }
    // The descriptors are read again and again by the cursors: pull them into
    // L1 once.
    for (int off = threadIdx.x * 128; off < sa.n_gemv * (int)sizeof(StackGemv); off += NT * 128)
        prefetch_l1(reinterpret_cast<const uint8_t*>(sa.gemv) + off);
    __syncthreads();

    StreamProducer<R, C> prod;
    prod.start(sa, gw);
    int consumed = 0;
    prod.fill(sa, gw, consumed, stage0, wbars, lane);

    bool ok = true;
    float s_prev = 1.f;                   // output scale of GEMV i-1
    int xphases = 0;                      // phases of the copy barrier completed
    for (int i = 0; i < sa.n_gemv && ok; ++i) {
        GemvArgs a = stack_view(sa, i);
        a.ws = sa.ws + (size_t)(i & 1) * sa.ws_half;
        // The warp's share of GEMV i depends on no data: set it up before the
        // barrier.  Finished output blocks go out pre-quantised for GEMV i+1.
        Dp2aConsumer<1> cons;
        cons.init(a, gw, xs, rec, park + (size_t)warp * 2 * 32);
        if (i + 1 < sa.n_gemv && !(GATED && sa.gemv[i + 1].gated)) {
            uint8_t* ob = sa.xq + (size_t)((i + 1) & 1) * sa.xq_half;
            cons.qo.x = reinterpret_cast<int16_t*>(ob);
            cons.qo.rec = reinterpret_cast<uint2*>(ob + (size_t)sa.kmax * 2);
            cons.qo.sq = reinterpret_cast<float*>(ob + (size_t)sa.kmax * 3);
            cons.qo.nb = sa.gemv[i + 1].K / 32;
        }
        if (i > 0)
            ok = grid_wait(sa.sync, i * (int)gridDim.x + (i == 1 ? sa.unreachable : 0), sa.err, &flag,
                           sa.poll_limit);
        if (!ok) break;
        if (i == 0) {
            if (a.K <= 2 * NT * 8) stage_activations<1, NT, 2>(a, xs, rec, sq);
            else stage_activations<1, NT, kStackXChunks>(a, xs, rec, sq);
        } else {
            const StackGemv& pd = sa.gemv[i - 1];
            SplitFix<WARPS> fix;
            fix.ws = sa.ws + (size_t)((i - 1) & 1) * sa.ws_half;
            fix.sc = pd.sc;
            fix.KB = pd.K / 32;
            fix.oscale = s_prev;
            fix.fill_y = pd.fill_y ? pd.y : nullptr;
            fix.fill_n = pd.N;
            fix.fill_all = false;
            if (GATED && sa.gemv[i].gated) {
                if (a.K <= 2 * NT * 8) stage_gated<WARPS, NT, 2>(sa, a.K, fix, pd.y, xs, rec, sq);
                else stage_gated<WARPS, NT, kStackXChunks>(sa, a.K, fix, pd.y, xs, rec, sq);
            } else {
                // the copy barrier completes one phase per pre-converted staging
                const uint32_t parity = GATED ? (uint32_t)(xphases & 1) : (uint32_t)((i - 1) & 1);
                stage_prequant<WARPS, NT>(sa, i, a.K, fix, xs, rec, sq, &xbar, parity);
                ++xphases;
            }
            cons.oscale = unit_rms_scale(sq, a.KB, a.K);
        }
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
        cons.flush_last(a);
        __syncthreads();
        int xt[2], xcf[2], xcl[2];   // tiles shared with other CTAs: combined by their readers
        cons.template combine_cta<WARPS>(a, park, a.ws, xt, xcf, xcl);
        s_prev = cons.oscale;
        // This CTA is done with GEMV i (outputs, CTA partials and the next
        // input's blocks written; the latter are read by bulk copies).
        fence_proxy_async_global();
        __syncthreads();
        if (threadIdx.x == 0) red_add_release_gpu(sa.sync, 1);
    }
    if (ok) ok = grid_wait(sa.sync, sa.n_gemv * (int)gridDim.x, sa.err, &flag, sa.poll_limit);
    if (ok) {
        const int il = sa.n_gemv - 1;
        const StackGemv& ld = sa.gemv[il];
        if (blockIdx.x == 0) {
            SplitFix<WARPS> fix;
            fix.ws = sa.ws + (size_t)(il & 1) * sa.ws_half;
            fix.sc = ld.sc;
            fix.KB = ld.K / 32;
            fix.oscale = s_prev;
            fix.fill_y = ld.fill_y ? ld.y : nullptr;
            fix.fill_n = ld.N;
            fix.fill_all = true;
            renorm_block<NT, kStackXChunks, true>(ld.y, sa.x_out, sa.hidden, sq, fix, xs);
        }
        // Traced inputs: GEMV j read x_in (j = 0) or GEMV j-1's output, all
        // complete now (j - 1 is not the last GEMV).
        for (int j = blockIdx.x; j < sa.n_gemv; j += gridDim.x) {
            const StackGemv& d = sa.gemv[j];
            if (d.trace_x == nullptr) continue;
            const __half* src = j == 0 ? sa.x_in : sa.gemv[j - 1].y;
            for (int q = threadIdx.x; q < d.K / 8; q += NT)
                reinterpret_cast<uint4*>(d.trace_x)[q] = __ldcg(reinterpret_cast<const uint4*>(src) + q);
        }
        return;
    }
    // Abort: let this warp's copies in flight land (bounded) before leaving.
    for (; consumed < prod.issued; ++consumed)
        mbar_wait_bounded(wbars + consumed % R, (uint32_t)((consumed / R) & 1), 1u << 22);
}

}  // namespace q4
