// Q4_0 / Q8_0 GEMM for M = 17..256 activation vectors (prefill chunks; Q8_0
// also for M = 3..16 and wide K) on the 5th-generation tensor cores:
// Y[m][n] = sum_k W[n][k] * X[m][k].
//
// Dequantise-then-multiply, the reading of "dequantise a weight tile once and
// apply it to every vector".  A weight w = q * d (q = the nibble - 8, or the
// signed byte) has up to 14 (Q4_0) or 18 (Q8_0) significant bits, more than
// binary16 holds, so it is split exactly into two binary16 values:
// main = RN(w) and rest = w - main (a multiple of d's last bit below main's
// last bit, so it has at most 7 significant bits and is representable unless
// main overflowed).
// Both parts multiply the same activations, so every weight costs two f16
// products; these are exact in fp32 and accumulate in fp32 in tensor memory,
// which leaves fp32 summation as the only error before the output rounding.
// With this many vectors the work is a dense contraction (4 * M tensor flops
// per 0.5625 weight bytes), so it runs on tcgen05.mma, not the CUDA cores.
//
// One CTA computes 256 output rows (two M = 128 accumulators) for all vectors
// over its share of K (a split of the K steps when N alone gives too few CTAs):
//   warps 0..7  dequantise the stage's weights into the A tiles (main and
//               rest parts, one tile each per accumulator) and, at the
//               end, read the accumulators back (warp w: accumulator w / 4,
//               TMEM lanes 32 (w % 4) ..);
//   warp 8      issues the bulk copies of each K step into a ring of L load
//               stages: the step's packed segments (the 576-byte Q4_0 or
//               1088-byte Q8_0 tiles of 32 rows x one block) and its slice of
//               the activation image;
//   warp 9      one thread issues the MMAs and commits them to the load
//               stage's and the A buffer's "empty" barriers, finally to the
//               accumulator barrier.
// A K step covers 64 columns (two blocks).  The A tiles (main and rest parts
// of 256 rows, 64 KB) are double-buffered apart from the load ring, so the
// copies run L steps ahead while dequantising step i + 1 overlaps the MMAs of
// step i.  Operands sit in shared memory in
// the K-major, 128-byte-swizzled canonical layout: row r of a tile is 128
// bytes at r * 128, its 16-byte chunk c stored at chunk position c ^ (r % 8);
// groups of 8 rows are 1024 bytes apart.  The activation image (written by
// tc_ximg_kernel) already holds each stage's [Mp][64] slice in that byte
// order, so one bulk copy brings it in.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

#include "device_common.cuh"

namespace q4 {

constexpr int kTcAcc = 2;                       // 128-row accumulators per CTA
constexpr int kTcRows = 128 * kTcAcc;           // output rows per CTA
constexpr int kTcTiles = kTcRows / 32;          // packed 32-row tiles per CTA
constexpr int kTcDqWarps = 4 * kTcAcc;          // dequantise / epilogue warps
constexpr int kTcIssuers = 2;                   // MMA-issuing warps (alternate K steps)
constexpr int kTcThreads = 32 * (kTcDqWarps + 1 + kTcIssuers);
constexpr int kTcMaxVec = 256;                  // MMA N limit (vectors)
constexpr int kTcAccCols = 256;                 // TMEM columns per accumulator
constexpr int kTcTmemCols = kTcAcc * kTcAccCols;
constexpr int kTcATile = 128 * 128;             // bytes of one 128-row A tile
// Packed segment of one 32-row tile and one block: Q4_0 576 bytes (codes at
// 16 (4g + c) + 4i, scales at 512), Q8_0 1088 bytes (codes at 32 (4g + c) + 8i,
// scales at 1024); a load stage holds two segments of each of the CTA's tiles.
__host__ __device__ constexpr int tc_seg_bytes(bool q8) { return q8 ? 1088 : 576; }
__host__ __device__ constexpr int tc_raw_bytes(bool q8) { return kTcTiles * 2 * tc_seg_bytes(q8); }

constexpr int kTcABytes = 2 * kTcAcc * kTcATile; // main + rest tiles of one A buffer
constexpr int kTcABufs = 2;                      // A buffers: dequantise one, multiply the other

// Bytes of one load stage for Mp vectors (the activation slice, then the
// packed bytes), a multiple of 1024 so every slice starts on a swizzle-pattern
// boundary.
__host__ __device__ constexpr uint32_t tc_load_stage_bytes(int Mp, bool q8 = false) {
    return (uint32_t)((Mp * 128 + tc_raw_bytes(q8) + 1023) / 1024 * 1024);
}
// Dynamic shared memory of the kernel with L load stages: 1024 bytes of
// alignment slack, the A buffers, the load stages, the barriers (2 per load
// stage, 2 per A buffer, 1), the TMEM address word and the abort flag.
__host__ __device__ constexpr uint32_t tc_smem_bytes(int Mp, int L, bool q8 = false, bool at = false) {
    return 1024 + (at ? 0u : (uint32_t)(kTcABufs * kTcABytes)) + (uint32_t)L * tc_load_stage_bytes(Mp, q8) +
           8u * (2 * L + 2 * kTcABufs + 1) + 16;
}
// With A in tensor memory (MMA width Mp <= 128): accumulators at columns
// 128 acc, the two A buffers at 256 + 128 b (per accumulator 64 columns: the
// main part's 64 K values, then the rest part's).
constexpr int kTcAtMaxVec = 128;

// Instruction descriptor of tcgen05.mma kind::f16: f16 A and B, both K-major,
// fp32 accumulator, no negation or sparsity, shape m x n.
__host__ __device__ constexpr uint32_t tc_idesc_f16(int m, int n) {
    return (1u << 4)                         // accumulator format: f32
           | (0u << 7) | (0u << 10)          // A, B format: f16
           | (0u << 15) | (0u << 16)         // A, B: K-major
           | ((uint32_t)(n >> 3) << 17)      // N / 8
           | ((uint32_t)(m >> 4) << 24);     // M / 16
}

// Shared-memory matrix descriptor of a K-major, 128-byte-swizzled operand
// whose 8-row groups are 1024 bytes apart, starting at shared address `saddr`.
__host__ __device__ constexpr uint64_t tc_sdesc_sw128(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu)          // start address / 16
           | ((uint64_t)1 << 16)                       // leading offset (unused when swizzled)
           | ((uint64_t)(1024 >> 4) << 32)             // stride offset: next 8-row group
           | ((uint64_t)1 << 46)                       // descriptor version (sm_100)
           | ((uint64_t)2 << 61);                      // 128-byte swizzle
}

// ---- tcgen05 wrappers -----------------------------------------------------

__device__ __forceinline__ void tc_alloc(uint32_t* slot, uint32_t ncols) {   // whole warp
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_addr(slot)), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_dealloc(uint32_t taddr, uint32_t ncols) {   // whole warp
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                 :: "r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D (+)= A * B^T for one 16-column K slice; `acc` = 0 overwrites D.
__device__ __forceinline__ void tc_mma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc, uint32_t acc) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 :: "r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc) : "memory");
}
// D (+)= A * B^T for one 16-column K slice with A in tensor memory (`tmem_a`:
// lane = row, 8 columns = 16 f16 K values in order); `acc` = 0 overwrites D.
__device__ __forceinline__ void tc_mma_f16_ta(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc,
                                              uint32_t idesc, uint32_t acc) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
                 :: "r"(tmem_d), "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(acc) : "memory");
}
// Eight registers into the tcgen05.st 16x256b fragment, two repetitions:
// thread 4g + c writes TMEM lanes g (r0, r1, r4, r5) and g + 8 (r2, r3, r6,
// r7) of the 16-lane group at `taddr`, 32-bit columns 2c, 2c + 1 (r0..r3)
// and 8 + 2c, 9 + 2c (r4..r7).
__device__ __forceinline__ void tc_st16x256b_x2(uint32_t taddr, uint2 a0, uint2 a1, uint2 b0, uint2 b1) {
    asm volatile("tcgen05.st.sync.aligned.16x256b.x2.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
                 ::"r"(taddr), "r"(a0.x), "r"(a0.y), "r"(a1.x), "r"(a1.y), "r"(b0.x), "r"(b0.y),
                   "r"(b1.x), "r"(b1.y)
                 : "memory");
}
__device__ __forceinline__ void tc_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// Arrives once on `bar` when every MMA this thread issued so far has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(smem_addr(bar)) : "memory");
}
// 16 consecutive fp32 columns of this thread's TMEM lane, waited for in the
// same statement so no use of the registers can move above the wait.
__device__ __forceinline__ void tc_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
                 "tcgen05.wait::ld.sync.aligned;"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                   "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]),
                   "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
                 : "r"(taddr) : "memory");
}

__device__ __forceinline__ int ld_acquire_cta_shared(const int* p) {
    int v;
    asm volatile("ld.acquire.cta.shared::cta.b32 %0, [%1];" : "=r"(v) : "r"(smem_addr(p)) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_cta_shared(int* p, int v) {
    asm volatile("st.release.cta.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(p)), "r"(v) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_addr(bar)) : "memory");
}

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    for (uint32_t i = 0; i < (1u << 22); ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63) == 63 && *abort_flag) return false;
    }
    return false;
}

struct TcArgs {
    const uint8_t* W;    // packed Q4_0 (576-byte segments) or Q8_0 (1088-byte) matrix
    const uint8_t* xi;   // activation image: [nk][Mp][128 bytes], swizzled rows
    __half* y;           // [M][N] (P == 1)
    float* ypart;        // [P][M][N] fp32 split sums (P > 1)
    int* err;
    int64_t N;
    int KB, T;           // blocks per row, packed tiles ceil(N / 32)
    int M, Mp;           // vectors; MMA N = Mp = M rounded up to 16
    int nk, nkp, P;      // K steps, steps per split, splits
    int L;               // load stages
    uint32_t idesc;      // tc_idesc_f16(128, Mp)
};

// Exact split of one (q - 8) * d pair: main = RN(q * d), rest = q * d - main
// (the fused multiply-add rounds the exact remainder, which is representable).
__device__ __forceinline__ void tc_split2(__half2 q, __half2 dd, uint32_t& m, uint32_t& r) {
    const __half2 hm = __hmul2(q, dd);
    const __half2 hr = __hfma2(q, dd, __hneg2(hm));
    m = *reinterpret_cast<const uint32_t*>(&hm);
    r = *reinterpret_cast<const uint32_t*>(&hr);
}

// Four weights of one packed word (bytes e = 0..3; low nibbles are codes
// 4c + e, high nibbles codes 16 + 4c + e), in code order, 8 bytes per set:
// lm / lr = main / rest parts of the low-nibble weights, hm / hr of the high.
// 0x6400 | q is the f16 1024 + q; 0x5400 | (q << 4) is the f16 64 + q; the
// subtractions leave q - 8 exactly.
__device__ __forceinline__ void tc_dequant_word(uint32_t w, __half2 dd, uint2& lm, uint2& lr,
                                                uint2& hm, uint2& hr) {
    const uint32_t p01 = __byte_perm(w, 0u, 0x4140);   // bytes 0, 1 -> 16-bit lanes
    const uint32_t p23 = __byte_perm(w, 0u, 0x4342);   // bytes 2, 3
    const __half2 k1032 = __half2half2(__ushort_as_half((unsigned short)0x6408));   // 1032
    const __half2 k72 = __half2half2(__ushort_as_half((unsigned short)0x5480));     // 72
    const uint32_t l01 = (p01 & 0x000F000Fu) | 0x64006400u;
    const uint32_t l23 = (p23 & 0x000F000Fu) | 0x64006400u;
    const uint32_t h01 = (p01 & 0x00F000F0u) | 0x54005400u;
    const uint32_t h23 = (p23 & 0x00F000F0u) | 0x54005400u;
    tc_split2(__hsub2(*reinterpret_cast<const __half2*>(&l01), k1032), dd, lm.x, lr.x);
    tc_split2(__hsub2(*reinterpret_cast<const __half2*>(&l23), k1032), dd, lm.y, lr.y);
    tc_split2(__hsub2(*reinterpret_cast<const __half2*>(&h01), k72), dd, hm.x, hr.x);
    tc_split2(__hsub2(*reinterpret_cast<const __half2*>(&h23), k72), dd, hm.y, hr.y);
}

// Four signed 8-bit codes of one word (byte e = code e), as f16 q * d in code
// order, split into main and rest parts (8 bytes each).  (b ^ 0x80) | 0x6400 is
// the f16 1024 + (q + 128); subtracting 1152 leaves q exactly.
__device__ __forceinline__ void tc_dequant_word_q8(uint32_t w, __half2 dd, uint2& m, uint2& r) {
    const __half2 k1152 = __half2half2(__ushort_as_half((unsigned short)0x6480));   // 1152
    const uint32_t p01 = (__byte_perm(w, 0u, 0x4140) ^ 0x00800080u) | 0x64006400u;
    const uint32_t p23 = (__byte_perm(w, 0u, 0x4342) ^ 0x00800080u) | 0x64006400u;
    tc_split2(__hsub2(*reinterpret_cast<const __half2*>(&p01), k1152), dd, m.x, r.x);
    tc_split2(__hsub2(*reinterpret_cast<const __half2*>(&p23), k1152), dd, m.y, r.y);
}

// AT: the A tiles in tensor memory (Mp <= 128) instead of shared memory.
template <bool Q8, bool AT = false>
__global__ void __launch_bounds__(kTcThreads, 1) gemm_tc_kernel(const TcArgs a) {
    constexpr int SEG = tc_seg_bytes(Q8), SCL = Q8 ? 1024 : 512;
    constexpr uint32_t kAccCols = AT ? (uint32_t)kTcAtMaxVec : (uint32_t)kTcAccCols;
    extern __shared__ uint8_t tc_smem_raw[];
    const int L = a.L;
    const uint32_t ld_bytes = tc_load_stage_bytes(a.Mp, Q8);
    const uint32_t raw0 = smem_addr(tc_smem_raw);
    const uint32_t base = (raw0 + 1023u) & ~1023u;               // swizzle needs 1024-byte tiles
    const uint32_t ld0 = base + (AT ? 0u : (uint32_t)(kTcABufs * kTcABytes));  // first load stage
    uint8_t* gbar = tc_smem_raw + (ld0 - raw0) + (size_t)L * ld_bytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(gbar);          // [L] copies landed
    uint64_t* lempty = full + L;                                 // [L] MMAs done with the stage
    uint64_t* aready = lempty + L;                               // [2] A buffer written
    uint64_t* aempty = aready + kTcABufs;                        // [2] MMAs done with the buffer
    uint64_t* accbar = aempty + kTcABufs;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(accbar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
    __shared__ int mma_turn_word;                                // next K step whose MMAs may be issued
    int* mma_turn = &mma_turn_word;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = blockIdx.x * kTcTiles;                       // first packed tile
    const int p = blockIdx.y;
    const int k0 = p * a.nkp;
    const int ns = min(a.nk, k0 + a.nkp) - k0;                  // this split's K steps (>= 1)
    const uint32_t bbytes = (uint32_t)a.Mp * 128u;

    if (threadIdx.x == 0) {
        for (int j = 0; j < L; ++j) {
            mbar_init(full + j, 1);
            mbar_init(lempty + j, 1);
        }
        for (int b = 0; b < kTcABufs; ++b) {
            mbar_init(aready + b, kTcDqWarps);
            mbar_init(aempty + b, 1);
        }
        mbar_init(accbar, kTcIssuers);
        *abort_flag = 0;
        *mma_turn = 0;
        fence_barrier_init();
    }
    if (warp == 0) tc_alloc(tslot, kTcTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    if (warp == kTcDqWarps) {
        // ---- producer: bulk copies of each K step into load stage i % L ----
        if (lane == 0) {
            // Launched as a dependent of the activation-image kernel: the
            // image (and anything earlier in the stream) is complete and
            // visible after this wait; the prologue above overlapped it.
            pdl_wait();
            const int ntiles = min(kTcTiles, a.T - t0);
            int i = 0;
            for (; i < ns; ++i) {
                const int j = i % L;
                if (i >= L && !tc_wait(lempty + j, (uint32_t)((i / L - 1) & 1), abort_flag)) {
                    *abort_flag = 1;
                    set_device_error(a.err, kDevTimeout);
                    break;
                }
                const int ks = k0 + i, b0 = 2 * ks;
                const int nb = min(2, a.KB - b0);
                const uint32_t sB = ld0 + (uint32_t)j * ld_bytes, sraw = sB + bbytes;
                mbar_arrive_expect_tx(full + j, (uint32_t)(ntiles * nb * SEG) + bbytes);
                for (int t = 0; t < ntiles; ++t)
                    bulk_g2s_addr(sraw + (uint32_t)(t * 2 * SEG),
                                  a.W + ((size_t)(t0 + t) * a.KB + b0) * SEG, (uint32_t)(nb * SEG),
                                  full + j);
                bulk_g2s_addr(sB, a.xi + (size_t)ks * bbytes, bbytes, full + j);
            }
            // Copies still in flight must land before the CTA exits: wait for
            // the last phase issued on every stage (already complete normally).
            for (int j = 0; j < L && j < i; ++j) {
                const int last = j + ((i - 1 - j) / L) * L;
                mbar_wait_bounded(full + j, (uint32_t)((last / L) & 1), 1u << 22);
            }
        }
    } else if (warp > kTcDqWarps) {
        // ---- MMA issuers: issuer q takes the K steps i with i % 2 == q.  It
        // waits for its step's operands while the other issues, then for its
        // turn (the MMAs enter the tensor pipe in step order, so the
        // accumulation order is the step order and step 0's MMAs overwrite
        // first); a tcgen05 fence before handing the turn on and after taking
        // it orders the two threads' MMAs. ----
        const int q = warp - (kTcDqWarps + 1);
        if (lane == 0) {
            for (int i = q; i < ns; i += kTcIssuers) {
                const int j = i % L, b = i & 1;
                bool got = tc_wait(aready + b, (uint32_t)((i >> 1) & 1), abort_flag) &&
                           tc_wait(full + j, (uint32_t)((i / L) & 1), abort_flag);
                for (uint32_t it = 0; got; ++it) {
                    if (ld_acquire_cta_shared(mma_turn) == i) break;
                    if (it >= (1u << 24) || ((it & 63) == 63 && *abort_flag)) got = false;
                }
                if (!got) {
                    *abort_flag = 1;
                    set_device_error(a.err, kDevTimeout);
                    break;
                }
                tc_fence_after();
                const uint32_t sA = base + (uint32_t)(b * kTcABytes);
                const uint32_t sB = ld0 + (uint32_t)j * ld_bytes;
                if constexpr (AT) {
                    const uint32_t tA = tmem + 256u + (uint32_t)b * 128u;
#pragma unroll
                    for (int acc = 0; acc < kTcAcc; ++acc)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t bdesc = tc_sdesc_sw128(sB + (uint32_t)(32 * kk));
                            const uint32_t ta = tA + (uint32_t)(acc * 64 + 8 * kk);
                            tc_mma_f16_ta(tmem + (uint32_t)(acc * kAccCols), ta, bdesc, a.idesc,
                                          (uint32_t)(i | kk));
                            tc_mma_f16_ta(tmem + (uint32_t)(acc * kAccCols), ta + 32u, bdesc, a.idesc, 1u);
                        }
                } else
#pragma unroll
                for (int acc = 0; acc < kTcAcc; ++acc)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t bdesc = tc_sdesc_sw128(sB + (uint32_t)(32 * kk));
                        const uint32_t am = sA + (uint32_t)(acc * kTcATile + 32 * kk);
                        tc_mma_f16(tmem + (uint32_t)(acc * kTcAccCols), tc_sdesc_sw128(am), bdesc,
                                   a.idesc, (uint32_t)(i | kk));
                        tc_mma_f16(tmem + (uint32_t)(acc * kTcAccCols),
                                   tc_sdesc_sw128(am + (uint32_t)(kTcAcc * kTcATile)), bdesc,
                                   a.idesc, 1u);
                    }
                tc_commit(lempty + j);
                tc_commit(aempty + b);
                tc_fence_before();
                st_release_cta_shared(mma_turn, i + 1);
            }
            tc_commit(accbar);        // also after an abort: tracks every MMA this thread issued
        }
    } else {
        // ---- dequantise: the thread with pair (g, c) takes the 16 bytes at
        // 16 (4g + c) of tile w's segments: rows g + 8i (i = 0..3), codes
        // 4c..4c+3 and 16+4c..16+4c+3 of each block.  The lane -> (g, c) map
        // (g bits: lane bit 0, bit 3, bit 0 ^ bit 4; c: lane bits 1-2) makes
        // every quarter-warp's 16-byte loads and every half-warp's 8-byte
        // swizzled stores hit distinct banks ----
        if constexpr (AT) {
        // With A in tensor memory the thread is 4g + c (the tcgen05.st
        // 16x256b fragment: TMEM lanes g and g + 8, columns 2c, 2c + 1 and
        // 8 + 2c, 9 + 2c) and its 16 bytes are at 16 (4g + c): a warp's loads
        // cover 512 contiguous bytes.  Columns 16h + 2c.. then hold K values
        // 32h + 4c + e and columns 16h + 8 + 2c.. K values 32h + 16 + 4c + e:
        // the natural K order, as in the activation image.
        const int g = lane >> 2;
        const int acc = warp >> 2;
        const uint32_t trows = (uint32_t)(32 * (warp & 3)) << 16;
        for (int i = 0; i < ns; ++i) {
            const int j = i % L, b = i & 1;
            const bool got = tc_wait(full + j, (uint32_t)((i / L) & 1), abort_flag) &&
                             (i < kTcABufs ||
                              tc_wait(aempty + b, (uint32_t)(((i >> 1) - 1) & 1), abort_flag));
            if (!__all_sync(0xFFFFFFFFu, got)) {       // the warp leaves together
                *abort_flag = 1;
                set_device_error(a.err, kDevTimeout);
                break;
            }
            tc_fence_after();
            const uint32_t tA = tmem + trows + 256u + (uint32_t)b * 128u + (uint32_t)acc * 64u;
            const uint32_t sraw = ld0 + (uint32_t)j * ld_bytes + bbytes + (uint32_t)(warp * 2 * SEG);
            const int nb = min(2, a.KB - 2 * (k0 + i));
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t wv[Q8 ? 8 : 4];
                uint2 sc = make_uint2(0, 0);
                if (h < nb) {
                    const uint32_t seg = sraw + (uint32_t)(h * SEG);
                    if constexpr (Q8) {
                        const uint4 u0 = lds128(seg + (uint32_t)(32 * lane));
                        const uint4 u1 = lds128(seg + (uint32_t)(32 * lane + 16));
                        wv[0] = u0.x; wv[1] = u0.y; wv[2] = u0.z; wv[3] = u0.w;
                        wv[4] = u1.x; wv[5] = u1.y; wv[6] = u1.z; wv[7] = u1.w;
                    } else {
                        const uint4 u0 = lds128(seg + (uint32_t)(16 * lane));
                        wv[0] = u0.x; wv[1] = u0.y; wv[2] = u0.z; wv[3] = u0.w;
                    }
                    sc = lds64(seg + (uint32_t)(SCL + 8 * g));
                } else {
#pragma unroll
                    for (int e = 0; e < (Q8 ? 8 : 4); ++e) wv[e] = 0;
                }
                const uint32_t sv[4] = {sc.x, sc.x >> 16, sc.y, sc.y >> 16};
                uint2 lm[4], lr[4], hm[4], hr[4];            // rows g + 8ii
#pragma unroll
                for (int ii = 0; ii < 4; ++ii) {
                    const __half2 dd = __half2half2(__ushort_as_half((unsigned short)(sv[ii] & 0xFFFFu)));
                    if constexpr (Q8) {
                        tc_dequant_word_q8(wv[2 * ii], dd, lm[ii], lr[ii]);
                        tc_dequant_word_q8(wv[2 * ii + 1], dd, hm[ii], hr[ii]);
                    } else {
                        tc_dequant_word(wv[ii], dd, lm[ii], lr[ii], hm[ii], hr[ii]);
                    }
                    if (h >= nb) { lm[ii] = make_uint2(0, 0); lr[ii] = lm[ii]; hm[ii] = lm[ii]; hr[ii] = lm[ii]; }
                }
                const uint32_t col = tA + (uint32_t)(16 * h);
                tc_st16x256b_x2(col, lm[0], lm[1], hm[0], hm[1]);                       // main, rows g, g + 8
                tc_st16x256b_x2(col + 32u, lr[0], lr[1], hr[0], hr[1]);                 // rest
                tc_st16x256b_x2(col + (16u << 16), lm[2], lm[3], hm[2], hm[3]);         // rows g + 16, g + 24
                tc_st16x256b_x2(col + (16u << 16) + 32u, lr[2], lr[3], hr[2], hr[3]);
            }
            tc_wait_st();
            tc_fence_before();            // tensor-memory writes -> the MMAs
            __syncwarp();
            if (lane == 0) mbar_arrive(aready + b);
        }
        } else {
        const int g = (lane & 1) | ((lane >> 2) & 2) | (((lane ^ (lane >> 4)) & 1) << 2);
        const int c = (lane >> 1) & 3;
        const int acc = warp >> 2;
        const uint32_t arow0 = (uint32_t)((warp & 3) * 32 + g);      // A row of i = 0
        for (int i = 0; i < ns; ++i) {
            const int j = i % L, b = i & 1;
            const bool got = tc_wait(full + j, (uint32_t)((i / L) & 1), abort_flag) &&
                             (i < kTcABufs ||
                              tc_wait(aempty + b, (uint32_t)(((i >> 1) - 1) & 1), abort_flag));
            if (!__all_sync(0xFFFFFFFFu, got)) {       // the warp leaves together
                *abort_flag = 1;
                set_device_error(a.err, kDevTimeout);
                break;
            }
            const uint32_t sA = base + (uint32_t)(b * kTcABytes + acc * kTcATile);   // main part
            const uint32_t sR = sA + (uint32_t)(kTcAcc * kTcATile);                 // rest part
            const uint32_t sraw = ld0 + (uint32_t)j * ld_bytes + bbytes + (uint32_t)(warp * 2 * SEG);
            const int nb = min(2, a.KB - 2 * (k0 + i));
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                // Q4_0: one 16-byte word per row i (row g + 8i), low nibbles codes
                // 4c.., high nibbles 16 + 4c..; Q8_0: two words per row, codes 4c..
                // then 16 + 4c...
                uint32_t wv[Q8 ? 8 : 4];
                uint2 sc = make_uint2(0, 0);
                if (h < nb) {
                    const uint32_t seg = sraw + (uint32_t)(h * SEG);
                    if constexpr (Q8) {
                        const uint4 u0 = lds128(seg + (uint32_t)(32 * (4 * g + c)));
                        const uint4 u1 = lds128(seg + (uint32_t)(32 * (4 * g + c) + 16));
                        wv[0] = u0.x; wv[1] = u0.y; wv[2] = u0.z; wv[3] = u0.w;
                        wv[4] = u1.x; wv[5] = u1.y; wv[6] = u1.z; wv[7] = u1.w;
                    } else {
                        const uint4 u0 = lds128(seg + (uint32_t)(16 * (4 * g + c)));
                        wv[0] = u0.x; wv[1] = u0.y; wv[2] = u0.z; wv[3] = u0.w;
                    }
                    sc = lds64(seg + (uint32_t)(SCL + 8 * g));
                } else {
#pragma unroll
                    for (int e = 0; e < (Q8 ? 8 : 4); ++e) wv[e] = 0;
                }
                const uint32_t sv[4] = {sc.x, sc.x >> 16, sc.y, sc.y >> 16};
#pragma unroll
                for (int ii = 0; ii < 4; ++ii) {
                    const __half2 dd = __half2half2(__ushort_as_half((unsigned short)(sv[ii] & 0xFFFFu)));
                    uint2 lm, lr, hm, hr;
                    if constexpr (Q8) {
                        tc_dequant_word_q8(wv[2 * ii], dd, lm, lr);
                        tc_dequant_word_q8(wv[2 * ii + 1], dd, hm, hr);
                    } else {
                        tc_dequant_word(wv[ii], dd, lm, lr, hm, hr);
                    }
                    if (h >= nb) { lm = make_uint2(0, 0); lr = lm; hm = lm; hr = lm; }
                    const uint32_t r = arow0 + 8u * (uint32_t)ii;    // r % 8 == g
                    const uint32_t off = r * 128u + (uint32_t)(c & 1) * 8u;
                    const uint32_t chl = (uint32_t)(4 * h + (c >> 1));   // columns 32h + 4c ..
                    const uint32_t chh = chl + 2u;                       // columns 32h + 16 + 4c ..
                    const uint32_t ol = off + ((chl ^ (uint32_t)g) << 4);
                    const uint32_t oh = off + ((chh ^ (uint32_t)g) << 4);
                    sts64(sA + ol, lm);
                    sts64(sA + oh, hm);
                    sts64(sR + ol, lr);
                    sts64(sR + oh, hr);
                }
            }
            fence_proxy_async_smem();      // this thread's tile writes -> tensor-core reads
            __syncwarp();
            if (lane == 0) mbar_arrive(aready + b);
        }

        }

        // ---- epilogue: accumulator rows -> y (or the split's fp32 sums) ----
        // tcgen05.ld is warp-collective: the decision to read is made per warp.
        const int acc = warp >> 2;
        const bool ok = __all_sync(0xFFFFFFFFu, tc_wait(accbar, 0u, abort_flag) && !*abort_flag);
        tc_fence_after();
        if (ok) {
            const int64_t n = (int64_t)blockIdx.x * kTcRows + acc * 128 + (warp & 3) * 32 + lane;
            const uint32_t taddr = tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(acc * kAccCols);
            for (int c0 = 0; c0 < a.Mp; c0 += 16) {
                uint32_t v[16];
                tc_ld16(taddr + (uint32_t)c0, v);
                if (n < a.N) {
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) {
                        const int m = c0 + jj;
                        if (m < a.M) {
                            const float f = __uint_as_float(v[jj]);
                            if (a.P == 1)
                                a.y[(size_t)m * a.N + n] = __float2half_rn(f);
                            else
                                a.ypart[((size_t)p * a.M + m) * a.N + n] = f;
                        }
                    }
                }
            }
        } else if (threadIdx.x == 0) {
            set_device_error(a.err, kDevTimeout);
        }
    }

    __syncwarp();        // single-lane roles rejoin their warps
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tc_dealloc(tmem, kTcTmemCols);
    }
}

// Activation image of x[M][K] for gemm_tc_kernel: for each 64-column step ks,
// Mp rows of 128 bytes, row m's 16-byte chunk c (columns 64 ks + 8c ..) at
// chunk position c ^ (m % 8); rows m >= M and columns >= K are zero.
static __global__ void __launch_bounds__(256) tc_ximg_kernel(const __half* __restrict__ x,
                                                           uint8_t* __restrict__ img, int M, int K,
                                                           int Mp, int nk) {
    pdl_launch_dependents();      // the GEMM may start its prologue now
    const int64_t total = (int64_t)nk * Mp * 8;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < total; q += stride) {
        const int64_t ks = q / ((int64_t)Mp * 8);
        const int rem = (int)(q - ks * Mp * 8);
        const int m = rem >> 3, c = rem & 7;
        const int64_t k = ks * 64 + c * 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (m < M && k < K) v = *reinterpret_cast<const uint4*>(x + (size_t)m * K + k);
        *reinterpret_cast<uint4*>(img + ((size_t)ks * Mp + m) * 128 + ((c ^ (m & 7)) << 4)) = v;
    }
}

}  // namespace q4
