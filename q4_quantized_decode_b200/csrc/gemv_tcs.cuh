// Q4_0 GEMV for a few activation vectors (M <= 16) on the 5th-generation
// tensor cores: tcgen05.mma kind::i8 with the weights in tensor memory and
// exact int32 block sums in tensor memory.
//
// Speculative verification applies the decode weights to a handful of draft
// tokens, and prefill chunks to 16 or so (aipolix en-US page, section
// "Speculation is used to amortize network round trips"; originshq.com page,
// section "Multi-Device Performance and the Network Penalty").  The weight
// stream is the decode stream; only the work per weight grows with M.  Here
// one unit -- 128 rows (four packed 32-row tiles) of one 32-column block --
// is ONE tensor-core instruction (K = 32):
//   A (128 x 32, signed 8-bit, in tensor memory: lane = row): 16 (q - 8), the
//     nibble moved to the top of its byte with the top bit flipped -- one
//     LOP3 (and a shift) per four codes;
//   B (2V x 32, signed 8-bit, shared memory): per vector m the block's
//     activations as integers X = rint(v 2^(14-E)) (E: the block maximum is
//     below 2^E, so |X| <= 2^14; exact for the block maximum and every entry
//     within a factor 2^3 of it, 2^-15 of the maximum otherwise -- the
//     conversion of the M <= 2 path), split exactly as X = 256 Xh + Xl with
//     Xh = (X + 128) >> 8 in [-64, 64] and Xl in [-128, 127]: rows 2m (Xl)
//     and 2m + 1 (Xh); V = 8 or 16 vectors;
//   D (128 x 2V, int32, tensor memory, a fresh accumulator per unit): columns
//     2m and 2m + 1 hold 16 sum (q - 8) Xl and 16 sum (q - 8) Xh, so
//     T = D[2m] + 256 D[2m + 1] = 16 sum_j (q_nj - 8) X_mj exactly (|T| <=
//     2^26 with four trailing zeros: exact in fp32).
// The epilogue adds T * (d_n * 2^(E_m - 14) / 16) to an fp32 sum per row and
// vector (one FMA after the integer combine), over the blocks in order.
//
// A tensor-core instruction costs about the same time at N = 16 as at twice
// that, so the kernel is built around issuing as few as possible: 8-bit
// operands cover K = 32 per instruction (f16 covers 16).  A is written to
// tensor memory (tcgen05.st), not shared memory: shared memory carries only
// the packed weights (bulk copy in, one read) and the activation image.
//
// The CTA walks its units in load stages of up to kTcsS consecutive units of
// one 128-row block; every role synchronises once per stage, not per unit:
//   8 warps    dequantise (two groups of four taking alternate stages; warp t
//              of a group the packed tile t of each unit of the stage) into
//              an A group in tensor memory, TMEM lanes 32t.. (a warp reaches
//              only its own quarter of the lanes), with the rows' block scales
//              and the vectors' block scales into shared memory;
//   4 warps    read back the stage's accumulator group (tcgen05.ld; epilogue
//              warp e reads TMEM lanes 32e.., the rows of tile e), scale and
//              sum as above, and release the accumulator group and the scale
//              slot;
//   2 warps    issue the bulk copies of alternate load stages (one contiguous
//              run of segments per tile, and the activation image of its
//              blocks; one thread issues a bulk copy only every ~200 cycles);
//   2 warps    issue the MMAs (one per unit; the two take alternate stages)
//              and commit them once per stage: the stage's completion frees
//              its accumulator group for the epilogue, its A group and its
//              load stage (B is read from the stage).  A commit occupies the
//              tensor pipe about as long as a small MMA, so there is one.
// Independent rings -- load stages, A groups and accumulator groups in
// tensor memory, scale slots, stage completions -- so no role waits on a
// chain of the others longer than one hand-off.  Barrier waits test the
// phase first and otherwise sleep in try_wait.
//
// The units u = row block * KB + block (row-block major) are split flat over
// the CTAs (every SM streams the same bytes).  A row block whose blocks lie in
// one CTA is written directly; otherwise each contributing CTA leaves an fp32
// partial per row and warp, and the last to arrive -- per (row block, warp)
// counter -- sums them in CTA order, writes y and re-arms the counter: the
// result does not depend on the arrival order.
//
// The K order inside a block is permuted the same way in A and B (a dot
// product does not depend on the order of its terms): K slot s holds code
// 4 (s / 8) + s % 4 for s % 8 < 4 and 16 + 4 (s / 8) + s % 4 otherwise -- the
// low and high nibbles of word s / 8 of the row, as the tcgen05.st 16x256b
// fragment places them (thread 4g + c: TMEM lanes g and g + 8, 32-bit
// columns 2c (low nibbles) and 2c + 1 (high nibbles); a column holds K slots
// 4col .. 4col + 3, one per byte).
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

#include "gemm_tc.cuh"
#include "partition.cuh"

namespace q4 {

constexpr int kTcsS = 4;                             // units per load stage (at most)
constexpr int kTcsG = 2;                             // dequantise groups
constexpr int kTcsDq = 4 * kTcsG;                    // dequantise warps
constexpr int kTcsEp = 4;                            // epilogue warps
constexpr int kTcsIss = 2;                           // MMA-issuing warps (alternate stages)
constexpr int kTcsProd = 2;                          // bulk-copy warps (alternate stages)
constexpr int kTcsThreads = 32 * (kTcsDq + kTcsEp + kTcsProd + kTcsIss);
constexpr int kTcsL = 10;                            // load stages
constexpr int kTcsNSB = 8;                           // scale slots in shared memory (one stage each)
// "Stage's MMAs completed" barriers (one commit per stage, awaited by the
// epilogue, the dequantise warps reusing the A group and the bulk-copy warp
// reusing the load stage): a ring longer than the load ring, so no slot can
// complete again before its slowest waiter (the copy warp, kTcsL stages
// behind) has seen it.
constexpr int kTcsNM = kTcsL + 2;
constexpr int kTcsACols = 8;                         // TMEM columns of one unit's A (32 bytes a row)
constexpr int kTcsTmemCols = 512;
constexpr int kTcsSBytes = kTcsS * (128 + 16) * 4;   // one stage's row scales and vector scales
// Tensor-memory rings (one stage each): accumulator groups of 4 x 2V columns
// and A groups of 4 x 8 columns, as many as fit in the 512 columns.
__host__ __device__ constexpr int tcs_ndg(int V) { return V == 8 ? 4 : 3; }
__host__ __device__ constexpr int tcs_nag(int V) { return V == 8 ? 6 : 4; }

// Vectors the MMA covers: 8 (M <= 8) or 16 (M <= 16); the MMA width is twice.
__host__ __device__ constexpr int tcs_vecs(int M) { return M <= 8 ? 8 : 16; }
// Activation image of one block: 2V rows of 32 bytes in 8-row x 16-byte core
// matrices (tcs_core_off), then V fp32 vector scales 2^(E - 14) / 16.
__host__ __device__ constexpr int tcs_img_blk(int V) { return 2 * V * 32 + V * 4; }
// One load stage: 4 tile runs of kTcsS segments, then the image of kTcsS blocks.
__host__ __device__ constexpr int tcs_stage_bytes(int V) { return kTcsS * (4 * 576 + tcs_img_blk(V)); }
__host__ __device__ constexpr int tcs_smem_bytes(int V) {
    return 128 + kTcsL * tcs_stage_bytes(V) + kTcsNSB * kTcsSBytes +
           8 * (kTcsL + kTcsNM + tcs_nag(V) + tcs_ndg(V) + 2 * kTcsNSB + kTcsIss) + 16;
}

// Shared-memory matrix descriptor of a K-major operand without swizzle with
// 32-byte rows (K = 32 8-bit values) in 8-row x 16-byte core matrices: core
// matrix (8-row group r, 16-byte K chunk k) at saddr + (2 r + k) * 128, i.e.
// the K-adjacent core matrix 128 bytes on (leading offset) and the next 8-row
// group 256 bytes on (stride offset).
__host__ __device__ constexpr uint64_t tcs_sdesc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu)      // start address / 16
           | ((uint64_t)(128 >> 4) << 16)          // leading offset: next K chunk
           | ((uint64_t)(256 >> 4) << 32)          // stride offset: next 8-row group
           | ((uint64_t)1 << 46);                  // descriptor version (sm_100); no swizzle
}
// Byte offset of (row r, K chunk k) in that layout.
__host__ __device__ constexpr uint32_t tcs_core_off(int r, int k) {
    return (uint32_t)(((r >> 3) * 2 + k) * 128 + (r & 7) * 16);
}
// Instruction descriptor of tcgen05.mma kind::i8: signed 8-bit A and B, both
// K-major, int32 accumulator, M = 128, width n.
__host__ __device__ constexpr uint32_t tcs_idesc_i8(int n) {
    return (2u << 4)                         // accumulator format: S32
           | (1u << 7) | (1u << 10)          // A, B: signed 8-bit
           | (0u << 15) | (0u << 16)         // A, B: K-major
           | ((uint32_t)(n >> 3) << 17)      // N / 8
           | ((uint32_t)(128 >> 4) << 24);   // M / 16
}

// NC = 8, 16, 32 or 64 consecutive fp32 columns of this thread's TMEM lane,
// waited for in the same statement.
template <int NC>
__device__ __forceinline__ void tcs_ld(uint32_t taddr, uint32_t (&v)[NC]) {
    if constexpr (NC == 64) {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x64.b32 "
                     "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                     "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
                     "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
                     "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
                     "tcgen05.wait::ld.sync.aligned;"
                     : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
                       "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
                       "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
                       "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
                       "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
                       "=r"(v[31]), "=r"(v[32]), "=r"(v[33]), "=r"(v[34]), "=r"(v[35]), "=r"(v[36]),
                       "=r"(v[37]), "=r"(v[38]), "=r"(v[39]), "=r"(v[40]), "=r"(v[41]), "=r"(v[42]),
                       "=r"(v[43]), "=r"(v[44]), "=r"(v[45]), "=r"(v[46]), "=r"(v[47]), "=r"(v[48]),
                       "=r"(v[49]), "=r"(v[50]), "=r"(v[51]), "=r"(v[52]), "=r"(v[53]), "=r"(v[54]),
                       "=r"(v[55]), "=r"(v[56]), "=r"(v[57]), "=r"(v[58]), "=r"(v[59]), "=r"(v[60]),
                       "=r"(v[61]), "=r"(v[62]), "=r"(v[63])
                     : "r"(taddr) : "memory");
    } else if constexpr (NC == 32) {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                     "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                     "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
                     "tcgen05.wait::ld.sync.aligned;"
                     : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                       "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]),
                       "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]),
                       "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
                       "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]),
                       "=r"(v[30]), "=r"(v[31])
                     : "r"(taddr) : "memory");
    } else if constexpr (NC == 16) {
        tc_ld16(taddr, v);
    } else {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n\t"
                     "tcgen05.wait::ld.sync.aligned;"
                     : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                       "=r"(v[6]), "=r"(v[7])
                     : "r"(taddr) : "memory");
    }
}

// Four registers into the 16x256b fragment: thread 4g + c writes TMEM lanes
// g (r.x, r.y) and g + 8 (r.z, r.w) of the 16-lane group at `taddr`, 32-bit
// columns 2c (r.x, r.z) and 2c + 1 (r.y, r.w).
__device__ __forceinline__ void tcs_st16x256b(uint32_t taddr, uint4 r) {
    asm volatile("tcgen05.st.sync.aligned.16x256b.x1.b32 [%0], {%1,%2,%3,%4};"
                 ::"r"(taddr), "r"(r.x), "r"(r.y), "r"(r.z), "r"(r.w) : "memory");
}
__device__ __forceinline__ void tcs_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// D = A * B^T (int32, overwriting D) with A in tensor memory (`tmem_a`:
// lane = row, K along columns) and B described in shared memory.
__device__ __forceinline__ void tcs_mma_i8(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc,
                                           uint32_t idesc) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, 0, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}"
                 :: "r"(tmem_d), "r"(tmem_a), "l"(bdesc), "r"(idesc) : "memory");
}

__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ float lds_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ void sts_f32(uint32_t addr, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// One 32-bit word of packed codes (byte e: low nibble code 4c + e, high
// nibble code 16 + 4c + e) -> 16 (q - 8) as signed bytes: .x the low
// nibbles, .y the high ones.
__device__ __forceinline__ uint2 tcs_dequant_word(uint32_t w) {
    return make_uint2(((w << 4) & 0xF0F0F0F0u) ^ 0x80808080u, (w & 0xF0F0F0F0u) ^ 0x80808080u);
}

// The CTA's load stages, walked without division: stage = units [k, k + n)
// of row block rb from block b on; at most kTcsS units, never past the end
// of a row block.
struct TcsWalk {
    int k, n, rb, b, nu, KB;
    __device__ __forceinline__ void init(int u0, int nu_, int KB_) {
        nu = nu_;
        KB = KB_;
        rb = u0 / KB;
        b = u0 - rb * KB;
        k = 0;
        n = min(min(kTcsS, nu), KB - b);
    }
    __device__ __forceinline__ bool valid() const { return k < nu; }
    __device__ __forceinline__ void step() {
        k += n;
        b += n;
        if (b == KB) {
            b = 0;
            ++rb;
        }
        n = min(min(kTcsS, nu - k), KB - b);
    }
    // the last stage of its row block in this CTA
    __device__ __forceinline__ bool closes_row_block() const { return b + n == KB || k + n == nu; }
};

struct TcsArgs {
    const uint8_t* W;     // packed Q4_0 matrix (576-byte segments)
    const uint8_t* xi;    // activation image: [KB][tcs_img_blk(V)]
    __half* y;            // [M][N]
    float* ws;            // CTA partials [CTAs][2][16][128]
    int* cnt;             // per (row block, epilogue warp) arrival counters, zero between calls
    int* err;
    int64_t N;
    int KB, T, M;         // blocks per row, packed tiles, vectors
    SplitConsts sc;       // make_split(row blocks * KB, CTAs)
};

// Bounded wait on an mbarrier phase: a non-blocking test first (the common
// case in a pipeline that runs ahead), then try_wait, which may suspend the
// thread for up to 20 us (woken when the phase completes), so waiting roles
// leave the issue slots to the dequantise warps.  Gives up after about 0.3 s,
// or as soon as another role aborted.
__device__ __forceinline__ bool tcs_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity) : "memory");
    if (ok) return true;
    for (uint32_t i = 0; i < (1u << 14); ++i) {
        asm volatile("{\n\t.reg .pred p;\n\t"
                     "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}"
                     : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity), "r"(20000u) : "memory");
        if (ok) return true;
        if (*abort_flag) return false;
    }
    return false;
}

// V: vectors the MMA covers (8 or 16; MMA width 2V).
template <int V>
__global__ void __launch_bounds__(kTcsThreads, 1) gemv_tcs_kernel(const TcsArgs a) {
    constexpr int N2 = 2 * V;                              // MMA width / accumulator columns per unit
    constexpr int L = kTcsL, NAG = tcs_nag(V), NDG = tcs_ndg(V), NSB = kTcsNSB, NM = kTcsNM;
    static_assert(NAG < NM && L < NM, "a stage's completion barrier outlives its waiters");
    constexpr uint32_t kImg = tcs_img_blk(V);
    constexpr uint32_t kStage = tcs_stage_bytes(V);
    constexpr uint32_t kRun = kTcsS * 576;                 // one tile's run inside a stage
    constexpr uint32_t kDGroupCols = kTcsS * N2;           // accumulator group: 64 or 128 columns
    constexpr uint32_t kAcol0 = NDG * kDGroupCols;         // first TMEM column of the A groups
    static_assert(kAcol0 + NAG * kTcsS * kTcsACols <= (uint32_t)kTcsTmemCols, "tensor memory");

    extern __shared__ uint8_t tcs_raw[];
    const uint32_t raw0 = smem_addr(tcs_raw);
    const uint32_t st0 = (raw0 + 127u) & ~127u;
    const uint32_t sbuf0 = st0 + (uint32_t)L * kStage;    // per slot: [S][128] row scales, [S][16] vector scales
    uint8_t* bar0 = tcs_raw + (sbuf0 - raw0) + (size_t)NSB * kTcsSBytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(bar0);   // [L] copies landed
    uint64_t* mdone = full + L;                             // [NM] the stage's MMAs completed
    uint64_t* afull = mdone + NM;                           // [NAG] A group written
    uint64_t* dempty = afull + NAG;                         // [NDG] accumulator group read back
    uint64_t* sfull = dempty + NDG;                         // [NSB] scale slot written
    uint64_t* sfree = sfull + NSB;                          // [NSB] scale slot read
    uint64_t* fin = sfree + NSB;                            // [kTcsIss] every MMA an issuer issued has completed
    uint32_t* tslot = reinterpret_cast<uint32_t*>(fin + kTcsIss);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = a.KB;
    const int u0 = seg_begin((int)blockIdx.x, a.sc), u1 = seg_begin((int)blockIdx.x + 1, a.sc);
    const int nu = u1 - u0;
    constexpr int kProducer = kTcsDq + kTcsEp, kIssuer = kProducer + kTcsProd;   // kProducer.., kIssuer..

    if (threadIdx.x == 0) {
        for (int j = 0; j < L; ++j) mbar_init(full + j, 1);
        for (int j = 0; j < NM; ++j) mbar_init(mdone + j, 1);
        for (int j = 0; j < NAG; ++j) mbar_init(afull + j, 4);
        for (int j = 0; j < NDG; ++j) mbar_init(dempty + j, kTcsEp);
        for (int j = 0; j < NSB; ++j) {
            mbar_init(sfull + j, 4);
            mbar_init(sfree + j, kTcsEp);
        }
        for (int j = 0; j < kTcsIss; ++j) mbar_init(fin + j, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kIssuer) tc_alloc(tslot, kTcsTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    auto fail_here = [&]() {
        *abort_flag = 1;
        set_device_error(a.err, kDevTimeout);
    };
    // phase parity of the n-th use of a ring slot (n = s / ring size)
    auto par = [](int n) { return (uint32_t)(n & 1); };

    TcsWalk w;
    w.init(u0, nu, KB);

    if (warp >= kProducer && warp < kIssuer) {
        // ---- bulk copies: producer pi takes the stages s with s % kTcsProd
        // == pi (one thread issues a bulk copy about every 200 cycles) ----
        const int pi = warp - kProducer;
        if (lane == 0) {
            // Launched as a dependent of the activation-image kernel: the image
            // is complete and visible after this wait.
            pdl_wait();
            int s = 0;
            for (; w.valid(); ++s, w.step()) {
                if (s % kTcsProd != pi) continue;
                const int j = s % L;
                if (s >= L && !tcs_wait(mdone + (s - L) % NM, par((s - L) / NM), abort_flag)) {
                    fail_here();
                    break;
                }
                const int ntiles = min(4, a.T - 4 * w.rb);
                const uint32_t sb = st0 + (uint32_t)j * kStage;
                mbar_arrive_expect_tx(full + j, (uint32_t)(ntiles * w.n * 576) + (uint32_t)w.n * kImg);
                for (int t = 0; t < ntiles; ++t)
                    bulk_g2s_addr(sb + (uint32_t)t * kRun, a.W + ((size_t)(4 * w.rb + t) * KB + w.b) * 576,
                                  (uint32_t)(w.n * 576), full + j);
                bulk_g2s_addr(sb + 4u * kRun, a.xi + (size_t)w.b * kImg, (uint32_t)w.n * kImg, full + j);
            }
            // this producer's copies still in flight land before the CTA exits
            for (int s2 = s - 1; s2 >= 0 && s2 >= s - L; --s2)
                if (s2 % kTcsProd == pi) mbar_wait_bounded(full + s2 % L, par(s2 / L), 1u << 22);
        }
    } else if (warp >= kIssuer) {
        // ---- MMA issuers: issuer ii takes the stages s with s % kTcsIss ==
        // ii (a tcgen05.commit tracks the MMAs of its own thread); stage s,
        // A group s % NAG, accumulator group s % NDG; unit i: A columns 8i..,
        // accumulator columns 2V i.. ----
        const int ii = warp - kIssuer;
        if (lane == 0) {
            const uint32_t idesc = tcs_idesc_i8(N2);
            int s = 0;
            for (; w.valid(); ++s, w.step()) {
                if (s % kTcsIss != ii) continue;
                const int j = s % L, ga = s % NAG, gd = s % NDG;
                if (!tcs_wait(afull + ga, par(s / NAG), abort_flag) ||
                    (s >= NDG && !tcs_wait(dempty + gd, par(s / NDG - 1), abort_flag))) {
                    fail_here();
                    break;
                }
                tc_fence_after();
                // Shared addresses stay below 2^18, so the start-address field
                // (address / 16, 14 bits) takes offsets by plain addition.
                const uint64_t b0 = tcs_sdesc(st0 + (uint32_t)j * kStage + 4u * kRun);
                const uint32_t d0 = tmem + (uint32_t)gd * kDGroupCols;
                const uint32_t a0 = tmem + kAcol0 + (uint32_t)ga * (kTcsS * kTcsACols);
                for (int i = 0; i < w.n; ++i)
                    tcs_mma_i8(d0 + (uint32_t)(N2 * i), a0 + (uint32_t)(kTcsACols * i),
                               b0 + (uint64_t)((i * kImg) >> 4), idesc);
                tc_commit(mdone + s % NM);     // accumulators, A group and load stage (B)
            }
            tc_commit(fin + ii);     // also after an abort: tracks every MMA this thread issued
            mbar_wait_bounded(fin + ii, 0u, 1u << 22);
        }
    } else if (warp < kTcsDq) {
        // ---- dequantise: group gi = warp / 4 takes the stages s with
        // s % kTcsG == gi; warp t = warp % 4 the packed tile t of each unit,
        // written to TMEM lanes 32t.. (A rows 32t..) ----
        // Thread 4g + c loads the 16 bytes at 16 (4g + c) of a segment (a
        // warp's loads cover 512 contiguous bytes): word c of rows g, g+8,
        // g+16, g+24, and the scale of row g + 8c.
        const int gi = warp >> 2, t = warp & 3;
        const int g = lane >> 2, c = lane & 3;
        const uint32_t t_rows = (uint32_t)(32 * t) << 16;
        const uint32_t d_off = 512u + 8u * (uint32_t)g + 2u * (uint32_t)c;   // scale of row g + 8c
        int s = 0;
        for (; w.valid(); ++s, w.step()) {
            if (s % kTcsG != gi) continue;
            const int j = s % L, ga = s % NAG, gs = s % NSB, n = w.n;
            const bool got = tcs_wait(full + j, par(s / L), abort_flag) &&
                             (s < NAG || tcs_wait(mdone + (s - NAG) % NM, par((s - NAG) / NM), abort_flag)) &&
                             (s < NSB || tcs_wait(sfree + gs, par(s / NSB - 1), abort_flag));
            if (!__all_sync(0xFFFFFFFFu, got)) {      // the warp leaves together
                fail_here();
                break;
            }
            tc_fence_after();
            const int ntiles = min(4, a.T - 4 * w.rb);
            const uint32_t sb = st0 + (uint32_t)j * kStage;
            const uint32_t ta = tmem + t_rows + kAcol0 + (uint32_t)ga * (kTcsS * kTcsACols);
            const uint32_t sg = sbuf0 + (uint32_t)gs * kTcsSBytes;
#pragma unroll
            for (int i = 0; i < kTcsS; ++i) {
                if (i < n) {
                    uint4 u = make_uint4(0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u);
                    uint32_t dbits = 0;
                    if (t < ntiles) {
                        const uint32_t seg = sb + (uint32_t)t * kRun + (uint32_t)i * 576u;
                        u = lds128(seg + 16u * (uint32_t)lane);
                        dbits = lds_u16(seg + d_off);
                    }
                    sts_f32(sg + (uint32_t)(i * 128 + 32 * t + g + 8 * c) * 4u,
                            __half2float(__ushort_as_half((unsigned short)dbits)));
                    if (t == 0 && lane < V)                // the block's vector scales
                        sts_f32(sg + (uint32_t)(kTcsS * 128 + i * 16 + lane) * 4u,
                                lds_f32(sb + 4u * kRun + (uint32_t)i * kImg + (uint32_t)(N2 * 32 + 4 * lane)));
                    const uint2 r0 = tcs_dequant_word(u.x);   // row g
                    const uint2 r1 = tcs_dequant_word(u.y);   // row g + 8
                    const uint2 r2 = tcs_dequant_word(u.z);   // row g + 16
                    const uint2 r3 = tcs_dequant_word(u.w);   // row g + 24
                    const uint32_t col = ta + (uint32_t)(kTcsACols * i);
                    tcs_st16x256b(col, make_uint4(r0.x, r0.y, r1.x, r1.y));
                    tcs_st16x256b(col + (16u << 16), make_uint4(r2.x, r2.y, r3.x, r3.y));
                }
            }
            tcs_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(afull + ga);
                mbar_arrive(sfull + gs);
            }
        }
    } else {
        // ---- epilogue: accumulator group s % NDG (TMEM lanes 32e..) ----
        const int e = warp - kTcsDq;
        const uint32_t t_lane = ((uint32_t)(32 * e) << 16);
        const int rb_first = w.rb;
        float acc[V];
#pragma unroll
        for (int m = 0; m < V; ++m) acc[m] = 0.f;

        // Row block rb's sums -> y (whole in this CTA) or a partial + arrival.
        auto flush = [&](int rb) {
            const int64_t n = (int64_t)rb * 128 + 32 * e + lane;
            const bool whole = rb * KB >= u0 && (rb + 1) * KB <= u1;
            if (whole) {
                if (n < a.N)
#pragma unroll
                    for (int m = 0; m < V; ++m)
                        if (m < a.M) a.y[(size_t)m * a.N + n] = __float2half_rn(acc[m]);
            } else {
                const int slot = rb == rb_first ? 0 : 1;
                float* wp = a.ws + ((size_t)blockIdx.x * 2 + slot) * 16 * 128 + 32 * e + lane;
#pragma unroll
                for (int m = 0; m < V; ++m)
                    if (m < a.M) wp[m * 128] = acc[m];
                __threadfence();
                __syncwarp();
                int* cn = a.cnt + (size_t)rb * kTcsEp + e;
                int old = 0;
                if (lane == 0) old = atom_add_acq_rel_gpu(cn, 1);
                old = __shfl_sync(0xFFFFFFFFu, old, 0);
                __syncwarp();                      // the lanes' reads follow lane 0's acquire
                const int cf = warp_of_seg(rb * KB, a.sc), cl = warp_of_seg(rb * KB + KB - 1, a.sc);
                const int need = cl - cf + 1;
                if (old == need - 1) {
                    float sum[V];
#pragma unroll
                    for (int m = 0; m < V; ++m) sum[m] = 0.f;
                    for (int cc = cf; cc <= cl; ++cc) {
                        const int sl = rb == seg_begin(cc, a.sc) / KB ? 0 : 1;
                        const float* rp = a.ws + ((size_t)cc * 2 + sl) * 16 * 128 + 32 * e + lane;
#pragma unroll
                        for (int m = 0; m < V; ++m)
                            if (m < a.M) sum[m] += ld_relaxed_gpu(rp + m * 128);
                    }
                    if (n < a.N)
#pragma unroll
                        for (int m = 0; m < V; ++m)
                            if (m < a.M) a.y[(size_t)m * a.N + n] = __float2half_rn(sum[m]);
                    if (lane == 0) *cn = 0;
                } else if (old >= need && lane == 0) {
                    set_device_error(a.err, kDevConcurrent);
                }
            }
#pragma unroll
            for (int m = 0; m < V; ++m) acc[m] = 0.f;
        };

        int s = 0;
        for (; w.valid(); ++s, w.step()) {
            const int gd = s % NDG, gs = s % NSB, n = w.n;
            const bool got = tcs_wait(mdone + s % NM, par(s / NM), abort_flag) &&
                             tcs_wait(sfull + gs, par(s / NSB), abort_flag);
            if (!__all_sync(0xFFFFFFFFu, got)) {
                fail_here();
                break;
            }
            tc_fence_after();
            const uint32_t sg = sbuf0 + (uint32_t)gs * kTcsSBytes;
            float dv[kTcsS];
#pragma unroll
            for (int i = 0; i < kTcsS; ++i)
                dv[i] = i < n ? lds_f32(sg + (uint32_t)(i * 128 + 32 * e + lane) * 4u) : 0.f;
            // 64 columns (4 units of 16 or 2 of 32) per read-back; unit i:
            // T_m = D[2m] + 256 D[2m + 1], acc[m] += T_m * d * s_m.
            constexpr int UPL = 64 / N2;
#pragma unroll
            for (int i0 = 0; i0 < kTcsS; i0 += UPL) {
                if (i0 < n) {
                    uint32_t v[64];
                    tcs_ld<64>(tmem + t_lane + (uint32_t)gd * kDGroupCols + (uint32_t)(N2 * i0), v);
#pragma unroll
                    for (int ii = 0; ii < UPL; ++ii) {
                        const int i = i0 + ii;
                        if (i < n) {
#pragma unroll
                            for (int m = 0; m < V; ++m) {
                                const int T = (int)v[N2 * ii + 2 * m] + 256 * (int)v[N2 * ii + 2 * m + 1];
                                const float sc = dv[i] * lds_f32(sg + (uint32_t)(kTcsS * 128 + i * 16 + m) * 4u);
                                acc[m] = fmaf(__int2float_rn(T), sc, acc[m]);
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(dempty + gd);
                mbar_arrive(sfree + gs);
            }
            if (w.closes_row_block()) flush(w.rb);
        }
    }

    __syncwarp();        // single-lane roles rejoin their warps
    tc_fence_before();
    __syncthreads();
    if (warp == kIssuer) {
        tc_fence_after();
        tc_dealloc(tmem, kTcsTmemCols);
    }
}

// Activation image of x[M][K] for gemv_tcs_kernel (V = 8 or 16 vectors): per
// block b, 2V rows of 32 signed bytes in 8-row x 16-byte core matrices
// (tcs_core_off) -- rows 2m and 2m + 1 the low and high parts Xl, Xh of
// X = rint(x[m][32b + j] 2^(14 - E)), E the exponent with every |x| of the
// block below 2^E, in the kernel's K order -- then the V fp32 scales
// 2^(E - 14) / 16 (NaN for a block holding a NaN or an infinity, whose
// outputs are then NaN; 0 for rows m >= M and all-zero blocks).  One thread
// per (block, vector).
static __global__ void __launch_bounds__(256) tcs_ximg_kernel(const __half* __restrict__ x,
                                                             uint8_t* __restrict__ img, int M,
                                                             int K, int V, int KB) {
    pdl_launch_dependents();      // the GEMV may start its prologue now
    const int total = KB * V;
    const int blk = 2 * V * 32 + V * 4;
    for (int q = blockIdx.x * blockDim.x + threadIdx.x; q < total; q += gridDim.x * blockDim.x) {
        const int b = q / V, m = q - b * V;
        uint8_t* out = img + (size_t)b * blk;
        float scale = 0.f;
        uint32_t lo[8], hi[8];                 // K slots 4w..4w+3 of rows 2m, 2m + 1
#pragma unroll
        for (int w = 0; w < 8; ++w) lo[w] = hi[w] = 0;
        if (m < M) {
            const __half* p = x + (size_t)m * K + 32 * b;
            float v[32];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const uint4 u = *reinterpret_cast<const uint4*>(p + 8 * h);
                const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const __half2 h2 = *reinterpret_cast<const __half2*>(&wv[e]);
                    v[8 * h + 2 * e] = __low2float(h2);
                    v[8 * h + 2 * e + 1] = __high2float(h2);
                }
            }
            float amax = 0.f;
            bool finite = true;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                finite = finite && isfinite(v[j]);
                amax = fmaxf(amax, fabsf(v[j]));
            }
            if (!finite) {
                scale = __int_as_float(0x7FC00000);    // NaN
            } else if (amax > 0.f) {
                int E;
                frexpf(amax, &E);                      // amax < 2^E
                scale = ldexpf(1.f, E - 18);           // 2^(E - 14) / 16
#pragma unroll
                for (int sl = 0; sl < 32; ++sl) {
                    // K slot sl holds code 4 (sl / 8) + sl % 4, plus 16 when sl % 8 >= 4
                    const int code = 4 * (sl >> 3) + (sl & 3) + ((sl & 4) ? 16 : 0);
                    const int X = (int)rintf(ldexpf(v[code], 14 - E));
                    const int Xh = (X + 128) >> 8, Xl = X - 256 * Xh;
                    lo[sl >> 2] |= ((uint32_t)Xl & 0xFFu) << (8 * (sl & 3));
                    hi[sl >> 2] |= ((uint32_t)Xh & 0xFFu) << (8 * (sl & 3));
                }
            }
        }
        *reinterpret_cast<uint4*>(out + tcs_core_off(2 * m, 0)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        *reinterpret_cast<uint4*>(out + tcs_core_off(2 * m, 1)) = make_uint4(lo[4], lo[5], lo[6], lo[7]);
        *reinterpret_cast<uint4*>(out + tcs_core_off(2 * m + 1, 0)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(out + tcs_core_off(2 * m + 1, 1)) = make_uint4(hi[4], hi[5], hi[6], hi[7]);
        reinterpret_cast<float*>(out + 2 * V * 32)[m] = scale;
    }
}

}  // namespace q4
