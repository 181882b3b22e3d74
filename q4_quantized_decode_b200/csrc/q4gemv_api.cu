// Host side of the q4gemv C ABI (see include/q4gemv.h): argument validation,
// workspace ownership, kernel selection and launch, and the CUDA-graph
// decode-step runner.
#include <cuda_runtime.h>
#include <dlfcn.h>
#include <nccl.h>   // types only: the functions are resolved at run time

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/q4gemv.h"
#include "gemv_dp2a.cuh"
#include "gemm_tc.cuh"
#include "gemv_mma.cuh"
#include "gemv_swiglu.cuh"
#include "gemv_tcs.cuh"
#include "stack.cuh"

namespace {

constexpr int kWarps = 16;                 // warps per CTA of the GEMV kernels
constexpr int kThreads = kWarps * 32;
// Per-warp TMA ring (stages x segments per stage) of each kernel.
constexpr int kR1 = 3, kC1 = 6;            // M = 1 and the decode step
constexpr int kR2 = 2, kC2 = 4;            // M = 2
constexpr int kRm1 = 2, kCm1 = 7;          // tensor-core kernel, M <= 8
constexpr int kRm2 = 2, kCm2 = 3;          // tensor-core kernel, M <= 16
constexpr int kMinSegsPerWarp = 4;         // small problems use fewer warps
constexpr int kMaxTiles = Q4GEMV_MAX_N / 32;
constexpr size_t kMaxDynSmem = 224 * 1024;   // opt-in dynamic shared memory per CTA
constexpr size_t kYaccPrealloc = (size_t)1 << 21;   // fp32 panel accumulator floats at create
constexpr size_t kXimgPrealloc = (size_t)1 << 24;   // GEMM activation image bytes at create
static_assert(q4::kTcMaxVec == Q4GEMV_MAX_M, "the GEMM's MMA width bounds M");

#define Q4_DP2A_KERNEL_1 q4::gemv_dp2a_kernel<1, kWarps, kR1, kC1>
#define Q4_DP2A_KERNEL_2 q4::gemv_dp2a_kernel<2, kWarps, kR2, kC2>
// Q8_0 (1088-byte segments): stages of three segments, about the bytes of
// six Q4_0 ones.
constexpr int kRq1 = 3, kCq1 = 3, kRq2 = 2, kCq2 = 3;
#define Q4_Q8_KERNEL_1 q4::gemv_dp2a_kernel<1, kWarps, kRq1, kCq1, true>
#define Q4_Q8_KERNEL_2 q4::gemv_dp2a_kernel<2, kWarps, kRq2, kCq2, true>
#define Q4_MMA_KERNEL_1 q4::gemv_mma_kernel<1, kWarps, kRm1, kCm1>
#define Q4_MMA_KERNEL_2 q4::gemv_mma_kernel<2, kWarps, kRm2, kCm2>
// The same for Q8_0 (1088-byte segments: stages of about the same bytes).
constexpr int kRmq1 = 2, kCmq1 = 4, kRmq2 = 2, kCmq2 = 2;
#define Q4_MMA_Q8_KERNEL_1 q4::gemv_mma_kernel<1, kWarps, kRmq1, kCmq1, true>
#define Q4_MMA_Q8_KERNEL_2 q4::gemv_mma_kernel<2, kWarps, kRmq2, kCmq2, true>
#define Q4_STACK_KERNEL q4::stack_kernel<kWarps, kR1, kC1>
#define Q4_STACK_KERNEL_GATED q4::stack_kernel<kWarps, kR1, kC1, true>
#define Q4_SWIGLU_KERNEL q4::gemv_swiglu_kernel<kWarps, kR1, kC1>
static_assert(Q4GEMV_MAX_M_GEMV == 16, "the small-M tensor-core kernel reads 16 accumulator columns");
// Largest input of a GEMV in the persistent step (its staging holds up to
// kStackXChunks 16-byte chunks per thread).
constexpr int kStackKmax = q4::kStackXChunks * 8 * kThreads;

enum StackMode { kStackPersistent = 0, kStackKernels = 1 };
// Kernel of the Q4_0 GEMVs with 3..16 vectors (and of M <= 2 with K beyond
// the dp2a kernel's staging): the mma.sync kernel (default; the faster of the
// two on every measured shape) or the tcgen05 kernel (Q4GEMV_SMALL_M = tcs,
// read at create).
enum SmallM { kSmallMma = 0, kSmallTcs = 1 };

size_t dp2a_smem(int M, int64_t K, bool q8 = false) {
    if (q8)
        return M == 1 ? q4::gemv_dp2a_smem_bytes(1, (int)K, kWarps, kRq1, kCq1, q4::kSegBytesQ8)
                      : q4::gemv_dp2a_smem_bytes(2, (int)K, kWarps, kRq2, kCq2, q4::kSegBytesQ8);
    return M == 1 ? q4::gemv_dp2a_smem_bytes(1, (int)K, kWarps, kR1, kC1)
                  : q4::gemv_dp2a_smem_bytes(2, (int)K, kWarps, kR2, kC2);
}

enum Fault { kFaultNone = 0, kFaultAlloc, kFaultLaunch, kFaultGraph, kFaultTimeout };

struct StackKey {
    std::vector<q4gemv_layer> layers;
    int64_t hidden = 0, qkv_n = 0, ffn = 0;
    const void* x_in = nullptr;
    void* x_out = nullptr;
    void* trace_x = nullptr;
    void* trace_y = nullptr;
    bool gated = false;
    bool operator==(const StackKey& o) const {
        if (layers.size() != o.layers.size()) return false;
        for (size_t i = 0; i < layers.size(); ++i) {
            const q4gemv_layer& a = layers[i];
            const q4gemv_layer& b = o.layers[i];
            if (a.qkv != b.qkv || a.o != b.o || a.gate_up != b.gate_up || a.down != b.down)
                return false;
        }
        return hidden == o.hidden && qkv_n == o.qkv_n && ffn == o.ffn && x_in == o.x_in &&
               x_out == o.x_out && trace_x == o.trace_x && trace_y == o.trace_y && gated == o.gated;
    }
};

}  // namespace

struct q4gemv_ctx {
    int device = 0;
    int sms = 0;
    int fault = kFaultNone;
    float* ws = nullptr;          // [ws_warps][2][MAX_M_GEMV][32] fp32
    int ws_warps = 0;
    int* cnt = nullptr;           // arrival counters, zero between calls
    int64_t cnt_elems = 0;
    int* err = nullptr;           // device error word
    __half* act = nullptr;        // stack intermediates
    size_t act_elems = 0;
    cudaStream_t cap = nullptr;   // private capture stream
    cudaGraphExec_t exec = nullptr;
    StackKey key;
    int stack_mode = kStackPersistent;
    int small_m = kSmallMma;
    q4::StackGemv* desc = nullptr;   // device descriptors of the persistent step
    int desc_cap = 0;
    StackKey desc_key;
    bool desc_valid = false;
    int* sync = nullptr;             // grid barrier words of the persistent step
    uint8_t* xq = nullptr;           // pre-quantised inputs of the persistent step (two halves)
    uint4* gscr = nullptr;           // gated persistent step: per-CTA combined shared tiles
    float* yacc = nullptr;           // fp32 panel sums of wide tensor-core GEMVs
    size_t yacc_floats = 0;
    __half* hio = nullptr;           // device copies of host x_in / x_out of run_stack
    uint8_t* ximg = nullptr;         // activation image of the tensor-core GEMM
    size_t ximg_bytes = 0;
    int64_t hio_elems = 0;           // per vector
    // Row-sharded decode step (one rank of `world`).
    ncclComm_t comm = nullptr;
    int world = 1, rank = 0;
    __half* sh_slice[4] = {nullptr, nullptr, nullptr, nullptr};    // this rank's output rows, per matrix type
    __half* sh_gather[4] = {nullptr, nullptr, nullptr, nullptr};   // all ranks' rows, per matrix type
    int64_t sh_chunk[4] = {0, 0, 0, 0};
    cudaGraphExec_t sh_exec = nullptr;
    StackKey sh_key;
    // Peer-memory exchange of the row-sharded step (q4gemv_peer_*).
    uint8_t* px_base = nullptr;          // this rank's exchange buffer
    int64_t px_off[6] = {0, 0, 0, 0, 0, 0};
    int px_world = 0, px_rank = 0;
    int64_t px_hidden = 0, px_qkv = 0, px_ffn = 0;
    uint8_t* px_remote[Q4GEMV_PEER_MAX_WORLD] = {};   // mapped peer buffers (not this rank's)
    uint32_t** px_ytab = nullptr;        // device: [4][world] this rank's slice in each buffer
    int* px_cnt = nullptr;               // arrival counts of the step's four matrices [4][tiles]
    int64_t px_cnt_elems = 0;
    int px_cnt_layers = 0;               // layers of the steps counted since they were zeroed
    bool px_open = false;
    unsigned char px_blob[Q4GEMV_PEER_BLOB_BYTES] = {};
    std::string last_error;
};

namespace {

int fail(q4gemv_ctx* h, int status, const char* fmt, ...) {
    if (h) {
        char buf[512];
        va_list ap;
        va_start(ap, fmt);
        vsnprintf(buf, sizeof buf, fmt, ap);
        va_end(ap);
        h->last_error = buf;
    }
    return status;
}

int cuda_fail(q4gemv_ctx* h, cudaError_t e, const char* what) {
    return fail(h, Q4_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define Q4_CUDA(h, call)                                          \
    do {                                                          \
        cudaError_t e_ = (call);                                  \
        if (e_ != cudaSuccess) return cuda_fail((h), e_, #call);  \
    } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Host memory (pinned or pageable) rather than device or managed memory.
bool is_host_pointer(const void* p) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();           // clear: an unknown pointer is pageable host memory
        return true;
    }
    return at.type == cudaMemoryTypeHost || at.type == cudaMemoryTypeUnregistered;
}

int check_shape(int64_t N, int64_t K) {
    if (N <= 0 || K <= 0 || K % 32 != 0) return Q4_ESHAPE;
    if (N > Q4GEMV_MAX_N || K > Q4GEMV_MAX_K) return Q4_ESHAPE;
    const int64_t T = (N + 31) / 32;
    if (T * (K / 32) >= (int64_t(1) << 31)) return Q4_ESHAPE;
    return Q4_OK;
}

int parse_fault(const char* s) {
    if (!s || !*s || !strcmp(s, "none")) return kFaultNone;
    if (!strcmp(s, "alloc")) return kFaultAlloc;
    if (!strcmp(s, "launch")) return kFaultLaunch;
    if (!strcmp(s, "graph")) return kFaultGraph;
    if (!strcmp(s, "timeout")) return kFaultTimeout;
    return -1;
}

template <typename F>
int set_smem_attr(F* kernel) {
    const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)kMaxDynSmem);
    return e == cudaSuccess ? 0 : -1;
}

// Launch one GEMV (M <= 2 path).  `pdl` adds the programmatic-dependent-
// launch attribute (only used between the library's own kernels).
int launch_gemv(q4gemv_ctx* h, const void* W, const __half* x, __half* y, int M, int64_t N,
                int64_t K, int renorm, __half* trace_x, cudaStream_t st, bool pdl, bool q8 = false,
                bool swiglu = false, const q4::PeerArgs* peer = nullptr, int* cnt = nullptr,
                float* ws = nullptr) {
    if (h->fault == kFaultLaunch) return fail(h, Q4_EFAULTINJ, "injected launch failure");
    const int KB = (int)(K / 32);
    const int T = (int)((N + 31) / 32);
    const int S = T * KB;
    int ctas = h->sms;
    const int want_warps = (S + kMinSegsPerWarp - 1) / kMinSegsPerWarp;
    if (want_warps < ctas * kWarps) ctas = (want_warps + kWarps - 1) / kWarps;
    if (ctas < 1) ctas = 1;
    q4::GemvArgs a;
    a.W = static_cast<const uint8_t*>(W);
    a.x = x;
    a.y = y;
    a.ws = h->ws;
    a.cnt = h->cnt;
    a.err = h->err;
    a.trace_x = trace_x;
    a.N = N;
    a.K = (int)K;
    a.KB = KB;
    a.T = T;
    a.S = S;
    a.G = ctas * kWarps < S ? ctas * kWarps : S;   // every owning warp gets >= 1 segment
    a.renorm = renorm;
    a.sc = q4::make_split(a.S, a.G);
    if (peer) a.peer = *peer;
    if (cnt) a.cnt = cnt;
    if (ws) a.ws = ws;
    const size_t smem = dp2a_smem(M, K, q8);

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ctas);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    cudaError_t e;
    if (swiglu)
        e = cudaLaunchKernelEx(&cfg, Q4_SWIGLU_KERNEL, a);   // M == 1, gated input
    else if (q8)
        e = M == 1 ? cudaLaunchKernelEx(&cfg, Q4_Q8_KERNEL_1, a) : cudaLaunchKernelEx(&cfg, Q4_Q8_KERNEL_2, a);
    else if (M == 1)
        e = cudaLaunchKernelEx(&cfg, Q4_DP2A_KERNEL_1, a);
    else
        e = cudaLaunchKernelEx(&cfg, Q4_DP2A_KERNEL_2, a);
    if (e != cudaSuccess) return cuda_fail(h, e, "gemv launch");
    return Q4_OK;
}

// Grows the split-tile workspace to hold `warps` warps (never during capture).
int ensure_ws(q4gemv_ctx* h, int warps, cudaStream_t st) {
    if (warps <= h->ws_warps) return Q4_OK;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    Q4_CUDA(h, cudaStreamIsCapturing(st, &cs));
    if (cs != cudaStreamCaptureStatusNone)
        return fail(h, Q4_EUNSUPPORTED,
                    "the first call with this shape must come outside stream capture (workspace growth)");
    if (h->fault == kFaultAlloc) return fail(h, Q4_EFAULTINJ, "injected allocation failure");
    Q4_CUDA(h, cudaDeviceSynchronize());
    cudaFree(h->ws);
    h->ws = nullptr;
    h->ws_warps = 0;
    if (cudaMalloc(&h->ws, (size_t)warps * 2 * Q4GEMV_MAX_M_GEMV * 32 * sizeof(float)) != cudaSuccess)
        return fail(h, Q4_ENOMEM, "workspace growth to %d warps failed", warps);
    h->ws_warps = warps;
    return Q4_OK;
}

// Ring bytes of the tensor-core kernel (nt8 = 1: up to 8 vectors, 2: up to 16).
size_t mma_ring(int nt8, bool q8 = false) {
    if (q8)
        return nt8 == 1 ? q4::ring_bytes(kWarps, kRmq1, kCmq1, q4::kSegBytesQ8)
                        : q4::ring_bytes(kWarps, kRmq2, kCmq2, q4::kSegBytesQ8);
    return nt8 == 1 ? q4::ring_bytes(kWarps, kRm1, kCm1) : q4::ring_bytes(kWarps, kRm2, kCm2);
}

// Largest block count one CTA may stage beside the ring.
int mma_xcap(int nt8, int M, bool q8 = false) {
    const size_t ring = mma_ring(nt8, q8);
    int xcap = 1;
    while (ring + q4::gemv_mma_smem_bytes(M, xcap + 1) <= kMaxDynSmem) ++xcap;
    return xcap;
}

// fp32 panel sums of a tensor-core GEMV run as several column panels.
int ensure_yacc(q4gemv_ctx* h, size_t floats, cudaStream_t st) {
    if (floats <= h->yacc_floats) return Q4_OK;
    if (h->fault == kFaultAlloc) return fail(h, Q4_EFAULTINJ, "injected allocation failure");
    cudaStreamSynchronize(st);
    cudaFree(h->yacc);
    h->yacc = nullptr;
    h->yacc_floats = 0;
    if (cudaMalloc(&h->yacc, floats * sizeof(float)) != cudaSuccess)
        return fail(h, Q4_ENOMEM, "panel sums of %zu floats failed", floats);
    h->yacc_floats = floats;
    return Q4_OK;
}

// Arrival counters for `n` (panel, tile) pairs, zero between calls.
int ensure_cnt(q4gemv_ctx* h, int64_t n, cudaStream_t st) {
    if (n <= h->cnt_elems) return Q4_OK;
    if (h->fault == kFaultAlloc) return fail(h, Q4_EFAULTINJ, "injected allocation failure");
    cudaStreamSynchronize(st);
    cudaFree(h->cnt);
    h->cnt = nullptr;
    h->cnt_elems = 0;
    if (cudaMalloc(&h->cnt, (size_t)n * sizeof(int)) != cudaSuccess ||
        cudaMemset(h->cnt, 0, (size_t)n * sizeof(int)) != cudaSuccess)
        return fail(h, Q4_ENOMEM, "arrival counters for %lld tiles failed", (long long)n);
    h->cnt_elems = n;
    return Q4_OK;
}

// Launch one GEMV on the tensor-core path (any M in 1..16, any K) as a grid
// of P column panels × CTAs.  P makes every panel fit one CTA's activation
// staging and keeps the staged slice (panel width × 8 or 16 vectors × 64 B)
// at most half the weight bytes a CTA streams; P > 1 adds a reduce launch.
int launch_gemv_mma(q4gemv_ctx* h, const void* W, const __half* x, __half* y, int M, int64_t N,
                    int64_t K, cudaStream_t st, bool q8 = false) {
    if (h->fault == kFaultLaunch) return fail(h, Q4_EFAULTINJ, "injected launch failure");
    const int nt8 = M <= 8 ? 1 : 2;
    const int KB = (int)(K / 32);
    const int T = (int)((N + 31) / 32);
    const int xcap = mma_xcap(nt8, M, q8);
    const int64_t seg = q8 ? q4::kSegBytesQ8 : q4::kSegBytes;
    int64_t P = (KB + xcap - 1) / xcap;
    // staging per CTA <= half its weights: P >= 2 * 64 * M * sms / (seg * T)
    const int64_t p_ratio = (2 * 64 * (int64_t)M * h->sms + seg * (int64_t)T - 1) / (seg * (int64_t)T);
    if (P < p_ratio) P = p_ratio;
    if (P > KB) P = KB;
    if (P > h->sms) P = h->sms;
    const int Wf = (int)((KB + P - 1) / P);          // panel width
    P = (KB + Wf - 1) / Wf;                          // no empty panel
    const int Wl = KB - (int)(P - 1) * Wf;           // the last panel's width
    int64_t cpp = h->sms / P;                        // CTAs per panel: about one wave in all
    const int64_t S = (int64_t)T * Wf, S_last = (int64_t)T * Wl;
    const int64_t cap = S_last / (kWarps * kMinSegsPerWarp);
    if (cpp > cap) cpp = cap;
    if (cpp < 1) cpp = 1;
    const int64_t Gmax = cpp * kWarps;
    const int64_t G = Gmax < S ? Gmax : S, G_last = Gmax < S_last ? Gmax : S_last;
    int rc = ensure_ws(h, (int)(P * (Gmax + cpp)), st);
    if (rc != Q4_OK) return rc;
    rc = ensure_cnt(h, P * T, st);
    if (rc != Q4_OK) return rc;
    if (P > 1) {
        rc = ensure_yacc(h, (size_t)P * M * (size_t)N, st);
        if (rc != Q4_OK) return rc;
    }
    q4::MmaArgs a;
    a.W = static_cast<const uint8_t*>(W);
    a.x = x;
    a.y = y;
    a.ws = h->ws;
    a.cnt = h->cnt;
    a.err = h->err;
    a.ypart = h->yacc;
    a.N = N;
    a.K = (int)K;
    a.KB = KB;
    a.T = T;
    a.S = (int)S;
    a.G = (int)G;
    a.KBv = Wf;
    a.p0 = 0;
    a.M = M;
    a.sc = q4::make_split(a.S, a.G);
    a.P = (int)P;
    a.S_last = (int)S_last;
    a.G_last = (int)G_last;
    a.sc_last = q4::make_split(a.S_last, a.G_last);
    a.ws_panel = (Gmax + cpp) * 2 * 16 * 32;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cpp, (unsigned)P);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = mma_ring(nt8, q8) + q4::gemv_mma_smem_bytes(M, Wf);
    cfg.stream = st;
    // The weight stream starts before the wait for the previous kernel.
    cudaLaunchAttribute pattr[1];
    pattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pattr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = pattr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (q8)
        e = nt8 == 1 ? cudaLaunchKernelEx(&cfg, Q4_MMA_Q8_KERNEL_1, a) : cudaLaunchKernelEx(&cfg, Q4_MMA_Q8_KERNEL_2, a);
    else
        e = nt8 == 1 ? cudaLaunchKernelEx(&cfg, Q4_MMA_KERNEL_1, a) : cudaLaunchKernelEx(&cfg, Q4_MMA_KERNEL_2, a);
    if (e != cudaSuccess) return cuda_fail(h, e, "gemv (mma) launch");
    if (P > 1) {
        const int64_t MN = (int64_t)M * N;
        int64_t blocks = (MN + 255) / 256;
        if (blocks > (int64_t)h->sms * 8) blocks = (int64_t)h->sms * 8;
        cudaLaunchConfig_t rcfg = {};
        rcfg.gridDim = dim3((unsigned)blocks);
        rcfg.blockDim = dim3(256);
        rcfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        rcfg.attrs = attr;
        rcfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&rcfg, q4::panel_reduce_kernel, (const float*)h->yacc, y, (int)P, MN);
        if (e != cudaSuccess) return cuda_fail(h, e, "panel reduce launch");
    }
    return Q4_OK;
}

// Activation image of the tensor-core GEMM (grows like the panel sums).
int ensure_ximg(q4gemv_ctx* h, size_t bytes, cudaStream_t st) {
    if (bytes <= h->ximg_bytes) return Q4_OK;
    if (h->fault == kFaultAlloc) return fail(h, Q4_EFAULTINJ, "injected allocation failure");
    cudaStreamSynchronize(st);
    cudaFree(h->ximg);
    h->ximg = nullptr;
    h->ximg_bytes = 0;
    if (cudaMalloc(&h->ximg, bytes) != cudaSuccess)
        return fail(h, Q4_ENOMEM, "activation image of %zu bytes failed", bytes);
    h->ximg_bytes = bytes;
    return Q4_OK;
}

// Launch a Q4_0 GEMV with M <= 16 on the tcgen05 small-M kernel: the
// activation image, then the GEMV over min(SMs, units) CTAs (units = 128-row
// blocks x 32-column blocks, split flat) as its programmatic dependent.
int launch_gemv_tcs(q4gemv_ctx* h, const void* W, const __half* x, __half* y, int M, int64_t N,
                    int64_t K, cudaStream_t st) {
    if (h->fault == kFaultLaunch) return fail(h, Q4_EFAULTINJ, "injected launch failure");
    const int KB = (int)(K / 32);
    const int64_t T = (N + 31) / 32;
    const int64_t RB = (T + 3) / 4;
    const int64_t U = RB * KB;
    if (U >= ((int64_t)1 << 31) - 1) return fail(h, Q4_EUNSUPPORTED, "small-M GEMV: too many units");
    const int grid = (int)(U < h->sms ? U : h->sms);
    const int V = q4::tcs_vecs(M);
    // CTA partials: grid x 2 slots x 16 vectors x 128 rows (4 of the
    // split-tile workspace's per-warp shares each).
    int rc = ensure_ws(h, 4 * grid, st);
    if (rc != Q4_OK) return rc;
    rc = ensure_cnt(h, RB * q4::kTcsEp, st);
    if (rc != Q4_OK) return rc;
    rc = ensure_ximg(h, (size_t)KB * q4::tcs_img_blk(V), st);
    if (rc != Q4_OK) return rc;
    int64_t blocks = ((int64_t)KB * V + 255) / 256;
    if (blocks > (int64_t)h->sms * 8) blocks = (int64_t)h->sms * 8;
    q4::tcs_ximg_kernel<<<(unsigned)blocks, 256, 0, st>>>(x, h->ximg, M, (int)K, V, KB);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(h, e, "activation image launch");
    q4::TcsArgs a;
    a.W = static_cast<const uint8_t*>(W);
    a.xi = h->ximg;
    a.y = y;
    a.ws = h->ws;
    a.cnt = h->cnt;
    a.err = h->err;
    a.N = N;
    a.KB = KB;
    a.T = (int)T;
    a.M = M;
    a.sc = q4::make_split((int)U, grid);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(q4::kTcsThreads);
    // One CTA per SM: two would fit beside each other and leave SMs idle.
    size_t smem = (size_t)q4::tcs_smem_bytes(V);
    if (smem < 116 * 1024) smem = 116 * 1024;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = V == 8 ? cudaLaunchKernelEx(&cfg, q4::gemv_tcs_kernel<8>, a)
               : cudaLaunchKernelEx(&cfg, q4::gemv_tcs_kernel<16>, a);
    if (e != cudaSuccess) return cuda_fail(h, e, "gemv (tcgen05 small-M) launch");
    return Q4_OK;
}

// Launch the M = 17..256 product on the tcgen05 tensor cores: the activation
// image, the GEMM over ceil(N/256) row tiles x P splits of the K steps (P as
// large as keeps the grid within one wave of the SMs), and for P > 1 the
// reduce of the fp32 split sums in split order.
int launch_gemm_tc(q4gemv_ctx* h, const void* W, const __half* x, __half* y, int M, int64_t N,
                   int64_t K, cudaStream_t st, bool q8 = false) {
    if (h->fault == kFaultLaunch) return fail(h, Q4_EFAULTINJ, "injected launch failure");
    const int KB = (int)(K / 32);
    const int nk = (KB + 1) / 2;
    const int Mp = (M + 15) / 16 * 16;
    const int64_t tiles = (N + q4::kTcRows - 1) / q4::kTcRows;
    int64_t P = h->sms / tiles;
    if (P < 1) P = 1;
    if (P > nk) P = nk;
    const int nkp = (int)((nk + P - 1) / P);
    P = (nk + nkp - 1) / nkp;                        // every split has steps
    // Up to 128 vectors the A tiles live in tensor memory beside the
    // accumulators (no shared-memory round trip); beyond, in shared memory.
    const bool at = Mp <= q4::kTcAtMaxVec;
    // Load stages: as many as fit beside the A buffers, if any (2..8; Q8_0
    // with more than 240 vectors fits one, which serialises copies and MMAs).
    const size_t fixed = q4::tc_smem_bytes(Mp, 0, q8, at);
    const size_t lsb = q4::tc_load_stage_bytes(Mp, q8) + 16;
    int L = (int)((kMaxDynSmem - fixed) / lsb);
    if (L > 8) L = 8;
    if (L < 1) L = 1;
    size_t smem = q4::tc_smem_bytes(Mp, L, q8, at);
    // One CTA per SM: each holds all 512 TMEM columns.
    if (smem < 116 * 1024) smem = 116 * 1024;
    int rc = ensure_ximg(h, (size_t)nk * Mp * 128, st);
    if (rc != Q4_OK) return rc;
    if (P > 1) {
        rc = ensure_yacc(h, (size_t)P * M * (size_t)N, st);
        if (rc != Q4_OK) return rc;
    }
    const int64_t chunks = (int64_t)nk * Mp * 8;
    int64_t blocks = (chunks + 255) / 256;
    if (blocks > (int64_t)h->sms * 8) blocks = (int64_t)h->sms * 8;
    q4::tc_ximg_kernel<<<(unsigned)blocks, 256, 0, st>>>(x, h->ximg, M, (int)K, Mp, nk);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(h, e, "activation image launch");
    q4::TcArgs a;
    a.W = static_cast<const uint8_t*>(W);
    a.xi = h->ximg;
    a.y = y;
    a.ypart = h->yacc;
    a.err = h->err;
    a.N = N;
    a.KB = KB;
    a.T = (int)((N + 31) / 32);
    a.M = M;
    a.Mp = Mp;
    a.nk = nk;
    a.nkp = nkp;
    a.P = (int)P;
    a.L = L;
    a.idesc = q4::tc_idesc_f16(128, Mp);
    cudaLaunchConfig_t gcfg = {};
    gcfg.gridDim = dim3((unsigned)tiles, (unsigned)P);
    gcfg.blockDim = dim3(q4::kTcThreads);
    gcfg.dynamicSmemBytes = smem;
    gcfg.stream = st;
    cudaLaunchAttribute gattr[1];
    gattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    gattr[0].val.programmaticStreamSerializationAllowed = 1;
    gcfg.attrs = gattr;
    gcfg.numAttrs = 1;
    if (at)
        e = q8 ? cudaLaunchKernelEx(&gcfg, q4::gemm_tc_kernel<true, true>, a)
               : cudaLaunchKernelEx(&gcfg, q4::gemm_tc_kernel<false, true>, a);
    else
        e = q8 ? cudaLaunchKernelEx(&gcfg, q4::gemm_tc_kernel<true>, a)
               : cudaLaunchKernelEx(&gcfg, q4::gemm_tc_kernel<false>, a);
    if (e != cudaSuccess) return cuda_fail(h, e, "gemm (tcgen05) launch");
    if (P > 1) {
        const int64_t MN = (int64_t)M * N;
        int64_t rb = (MN + 255) / 256;
        if (rb > (int64_t)h->sms * 8) rb = (int64_t)h->sms * 8;
        cudaLaunchConfig_t rcfg = {};
        rcfg.gridDim = dim3((unsigned)rb);
        rcfg.blockDim = dim3(256);
        rcfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        rcfg.attrs = attr;
        rcfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&rcfg, q4::panel_reduce_kernel, (const float*)h->yacc, y, (int)P, MN);
        if (e != cudaSuccess) return cuda_fail(h, e, "split reduce launch");
    }
    return Q4_OK;
}

int launch_renorm(q4gemv_ctx* h, const __half* in, __half* out, int len, cudaStream_t st,
                  bool pdl) {
    if (h->fault == kFaultLaunch) return fail(h, Q4_EFAULTINJ, "injected launch failure");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, q4::renorm_kernel<kWarps>, in, out, len);
    if (e != cudaSuccess) return cuda_fail(h, e, "renorm launch");
    return Q4_OK;
}

// The M <= 2 kernel holds the staged activations in registers (up to
// kXChunksPerThread 16-byte chunks per thread) and its ring plus the int16
// activations in shared memory.
bool dp2a_fits(int M, int64_t K) {
    return M <= 2 && M * K <= (int64_t)q4::kXChunksPerThread * 8 * kThreads &&
           dp2a_smem(M, K) <= kMaxDynSmem;
}

// Q8_0: the CUDA-core kernel for M <= 2 where its activation staging fits,
// the tensor-core GEMM otherwise.
bool q8_dp2a_fits(int M, int64_t K) {
    return M <= 2 && M * K <= (int64_t)q4::kXChunksPerThread * 8 * kThreads &&
           dp2a_smem(M, K, true) <= kMaxDynSmem;
}

// NCCL, loaded on first use (the library has no link-time dependency on it;
// in a process that already uses NCCL the loaded copy is shared).
struct NcclApi {
    void* lib = nullptr;
    ncclResult_t (*GetUniqueId)(ncclUniqueId*) = nullptr;
    ncclResult_t (*CommInitRank)(ncclComm_t*, int, ncclUniqueId, int) = nullptr;
    ncclResult_t (*AllGather)(const void*, void*, size_t, ncclDataType_t, ncclComm_t, cudaStream_t) = nullptr;
    ncclResult_t (*CommDestroy)(ncclComm_t) = nullptr;
    const char* (*GetErrorString)(ncclResult_t) = nullptr;
};
std::mutex g_nccl_mu;
NcclApi g_nccl;

bool nccl_load() {
    std::lock_guard<std::mutex> lock(g_nccl_mu);
    if (g_nccl.lib) return true;
    void* lib = dlopen("libnccl.so.2", RTLD_NOW | RTLD_GLOBAL);
    if (!lib) return false;
    NcclApi a;
    a.lib = lib;
    a.GetUniqueId = reinterpret_cast<decltype(a.GetUniqueId)>(dlsym(lib, "ncclGetUniqueId"));
    a.CommInitRank = reinterpret_cast<decltype(a.CommInitRank)>(dlsym(lib, "ncclCommInitRank"));
    a.AllGather = reinterpret_cast<decltype(a.AllGather)>(dlsym(lib, "ncclAllGather"));
    a.CommDestroy = reinterpret_cast<decltype(a.CommDestroy)>(dlsym(lib, "ncclCommDestroy"));
    a.GetErrorString = reinterpret_cast<decltype(a.GetErrorString)>(dlsym(lib, "ncclGetErrorString"));
    if (!a.GetUniqueId || !a.CommInitRank || !a.AllGather || !a.CommDestroy || !a.GetErrorString) {
        dlclose(lib);
        return false;
    }
    g_nccl = a;
    return true;
}

// Frees the sharded step's communicator, buffers and graph.
void shard_release(q4gemv_ctx* h) {
    if (h->sh_exec) cudaGraphExecDestroy(h->sh_exec);
    h->sh_exec = nullptr;
    for (int t = 0; t < 4; ++t) {
        cudaFree(h->sh_slice[t]);
        cudaFree(h->sh_gather[t]);
        h->sh_slice[t] = h->sh_gather[t] = nullptr;
        h->sh_chunk[t] = 0;
    }
    if (h->comm && g_nccl.CommDestroy) g_nccl.CommDestroy(h->comm);
    h->comm = nullptr;
}

// Rows per rank of an N-row matrix split over `world` ranks: whole 32-row
// tiles, the same count for every rank (the all-gather sends equal pieces).
// Unmaps the peers' exchange buffers and frees this rank's.
void peer_release(q4gemv_ctx* h) {
    if (h->sh_exec) cudaGraphExecDestroy(h->sh_exec);
    h->sh_exec = nullptr;
    for (int p = 0; p < Q4GEMV_PEER_MAX_WORLD; ++p) {
        if (h->px_remote[p]) cudaIpcCloseMemHandle(h->px_remote[p]);
        h->px_remote[p] = nullptr;
    }
    cudaFree(h->px_ytab);
    cudaFree(h->px_cnt);
    cudaFree(h->px_base);
    h->px_ytab = nullptr;
    h->px_cnt = nullptr;
    h->px_cnt_elems = 0;
    h->px_cnt_layers = 0;
    h->px_base = nullptr;
    h->px_open = false;
    h->px_world = 0;
}

int64_t shard_chunk(int64_t N, int world) {
    const int64_t unit = 32 * (int64_t)world;
    return (N + unit - 1) / unit * 32;
}

}  // namespace

extern "C" {

int q4gemv_version(void) { return (0 << 16) | 1; }

const char* q4gemv_strerror(int status) {
    switch (status) {
        case Q4_OK: return "ok";
        case Q4_EINVAL: return "invalid argument";
        case Q4_ESHAPE: return "invalid shape (N, K > 0, K % 32 == 0, within limits)";
        case Q4_EALIGN: return "device pointer not 16-byte aligned";
        case Q4_ENOMEM: return "out of memory";
        case Q4_ECUDA: return "CUDA runtime error";
        case Q4_EUNSUPPORTED: return "unsupported configuration";
        case Q4_ETIMEOUT: return "bounded device wait timed out";
        case Q4_EFAULTINJ: return "injected fault";
        case Q4_ECONCURRENT: return "overlapping calls on one handle";
        default: return "unknown status";
    }
}

const char* q4gemv_last_error(q4gemv_t h) { return h ? h->last_error.c_str() : ""; }

size_t q4gemv_gguf_bytes(int64_t N, int64_t K) {
    if (check_shape(N, K) != Q4_OK) return 0;
    return (size_t)N * (size_t)(K / 32) * 18;
}

size_t q4gemv_packed_bytes(int64_t N, int64_t K) {
    if (check_shape(N, K) != Q4_OK) return 0;
    return (size_t)((N + 31) / 32 * 32) * (size_t)(K / 32) * 18;
}

int q4gemv_validate(int M, int64_t N, int64_t K, const void* W, const void* x, const void* y) {
    if (M < 1 || M > Q4GEMV_MAX_M) return Q4_EUNSUPPORTED;
    const int sh = check_shape(N, K);
    if (sh != Q4_OK) return sh;
    if (!W || !x || !y) return Q4_EINVAL;
    if (!aligned16(W) || !aligned16(x) || !aligned16(y)) return Q4_EALIGN;
    return Q4_OK;
}

int q4gemv_set_fault(q4gemv_t h, const char* which) {
    if (!h) return Q4_EINVAL;
    const int f = parse_fault(which);
    if (f < 0) return fail(h, Q4_EINVAL, "unknown fault name");
    if (f != h->fault && h->sh_exec) {   // the sharded step's graph holds the knob's values
        Q4_CUDA(h, cudaSetDevice(h->device));
        Q4_CUDA(h, cudaDeviceSynchronize());
        cudaGraphExecDestroy(h->sh_exec);
        h->sh_exec = nullptr;
    }
    h->fault = f;
    return Q4_OK;
}

int q4gemv_create(q4gemv_t* out, int device) {
    if (!out) return Q4_EINVAL;
    *out = nullptr;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev)
        return Q4_EINVAL;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, device) != cudaSuccess) return Q4_ECUDA;
    if (prop.major != 10) return Q4_EUNSUPPORTED;
    q4gemv_ctx* h = new (std::nothrow) q4gemv_ctx;
    if (!h) return Q4_ENOMEM;
    h->device = device;
    h->sms = prop.multiProcessorCount;
    const int f = parse_fault(getenv("Q4GEMV_FAULT"));
    h->fault = f < 0 ? kFaultNone : f;
    int rc = Q4_OK;
    cudaError_t e = cudaSetDevice(device);
    if (e != cudaSuccess) rc = cuda_fail(h, e, "cudaSetDevice");
    if (rc == Q4_OK && h->fault == kFaultAlloc) rc = fail(h, Q4_EFAULTINJ, "injected allocation failure");
    if (rc == Q4_OK) {
        h->ws_warps = h->sms * kWarps;
        const size_t ws_bytes = (size_t)h->ws_warps * 2 * Q4GEMV_MAX_M_GEMV * 32 * sizeof(float);
        if (cudaMalloc(&h->ws, ws_bytes) != cudaSuccess ||
            cudaMalloc(&h->cnt, (size_t)kMaxTiles * sizeof(int)) != cudaSuccess ||
            cudaMalloc(&h->err, sizeof(int)) != cudaSuccess ||
            cudaMalloc(&h->sync, 4 * sizeof(int)) != cudaSuccess ||
            cudaMalloc(&h->xq, 2 * q4::stack_xq_half_bytes(kStackKmax)) != cudaSuccess ||
            cudaMalloc(&h->yacc, kYaccPrealloc * sizeof(float)) != cudaSuccess ||
            cudaMalloc(&h->ximg, kXimgPrealloc) != cudaSuccess)
            rc = fail(h, Q4_ENOMEM, "workspace allocation failed");
        else {
            h->yacc_floats = kYaccPrealloc;
            h->ximg_bytes = kXimgPrealloc;
            h->cnt_elems = kMaxTiles;
        }
        const char* mode = getenv("Q4GEMV_STACK_MODE");
        if (mode && !strcmp(mode, "kernels")) h->stack_mode = kStackKernels;
        const char* sm = getenv("Q4GEMV_SMALL_M");
        if (sm && !strcmp(sm, "tcs")) h->small_m = kSmallTcs;
    }
    if (rc == Q4_OK) {
        if (cudaMemset(h->cnt, 0, (size_t)kMaxTiles * sizeof(int)) != cudaSuccess ||
            cudaMemset(h->err, 0, sizeof(int)) != cudaSuccess)
            rc = fail(h, Q4_ECUDA, "workspace initialisation failed");
    }
    if (rc == Q4_OK) {
        if (set_smem_attr(Q4_DP2A_KERNEL_1) || set_smem_attr(Q4_DP2A_KERNEL_2) ||
            set_smem_attr(Q4_Q8_KERNEL_1) || set_smem_attr(Q4_Q8_KERNEL_2) ||
            set_smem_attr(Q4_MMA_KERNEL_1) || set_smem_attr(Q4_MMA_KERNEL_2) ||
            set_smem_attr(Q4_MMA_Q8_KERNEL_1) || set_smem_attr(Q4_MMA_Q8_KERNEL_2) ||
            set_smem_attr(Q4_STACK_KERNEL) || set_smem_attr(Q4_STACK_KERNEL_GATED) ||
            set_smem_attr(Q4_SWIGLU_KERNEL) ||
            set_smem_attr(q4::gemm_tc_kernel<false>) ||
            set_smem_attr(q4::gemm_tc_kernel<true>) ||
            set_smem_attr(q4::gemm_tc_kernel<false, true>) ||
            set_smem_attr(q4::gemm_tc_kernel<true, true>) ||
            set_smem_attr(q4::gemv_tcs_kernel<8>) || set_smem_attr(q4::gemv_tcs_kernel<16>) ||
            0)
            rc = fail(h, Q4_ECUDA, "cudaFuncSetAttribute failed");
    }
    if (rc == Q4_OK) {
        e = cudaStreamCreateWithFlags(&h->cap, cudaStreamNonBlocking);
        if (e != cudaSuccess) rc = cuda_fail(h, e, "cudaStreamCreate");
    }
    if (rc == Q4_OK) {
        e = cudaDeviceSynchronize();
        if (e != cudaSuccess) rc = cuda_fail(h, e, "cudaDeviceSynchronize");
    }
    if (rc != Q4_OK) {
        cudaFree(h->ws);
        cudaFree(h->cnt);
        cudaFree(h->err);
        cudaFree(h->sync);
        cudaFree(h->xq);
        cudaFree(h->yacc);
        cudaFree(h->ximg);
        if (h->cap) cudaStreamDestroy(h->cap);
        delete h;
        return rc;
    }
    *out = h;
    return Q4_OK;
}

int q4gemv_destroy(q4gemv_t h) {
    if (!h) return Q4_OK;
    cudaSetDevice(h->device);
    cudaDeviceSynchronize();
    if (h->exec) cudaGraphExecDestroy(h->exec);
    if (h->cap) cudaStreamDestroy(h->cap);
    cudaFree(h->ws);
    cudaFree(h->cnt);
    cudaFree(h->err);
    cudaFree(h->act);
    cudaFree(h->desc);
    cudaFree(h->sync);
    cudaFree(h->xq);
    cudaFree(h->yacc);
    cudaFree(h->hio);
    cudaFree(h->ximg);
    cudaFree(h->gscr);
    shard_release(h);
    peer_release(h);
    delete h;
    return Q4_OK;
}

int q4gemv_repack(q4gemv_t h, const void* gguf, void* packed, int64_t N, int64_t K,
                  q4gemv_stream_t stream) {
    if (!h) return Q4_EINVAL;
    const int sh = check_shape(N, K);
    if (sh != Q4_OK) return fail(h, sh, "repack: invalid shape N=%lld K=%lld", (long long)N, (long long)K);
    if (!gguf || !packed) return fail(h, Q4_EINVAL, "repack: null pointer");
    if ((reinterpret_cast<uintptr_t>(gguf) & 1u) || !aligned16(packed))
        return fail(h, Q4_EALIGN, "repack: misaligned pointer");
    const uintptr_t g0 = reinterpret_cast<uintptr_t>(gguf), g1 = g0 + q4gemv_gguf_bytes(N, K);
    const uintptr_t p0 = reinterpret_cast<uintptr_t>(packed), p1 = p0 + q4gemv_packed_bytes(N, K);
    if (g0 < p1 && p0 < g1) return fail(h, Q4_EINVAL, "repack: gguf and packed overlap");
    if (h->fault == kFaultLaunch) return fail(h, Q4_EFAULTINJ, "injected launch failure");
    Q4_CUDA(h, cudaSetDevice(h->device));
    const int KB = (int)(K / 32);
    const int64_t T = (N + 31) / 32;
    const int64_t S = T * KB;
    int64_t blocks = (S + 7) / 8;
    if (blocks > (int64_t)h->sms * 32) blocks = (int64_t)h->sms * 32;
    q4::repack_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint8_t*>(gguf), static_cast<uint8_t*>(packed), N, KB, S);
    Q4_CUDA(h, cudaGetLastError());
    return Q4_OK;
}

int q4gemv_run(q4gemv_t h, const void* W, const void* x, void* y, int M, int64_t N, int64_t K,
               q4gemv_stream_t stream) {
    if (!h) return Q4_EINVAL;
    const int v = q4gemv_validate(M, N, K, W, x, y);
    if (v != Q4_OK)
        return fail(h, v, "run: %s (M=%d N=%lld K=%lld)", q4gemv_strerror(v), M, (long long)N,
                    (long long)K);
    Q4_CUDA(h, cudaSetDevice(h->device));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (M > Q4GEMV_MAX_M_GEMV)
        return launch_gemm_tc(h, W, static_cast<const __half*>(x), static_cast<__half*>(y), M, N,
                              K, st);
    if (dp2a_fits(M, K))
        return launch_gemv(h, W, static_cast<const __half*>(x), static_cast<__half*>(y), M, N, K,
                           0, nullptr, st, true);
    if (h->small_m == kSmallTcs)
        return launch_gemv_tcs(h, W, static_cast<const __half*>(x), static_cast<__half*>(y), M, N,
                               K, st);
    return launch_gemv_mma(h, W, static_cast<const __half*>(x), static_cast<__half*>(y), M, N, K,
                           st);
}
 
int q4gemv_run_swiglu(q4gemv_t h, const void* W, const void* gate_up, void* y, int64_t N,
                      int64_t K, q4gemv_stream_t stream) {
    if (!h) return Q4_EINVAL;
    int v = q4gemv_validate(1, N, K, W, gate_up, y);
    if (v == Q4_OK && !dp2a_fits(1, K)) v = Q4_EUNSUPPORTED;
    if (v != Q4_OK)
        return fail(h, v, "run_swiglu: %s (N=%lld K=%lld)", q4gemv_strerror(v), (long long)N,
                    (long long)K);
    Q4_CUDA(h, cudaSetDevice(h->device));
    return launch_gemv(h, W, static_cast<const __half*>(gate_up), static_cast<__half*>(y), 1, N, K,
                       0, nullptr, static_cast<cudaStream_t>(stream), true, false, true);
}

size_t q4gemv_q8_0_gguf_bytes(int64_t N, int64_t K) {
    if (check_shape(N, K) != Q4_OK) return 0;
    return (size_t)N * (size_t)(K / 32) * 34;
}

size_t q4gemv_q8_0_packed_bytes(int64_t N, int64_t K) {
    if (check_shape(N, K) != Q4_OK) return 0;
    return (size_t)((N + 31) / 32 * 32) * (size_t)(K / 32) * 34;
}

int q4gemv_q8_0_repack(q4gemv_t h, const void* gguf, void* packed, int64_t N, int64_t K,
                       q4gemv_stream_t stream) {
    if (!h) return Q4_EINVAL;
    const int sh = check_shape(N, K);
    if (sh != Q4_OK) return fail(h, sh, "q8_0 repack: invalid shape N=%lld K=%lld", (long long)N, (long long)K);
    if (!gguf || !packed) return fail(h, Q4_EINVAL, "q8_0 repack: null pointer");
    if ((reinterpret_cast<uintptr_t>(gguf) & 1u) || !aligned16(packed))
        return fail(h, Q4_EALIGN, "q8_0 repack: misaligned pointer");
    const uintptr_t g0 = reinterpret_cast<uintptr_t>(gguf), g1 = g0 + q4gemv_q8_0_gguf_bytes(N, K);
    const uintptr_t p0 = reinterpret_cast<uintptr_t>(packed), p1 = p0 + q4gemv_q8_0_packed_bytes(N, K);
    if (g0 < p1 && p0 < g1) return fail(h, Q4_EINVAL, "q8_0 repack: gguf and packed overlap");
    if (h->fault == kFaultLaunch) return fail(h, Q4_EFAULTINJ, "injected launch failure");
    Q4_CUDA(h, cudaSetDevice(h->device));
    const int KB = (int)(K / 32);
    const int64_t S = (N + 31) / 32 * KB;
    int64_t blocks = (S + 7) / 8;
    if (blocks > (int64_t)h->sms * 32) blocks = (int64_t)h->sms * 32;
    q4::repack_q8_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint8_t*>(gguf), static_cast<uint8_t*>(packed), N, KB, S);
    Q4_CUDA(h, cudaGetLastError());
    return Q4_OK;
}

int q4gemv_q8_0_validate(int M, int64_t N, int64_t K, const void* W, const void* x, const void* y) {
    if (M < 1 || M > Q4GEMV_MAX_M) return Q4_EUNSUPPORTED;
    const int sh = check_shape(N, K);
    if (sh != Q4_OK) return sh;
    if (!W || !x || !y) return Q4_EINVAL;
    if (!aligned16(W) || !aligned16(x) || !aligned16(y)) return Q4_EALIGN;
    return Q4_OK;
}

int q4gemv_q8_0_run(q4gemv_t h, const void* W, const void* x, void* y, int M, int64_t N, int64_t K,
                    q4gemv_stream_t stream) {
    if (!h) return Q4_EINVAL;
    const int v = q4gemv_q8_0_validate(M, N, K, W, x, y);
    if (v != Q4_OK)
        return fail(h, v, "q8_0 run: %s (M=%d N=%lld K=%lld)", q4gemv_strerror(v), M, (long long)N,
                    (long long)K);
    Q4_CUDA(h, cudaSetDevice(h->device));
    if (q8_dp2a_fits(M, K))
        return launch_gemv(h, W, static_cast<const __half*>(x), static_cast<__half*>(y), M, N, K, 0,
                           nullptr, static_cast<cudaStream_t>(stream), true, true);
    if (M <= Q4GEMV_MAX_M_GEMV)
        return launch_gemv_mma(h, W, static_cast<const __half*>(x), static_cast<__half*>(y), M, N, K,
                               static_cast<cudaStream_t>(stream), true);
    return launch_gemm_tc(h, W, static_cast<const __half*>(x), static_cast<__half*>(y), M, N, K,
                          static_cast<cudaStream_t>(stream), true);
}

namespace {

// After a step whose x_out is host memory: copy the device result out on
// the same stream.
int finish_host_out(q4gemv_ctx* h, int rc, bool host_out, void* user_out, const void* dev_out,
                    int64_t hidden, cudaStream_t st) {
    if (rc != Q4_OK || !host_out) return rc;
    Q4_CUDA(h, cudaMemcpyAsync(user_out, dev_out, hidden * sizeof(__half), cudaMemcpyDeviceToHost, st));
    return Q4_OK;
}

// Enqueue the whole decode step on `st`.
int enqueue_stack(q4gemv_ctx* h, const StackKey& k, cudaStream_t st) {
    const int64_t hidden = k.hidden, qkv_n = k.qkv_n, ffn = k.ffn;
    const int64_t kmax = hidden > ffn ? hidden : ffn;
    int64_t nmax = qkv_n > hidden ? qkv_n : hidden;
    if (2 * ffn > nmax) nmax = 2 * ffn;
    // Intermediate outputs: QKV, O, gate_up, down (rounded up to 16 bytes).
    const int64_t n_of[4] = {qkv_n, hidden, 2 * ffn, hidden};
    const int64_t k_of[4] = {hidden, hidden, hidden, ffn};
    __half* buf[4];
    size_t off = 0;
    for (int t = 0; t < 4; ++t) {
        buf[t] = h->act + off;
        off += (size_t)((n_of[t] + 7) / 8 * 8);
    }
    const int n_gemv = 4 * (int)k.layers.size();
    const __half* prev = nullptr;
    for (int i = 0; i < n_gemv; ++i) {
        const int l = i / 4, t = i % 4;
        const q4gemv_layer& L = k.layers[l];
        const void* W = t == 0 ? L.qkv : t == 1 ? L.o : t == 2 ? L.gate_up : L.down;
        __half* yout = k.trace_y ? static_cast<__half*>(k.trace_y) + (size_t)i * nmax : buf[t];
        __half* tx = k.trace_x ? static_cast<__half*>(k.trace_x) + (size_t)i * kmax : nullptr;
        const __half* xin = (i == 0) ? static_cast<const __half*>(k.x_in) : prev;
        const bool gated = k.gated && t == 3;   // SiLU(gate) * up of the 2K gate+up outputs
        const int rc = launch_gemv(h, W, xin, yout, 1, n_of[t], k_of[t], i == 0 ? 0 : 1, tx, st,
                                   i != 0, false, gated);
        if (rc != Q4_OK) return rc;
        prev = yout;
    }
    return launch_renorm(h, prev, static_cast<__half*>(k.x_out), (int)hidden, st, true);
}

// Descriptors of the persistent step for key k (host side).
void build_descriptors(q4gemv_ctx* h, const StackKey& k, std::vector<q4::StackGemv>& out) {
    const int64_t hidden = k.hidden, qkv_n = k.qkv_n, ffn = k.ffn;
    const int64_t kmax = hidden > ffn ? hidden : ffn;
    int64_t nmax = qkv_n > hidden ? qkv_n : hidden;
    if (2 * ffn > nmax) nmax = 2 * ffn;
    const int64_t n_of[4] = {qkv_n, hidden, 2 * ffn, hidden};
    const int64_t k_of[4] = {hidden, hidden, hidden, ffn};
    __half* buf[4];
    size_t off = 0;
    for (int t = 0; t < 4; ++t) {
        buf[t] = h->act + off;
        off += (size_t)((n_of[t] + 7) / 8 * 8);
    }
    const int n_gemv = 4 * (int)k.layers.size();
    out.resize(n_gemv);
    for (int i = 0; i < n_gemv; ++i) {
        const int l = i / 4, t = i % 4;
        const q4gemv_layer& L = k.layers[l];
        q4::StackGemv& d = out[i];
        d.W = static_cast<const uint8_t*>(t == 0 ? L.qkv : t == 1 ? L.o : t == 2 ? L.gate_up : L.down);
        d.y = k.trace_y ? static_cast<__half*>(k.trace_y) + (size_t)i * nmax : buf[t];
        d.trace_x = k.trace_x ? static_cast<__half*>(k.trace_x) + (size_t)i * kmax : nullptr;
        d.N = (int)n_of[t];
        d.K = (int)k_of[t];
        d.renorm = i == 0 ? 0 : 1;
        d.fill_y = k.trace_y ? 1 : 0;
        d.gated = k.gated && t == 3 ? 1 : 0;
        const int S = (int)((n_of[t] + 31) / 32 * (k_of[t] / 32));
        const int gmax = h->sms * kWarps;
        d.sc = q4::make_split(S, gmax < S ? gmax : S);
    }
}

// The whole step as one cooperative launch (plus the barrier reset).
int enqueue_stack_persistent(q4gemv_ctx* h, const StackKey& k, cudaStream_t st) {
    if (h->fault == kFaultLaunch) return fail(h, Q4_EFAULTINJ, "injected launch failure");
    const int64_t kmax = k.hidden > k.ffn ? k.hidden : k.ffn;
    Q4_CUDA(h, cudaMemsetAsync(h->sync, 0, 4 * sizeof(int), st));
    q4::StackArgs sa;
    sa.gemv = h->desc;
    sa.n_gemv = 4 * (int)k.layers.size();
    sa.x_in = static_cast<const __half*>(k.x_in);
    sa.x_out = static_cast<__half*>(k.x_out);
    sa.hidden = (int)k.hidden;
    sa.ws = h->ws;
    sa.ws_half = h->sms * 2 * 32;   // [CTAs][2][32] per GEMV parity (ws holds sms * 16 warps * 1 KB)
    sa.err = h->err;
    sa.sync = h->sync;
    sa.xq = h->xq;
    sa.xq_half = (int)q4::stack_xq_half_bytes(kStackKmax);
    sa.kmax = (int)kmax;
    // A test of the device-side timeout: few polls, and a first grid wait
    // that no arrival count satisfies.
    sa.poll_limit = h->fault == kFaultTimeout ? (1u << 10) : (1u << 26);
    sa.unreachable = h->fault == kFaultTimeout ? 1 : 0;
    sa.gscr = h->gscr;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(h->sms);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = q4::stack_smem_bytes((int)kmax, kWarps, kR1, kC1);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = k.gated ? cudaLaunchKernelEx(&cfg, Q4_STACK_KERNEL_GATED, sa, (int)kmax)
                                  : cudaLaunchKernelEx(&cfg, Q4_STACK_KERNEL, sa, (int)kmax);
    if (e != cudaSuccess) return cuda_fail(h, e, "decode-step launch");
    return Q4_OK;
}

}  // namespace

namespace {
int run_stack_impl(q4gemv_ctx* h, const q4gemv_layer* layers, int n_layers, int64_t hidden,
                   int64_t qkv_n, int64_t ffn, const void* x_in, void* x_out, void* trace_x,
                   void* trace_y, q4gemv_stream_t stream, bool gated) {
    if (!h) return Q4_EINVAL;
    if (!layers || !x_in || !x_out) return fail(h, Q4_EINVAL, "run_stack: null pointer");
    if (n_layers < 1 || n_layers > 4096) return fail(h, Q4_ESHAPE, "run_stack: n_layers out of range");
    if (qkv_n < hidden) return fail(h, Q4_ESHAPE, "run_stack: qkv_n < hidden");
    if (qkv_n % 8 != 0)   // trace_y rows must start on 16-byte boundaries
        return fail(h, Q4_ESHAPE, "run_stack: qkv_n must be a multiple of 8");
    const int64_t dims[4][2] = {{qkv_n, hidden}, {hidden, hidden}, {2 * ffn, hidden}, {hidden, ffn}};
    for (auto& d : dims) {
        const int s = check_shape(d[0], d[1]);
        if (s != Q4_OK) return fail(h, s, "run_stack: invalid matrix shape");
        if (!dp2a_fits(1, d[1])) return fail(h, Q4_EUNSUPPORTED, "run_stack: K too large");
    }
    // x_in / x_out may be host memory (pinned or pageable): staged through
    // device copies on the same stream, inside this call.
    const bool host_in = is_host_pointer(x_in), host_out = is_host_pointer(x_out);
    if ((!host_in && !aligned16(x_in)) || (!host_out && !aligned16(x_out)) || !aligned16(trace_x) ||
        !aligned16(trace_y))
        return fail(h, Q4_EALIGN, "run_stack: misaligned pointer");
    for (int l = 0; l < n_layers; ++l) {
        const q4gemv_layer& L = layers[l];
        if (!L.qkv || !L.o || !L.gate_up || !L.down)
            return fail(h, Q4_EINVAL, "run_stack: null matrix in layer %d", l);
        if (!aligned16(L.qkv) || !aligned16(L.o) || !aligned16(L.gate_up) || !aligned16(L.down))
            return fail(h, Q4_EALIGN, "run_stack: misaligned matrix in layer %d", l);
    }
    Q4_CUDA(h, cudaSetDevice(h->device));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    void* x_out_user = x_out;
    if (host_in || host_out) {
        cudaStreamCaptureStatus cs0 = cudaStreamCaptureStatusNone;
        Q4_CUDA(h, cudaStreamIsCapturing(st, &cs0));
        if (cs0 != cudaStreamCaptureStatusNone)
            return fail(h, Q4_EUNSUPPORTED, "run_stack: host vectors cannot be used during stream capture");
        if (hidden > h->hio_elems) {
            if (h->fault == kFaultAlloc) return fail(h, Q4_EFAULTINJ, "injected allocation failure");
            Q4_CUDA(h, cudaStreamSynchronize(st));
            cudaFree(h->hio);
            h->hio = nullptr;
            h->hio_elems = 0;
            const int64_t n = (hidden + 7) / 8 * 8;
            if (cudaMalloc(&h->hio, 2 * n * sizeof(__half)) != cudaSuccess)
                return fail(h, Q4_ENOMEM, "run_stack: host-vector staging allocation failed");
            h->hio_elems = n;
        }
        if (host_in) {
            Q4_CUDA(h, cudaMemcpyAsync(h->hio, x_in, hidden * sizeof(__half), cudaMemcpyHostToDevice, st));
            x_in = h->hio;
        }
        if (host_out) x_out = h->hio + h->hio_elems;
    }

    StackKey k;
    k.layers.assign(layers, layers + n_layers);
    k.hidden = hidden;
    k.qkv_n = qkv_n;
    k.ffn = ffn;
    k.x_in = x_in;
    k.x_out = x_out;
    k.trace_x = trace_x;
    k.trace_y = trace_y;
    k.gated = gated;

    // Intermediate buffers (outside any capture: allocation is not captured).
    const size_t need = (size_t)((qkv_n + 7) / 8 * 8 + (hidden + 7) / 8 * 8 +
                                 (2 * ffn + 7) / 8 * 8 + (hidden + 7) / 8 * 8);
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    Q4_CUDA(h, cudaStreamIsCapturing(st, &cs));
    if (need > h->act_elems) {
        if (cs != cudaStreamCaptureStatusNone)
            return fail(h, Q4_EUNSUPPORTED,
                        "run_stack: first call with these sizes must happen outside stream capture");
        if (h->fault == kFaultAlloc) return fail(h, Q4_EFAULTINJ, "injected allocation failure");
        Q4_CUDA(h, cudaStreamSynchronize(st));
        cudaFree(h->act);
        h->act = nullptr;
        h->act_elems = 0;
        if (cudaMalloc(&h->act, need * sizeof(__half)) != cudaSuccess)
            return fail(h, Q4_ENOMEM, "run_stack: activation buffer allocation failed");
        h->act_elems = need;
    }

    const int64_t kmax_step = hidden > ffn ? hidden : ffn;
    if (h->stack_mode == kStackPersistent && kmax_step <= (int64_t)kStackKmax &&
        q4::stack_smem_bytes((int)kmax_step, kWarps, kR1, kC1) <= kMaxDynSmem &&
        (!gated || h->sms <= q4::kStackMaxCtas)) {
        if (!h->desc_valid || !(h->desc_key == k)) {
            if (cs != cudaStreamCaptureStatusNone)
                return fail(h, Q4_EUNSUPPORTED,
                            "run_stack: first call with these arguments must happen outside stream capture");
            if (gated && !h->gscr) {
                if (h->fault == kFaultAlloc) return fail(h, Q4_EFAULTINJ, "injected allocation failure");
                if (cudaMalloc(&h->gscr, (size_t)h->sms * q4::kStackMaxCtas * 4 * sizeof(uint4)) != cudaSuccess) {
                    h->gscr = nullptr;
                    return fail(h, Q4_ENOMEM, "run_stack: gated scratch allocation failed");
                }
            }
            std::vector<q4::StackGemv> desc;
            build_descriptors(h, k, desc);
            if ((int)desc.size() > h->desc_cap) {
                if (h->fault == kFaultAlloc) return fail(h, Q4_EFAULTINJ, "injected allocation failure");
                Q4_CUDA(h, cudaStreamSynchronize(st));
                cudaFree(h->desc);
                h->desc = nullptr;
                h->desc_cap = 0;
                if (cudaMalloc(&h->desc, desc.size() * sizeof(q4::StackGemv)) != cudaSuccess)
                    return fail(h, Q4_ENOMEM, "run_stack: descriptor allocation failed");
                h->desc_cap = (int)desc.size();
            }
            Q4_CUDA(h, cudaStreamSynchronize(st));
            Q4_CUDA(h, cudaMemcpy(h->desc, desc.data(), desc.size() * sizeof(q4::StackGemv),
                                  cudaMemcpyHostToDevice));
            h->desc_key = k;
            h->desc_valid = true;
        }
        return finish_host_out(h, enqueue_stack_persistent(h, k, st), host_out, x_out_user, x_out,
                               hidden, st);
    }
    if (cs != cudaStreamCaptureStatusNone) return enqueue_stack(h, k, st);

    if (!h->exec || !(h->key == k)) {
        if (h->fault == kFaultGraph) return fail(h, Q4_EFAULTINJ, "injected graph failure");
        if (h->exec) {
            cudaGraphExecDestroy(h->exec);
            h->exec = nullptr;
        }
        Q4_CUDA(h, cudaStreamBeginCapture(h->cap, cudaStreamCaptureModeThreadLocal));
        const int rc = enqueue_stack(h, k, h->cap);
        cudaGraph_t graph = nullptr;
        const cudaError_t ee = cudaStreamEndCapture(h->cap, &graph);
        if (rc != Q4_OK) {
            if (graph) cudaGraphDestroy(graph);
            return rc;
        }
        if (ee != cudaSuccess) return cuda_fail(h, ee, "cudaStreamEndCapture");
        const cudaError_t ei = cudaGraphInstantiate(&h->exec, graph, 0);
        cudaGraphDestroy(graph);
        if (ei != cudaSuccess) {
            h->exec = nullptr;
            return cuda_fail(h, ei, "cudaGraphInstantiate");
        }
        h->key = k;
    }
    Q4_CUDA(h, cudaGraphLaunch(h->exec, st));
    return finish_host_out(h, Q4_OK, host_out, x_out_user, x_out, hidden, st);
}
}  // namespace

int q4gemv_run_stack(q4gemv_t h, const q4gemv_layer* layers, int n_layers, int64_t hidden,
                     int64_t qkv_n, int64_t ffn, const void* x_in, void* x_out, void* trace_x,
                     void* trace_y, q4gemv_stream_t stream) {
    return run_stack_impl(h, layers, n_layers, hidden, qkv_n, ffn, x_in, x_out, trace_x, trace_y, stream,
                          false);
}

int q4gemv_run_stack_gated(q4gemv_t h, const q4gemv_layer* layers, int n_layers, int64_t hidden,
                           int64_t qkv_n, int64_t ffn, const void* x_in, void* x_out,
                           q4gemv_stream_t stream) {
    return run_stack_impl(h, layers, n_layers, hidden, qkv_n, ffn, x_in, x_out, nullptr, nullptr, stream,
                          true);
}

int q4gemv_shard_rows(int64_t N, int world, int rank, int64_t* row0, int64_t* rows, int64_t* chunk) {
    if (N <= 0 || world < 1 || rank < 0 || rank >= world || !row0 || !rows) return Q4_EINVAL;
    const int64_t c = shard_chunk(N, world);
    const int64_t r0 = (int64_t)rank * c;
    *row0 = r0 < N ? r0 : N;
    *rows = N - r0 < 0 ? 0 : (N - r0 < c ? N - r0 : c);
    if (chunk) *chunk = c;
    return Q4_OK;
}

int q4gemv_comm_unique_id(void* id) {
    if (!id) return Q4_EINVAL;
    if (!nccl_load()) return Q4_EUNSUPPORTED;
    ncclUniqueId u;
    if (g_nccl.GetUniqueId(&u) != ncclSuccess) return Q4_ECUDA;
    memcpy(id, &u, sizeof u);
    return Q4_OK;
}

int q4gemv_comm_init(q4gemv_t h, int world, int rank, const void* id) {
    if (!h || !id) return Q4_EINVAL;
    if (world < 1 || rank < 0 || rank >= world) return fail(h, Q4_EINVAL, "comm_init: rank %d of %d", rank, world);
    if (!nccl_load()) return fail(h, Q4_EUNSUPPORTED, "comm_init: libnccl.so.2 could not be loaded");
    Q4_CUDA(h, cudaSetDevice(h->device));
    Q4_CUDA(h, cudaDeviceSynchronize());
    shard_release(h);
    ncclUniqueId u;
    memcpy(&u, id, sizeof u);
    ncclComm_t c = nullptr;
    const ncclResult_t r = g_nccl.CommInitRank(&c, world, u, rank);
    if (r != ncclSuccess) return fail(h, Q4_ECUDA, "ncclCommInitRank: %s", g_nccl.GetErrorString(r));
    h->comm = c;
    h->world = world;
    h->rank = rank;
    return Q4_OK;
}

namespace {
// The exchange blob (layout stated with q4gemv_peer_layout in the header).
struct PeerBlob {
    uint32_t magic, version;
    int32_t world, rank;
    int64_t hidden, qkv_n, ffn;
    uint64_t bytes;
    unsigned char handle[64];
    unsigned char pad[16];
};
static_assert(sizeof(PeerBlob) == Q4GEMV_PEER_BLOB_BYTES, "blob size");
constexpr uint32_t kPeerMagic = 0x51345045u, kPeerVersion = 1u;
int64_t align256(int64_t v) { return (v + 255) / 256 * 256; }
}  // namespace

int q4gemv_peer_layout(int world, int64_t hidden, int64_t qkv_n, int64_t ffn, int64_t* off) {
    if (!off || world < 1 || world > Q4GEMV_PEER_MAX_WORLD || hidden <= 0 || qkv_n <= 0 || ffn <= 0)
        return Q4_EINVAL;
    const int64_t n_of[4] = {qkv_n, hidden, 2 * ffn, hidden};
    int64_t o = 0;
    for (int t = 0; t < 4; ++t) {
        off[t] = o;                    // world * chunk stamped words
        o += align256((int64_t)world * shard_chunk(n_of[t], world) * 4);
    }
    off[4] = o;                        // steps run, arrival-count epoch
    o += 256;
    off[5] = o;
    return Q4_OK;
}

int q4gemv_peer_check(const void* blobs, int world) {
    if (!blobs || world < 1 || world > Q4GEMV_PEER_MAX_WORLD) return Q4_EINVAL;
    const PeerBlob* b = static_cast<const PeerBlob*>(blobs);
    for (int r = 0; r < world; ++r) {
        if (b[r].magic != kPeerMagic || b[r].version != kPeerVersion || b[r].world != world || b[r].rank != r)
            return Q4_EINVAL;
        if (b[r].hidden != b[0].hidden || b[r].qkv_n != b[0].qkv_n || b[r].ffn != b[0].ffn ||
            b[r].bytes != b[0].bytes)
            return Q4_EINVAL;
    }
    int64_t off[6];
    if (q4gemv_peer_layout(world, b[0].hidden, b[0].qkv_n, b[0].ffn, off) != Q4_OK) return Q4_EINVAL;
    return (uint64_t)off[5] == b[0].bytes ? Q4_OK : Q4_EINVAL;
}

int q4gemv_peer_export(q4gemv_t h, int world, int rank, int64_t hidden, int64_t qkv_n, int64_t ffn,
                       void* blob) {
    if (!h || !blob) return Q4_EINVAL;
    if (world < 1 || world > Q4GEMV_PEER_MAX_WORLD || rank < 0 || rank >= world)
        return fail(h, Q4_EINVAL, "peer_export: rank %d of %d", rank, world);
    int64_t off[6];
    if (q4gemv_peer_layout(world, hidden, qkv_n, ffn, off) != Q4_OK)
        return fail(h, Q4_EINVAL, "peer_export: invalid shapes");
    if (h->fault == kFaultAlloc) return fail(h, Q4_EFAULTINJ, "injected allocation failure");
    Q4_CUDA(h, cudaSetDevice(h->device));
    Q4_CUDA(h, cudaDeviceSynchronize());
    peer_release(h);
    if (cudaMalloc(&h->px_base, (size_t)off[5]) != cudaSuccess) {
        h->px_base = nullptr;
        return fail(h, Q4_ENOMEM, "peer_export: exchange buffer of %lld bytes", (long long)off[5]);
    }
    Q4_CUDA(h, cudaMemset(h->px_base, 0, (size_t)off[5]));
    Q4_CUDA(h, cudaDeviceSynchronize());
    PeerBlob b;
    memset(&b, 0, sizeof b);
    b.magic = kPeerMagic;
    b.version = kPeerVersion;
    b.world = world;
    b.rank = rank;
    b.hidden = hidden;
    b.qkv_n = qkv_n;
    b.ffn = ffn;
    b.bytes = (uint64_t)off[5];
    if (world > 1) {
        cudaIpcMemHandle_t ih;
        Q4_CUDA(h, cudaIpcGetMemHandle(&ih, h->px_base));
        static_assert(sizeof(ih) == sizeof(b.handle), "IPC handle size");
        memcpy(b.handle, &ih, sizeof ih);
    }
    memcpy(blob, &b, sizeof b);
    memcpy(h->px_blob, &b, sizeof b);
    for (int i = 0; i < 6; ++i) h->px_off[i] = off[i];
    h->px_world = world;
    h->px_rank = rank;
    h->px_hidden = hidden;
    h->px_qkv = qkv_n;
    h->px_ffn = ffn;
    return Q4_OK;
}

int q4gemv_peer_open(q4gemv_t h, const void* blobs) {
    if (!h || !blobs) return Q4_EINVAL;
    if (!h->px_base) return fail(h, Q4_EINVAL, "peer_open: no exchange exported");
    const int world = h->px_world, rank = h->px_rank;
    if (q4gemv_peer_check(blobs, world) != Q4_OK) return fail(h, Q4_EINVAL, "peer_open: inconsistent blobs");
    const PeerBlob* b = static_cast<const PeerBlob*>(blobs);
    if (memcmp(&b[rank], h->px_blob, sizeof(PeerBlob)) != 0)
        return fail(h, Q4_EINVAL, "peer_open: blob %d is not this handle's export", rank);
    Q4_CUDA(h, cudaSetDevice(h->device));
    uint8_t* base[Q4GEMV_PEER_MAX_WORLD];
    for (int p = 0; p < world; ++p) {
        if (p == rank) {
            base[p] = h->px_base;
            continue;
        }
        if (h->px_remote[p]) {
            cudaIpcCloseMemHandle(h->px_remote[p]);
            h->px_remote[p] = nullptr;
        }
        cudaIpcMemHandle_t ih;
        memcpy(&ih, b[p].handle, sizeof ih);
        void* ptr = nullptr;
        const cudaError_t e = cudaIpcOpenMemHandle(&ptr, ih, cudaIpcMemLazyEnablePeerAccess);
        if (e != cudaSuccess) return cuda_fail(h, e, "peer_open: cudaIpcOpenMemHandle");
        h->px_remote[p] = static_cast<uint8_t*>(ptr);
        base[p] = h->px_remote[p];
    }
    const int64_t n_of[4] = {h->px_qkv, h->px_hidden, 2 * h->px_ffn, h->px_hidden};
    uint32_t* ytab[4 * Q4GEMV_PEER_MAX_WORLD];
    for (int p = 0; p < world; ++p)
        for (int t = 0; t < 4; ++t)
            ytab[t * world + p] = reinterpret_cast<uint32_t*>(base[p] + h->px_off[t]) + rank * shard_chunk(n_of[t], world);
    cudaFree(h->px_ytab);
    h->px_ytab = nullptr;
    if (cudaMalloc(&h->px_ytab, sizeof(uint32_t*) * 4 * world) != cudaSuccess)
        return fail(h, Q4_ENOMEM, "peer_open: pointer table");
    Q4_CUDA(h, cudaMemcpy(h->px_ytab, ytab, sizeof(uint32_t*) * 4 * world, cudaMemcpyHostToDevice));
    if (h->sh_exec) cudaGraphExecDestroy(h->sh_exec);
    h->sh_exec = nullptr;
    h->px_open = true;
    return Q4_OK;
}

int q4gemv_peer_close(q4gemv_t h) {
    if (!h) return Q4_EINVAL;
    Q4_CUDA(h, cudaSetDevice(h->device));
    Q4_CUDA(h, cudaDeviceSynchronize());
    peer_release(h);
    return Q4_OK;
}

int q4gemv_run_stack_sharded(q4gemv_t h, const q4gemv_layer* layers, int n_layers, int64_t hidden,
                             int64_t qkv_n, int64_t ffn, const void* x_in, void* x_out,
                             q4gemv_stream_t stream) {
    if (!h) return Q4_EINVAL;
    const bool px = h->px_open && h->px_hidden == hidden && h->px_qkv == qkv_n && h->px_ffn == ffn;
    if (!px && !h->comm)
        return fail(h, Q4_EINVAL, "run_stack_sharded: no communicator and no peer exchange for these shapes");
    const int world = px ? h->px_world : h->world, rank = px ? h->px_rank : h->rank;
    if (!layers || !x_in || !x_out) return fail(h, Q4_EINVAL, "run_stack_sharded: null pointer");
    if (n_layers < 1 || n_layers > 4096) return fail(h, Q4_ESHAPE, "run_stack_sharded: n_layers out of range");
    if (qkv_n < hidden) return fail(h, Q4_ESHAPE, "run_stack_sharded: qkv_n < hidden");
    const int64_t n_of[4] = {qkv_n, hidden, 2 * ffn, hidden};
    const int64_t k_of[4] = {hidden, hidden, hidden, ffn};
    for (int t = 0; t < 4; ++t) {
        const int sc = check_shape(n_of[t], k_of[t]);
        if (sc != Q4_OK) return fail(h, sc, "run_stack_sharded: invalid matrix shape");
        if (!dp2a_fits(1, k_of[t])) return fail(h, Q4_EUNSUPPORTED, "run_stack_sharded: K too large");
    }
    if (is_host_pointer(x_in) || is_host_pointer(x_out))
        return fail(h, Q4_EINVAL, "run_stack_sharded: x_in and x_out must be device memory");
    if (!aligned16(x_in) || !aligned16(x_out)) return fail(h, Q4_EALIGN, "run_stack_sharded: misaligned vector");
    int64_t rows[4], chunk[4];
    for (int t = 0; t < 4; ++t) {
        int64_t r0 = 0;
        q4gemv_shard_rows(n_of[t], world, rank, &r0, &rows[t], &chunk[t]);
    }
    for (int l = 0; l < n_layers; ++l) {
        const q4gemv_layer& L = layers[l];
        const void* m[4] = {L.qkv, L.o, L.gate_up, L.down};
        for (int t = 0; t < 4; ++t) {
            if (rows[t] > 0 && !m[t]) return fail(h, Q4_EINVAL, "run_stack_sharded: null matrix in layer %d", l);
            if (!aligned16(m[t])) return fail(h, Q4_EALIGN, "run_stack_sharded: misaligned matrix in layer %d", l);
        }
    }
    Q4_CUDA(h, cudaSetDevice(h->device));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    Q4_CUDA(h, cudaStreamIsCapturing(st, &cs));
    if (cs != cudaStreamCaptureStatusNone)
        return fail(h, Q4_EUNSUPPORTED, "run_stack_sharded: not available inside a stream capture");
    // Buffers (NCCL exchange): this rank's rows (zero past them) and the
    // gathered vector, per matrix type.  The peer exchange uses its own.
    for (int t = 0; t < 4 && !px; ++t) {
        if (chunk[t] == h->sh_chunk[t] && h->sh_slice[t]) continue;
        if (h->fault == kFaultAlloc) return fail(h, Q4_EFAULTINJ, "injected allocation failure");
        Q4_CUDA(h, cudaStreamSynchronize(st));
        if (h->sh_exec) {
            cudaGraphExecDestroy(h->sh_exec);
            h->sh_exec = nullptr;
        }
        cudaFree(h->sh_slice[t]);
        cudaFree(h->sh_gather[t]);
        h->sh_slice[t] = h->sh_gather[t] = nullptr;
        h->sh_chunk[t] = 0;
        if (cudaMalloc(&h->sh_slice[t], chunk[t] * sizeof(__half)) != cudaSuccess ||
            cudaMalloc(&h->sh_gather[t], chunk[t] * h->world * sizeof(__half)) != cudaSuccess)
            return fail(h, Q4_ENOMEM, "run_stack_sharded: buffer allocation failed");
        Q4_CUDA(h, cudaMemset(h->sh_slice[t], 0, chunk[t] * sizeof(__half)));
        h->sh_chunk[t] = chunk[t];
    }
    // Peer exchange: arrival counts of the split tiles, one set per matrix
    // of the layer, counting on across layers and steps (zeroed, with their
    // step count, when they grow or the layer count changes).
    int64_t tmax = 0;
    for (int t = 0; t < 4; ++t) tmax = std::max(tmax, (rows[t] + 31) / 32);
    if (px && (4 * tmax > h->px_cnt_elems || n_layers != h->px_cnt_layers)) {
        if (h->fault == kFaultAlloc) return fail(h, Q4_EFAULTINJ, "injected allocation failure");
        Q4_CUDA(h, cudaStreamSynchronize(st));
        if (h->sh_exec) {
            cudaGraphExecDestroy(h->sh_exec);
            h->sh_exec = nullptr;
        }
        if (4 * tmax > h->px_cnt_elems) {
            cudaFree(h->px_cnt);
            h->px_cnt = nullptr;
            h->px_cnt_elems = 0;
            if (cudaMalloc(&h->px_cnt, (size_t)(4 * tmax) * sizeof(int)) != cudaSuccess)
                return fail(h, Q4_ENOMEM, "run_stack_sharded: arrival counts");
            h->px_cnt_elems = 4 * tmax;
        }
        Q4_CUDA(h, cudaMemset(h->px_cnt, 0, (size_t)h->px_cnt_elems * sizeof(int)));
        Q4_CUDA(h, cudaMemset(h->px_base + h->px_off[4] + 4, 0, 4));   // their step count
        Q4_CUDA(h, cudaDeviceSynchronize());
        h->px_cnt_layers = n_layers;
    }
    __half* gather[4];
    for (int t = 0; t < 4; ++t) gather[t] = px ? nullptr : h->sh_gather[t];
    StackKey k;
    k.layers.assign(layers, layers + n_layers);
    k.hidden = hidden;
    k.qkv_n = qkv_n;
    k.ffn = ffn;
    k.x_in = x_in;
    k.x_out = x_out;
    k.trace_x = px ? static_cast<void*>(h->px_base) : nullptr;   // the exchange is part of the key
    if (!h->sh_exec || !(h->sh_key == k)) {
        if (h->fault == kFaultGraph) return fail(h, Q4_EFAULTINJ, "injected graph failure");
        if (h->sh_exec) {
            cudaGraphExecDestroy(h->sh_exec);
            h->sh_exec = nullptr;
        }
        // Every rank enqueues the same sequence: per GEMV its rows (the
        // M = 1 kernel on its row slice, input scaled to unit RMS) and every
        // rank's rows gathered -- by the kernel's own stores into every
        // rank's buffer and a stamp (peer exchange), or an NCCL all-gather;
        // the step ends with the renorm.
        Q4_CUDA(h, cudaStreamBeginCapture(h->cap, cudaStreamCaptureModeThreadLocal));
        int rc = Q4_OK;
        unsigned* seq = px ? reinterpret_cast<unsigned*>(h->px_base + h->px_off[4]) : nullptr;
        const uint32_t* words[4];
        for (int t = 0; t < 4; ++t)
            words[t] = px ? reinterpret_cast<const uint32_t*>(h->px_base + h->px_off[t]) : nullptr;
        // the "timeout" test knob: every wait for a stamp nothing writes, short budget
        const unsigned poll_limit = h->fault == kFaultTimeout ? (1u << 10) : (1u << 26);
        const unsigned unreachable = h->fault == kFaultTimeout ? 1u : 0u;
        q4::PeerArgs pa = {};
        if (px) {
            pa.n = world;
            pa.seq = seq;
            pa.per_step = 4 * n_layers;
            pa.poll_limit = poll_limit;
            pa.unreachable = unreachable;
            q4::peer_step_kernel<<<1, 1, 0, h->cap>>>(seq);
            const cudaError_t e = cudaGetLastError();
            if (e != cudaSuccess) rc = cuda_fail(h, e, "peer step launch");
        }
        bool last_was_gemv = false;
        for (int i = 0; i < 4 * n_layers && rc == Q4_OK; ++i) {
            const int t = i % 4;
            const q4gemv_layer& L = layers[i / 4];
            const void* W = t == 0 ? L.qkv : t == 1 ? L.o : t == 2 ? L.gate_up : L.down;
            const __half* xin = i == 0 ? static_cast<const __half*>(x_in) : gather[(t + 3) % 4];
            if (px) {
                // Each GEMV stores its rows, stamped, into every rank's buffer t;
                // the next stages buffer t's words once they carry its stamp.
                // Launched programmatically after a GEMV: its weights stream in
                // while that one ends.  Arrival counts per matrix of the layer;
                // the split workspace alternates between two halves.
                pa.y = h->px_ytab + t * world;
                pa.xw = i > 0 ? words[(t + 3) % 4] : nullptr;
                pa.g = i;
                pa.wait = i > 0 ? 1 : 0;
                if (rows[t] > 0) {
                    rc = launch_gemv(h, W, xin, nullptr, 1, rows[t], k_of[t], i == 0 ? 0 : 1, nullptr,
                                     h->cap, last_was_gemv, false, false, &pa, h->px_cnt + (int64_t)t * tmax,
                                     h->ws + (size_t)(i & 1) * h->sms * 2 * 32);
                    last_was_gemv = true;
                } else {
                    last_was_gemv = false;   // no rows of this matrix here
                }
                continue;
            }
            if (rows[t] > 0)
                rc = launch_gemv(h, W, xin, h->sh_slice[t], 1, rows[t], k_of[t], i == 0 ? 0 : 1, nullptr,
                                 h->cap, false);
            if (rc == Q4_OK) {
                const ncclResult_t r = g_nccl.AllGather(h->sh_slice[t], h->sh_gather[t], (size_t)chunk[t],
                                                        ncclFloat16, h->comm, h->cap);
                if (r != ncclSuccess) rc = fail(h, Q4_ECUDA, "ncclAllGather: %s", g_nccl.GetErrorString(r));
            }
        }
        if (rc == Q4_OK && px) {
            // the last GEMV's words, every rank's rows, unpacked and renormalised
            pa.g = 4 * n_layers;
            q4::peer_renorm_kernel<kWarps><<<1, kThreads, 0, h->cap>>>(words[3], static_cast<__half*>(x_out),
                                                                     (int)hidden, pa, h->err);
            const cudaError_t e = cudaGetLastError();
            if (e != cudaSuccess) rc = cuda_fail(h, e, "peer renorm launch");
        } else if (rc == Q4_OK) {
            rc = launch_renorm(h, gather[3], static_cast<__half*>(x_out), (int)hidden, h->cap, false);
        }
        cudaGraph_t graph = nullptr;
        const cudaError_t ee = cudaStreamEndCapture(h->cap, &graph);
        if (rc != Q4_OK) {
            if (graph) cudaGraphDestroy(graph);
            return rc;
        }
        if (ee != cudaSuccess) return cuda_fail(h, ee, "cudaStreamEndCapture");
        const cudaError_t ei = cudaGraphInstantiate(&h->sh_exec, graph, 0);
        cudaGraphDestroy(graph);
        if (ei != cudaSuccess) {
            h->sh_exec = nullptr;
            return cuda_fail(h, ei, "cudaGraphInstantiate");
        }
        h->sh_key = k;
    }
    Q4_CUDA(h, cudaGraphLaunch(h->sh_exec, st));
    return Q4_OK;
}

int q4gemv_sync_status(q4gemv_t h, q4gemv_stream_t stream) {
    if (!h) return Q4_EINVAL;
    Q4_CUDA(h, cudaSetDevice(h->device));
    Q4_CUDA(h, cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    int word = 0;
    Q4_CUDA(h, cudaMemcpy(&word, h->err, sizeof(int), cudaMemcpyDeviceToHost));
    if (word != 0) {
        Q4_CUDA(h, cudaMemset(h->err, 0, sizeof(int)));
        if (word == q4::kDevTimeout) return fail(h, Q4_ETIMEOUT, "device wait timed out");
        if (word == q4::kDevConcurrent) return fail(h, Q4_ECONCURRENT, "overlapping calls detected");
        return fail(h, Q4_ECUDA, "device error word %d", word);
    }
    return Q4_OK;
}

}  // extern "C"
