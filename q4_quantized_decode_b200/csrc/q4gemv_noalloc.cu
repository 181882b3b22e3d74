// q4gemv_run_noalloc: the M <= 2 GEMV without a handle and without any
// device allocation, for callers that cannot allocate device memory.
//
// q4gemv_create allocates its workspace with cudaMalloc.  Some callers cannot
// do that: code that runs while a stream is being captured in global capture
// mode (where cudaMalloc is an error), code on a latency-critical thread that
// must not take the implicit device synchronisation cudaMalloc/cudaFree can
// cause, or a plug-in living inside a host application that owns all device
// memory and forbids allocations behind its back.  This entry point gives them
// the same kernel with its scratch (split-tile partial sums, per-tile arrival
// counters, the device error word) in a fixed file-scope device array instead.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/q4gemv.h"
#include "gemv_dp2a.cuh"

namespace {

constexpr int kNaWarps = 16;                    // warps per CTA, as in q4gemv_run
constexpr int kNaThreads = kNaWarps * 32;
constexpr int kNaR1 = 4, kNaC1 = 4;             // ring of the M = 1 kernel
constexpr int kNaR2 = 2, kNaC2 = 4;             // ring of the M = 2 kernel
constexpr int kNaMinSegsPerWarp = 4;
constexpr size_t kNaMaxDynSmem = 224 * 1024;

// Static scratch layout: partials for up to kNaMaxWarps warps (two slots, two
// vectors, 32 rows of fp32), then one arrival counter per 32-row tile, then
// the error word.
constexpr int kNaMaxWarps = 2560;
constexpr int kNaMaxTiles = Q4GEMV_NOALLOC_MAX_N / 32;
constexpr size_t kNaWsBytes = (size_t)kNaMaxWarps * 2 * 2 * 32 * sizeof(float);
constexpr size_t kNaCntOffset = kNaWsBytes;
constexpr size_t kNaErrOffset = kNaCntOffset + (size_t)kNaMaxTiles * sizeof(int);
constexpr size_t kNaScratchBytes = Q4GEMV_NOALLOC_SCRATCH_BYTES;
static_assert(kNaErrOffset + 256 <= kNaScratchBytes, "static scratch too small");

// One copy per device that loads the library; its contents persist between
// calls (the counters are re-armed by the kernel and cleared before each
// launch).
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNaScratchBytes];

struct NaDevice {
    bool ready = false;
    unsigned char* scratch = nullptr;   // device address of g_noalloc_scratch
    int sms = 0;
};
constexpr int kNaMaxDevices = 64;
NaDevice g_na_dev[kNaMaxDevices];
std::mutex g_na_mu;

#define Q4_NA_KERNEL_1 q4::gemv_dp2a_kernel<1, kNaWarps, kNaR1, kNaC1>
#define Q4_NA_KERNEL_2 q4::gemv_dp2a_kernel<2, kNaWarps, kNaR2, kNaC2>

size_t na_smem(int M, int64_t K) {
    return M == 1 ? q4::gemv_dp2a_smem_bytes(1, (int)K, kNaWarps, kNaR1, kNaC1)
                  : q4::gemv_dp2a_smem_bytes(2, (int)K, kNaWarps, kNaR2, kNaC2);
}

// Once per device, with that device current: resolve the array's device
// address (the host-side symbol is only a stand-in), read the SM count and
// allow the kernels their shared memory.
int na_setup(int dev, NaDevice** out) {
    std::lock_guard<std::mutex> lock(g_na_mu);
    NaDevice& d = g_na_dev[dev];
    if (!d.ready) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return Q4_ECUDA;
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return Q4_ECUDA;
        if (cudaFuncSetAttribute(Q4_NA_KERNEL_1, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kNaMaxDynSmem) != cudaSuccess ||
            cudaFuncSetAttribute(Q4_NA_KERNEL_2, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kNaMaxDynSmem) != cudaSuccess)
            return Q4_ECUDA;
        d.scratch = static_cast<unsigned char*>(p);
        d.sms = sms;
        d.ready = true;
    }
    *out = &d;
    return Q4_OK;
}

}  // namespace

extern "C" int q4gemv_run_noalloc(const void* W, const void* x, void* y, int M, int64_t N,
                                  int64_t K, q4gemv_stream_t stream) {
    if (M < 1 || M > 2) return Q4_EUNSUPPORTED;
    if (N <= 0 || K <= 0 || K % 32 != 0 || N > Q4GEMV_NOALLOC_MAX_N) return Q4_ESHAPE;
    if (M * K > (int64_t)q4::kXChunksPerThread * 8 * kNaThreads || na_smem(M, K) > kNaMaxDynSmem)
        return Q4_ESHAPE;
    if (!W || !x || !y) return Q4_EINVAL;
    if ((reinterpret_cast<uintptr_t>(W) | reinterpret_cast<uintptr_t>(x) |
         reinterpret_cast<uintptr_t>(y)) & 15u)
        return Q4_EALIGN;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNaMaxDevices) return Q4_ECUDA;
    NaDevice* d = nullptr;
    const int rc = na_setup(dev, &d);
    if (rc != Q4_OK) return rc;

    const int KB = (int)(K / 32);
    const int T = (int)((N + 31) / 32);
    const int S = T * KB;
    int ctas = d->sms;
    if (ctas * kNaWarps > kNaMaxWarps) ctas = kNaMaxWarps / kNaWarps;
    const int want_warps = (S + kNaMinSegsPerWarp - 1) / kNaMinSegsPerWarp;
    if (want_warps < ctas * kNaWarps) ctas = (want_warps + kNaWarps - 1) / kNaWarps;
    if (ctas < 1) ctas = 1;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int* cnt = reinterpret_cast<int*>(d->scratch + kNaCntOffset);
    // The array keeps the last call's contents: the counters must start at 0.
    if (cudaMemsetAsync(cnt, 0, (size_t)T * sizeof(int), st) != cudaSuccess) return Q4_ECUDA;

    q4::GemvArgs a;
    a.W = static_cast<const uint8_t*>(W);
    a.x = static_cast<const __half*>(x);
    a.y = static_cast<__half*>(y);
    a.ws = reinterpret_cast<float*>(d->scratch);
    a.cnt = cnt;
    a.err = reinterpret_cast<int*>(d->scratch + kNaErrOffset);
    a.trace_x = nullptr;
    a.N = N;
    a.K = (int)K;
    a.KB = KB;
    a.T = T;
    a.S = S;
    a.G = ctas * kNaWarps < S ? ctas * kNaWarps : S;
    a.renorm = 0;
    a.sc = q4::make_split(a.S, a.G);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ctas);
    cfg.blockDim = dim3(kNaThreads);
    cfg.dynamicSmemBytes = na_smem(M, K);
    cfg.stream = st;
    cfg.numAttrs = 0;
    const cudaError_t e = (M == 1) ? cudaLaunchKernelEx(&cfg, Q4_NA_KERNEL_1, a)
                                   : cudaLaunchKernelEx(&cfg, Q4_NA_KERNEL_2, a);
    return e == cudaSuccess ? Q4_OK : Q4_ECUDA;
}
