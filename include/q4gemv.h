/*
 * q4gemv -- Q4_0 dequantise-and-multiply matrix-vector products on NVIDIA
 * B200 (sm_100a), the memory-bound core of quantised LLM decode.
 *
 * The operation (SwarmLLM coverage, originshq.com page, section "The Engine:
 * ~50 WGSL Kernels Written From Scratch"): decode reads every weight once per
 * token, dequantises the 4-bit values and accumulates the matrix-vector
 * product; speculative verification and prefill apply the same weights to a
 * handful of activation vectors (aipolix en-US page, section "Speculation is
 * used to amortize network round trips"; originshq.com page, section
 * "Multi-Device Performance and the Network Penalty", 16 tokens per round
 * trip).
 *
 *   y[m][n] = sum_k W[n][k] * x[m][k],   0 <= m < M, 0 <= n < N, 0 <= k < K
 *
 * W is Q4_0: the pages name the format (taozi.news page, section
 * "支持模型与限制") without laying it out; the GGUF block is used.  Each row
 * holds K/32 blocks of 18 bytes: an f16 scale d (little-endian) and 16 bytes
 * qs; weight j of a block has code q_j = qs[j] & 15 (j < 16) or
 * qs[j-16] >> 4 (j >= 16) and value (q_j - 8) * d.  x and y are row-major
 * IEEE binary16.
 *
 * Conventions for every entry point
 *  - All buffers are caller-owned device memory (except where a parameter
 *    says "host"); the library never frees them.  Pointers to device data
 *    must be 16-byte aligned.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *    default stream) and perform no implicit device synchronisation, except
 *    q4gemv_create, q4gemv_destroy and q4gemv_sync_status.
 *  - Every call returns a q4gemv_status.  Arguments are validated on the host
 *    before anything is launched; an invalid call launches nothing.  The
 *    library throws no C++ exception across this interface and never traps
 *    on the device.  The text of the last error of a handle is available from
 *    q4gemv_last_error.
 *  - A handle owns a small device workspace (split-K partial sums, per-tile
 *    arrival counters, an error word) and the cached CUDA graph of
 *    q4gemv_run_stack.  Calls on one handle must not overlap on the GPU: keep
 *    them on one stream, or order them with events.  Use one handle per
 *    concurrent stream.  Overlap that the kernels detect is reported as
 *    Q4_ECONCURRENT by the next q4gemv_sync_status.
 */
#ifndef Q4GEMV_H
#define Q4GEMV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define Q4GEMV_API __attribute__((visibility("default")))
#else
#define Q4GEMV_API
#endif

typedef struct q4gemv_ctx* q4gemv_t;   /* opaque, library-owned */
typedef void* q4gemv_stream_t;         /* a cudaStream_t */

typedef enum {
    Q4_OK = 0,
    Q4_EINVAL = -1,        /* null handle or pointer, bad enum value */
    Q4_ESHAPE = -2,        /* K % 32 != 0, N or K <= 0, sizes beyond the limits */
    Q4_EALIGN = -3,        /* a device pointer is not 16-byte aligned */
    Q4_ENOMEM = -4,        /* device or host allocation failed */
    Q4_ECUDA = -5,         /* a CUDA runtime call failed (see q4gemv_last_error) */
    Q4_EUNSUPPORTED = -6,  /* M outside [1, 256], or the device is not sm_100 */
    Q4_ETIMEOUT = -7,      /* a bounded device-side wait gave up */
    Q4_EFAULTINJ = -8,     /* a host step failed on purpose (fault injection) */
    Q4_ECONCURRENT = -9    /* kernels saw overlapping calls on one handle */
} q4gemv_status;

/* Limits checked by validation.  Besides these, ceil(N/32) * (K/32) must be
 * below 2^31. */
#define Q4GEMV_MAX_M 256            /* vectors per q4gemv_run call */
#define Q4GEMV_MAX_M_GEMV 16        /* above this, the tensor-core GEMM path */
#define Q4GEMV_MAX_N (1 << 22)     /* rows */
#define Q4GEMV_MAX_K (1 << 20)     /* columns */

/* Library version, (major << 16) | minor. */
Q4GEMV_API int q4gemv_version(void);

/* Creates a handle bound to CUDA device `device` (made current for the
 * call).  Queries the SM count and allocates the workspace.  Returns
 * Q4_EUNSUPPORTED on a device that is not compute capability 10.x. */
Q4GEMV_API int q4gemv_create(q4gemv_t* out, int device);

/* Synchronises the device, releases the workspace and cached graphs, frees
 * the handle.  Null is accepted (no-op). */
Q4GEMV_API int q4gemv_destroy(q4gemv_t h);

/* Bytes of a GGUF Q4_0 matrix: N * (K/32) * 18; 0 if the shape is invalid. */
Q4GEMV_API size_t q4gemv_gguf_bytes(int64_t N, int64_t K);

/* Bytes of the packed (repacked) matrix: Np * (K/32) * 18 with
 * Np = ceil(N/32)*32; 0 if the shape is invalid.
 *
 * Packed layout (the input of q4gemv_run).  Rows are padded to Np (padding
 * rows hold qs bytes 0x88 and d = +0, i.e. zero weights) and grouped into
 * tiles of 32 rows.  With KB = K/32, segment s = t*KB + b holds block b of
 * the rows of tile t and occupies the 576 bytes from 576*s; row
 * n = 32t + g + 8i (g in [0,8), i in [0,4)):
 *   segment bytes 16*(4g + c) + 4i + e  = qs[4c + e] of that block of row n
 *                                          (c, e in [0,4)), bytes [0, 512);
 *   segment bytes 512 + 8g + 2i, +1      = d of that block of row n
 *                                          (little-endian), bytes [512, 576).
 * A lane (g, c) of a warp thus finds qs word c of rows g, g+8, g+16, g+24 in
 * one 16-byte word and their four scales in one 8-byte word, and a run of
 * segments is one contiguous byte range (one bulk copy). */
Q4GEMV_API size_t q4gemv_packed_bytes(int64_t N, int64_t K);

/* Host-only check of q4gemv_run's arguments (no device access, no handle).
 * Returns the status q4gemv_run would return for these arguments before
 * launching anything. */
Q4GEMV_API int q4gemv_validate(int M, int64_t N, int64_t K, const void* W_packed,
                    const void* x, const void* y);

/* One-time repack of a GGUF Q4_0 matrix into the packed layout.
 *   gguf   : device, q4gemv_gguf_bytes(N, K) bytes (any alignment >= 2)
 *   packed : device, q4gemv_packed_bytes(N, K) bytes, 16-byte aligned,
 *            must not overlap gguf
 * Bit-exact: the packed bytes are a permutation of the GGUF bytes plus the
 * padding rows. */
Q4GEMV_API int q4gemv_repack(q4gemv_t h, const void* gguf, void* packed,
                  int64_t N, int64_t K, q4gemv_stream_t stream);

/* y[M][N] = W x[M][K]^T for a packed W.
 *   W_packed : device, q4gemv_packed_bytes(N, K) bytes
 *   x        : device, M*K binary16, row-major
 *   y        : device, M*N binary16, row-major (written, never read)
 * 1 <= M <= 256, K % 32 == 0.  Accumulation is fp32 or exact integer; y is
 * rounded to nearest even once.  Results beyond the binary16 range become
 * +-Inf; a non-finite x element makes the affected outputs NaN.  For M <= 2
 * the activations of each 32-column block are converted to 16-bit integers
 * with a power-of-two scale chosen so the block's largest magnitude is held
 * exactly (elements within a factor 16 of it are exact; others are rounded
 * to 2^-15 of the block maximum) and the per-block dot products are exact
 * integers.  Deterministic: the same inputs on the same device give the
 * same bits.
 * For 3 <= M <= 16 (and M <= 2 with K beyond the CUDA-core kernel's
 * activation staging) the mma.sync tensor-core kernel runs, as a grid of P
 * column panels whose
 * fp32 sums a second small kernel adds in panel order (P = 1 for large N and
 * K up to about 6,000 columns; more panels for narrow N, so a CTA stages a
 * short activation slice, and for wider K).  The panel sums live in a buffer
 * of P*M*N floats owned by the handle (preallocated for P*M*N <= 2^21; a
 * larger first call grows it, which synchronises the device and must not
 * happen during a stream capture).
 * With the environment variable Q4GEMV_SMALL_M=tcs (read at create) that
 * path runs on the tcgen05 tensor cores instead: kind::i8 MMAs, one per 128
 * rows x 32 columns, the weights dequantised to 16 (q - 8) in tensor memory
 * and the activations converted per block and vector to 15-bit integers X
 * (|X| <= 2^14, the block maximum exact) split into two signed bytes; the
 * int32 block sums are exact and scaled in fp32.  It keeps the same output
 * contract (non-finite inputs give NaN outputs for their vector) and uses
 * the same activation image buffer; it is slower than the mma.sync kernel on
 * the measured shapes and is kept for comparison.
 * For M = 17..256 (prefill chunks) a dense-contraction path on the tcgen05
 * tensor cores runs instead: "dequantise the weight tile, then multiply" --
 * each weight (q - 8) * d is split exactly into two binary16 parts (the
 * rounded value and its remainder), both multiply x (exact products), and
 * the sums accumulate in fp32.  Scales |d| >= 8192 overflow binary16 in the
 * split and give non-finite outputs.  A first kernel writes x into an
 * activation image owned by the handle (ceil(K/64) * Mp * 128 bytes, Mp = M
 * rounded up to 16; preallocated up to 16 MiB, grown like the panel sums);
 * the GEMM kernel covers 256 rows per CTA, and for narrow N splits K so the
 * grid fills the SMs, its fp32 split sums (P*M*N floats, the same buffer as
 * the panel sums) added in split order by the reduce kernel. */
Q4GEMV_API int q4gemv_run(q4gemv_t h, const void* W_packed, const void* x, void* y,
               int M, int64_t N, int64_t K, q4gemv_stream_t stream);

/* ---- Q8_0 matrices (the other GGUF format the pages name: taozi.news page,
 * section "支持模型与限制"; layout from GGUF).  A row holds K/32 blocks of 34
 * bytes: an f16 scale d (little-endian), then 32 signed 8-bit codes; weight
 * j of a block is qs[j] * d. */

/* The down GEMV fed directly by the gate+up GEMV: y[N] = W u for a packed
 * Q4_0 W (N x K), with u_k = SiLU(g_k) * up_k = g_k / (1 + e^-g_k) * up_k and
 * gate_up = [g | up] the 2K-entry binary16 output of the gate+up GEMV (gate
 * half first).  The pages name the model family (Qwen 3.8 27B: taozi.news
 * page, section "支持模型与限制"; originshq.com page, section "Limitations
 * and Open Questions") but not its FFN activation; this is that family's
 * gated unit.  u is computed in fp32 inside the kernel
 * (never written) and converted per 32-column block like any M = 1 input;
 * exact integer block sums, fp32 accumulation, y rounded once.
 *   gate_up : device, 2K binary16, 16-byte aligned
 *   y       : device, N binary16
 * Q4_EUNSUPPORTED for K beyond the M = 1 kernel's staging (K <= 36,864 and
 * its shared memory); otherwise errors as q4gemv_run.  Deterministic. */
Q4GEMV_API int q4gemv_run_swiglu(q4gemv_t h, const void* W_packed, const void* gate_up,
                      void* y, int64_t N, int64_t K, q4gemv_stream_t stream);

/* Bytes of a GGUF Q8_0 matrix: N * (K/32) * 34; 0 if the shape is invalid. */
Q4GEMV_API size_t q4gemv_q8_0_gguf_bytes(int64_t N, int64_t K);

/* Bytes of the packed Q8_0 matrix: Np * (K/32) * 34, Np = ceil(N/32)*32; 0 if
 * the shape is invalid.  Packed layout: rows padded to Np (padding rows hold
 * codes 0 and d = +0), tiles of 32 rows; segment s = t*KB + b (KB = K/32)
 * holds block b of the rows of tile t in the 1088 bytes from 1088*s; row
 * n = 32t + g + 8i (g in [0,8), i in [0,4)):
 *   segment bytes 32*(4g + c) + 8i + e      = qs[4c + e]       (c, e in [0,4))
 *   segment bytes 32*(4g + c) + 8i + 4 + e  = qs[16 + 4c + e]
 *   segment bytes 1024 + 8g + 2i, +1        = d (little-endian)
 * A lane (g, c) of a warp thus finds the codes it multiplies with the
 * activations' lane group c, for its four rows, in 32 contiguous bytes. */
Q4GEMV_API size_t q4gemv_q8_0_packed_bytes(int64_t N, int64_t K);

/* One-time repack of a GGUF Q8_0 matrix (arguments and errors as
 * q4gemv_repack; gguf any alignment >= 2).  Bit-exact. */
Q4GEMV_API int q4gemv_q8_0_repack(q4gemv_t h, const void* gguf, void* packed,
                       int64_t N, int64_t K, q4gemv_stream_t stream);

/* Host-only check of q4gemv_q8_0_run's arguments: Q4_EUNSUPPORTED for M
 * outside [1, 256], else as q4gemv_validate. */
Q4GEMV_API int q4gemv_q8_0_validate(int M, int64_t N, int64_t K, const void* W_packed,
                         const void* x, const void* y);

/* y[M][N] = W x[M][K]^T for a packed Q8_0 W, 1 <= M <= 256 (buffers as
 * q4gemv_run).  M <= 2 with M*K <= 36,864 (and the kernel's shared memory):
 * the activations are converted per 32-column block as for Q4_0 (exact for
 * the block maximum), each block's dot product with the 8-bit codes is an
 * exact integer, converted to fp32 once and scaled by d.  M <= 16 otherwise:
 * the mma.sync kernel of q4gemv_run's M = 3..16 path with Q8_0 segments (each
 * signed code exact in binary16, exact per-block sums in fp32, d applied once
 * per output and block; column panels for wide K).  M = 17..256: the
 * tcgen05 GEMM of q4gemv_run's M > 16 path runs with Q8_0 segments: each
 * weight q * d (up to 18 significant bits) is split exactly into two binary16
 * parts; scales |d| >= 512 overflow the split (non-finite outputs); its
 * activation image and split sums live in the same handle buffers.  fp32
 * accumulation; y rounded to binary16 once.  Deterministic. */
Q4GEMV_API int q4gemv_q8_0_run(q4gemv_t h, const void* W_packed, const void* x, void* y,
                    int M, int64_t N, int64_t K, q4gemv_stream_t stream);

/* One layer's packed matrices for q4gemv_run_stack. */
typedef struct {
    const void* qkv;      /* qkv_n  x hidden */
    const void* o;        /* hidden x hidden */
    const void* gate_up;  /* 2*ffn  x hidden (rows [0,ffn) gate, [ffn,2ffn) up) */
    const void* down;     /* hidden x ffn */
} q4gemv_layer;

/* One synthetic decode step (M = 1) through n_layers layers of four Q4_0
 * GEMVs each, the 27B-shaped workload of the pages (hidden 5120: taozi.news
 * page, section "技术架构"; 64 layers: originshq.com page, section "The
 * Architecture: Layers Distributed, Activations in Flight").  Every GEMV
 * output is rounded to binary16; the next GEMV reads its first K entries v
 * scaled to unit RMS by the real scalar s(v) = 1/sqrt(mean(v^2)) (0 for an
 * all-zero v), i.e. it computes f16(s(v) * (W v)):
 *     a = f16(QKV x),   b = f16(s(a') O a'),  a' = a[0:hidden]
 *     u = f16(s(b) gate_up b),   x' = f16(s(u') down u'),  u' = u[0:ffn]
 * and x_out = f16(s(x') x').  The pages give no layer math beyond the GEMVs,
 * so this chain (Q slice in place of attention, gate half without an
 * activation, a unit-RMS scale in place of the norm) is the reading adopted.
 * On the GPU s is taken in fp32: block sums of squares in a fixed binary tree,
 * blocks in a fixed order, the hardware's approximate reciprocal square root.
 *   layers  : HOST array of n_layers entries (device pointers inside)
 *   x_in    : hidden binary16 (not modified); device (16-byte aligned) or
 *             host memory, pinned or pageable: a host vector is copied to
 *             the device on `stream` inside the call
 *   x_out   : hidden binary16 (may alias x_in); device or host memory (a host
 *             vector is copied back on `stream` inside the call)
 *   trace_x : device or NULL; [4*n_layers][max(hidden, ffn)] binary16: the
 *             input vector of GEMV i = 4l + t (t = 0 QKV, 1 O, 2 gate_up,
 *             3 down), before its scale, in its first K_i entries
 *   trace_y : device or NULL; [4*n_layers][max(qkv_n, hidden, 2*ffn)]
 *             binary16: the raw output of GEMV i in its first N_i entries
 * Requires qkv_n >= hidden, qkv_n % 8 == 0, 1 <= n_layers <= 4096,
 * max(hidden, ffn) within one CTA's activation staging.  The step runs as ONE
 * cooperative persistent kernel (plus a 16-byte reset of its barrier words);
 * the first call with a given set of arguments uploads its descriptors and
 * must happen outside any stream capture, later calls only launch.  With the
 * environment variable Q4GEMV_STACK_MODE=kernels (read at create) the step
 * runs instead as a CUDA graph of one kernel per GEMV, captured on the first
 * call and replayed, or launched into the caller's capture when `stream` is
 * capturing; both modes give the same bits.  Host vectors are not accepted
 * while `stream` is capturing. */
Q4GEMV_API int q4gemv_run_stack(q4gemv_t h, const q4gemv_layer* layers, int n_layers,
                     int64_t hidden, int64_t qkv_n, int64_t ffn,
                     const void* x_in, void* x_out, void* trace_x,
                     void* trace_y, q4gemv_stream_t stream);

/* The decode step of q4gemv_run_stack with the feed-forward block's
 * activation: each layer's down GEMV takes u = SiLU(gate) * up of the whole
 * gate+up output (gate = rows [0, ffn), up = rows [ffn, 2 ffn); the pages
 * name the model family but not its activation -- taozi.news page, section
 * 支持模型与限制 -- so this is the common gated form, as in
 * q4gemv_run_swiglu), computed in fp32 inside the down GEMV's staging and
 * never written, and scaled to unit RMS like every input of the chain:
 * x' = f16(s(u) (down u)), s(u) = 1/sqrt(mean(u^2)).  Everything else,
 * arguments, modes and errors as q4gemv_run_stack (no traces). */
Q4GEMV_API int q4gemv_run_stack_gated(q4gemv_t h, const q4gemv_layer* layers, int n_layers,
                                      int64_t hidden, int64_t qkv_n, int64_t ffn,
                                      const void* x_in, void* x_out, q4gemv_stream_t stream);

/* ---- Row-sharded decode step over several GPUs (one process and one handle
 * per GPU).  The pages run the model split by contiguous layer ranges across
 * devices, passing the hidden state from one to the next (originshq.com page,
 * section "The Architecture: Layers Distributed, Activations in Flight";
 * taozi.news page, section "技术架构"); that pipelines tokens but does not
 * speed up one.  Here every GEMV of the step is split by output rows over
 * `world` GPUs and its output is all-gathered before the next GEMV, so one
 * token's step divides its weight bytes over the GPUs.
 *
 * Rows of an N-row matrix held by rank `rank`: [*row0, *row0 + *rows), whole
 * 32-row tiles, every rank holding *chunk = ceil(N / (32 world)) * 32 rows
 * or fewer (the last ranks: the remainder, possibly 0).  Host-only; no
 * device access.  Q4_EINVAL for N <= 0, world < 1 or rank outside
 * [0, world). */
Q4GEMV_API int q4gemv_shard_rows(int64_t N, int world, int rank, int64_t* row0, int64_t* rows,
                      int64_t* chunk);

/* An NCCL unique id (128 bytes, written to id) for q4gemv_comm_init: rank 0
 * calls it and sends the bytes to the other ranks.  NCCL (libnccl.so.2) is
 * loaded at run time; Q4_EUNSUPPORTED if it cannot be. */
Q4GEMV_API int q4gemv_comm_unique_id(void* id);

/* Binds the handle to rank `rank` of a `world`-GPU communicator created from
 * the unique id (every rank calls it with the same id; collective, blocks
 * until all ranks have joined).  Replaces an earlier communicator of the
 * handle. */
Q4GEMV_API int q4gemv_comm_init(q4gemv_t h, int world, int rank, const void* id);

/* Peer-memory exchange for the row-sharded step: instead of an NCCL
 * all-gather after every GEMV, each GEMV kernel stores its output rows
 * directly into every rank's gather buffer (CUDA IPC mappings over NVLink /
 * NVSwitch; plain stores, no multicast) and the next GEMV reads them there.
 * Every entry of a gather buffer is one 32-bit word, the binary16 value in
 * bits 0-15 and in bits 16-31 a stamp of the GEMV that wrote it: (steps run
 * x GEMVs per step + the GEMV's index in the step) mod 2^16.  A reader polls
 * (bounded) each word it needs until it carries the stamp it expects, so no
 * fence, flag or collective separates the GEMVs, and a GEMV starts (its
 * weights streaming) while the previous one ends.  The exchange buffer of a
 * rank (zeroed once) holds, for the four matrix types of the step (QKV, O,
 * gate+up, down), a gather buffer of world * chunk words (chunk from
 * q4gemv_shard_rows, rank r's rows at r * chunk), then the rank's step
 * count; offsets from q4gemv_peer_layout.
 *
 * Blob (Q4GEMV_PEER_BLOB_BYTES, little-endian): uint32 magic 0x51345045
 * ("EP4Q"), uint32 version 1, int32 world, int32 rank, int64 hidden, qkv_n,
 * ffn, uint64 buffer bytes, then the 64-byte cudaIpcMemHandle_t of the
 * buffer, zero padding to the end. */
#define Q4GEMV_PEER_BLOB_BYTES 128
#define Q4GEMV_PEER_MAX_WORLD 8

/* Byte offsets of the exchange buffer for these shapes: off[0..3] the gather
 * buffers of QKV, O, gate+up and down outputs, off[4] the step count, off[5]
 * the total size (six entries).  Host-only.  Q4_EINVAL for world outside
 * [1, Q4GEMV_PEER_MAX_WORLD] or non-positive shapes. */
Q4GEMV_API int q4gemv_peer_layout(int world, int64_t hidden, int64_t qkv_n, int64_t ffn,
                                  int64_t* off);

/* Checks `world` blobs (world * Q4GEMV_PEER_BLOB_BYTES bytes, rank order) for
 * one exchange: magic and version, the same world, shapes and buffer size in
 * all of them, blob r from rank r.  Host-only.  Q4_OK or Q4_EINVAL. */
Q4GEMV_API int q4gemv_peer_check(const void* blobs, int world);

/* Allocates (zeroed) this rank's exchange buffer for the step's shapes and
 * writes its blob.  Every rank calls it, sends its blob to all ranks (any
 * host channel) and then calls q4gemv_peer_open with all of them.  Replaces
 * an earlier exchange of the handle (synchronises the device). */
Q4GEMV_API int q4gemv_peer_export(q4gemv_t h, int world, int rank, int64_t hidden, int64_t qkv_n,
                                  int64_t ffn, void* blob);

/* Maps the other ranks' exchange buffers (cudaIpcOpenMemHandle) from the
 * `world` blobs of q4gemv_peer_export, in rank order, after q4gemv_peer_check
 * and a comparison with this handle's export.  From then on
 * q4gemv_run_stack_sharded with the exported shapes uses the peer-memory
 * exchange.  With world = 1 nothing is mapped (the rank's own buffer). */
Q4GEMV_API int q4gemv_peer_open(q4gemv_t h, const void* blobs);

/* Unmaps the peers' buffers and frees this rank's; every rank must stop
 * using the exchange first (no step of any rank in flight). */
Q4GEMV_API int q4gemv_peer_close(q4gemv_t h);

/* The decode step of q4gemv_run_stack, row-sharded: `layers` holds THIS
 * rank's row slices (q4gemv_shard_rows of each matrix, packed as q4gemv_run
 * matrices of `rows` rows; a slice of 0 rows may be NULL).  Per GEMV the rank
 * computes its rows f16(s(v) * W_slice v) from the full previous output v
 * (the M = 1 kernel; the scale as in q4gemv_run_stack), and every rank gets
 * the whole output: through the peer-memory exchange when it is open for
 * these shapes (stores by the GEMV kernel itself, above), else an NCCL
 * all-gather; x_out = f16(s(x') x') on every rank.  x_in, x_out: device
 * memory (hidden binary16), the same x_in on every rank.  Every rank must
 * make the same calls in the same order.  The step is captured as one CUDA
 * graph on the first call with these arguments (not inside the caller's
 * capture) and replayed.  Results agree with q4gemv_run_stack within the
 * GEMV tolerance (the row split changes the order of the partial sums, not
 * the arithmetic) and are the same bits on both exchanges.  Errors as
 * q4gemv_run_stack; Q4_EINVAL with neither a communicator nor an open
 * exchange for these shapes; a peer whose rows never come makes the waiting
 * GEMV report Q4_ETIMEOUT through q4gemv_sync_status (one time-out per step:
 * later waits of the step give up at once). */
Q4GEMV_API int q4gemv_run_stack_sharded(q4gemv_t h, const q4gemv_layer* layers_local,
                             int n_layers, int64_t hidden, int64_t qkv_n, int64_t ffn,
                             const void* x_in, void* x_out, q4gemv_stream_t stream);

/* Fixed limits of q4gemv_run_noalloc. */
#define Q4GEMV_NOALLOC_MAX_N (1 << 22)                 /* rows */
#define Q4GEMV_NOALLOC_SCRATCH_BYTES (2u << 20)        /* static device scratch */

/* q4gemv_run for M <= 2 without a handle and without allocating anything.
 * The paper has no counterpart; this is a library convenience.
 *
 * Who needs it: q4gemv_create obtains its workspace with cudaMalloc, which
 * some callers cannot do -- code that runs while a stream is captured in
 * global capture mode (cudaMalloc is then an error), threads that must not
 * take the implicit device synchronisation of cudaMalloc/cudaFree, and
 * plug-ins whose host application owns all device memory.  This entry point
 * runs the same kernel as q4gemv_run with its scratch (split-tile partial
 * sums, per-tile arrival counters, an error word) in one file-scope device
 * array of Q4GEMV_NOALLOC_SCRATCH_BYTES (2 MiB) that every GPU which loads
 * the library holds until the process exits.  It calls no cudaMalloc,
 * cudaFree or allocating library routine.
 *
 * Arguments as q4gemv_run (device pointers, 16-byte aligned, packed W), on
 * the current CUDA device, asynchronous on `stream`.  Limits: 1 <= M <= 2
 * (else Q4_EUNSUPPORTED); K % 32 == 0, N <= Q4GEMV_NOALLOC_MAX_N, and K <=
 * 24,896 for M = 1 or K <= 18,432 for M = 2 (the kernel's shared memory and
 * activation staging; else Q4_ESHAPE); at most 2560 warps are used.
 * Device-side error reports are not surfaced.
 *
 * The first call on a device sets that device up (resolves the array's
 * device address with cudaGetSymbolAddress, queries the SM count, sets the
 * kernels' shared-memory limit); make that first call before any stream
 * capture.  Every call shares the one array and clears its counters before
 * launching: calls that overlap on the GPU race and give wrong results, so
 * order them on one stream. */
Q4GEMV_API int q4gemv_run_noalloc(const void* W_packed, const void* x, void* y, int M,
                                  int64_t N, int64_t K, q4gemv_stream_t stream);

/* Synchronises `stream`, then reads and clears the handle's device error
 * word: Q4_OK, Q4_ETIMEOUT, Q4_ECONCURRENT, or Q4_ECUDA if an earlier
 * asynchronous error is pending on the device. */
Q4GEMV_API int q4gemv_sync_status(q4gemv_t h, q4gemv_stream_t stream);

/* Static text for a status code. */
Q4GEMV_API const char* q4gemv_strerror(int status);

/* Text of the handle's last error (empty if none).  Valid until the next
 * call on the handle. */
Q4GEMV_API const char* q4gemv_last_error(q4gemv_t h);

/* Fault injection for tests.  which: "none"; "alloc" (workspace or buffer
 * allocation), "launch" (kernel launch) or "graph" (graph capture or
 * instantiation) make that host step of later calls fail with
 * Q4_EFAULTINJ; "timeout" makes later persistent decode steps
 * (q4gemv_run_stack) give every bounded device wait a budget of 1,024 polls
 * and ask their first inter-GEMV wait for a condition that never holds, so
 * the wait gives up, the kernel records Q4_ETIMEOUT in the handle's error
 * word, every CTA returns (after its copies in flight have landed) and the
 * next q4gemv_sync_status reports Q4_ETIMEOUT; the handle stays usable.  No
 * GPU fault, trap or unbounded wait is involved.  The environment variable
 * Q4GEMV_FAULT sets the initial value at q4gemv_create. */
Q4GEMV_API int q4gemv_set_fault(q4gemv_t h, const char* which);

#ifdef __cplusplus
}
#endif

#endif /* Q4GEMV_H */
