/*
 * fg8.h -- C ABI of libfg8.so: fine-grained-scaled FP8 GEMM for NVIDIA B200
 * (sm_100a).
 *
 * The operation (fine-grained scaling "as proposed in DeepSeek-V3":
 * chujupifa.com "机器之心报道", opening summary; deepseek.csdn.net
 * "DeepGEMM：简洁、高效，用约300行CUDA代码重构AI计算的底层法则", section
 * "什么是DeepGEMM呢？"):
 *
 *   D[m,n] = bf16( sum_kb ( sum_{k in kb} A[m,k] * B[n,k] ) * sfa[m,kb] * sfb[n/128,kb] )
 *
 * with kb running over 128-wide blocks of K, A and B stored as E4M3 codes
 * (4 exponent bits, 3 mantissa bits: ai.abqq.net "DeepSeek开源周第三天…
 * DeepGEMM：FP8", section 3 "核心功能与特性"; OCP E4M3 "FN": max 448, no
 * infinities), one FP32 scale per 1x128 block of A (sfa) and per 128x128
 * block of B (sfb), and the result rounded to BF16 (round to nearest even).
 * "NT": both operands are K-major (row-major A [M,K] and B [N,K]).
 *
 * Three GEMM kinds are provided, the ones the pages list (ai.abqq.net section
 * 3; game.3loumao.org explainer, section "03 DeepSeek是如何创新的？"): normal,
 * contiguous-grouped MoE and masked-grouped MoE.  The helper functions mirror
 * the utilities of the csdn page, section "实用工具".
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never frees or retains them beyond the call (a small cache of TMA
 *    descriptors is keyed by pointer and shape).
 *  - Calls are asynchronous on `stream` (0 = legacy default stream) and never
 *    synchronise.  Errors detectable on the host are returned before anything
 *    is launched, and then D is untouched.
 *  - Errors detected on the device (a pipeline wait that timed out) are
 *    recorded in a per-device status word read by fg_get_last_device_status.
 *  - E4M3 operands: 1 byte per element.  Scales: IEEE fp32.  D: bf16.
 *  - Pointer alignment: A, B, D, sfa 16 bytes; sfb 4 bytes.
 *  - K must be a positive multiple of 128; N a positive multiple of 16.
 */
#ifndef FG8_H
#define FG8_H

#include <stddef.h>
#include <stdint.h>

/* The library is built with hidden symbol visibility; only the entry points
 * declared here (marked FG8_API) are exported. */
#if defined(__GNUC__)
#define FG8_API __attribute__((visibility("default")))
#else
#define FG8_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* fg_stream_t; /* same type as cudaStream_t */

typedef enum {
    FG_OK = 0,
    FG_ERR_INVALID_ARG = 1, /* null pointer, negative or inconsistent size */
    FG_ERR_ALIGNMENT = 2,   /* a pointer breaks the 16-byte rule above */
    FG_ERR_UNSUPPORTED = 3, /* K % 128 != 0, N % 16 != 0, size beyond limits */
    FG_ERR_NO_DEVICE = 4,   /* no CUDA device, or not an sm_100 device */
    FG_ERR_CUDA = 5,        /* a CUDA runtime / driver call failed */
    FG_ERR_TIMEOUT = 6      /* device side: a pipeline wait ran past its limit */
} fg_status;

/* Human-readable name of a status code (static string). */
FG8_API const char* fg_status_string(int status);

/* Library version, e.g. "fg8 0.1.0 sm_100a". */
FG8_API const char* fg_version(void);

/*
 * Normal GEMM, D = A . B^T with fine-grained scales.
 *   A   [M, K]   E4M3, row-major (row stride K bytes)
 *   sfa [K/128][M_pad] fp32: MN-major ("column-major, TMA-aligned") scales of
 *       A, M_pad = fg_get_tma_aligned_size(M, 4); sfa[kb*M_pad + m] scales
 *       A[m, 128*kb .. 128*kb+127].  Build it with fg_transform_sfa_to_tma_layout.
 *   B   [N, K]   E4M3, row-major
 *   sfb [ceil(N/128)][K/128] fp32 row-major: sfb[nb*(K/128) + kb] scales
 *       B[128*nb .. 128*nb+127, 128*kb .. 128*kb+127]
 *   D   [M, N]   bf16, row-major (row stride N elements), fully overwritten
 * M == 0 is a no-op.  Returns FG_OK or an error code.
 */
FG8_API fg_status fg_fp8_gemm_nt(const void* A, const float* sfa, const void* B, const float* sfb, void* D, int M,
                         int N, int K, fg_stream_t stream);

/*
 * Contiguous-grouped MoE GEMM (game.3loumao.org explainer section 03: the
 * rows of all experts "joined into one block").  Each expert's rows form one
 * segment of A; every segment is padded up to a multiple of
 * fg_get_m_alignment_for_contiguous_layout() rows and the segments are
 * concatenated along M.
 *   A         [M_tot, K] E4M3;   sfa [K/128][M_pad(M_tot)] MN-major
 *   B         [G, N, K]  E4M3;   sfb [G][ceil(N/128)][K/128]
 *   m_indices [M_tot] int32 (device): the expert of each row, or -1 on padding
 *   D         [M_tot, N] bf16
 * Row m of D is written iff 0 <= m_indices[m] < G, with
 *   D[m,:] = GEMM(A[m,:], B[m_indices[m]], sfb[m_indices[m]]).
 * Rows tagged -1 are never written.  Preconditions checked on the host:
 * M_tot % alignment == 0.  Preconditions NOT checked (device data): all rows
 * of one aligned block carry the same expert or -1, and a block's first row
 * is not -1 unless the whole block is padding; rows that break this are left
 * unwritten.
 */
FG8_API fg_status fg_m_grouped_fp8_gemm_nt_contiguous(const void* A, const float* sfa, const void* B,
                                              const float* sfb, void* D, const int* m_indices, int M_tot,
                                              int N, int K, int G, fg_stream_t stream);

/*
 * Masked-grouped MoE GEMM (game.3loumao.org explainer section 03: a mask
 * marks which rows to compute; empty rows are skipped).
 *   A        [G, M_max, K] E4M3;  sfa [G][K/128][M_pad(M_max)] MN-major
 *   B        [G, N, K]     E4M3;  sfb [G][ceil(N/128)][K/128]
 *   masked_m [G] int32 (device): rows r < min(masked_m[g], M_max) of group g
 *            are computed; the other rows of D[g] are never written, and a
 *            group with masked_m[g] <= 0 costs nothing (its B is not read).
 *   D        [G, M_max, N] bf16
 *   expected_m: host-side hint of the typical masked_m used to pick the tile
 *            shape (0 = M_max).  It never changes the result.
 */
FG8_API fg_status fg_m_grouped_fp8_gemm_nt_masked(const void* A, const float* sfa, const void* B, const float* sfb,
                                          void* D, const int* masked_m, int G, int M_max, int N, int K,
                                          int expected_m, fg_stream_t stream);

/* Maximum number of SMs the GEMM kernels use (csdn page, "实用工具":
 * set_num_sms / get_num_sms).  Process-global.  Default: the device's SM
 * count (or the FG_NUM_SMS environment variable).  fg_set_num_sms accepts
 * 1 .. device SM count and returns FG_ERR_INVALID_ARG otherwise. */
FG8_API int fg_get_num_sms(void);
FG8_API fg_status fg_set_num_sms(int n);

/* Row alignment of each expert segment in the contiguous layout (csdn page,
 * "实用工具": get_m_alignment_for_contiguous_layout).  Returns 128, the row
 * block of the kernels. */
FG8_API int fg_get_m_alignment_for_contiguous_layout(void);

/* Smallest n' >= n with n' * elem_bytes a multiple of 16 bytes, the TMA
 * stride rule (csdn page, "实用工具": get_tma_aligned_size).  elem_bytes must
 * divide 16; returns 0 otherwise. */
FG8_API size_t fg_get_tma_aligned_size(size_t n, size_t elem_bytes);

/* Scale layout transform (csdn page, "实用工具": get_col_major_tma_aligned_tensor).
 *   in  [G][M][KB] fp32 row-major (device)
 *   out [G][KB][M_pad] fp32 (device), M_pad = fg_get_tma_aligned_size(M, 4):
 *       out[g][kb][m] = in[g][m][kb] for m < M, 0 for M <= m < M_pad.
 * Both pointers 16-byte aligned (in: 4).  Runs one small kernel on stream. */
FG8_API fg_status fg_transform_sfa_to_tma_layout(const float* in, float* out, int G, int M, int KB, fg_stream_t stream);

/* Activation quantiser, the step that prepares A for the GEMMs (fine-grained
 * scaling, chujupifa.com "机器之心报道", opening summary; the scale layout of
 * get_col_major_tma_aligned_tensor, csdn page "实用工具").  For every 1 x 128
 * block of a row of x:
 *   scale = max(amax, 1e-4) / 448        in FP32 (448 = largest finite E4M3)
 *   q     = E4M3(x / scale)              FP32 division, round to nearest even,
 *                                        saturating at +-448
 *   x   [M, K] FP32 (x_is_bf16 = 0) or BF16 (x_is_bf16 = 1), row-major
 *   q   [M, K] E4M3 codes, row-major (written)
 *   sfa [K/128][M_pad] FP32, MN-major, M_pad = fg_get_tma_aligned_size(M, 4)
 *       (written, rows M .. M_pad-1 set to 0): the scale layout the GEMMs read.
 * K must be a positive multiple of 128; x, q and sfa 16-byte aligned.  M == 0
 * is a no-op.  Runs one kernel on stream. */
FG8_API fg_status fg_quantize_fp8_activations(const void* x, int x_is_bf16, void* q, float* sfa, int M, int K,
                                      fg_stream_t stream);

/* Reads and clears this device's status word after synchronising `stream`.
 * *code_out = 0 when no kernel recorded an error since the last call, else
 * FG_ERR_TIMEOUT; *detail_out (may be NULL) = (block << 8) | role of the
 * first failure (role 1 = TMA producer, 2 = MMA issuer, 3 = epilogue). */
FG8_API fg_status fg_get_last_device_status(fg_stream_t stream, int* code_out, int* detail_out);

/* Upper bound, in nanoseconds, on any single pipeline wait inside the GEMM
 * kernels (default 1e9 = 1 s; FG_WAIT_LIMIT_NS overrides at load).  A wait
 * that runs past it makes the kernel record FG_ERR_TIMEOUT, drain its copies
 * in flight, release tensor memory and return: it never hangs the GPU.
 * Values below 1000 are rejected. */
FG8_API fg_status fg_set_wait_limit_ns(unsigned long long ns);
FG8_API unsigned long long fg_get_wait_limit_ns(void);

/* The block width (BLOCK_N) the normal GEMM would use for (M, N, K) with the
 * current SM budget, negated when the tile runs on a pair of CTAs (256-row
 * tiles), or 0 for an unsupported shape.  Diagnostics. */
FG8_API int fg_query_block_n(int M, int N, int K);

/* The launch plan a GEMM call of these sizes would use with the current SM
 * budget and environment (diagnostics; launches nothing, allocates nothing).
 *   layout 0 = normal (rows = M, G = 1), 1 = contiguous (rows = M_tot, G
 *   experts), 2 = masked (rows = M_max, G groups, expected_m as in the call).
 * Outputs (all required):
 *   *kernel_out  0 = the tile kernel, 1 = the few-rows (decode) kernel
 *   *tile_n_out  BLOCK_N of the tile kernel, or the token-tile width of the
 *                decode kernel
 *   *pair_out    1 when tiles run on CTA pairs (256-row tiles)
 *   *splits_out  K splits per output tile (decode kernel, or the tile kernel's
 *                cluster split-K for few rows; 1 otherwise)
 *   *cluster_out CTAs per cluster (split-K reduction through distributed
 *                shared memory when equal to *splits_out > 1)
 * Returns FG_ERR_INVALID_ARG for a bad layout, non-positive sizes or a NULL
 * output, FG_ERR_UNSUPPORTED when K % 128 != 0 or N % 16 != 0. */
FG8_API fg_status fg_query_plan(int layout, int rows, int N, int K, int G, int expected_m, int* kernel_out,
                        int* tile_n_out, int* pair_out, int* splits_out, int* cluster_out);

/*
 * Runtime specialisation (the pages' library compiles its kernels at run time
 * per shape and caches them on disk: chujupifa.com "机器之心报道", opening
 * summary; deepseek.csdn.net "DeepGEMM：简洁、高效…", section "环境变量").
 * With FG_JIT=1 in the environment, the normal GEMM's tile kernel is compiled
 * with NVRTC for its block width, CTA pairing and K block count (a
 * compile-time constant of the kernel), once per process, and the cubin is
 * cached under FG_CACHE_DIR (default $HOME/.cache/fg8) for later processes.
 * If NVRTC (libnvrtc.so.12), the kernel sources (next to the library, in
 * csrc/) or a driver entry point is missing, the ahead-of-time kernel runs
 * instead.
 *
 * fg_jit_compile: compiles (or finds in the cache) the specialisation for
 *   block_n (16..256, multiple of 16), pair (0/1; block_n >= 32 when 1) and
 *   k_blocks (> 0) without a GPU, and writes the cubin's path into path_out
 *   (path_len bytes, NUL-terminated; may be NULL).  Returns FG_OK,
 *   FG_ERR_INVALID_ARG, FG_ERR_UNSUPPORTED (no NVRTC or sources) or
 *   FG_ERR_CUDA (compilation failed; FG_JIT_VERBOSE=1 prints the log).
 * fg_jit_stats: specialisations compiled / read from the disk cache by this
 *   process so far, and GEMM launches that ran a runtime-compiled kernel (any
 *   pointer may be NULL).
 */
FG8_API fg_status fg_jit_compile(int block_n, int pair, int k_blocks, char* path_out, size_t path_len);
FG8_API void fg_jit_stats(int* compiled, int* loaded_from_disk, int* launches);

/*
 * Few-rows normal GEMM that allocates nothing.  The pages have no counterpart
 * to this entry point: it is an addition of this library.
 *
 * Why: fg_fp8_gemm_nt, when it splits K over several CTAs for a small M, may
 * call cudaMalloc the first time it needs its split-K workspace on a device
 * and stream (or a larger one).  Some callers cannot let that happen: a
 * serving engine that reserved nearly all device memory for its own pool
 * up front (the allocation would fail), or a latency-critical loop in which
 * cudaMalloc / cudaFree, which may synchronise the device, are not allowed.
 * This entry point computes the same result as fg_fp8_gemm_nt, with the same
 * operands, layouts and alignment rules, but keeps its split-K partial sums
 * and arrival counters in a scratch array that the library defines as a
 * device variable: every GPU that loads the library holds one copy of it
 * (FG_NO_ALLOC_SCRATCH_BYTES) from module load until the process exits.  It
 * never calls cudaMalloc, cudaFree or any allocating routine; the caller
 * passes every input and output.  (Under CUDA's default lazy module loading
 * the driver places a kernel's code in device memory at its first launch; a
 * caller that must avoid even that at run time makes one call per shape
 * class first, or sets CUDA_MODULE_LOADING=EAGER.)
 *
 * Limits: 1 <= M <= FG_NO_ALLOC_MAX_M and N <= FG_NO_ALLOC_MAX_N; larger sizes
 * return FG_ERR_UNSUPPORTED and launch nothing.  The K split count is lowered
 * until the partial sums fit in FG_NO_ALLOC_PARTIAL_FLOATS floats (one split
 * needs no scratch).  M == 0 is a no-op.
 *
 * First call on a device: it looks up the scratch array's device address
 * (cudaGetSymbolAddress) with that device current, once per device; make
 * that first call before any stream capture.
 *
 * Sharing: every call on a device uses the same scratch and leaves its
 * contents behind (each call clears the counters it needs on `stream` before
 * its kernel runs).  Calls whose executions overlap on the GPU (other streams,
 * other host threads) race on the scratch and may return wrong results:
 * order them, e.g. on one stream.
 */
#define FG_NO_ALLOC_MAX_M 256
#define FG_NO_ALLOC_MAX_N 262144
#define FG_NO_ALLOC_PARTIAL_FLOATS (2u * 1024u * 1024u)
#define FG_NO_ALLOC_SCRATCH_BYTES ((FG_NO_ALLOC_MAX_N / 128) * 4u + FG_NO_ALLOC_PARTIAL_FLOATS * 4u)
FG8_API fg_status fg_fp8_gemm_nt_small_m_no_alloc(const void* A, const float* sfa, const void* B, const float* sfb, void* D,
                                          int M, int N, int K, fg_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FG8_H */
