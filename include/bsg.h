/*
 * bsg.h -- block-scaled grouped GEMM for NVIDIA B200 (sm_100a): the C ABI of libbsg.so.
 *
 * Two operations, both "C = A x B[g]^T with per-row expert routing", computed by hand-written
 * tcgen05 / TMA / TMEM kernels.  Everything is asynchronous on the caller's CUDA stream; nothing is
 * allocated, synchronised or retained by a call.  All pointers are CUDA device pointers owned by the
 * caller unless stated otherwise.  All tensors are dense, row-major, with no padding between rows.
 * Stream order is kept: a GEMM launch whose grid is smaller than the GPU is a programmatic dependent
 * of the previous kernel on the stream (it may start its set-up early) and waits on the device for
 * that kernel to complete before it reads or writes any operand.
 *
 * Error convention (after the argument checks of the FP8 page's host binding, "[flashinfer]
 * FlashInfer FP8 GEMM 최적화: 윈도우 세그먼트 KG1 프로그램으로 GPU 성능 극대화", section 1): every entry
 * point validates its arguments on the host before launching anything.  On a violation it returns a
 * negative bsg_status, launches nothing, and records a one-line description retrievable with
 * bsg_last_error() (per calling thread).  There is no fallback program and no CPU path.
 */
#ifndef BSG_H_
#define BSG_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* bsg_stream_t; /* a cudaStream_t; NULL is the legacy default stream */

typedef enum {
  BSG_OK = 0,
  BSG_ERR_INVALID_ARG = -1,       /* null pointer, non-positive size, bad routing pointer */
  BSG_ERR_ALIGNMENT = -2,         /* a base pointer or row pitch breaks the 16-byte rule */
  BSG_ERR_UNSUPPORTED_SHAPE = -3, /* outside the launch contract (M, N, K, G limits) */
  BSG_ERR_CUDA = -4,              /* a CUDA runtime / driver call failed (message has the code) */
  BSG_ERR_DEVICE_TIMEOUT = -5     /* a kernel gave up a bounded wait (see bsg_get_device_status) */
} bsg_status;

/*
 * FP8 grouped GEMM -- the operation of the FP8 page named above (introduction and section 1):
 * E4M3 inputs, FP32 scales per 128-element K block, BF16 output, rows grouped by m_indices, with
 * expert runs free to start inside a 128-row window (section 2).
 *
 *   for every row m with g = m_indices[m] in [0, G):
 *     C[m, n] = bf16( sum_kb a_scale[m, kb] * b_scale[g, n / 128, kb]
 *                            * sum_{k in block kb} A[m, k] * B[g, n, k] )        (kb = k / 128)
 *
 * A        uint8  [M, K]               E4M3 (FN) codes, row-major.
 * B        uint8  [G, N, K]            E4M3 codes, one K-major [N, K] matrix per expert.
 * a_scale  float  [M, K/128]           per row and K block.
 * b_scale  float  [G, ceil(N/128), K/128]  per expert, 128-row block of B[g] and K block.
 * m_indices int32 [M]                  expert of each row; a value < 0 or >= G means "skip the row:
 *                                      its C row is left untouched".  May be NULL only when G == 1
 *                                      (every row goes to expert 0).  Read on the device on every
 *                                      call, so a captured CUDA graph may be replayed after the
 *                                      indices (or any operand) change in place.
 * C        bf16   [M, N]               output; only routed rows are written.
 * Contract: 1 <= M <= 2^24, 64 <= N <= 2^19, N % 8 == 0, K % 128 == 0, 128 <= K <= 2^20,
 *           1 <= G <= 4096 (limits from the window program's launch contract, section 2 of the
 *           page, plus the 16-byte row rules of TMA); A, B, C 16-byte aligned; a_scale, b_scale,
 *           m_indices 4-byte aligned.
 * Rows are routed in runs: maximal stretches of consecutive rows with the same expert.  Any order
 * is correct; sorted (contiguous) runs are the fast case.
 */
bsg_status bsg_fp8_grouped_gemm(const void* A, const void* B, const float* a_scale, const float* b_scale,
                                const int32_t* m_indices, void* C, int64_t M, int64_t N, int64_t K,
                                int64_t G, bsg_stream_t stream);

/*
 * NVFP4 (grouped) GEMM -- the native FP4 x FP4 grouped GEMM of the page "[onnxruntime] ONNX Runtime:
 * Blackwell (SM120+)에서 NVFP4 QMoE를 위한 네이티브 FP4xFP4 Prefill 최적화", section 1: E2M1 codes
 * with one E4M3 scale per 16 K elements and an FP32 per-tensor factor.
 *
 *   for every row m with g = m_indices[m] in [0, G):
 *     C[m, n] = bf16( alpha[g] * sum_j sfa[m, j] * sfb[g, n, j]
 *                                    * sum_{k in block j} A[m, k] * B[g, n, k] )    (j = k / 16)
 *
 * A     uint8 [M, K/2]     E2M1 codes, two per byte, the lower-K element in the low nibble.
 * B     uint8 [G, N, K/2]  same packing, one K-major matrix per expert.
 * sfa   uint8 [M, K/16]    E4M3 scale codes (non-negative), row-major.
 * sfb   uint8 [G, N, K/16] E4M3 scale codes (non-negative), row-major.
 * alpha float [G]          device array: per-expert product of the two per-tensor scales.
 * m_indices, C             as for bsg_fp8_grouped_gemm.
 * Contract: 1 <= M <= 2^24, 64 <= N <= 2^19, N % 8 == 0, K % 256 == 0, 256 <= K <= 2^20,
 *           1 <= G <= 4096; A, B, sfa, sfb, C 16-byte aligned; alpha, m_indices 4-byte aligned.
 */
bsg_status bsg_nvfp4_gemm(const void* A, const void* B, const void* sfa, const void* sfb, const float* alpha,
                          const int32_t* m_indices, void* C, int64_t M, int64_t N, int64_t K, int64_t G,
                          bsg_stream_t stream);

/*
 * Activation quantisation into the A operand of the GEMMs above (the step just before the GEMM), with
 * an optional row gather -- the MoE "expand" that makes each expert's tokens contiguous, after the
 * expand-and-quantise of the input rows in the ONNX Runtime page cited above, section 1.
 *
 *   for every output row m with r = (src_rows ? src_rows[m] : m) in [0, M_in):
 *     FP8,   per 128-element block b:  a_scale[m,b] = amax / 448
 *                                      A[m,k] = e4m3(X[r,k] / a_scale[m,b])
 *     NVFP4, per 16-element block j:   sfa[m,j]   = ue4m3((amax / 6) / gs)
 *                                      A[m,k]     = e2m1(X[r,k] / (sfa[m,j] * gs))
 *   amax is the largest |X[r,k]| of the block; every step is an IEEE fp32 operation and each
 *   quotient the correctly rounded fp32 division (the codes are those of one division per element);
 *   e4m3 / e2m1 / ue4m3 round to the nearest value, ties to the even code, and saturate at 448 / 6 /
 *   448 (the saturating conversion of the page "[sglang] ROCm 아키텍처별 최적화: 런타임 디스패치로 성능
 *   극대화", section 1); a zero block gets scale 0 and zero codes.  Output rows whose source is
 *   outside [0, M_in) are not written.
 *
 * X         bf16  [M_in, K]  activations (finite values), row-major, 16-byte aligned.
 * src_rows  int32 [M]        source row of each output row, or NULL (then M <= M_in, row m <- row m).
 * A         FP8: uint8 [M, K] (16-byte aligned); NVFP4: uint8 [M, K/2], two codes per byte, the lower-K
 *           element in the low nibble (16-byte aligned) -- exactly the GEMMs' A layouts.
 * a_scale   float [M, K/128] (4-byte aligned).   sfa  uint8 [M, K/16].
 * global_scale  device float [1]: gs > 0 (for example amax(X) / (448 * 6)); read on the device.
 * Contract: 1 <= M, M_in <= 2^31 - 1; FP8: K % 128 == 0; NVFP4: K % 16 == 0; 16 <= K <= 2^20.
 * Asynchronous on `stream`; nothing is allocated or retained.
 */
bsg_status bsg_quantize_fp8_rows(const void* X, const int32_t* src_rows, void* A, float* a_scale, int64_t M_in,
                                 int64_t M, int64_t K, bsg_stream_t stream);
bsg_status bsg_quantize_nvfp4_rows(const void* X, const int32_t* src_rows, const float* global_scale, void* A,
                                   void* sfa, int64_t M_in, int64_t M, int64_t K, bsg_stream_t stream);

/*
 * MoE expand permutation -- the step before the quantiser: lay the routing entries out expert by
 * expert so that each expert's rows form one contiguous run of the grouped GEMM's A (the expanded
 * input rows of the ONNX Runtime page cited above, section 1).  A stable counting sort of the
 * n = T * top_k entries i = t * top_k + k (token-major) by their expert g = expert_ids[i]:
 *
 *   expert_offsets[g] = number of entries with an expert below g;  expert_offsets[G] = entries placed
 *   entry i with g in [0, G) takes the next position p of g's run, in increasing i:
 *       src_rows[p] = t,  m_indices[p] = g,  dst_rows[i] = p
 *   entry i with g outside [0, G) is dropped: dst_rows[i] = -1
 *   positions p in [expert_offsets[G], n): src_rows[p] = m_indices[p] = -1
 *
 * so bsg_quantize_*_rows(X, src_rows, ..., M_in = T, M = n) gathers the expanded activations (it
 * leaves the -1 rows untouched), the grouped GEMM takes m_indices as is (it skips the -1 rows), and
 * a later combine finds the output row of token t's choice k at dst_rows[t, k].
 *
 * expert_ids      int32 [T, top_k]  routing choices (any value; those outside [0, G) are dropped).
 * src_rows        int32 [n]         output: source token of each expanded row.
 * m_indices       int32 [n]         output: expert of each expanded row, non-decreasing, then -1.
 * dst_rows        int32 [T, top_k]  output: expanded row of each entry, or -1.
 * expert_offsets  int32 [G + 1]     output: start of each expert's run; [G] = rows placed.
 * workspace       device scratch of at least bsg_moe_permute_workspace_size() bytes, 16-byte
 *                 aligned, owned by the caller; its contents need not be initialised and are
 *                 overwritten.  Calls that share a workspace must not overlap on the GPU.  When
 *                 that size is 0 the workspace is not used and may be null.
 * Contract: T >= 1, 1 <= top_k <= 256, T * top_k <= 2^24, 1 <= G <= 4096; the int32 arrays 4-byte
 *           aligned.  Asynchronous on `stream`; nothing is allocated.  One kernel launch (one CTA,
 *           no scratch) when T * top_k <= 4096 and G <= 1024, three launches otherwise.
 * bsg_moe_permute_workspace_size() writes the scratch size for (T, top_k, G) to *bytes (0 for the
 * one-launch sizes, else 4 * G * min(512, ceil(T * top_k / 256)) up to rounding of the tiles, at most
 * 8 MiB) or returns an error for sizes outside the contract; it touches no GPU.
 */
bsg_status bsg_moe_permute_workspace_size(int64_t T, int64_t top_k, int64_t G, size_t* bytes);
bsg_status bsg_moe_permute(const int32_t* expert_ids, int64_t T, int64_t top_k, int64_t G, int32_t* src_rows,
                           int32_t* m_indices, int32_t* dst_rows, int32_t* expert_offsets, void* workspace,
                           size_t workspace_bytes, bsg_stream_t stream);

/*
 * bsg_moe_permute without a workspace argument, for callers that cannot allocate device memory:
 * a plugin whose host application owns every device allocation and hands it no allocator, a
 * serving loop that must not call cudaMalloc / cudaFree (they can synchronise the whole device and
 * stall the other streams), or a process that has to keep its device footprint fixed after start-up.
 * (This entry point has no counterpart in the pages the library follows; it is the same permutation
 * as bsg_moe_permute, with identical results.)
 *
 * The scratch is a fixed 2 MiB array that the library's device image carries on every GPU that loads
 * it, for as long as the process lives.  Limit: the sizes (T, top_k, G) whose
 * bsg_moe_permute_workspace_size() is at most 2 MiB -- every size with G <= 1024, and with more experts
 * T * top_k up to 65536 entries for G = 2048 or 32768 for G = 4096; larger sizes return
 * BSG_ERR_UNSUPPORTED_SHAPE with a message and launch nothing.  The first call on a device also looks
 * up that device's copy of the
 * array (with the device current), so make that first call before capturing any stream.
 * Every call on a device shares the one array and leaves its last contents behind; the kernels
 * overwrite every counter before they read it, so nothing needs clearing between calls, but calls
 * that overlap on the GPU (different streams, no ordering between them) race on the array and give
 * undefined results.  Nothing is allocated or freed, by this call or by anything it calls.
 * Arguments, outputs, contract and asynchrony otherwise as for bsg_moe_permute.
 */
bsg_status bsg_moe_permute_noalloc(const int32_t* expert_ids, int64_t T, int64_t top_k, int64_t G,
                                   int32_t* src_rows, int32_t* m_indices, int32_t* dst_rows,
                                   int32_t* expert_offsets, bsg_stream_t stream);

/* Description of the last failure on the calling thread ("" if none).  The string stays valid until
 * the next bsg_* call on the same thread. */
const char* bsg_last_error(void);

/*
 * Device-side status: every bounded wait in the kernels (pipeline barriers, TMA arrivals) gives up
 * after a time limit instead of hanging, records where it stopped in a device status word and makes
 * the kernel return.  This call synchronises `stream`, reads and clears the word of the current
 * device, and returns BSG_OK or BSG_ERR_DEVICE_TIMEOUT (details in bsg_last_error()).
 */
bsg_status bsg_get_device_status(bsg_stream_t stream);

/*
 * Wait limit of the kernels' bounded waits, in nanoseconds (default 2e9 = 2 s; applies to launches
 * made after the call, from any thread).  Returns the previous value.  0 restores the default.
 */
uint64_t bsg_set_wait_timeout_ns(uint64_t ns);

/*
 * Tile / grid chooser (the tactic ranking of the page "[flashinfer] FlashInfer의 FP4 GEMM 최적화:
 * 휴리스틱 개선과 Autotuning 효율화", section 2).  Tactic ids are small integers per kind (0 = FP8,
 * 1 = NVFP4); bsg_tactic_name() describes one.  bsg_tactic_score() is the page's score of a tactic
 * for a problem size (M rows, N, K, G experts, sm_count SMs), with the work-unit counts estimated
 * from the sizes alone; bsg_choose_tactic() returns the best-scored (or forced) tactic, or a
 * negative bsg_status.  bsg_set_tactic() forces a tactic for later calls of that kind (-1 = let the
 * chooser decide); the environment variable BSG_TACTIC does the same at load time.
 * FP8 tactics: 0 = one SM per 128-row window segment x 256 columns; 1 = an SM pair per 256 x 256
 * tile; 2, 3 = operand-swapped tiles for experts with few rows (128 or 256 output columns x a chunk
 * of at most 128 or 64 of one expert's rows; the page "[onnxruntime] ONNX Runtime: Blackwell
 * (SM120+)에서 NVFP4 QMoE를 위한 네이티브 FP4xFP4 Prefill 최적화", section 1, keeps decode shapes on a
 * path of their own); 4 = one SM per 128-row window segment x 64 columns (small problems, the
 * small-launch shapes of the FP8 page's section 2 table).  NVFP4 tactics: 0 = one SM, 1 = an SM pair.  Every tactic computes the same
 * result within the stated tolerance.
 */
int bsg_num_tactics(int kind);
const char* bsg_tactic_name(int kind, int tactic);
int bsg_choose_tactic(int kind, int64_t M, int64_t N, int64_t K, int64_t G, int sm_count);
double bsg_tactic_score(int kind, int tactic, int64_t M, int64_t N, int64_t K, int64_t G, int sm_count);
bsg_status bsg_set_tactic(int kind, int tactic);

/*
 * Runtime tactic selection by measurement (the autotuning of the score-ranked candidates on the page
 * "[flashinfer] FlashInfer의 FP4 GEMM 최적화: 휴리스틱 개선과 Autotuning 효율화", section 1; with at most
 * four tactics per kind the top-N of the ranking is all of them): runs every tactic of the kind on the
 * caller's operands -- one warm-up launch, then `reps` timed launches each,
 * CUDA events on `stream` -- records the fastest for these exact sizes (M, N, K, G) in a per-process
 * table that bsg_choose_tactic consults after a forced tactic and before the score, and returns its
 * id (or a negative bsg_status).  The arguments are those of the GEMM call; C receives the correct
 * result.  Synchronises `stream`; 1 <= reps <= 10000.  bsg_autotune_clear() empties the table.
 */
int bsg_autotune_fp8(const void* A, const void* B, const float* a_scale, const float* b_scale,
                     const int32_t* m_indices, void* C, int64_t M, int64_t N, int64_t K, int64_t G, int reps,
                     bsg_stream_t stream);
int bsg_autotune_nvfp4(const void* A, const void* B, const void* sfa, const void* sfb, const float* alpha,
                       const int32_t* m_indices, void* C, int64_t M, int64_t N, int64_t K, int64_t G, int reps,
                       bsg_stream_t stream);
void bsg_autotune_clear(void);

/*
 * Upper bound on the persistent grid of later calls of one kind (0 = FP8, 1 = NVFP4); 0 restores the
 * default (one CTA per SM, fewer when there are fewer work units).  Any value >= 1 gives the same
 * results, only slower: each CTA then walks more work units through the same pipelines.
 */
bsg_status bsg_set_max_ctas(int kind, int max_ctas);

/*
 * Test-only fault injection, for checking the bounded waits without faulting a GPU.  mode 0: off.
 * mode 1: in later launches the scheduler warp hands out no work, so the other warps' bounded waits
 * on the work queue expire after the wait limit; those launches issue no memory operation, release
 * their tensor memory and return, and bsg_get_device_status() then reports BSG_ERR_DEVICE_TIMEOUT.
 */
bsg_status bsg_debug_set_fault(int mode);

/* Library version string. */
const char* bsg_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BSG_H_ */
