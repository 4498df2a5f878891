/*
 * int8row -- LLM.int8() mixed-precision linear layer for NVIDIA B200 (sm_100a).
 *
 * C ABI.  Every pointer argument is a DEVICE pointer unless stated otherwise;
 * the caller owns every buffer, and no entry point allocates device memory.
 * Every compute entry point is asynchronous on the given stream and returns
 * as soon as its kernels are enqueued.  Matrices are row-major and contiguous
 * (leading dimension = number of columns).  fp16 data is IEEE binary16,
 * passed as `const void *` / `void *`.
 *
 * The method (web pages on LLM.int8()):
 *   "LLM.int8()" abstract, taxoreview.com/v/2/lake/expert/dblp:280/8696;
 *   "LLM.int8(): A Procedure for Int8 Matrix Multiplication in Transformer
 *   Language Models", summarizepaper.com/en/paper/2208.07339v1, sections
 *   "The LLM.int8() Methodology" and the summary bullets.
 * A linear layer Y = X W is computed in two parts.  Vector-wise quantisation:
 * every row of X and every output column of W gets its own absmax scale, so
 * each inner product has its own pair of normalisation constants.
 * Mixed-precision decomposition: the feature dimensions (columns of X) that
 * hold an outlier are multiplied in 16-bit together with the matching rows
 * of W; all other values are multiplied in int8 with int32 accumulation,
 * dequantised by the outer product of the two scale vectors and added to
 * the 16-bit partial result.
 *
 * Fixed choices where the pages give no number (one rule for all callers):
 *   - column k of X is an outlier when any |X[t,k]| >= alpha;
 *   - a scale is the absmax; a code is clamp(rhaz(v * fl32(127 / absmax)),
 *     -127, 127) with rhaz = round half away from zero, one fp32 division
 *     per row/column and one fp32 multiply per element; absmax 0 gives codes 0;
 *   - row scales of X are taken over the non-outlier columns only, and the
 *     outlier columns are 0 in the int8 operand;
 *   - column scales of W are taken over all K rows;
 *   - the 16-bit part uses the fp16 rows W16[k,:] for k in the outlier set,
 *     with fp32 accumulation; the result is rounded to fp16 (nearest-even).
 *
 * Shape rules shared by the entry points: T >= 0 (T == 0 is a no-op that
 * returns I8R_OK), 16 <= K <= 133144 (int32 accumulation is exact while
 * K * 127^2 < 2^31), K % 16 == 0, 16 <= N, N % 16 == 0, and every pointer
 * 16-byte aligned.  A violated rule is reported before anything is
 * enqueued, and nothing is written.
 *
 * Device-side anomalies (a pipeline wait that exceeded its time limit) do
 * not trap: the kernel records a code in a per-device status word and
 * returns early.  Read it with int8_read_and_clear_device_status().  While
 * the word is non-zero, the outputs of the calls made since it was last
 * cleared are undefined (a kernel that gave up left part of them unwritten).
 */
#ifndef INT8ROW_H
#define INT8ROW_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    I8R_OK = 0,
    I8R_EINVAL = 1,      /* null pointer, negative size, NaN or negative alpha */
    I8R_EALIGN = 2,      /* pointer not 16-byte aligned, K or N not a multiple of 16 */
    I8R_ERANGE = 3,      /* K > 133144, K < 16, N < 16, or a size beyond the library's limits */
    I8R_EWORKSPACE = 4,  /* workspace pointer null or smaller than the queried size */
    I8R_ECUDA = 5,       /* a CUDA runtime/driver call failed (see int8_last_cuda_error) */
    I8R_EDEVICE = 6,     /* the device status word holds a kernel-reported anomaly */
    I8R_EARCH = 7        /* the current device is not sm_100 (B200) */
} i8r_status;

/* Device status codes written by kernels (returned by
 * int8_read_and_clear_device_status). */
#define I8R_DEV_OK 0
#define I8R_DEV_PIPELINE_TIMEOUT 1   /* a shared-memory pipeline wait gave up */
#define I8R_DEV_TMEM_TIMEOUT 2       /* a tensor-memory hand-off wait gave up */

/* ---------------------------------------------------------------------------
 * Weight conversion.  The pages describe a 16/32-bit checkpoint converted to
 * Int8 at load time and used straight away, with one normalisation constant
 * per output column of W (LLM.int8() abstract; "The LLM.int8() Methodology").
 *
 *   W16 [K,N] fp16   input weight
 *   Wq  [K,N] int8   output codes, Wq[k,n] = clamp(rhaz(W16[k,n] * fl32(127/sW[n])), +-127)
 *   sW  [N]   fp32   output column absmax, sW[n] = max_k |W16[k,n]|
 * Enqueues two HBM-bound kernels; needs no workspace.
 * ------------------------------------------------------------------------- */
i8r_status int8_quantize_weight_colwise(const void *W16, int K, int N,
                                        int8_t *Wq, float *sW, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * The mixed-precision linear layer (LLM.int8() abstract; "The LLM.int8()
 * Methodology"; the summary's bullets on vector-wise quantisation and the
 * mixed-precision decomposition).
 *
 *   X   [T,K] fp16   activation
 *   Wq  [K,N] int8   and sW [N] fp32: from int8_quantize_weight_colwise
 *   W16 [K,N] fp16   the fp16 weight; only its rows in the outlier set are read
 *   alpha            outlier threshold (>= 0; +inf disables the 16-bit part)
 *   Y   [T,N] fp16   output, Y = fp16( acc*sX[t]*sW[n]/127^2 + X[:,O] W16[O,:] )
 *                    with acc the exact int32 product of the int8 codes
 *   workspace        device scratch of at least
 *                    int8_mixed_linear_workspace_size(T, K, N) bytes, 256-byte
 *                    aligned; its contents on entry are ignored and on return
 *                    are unspecified (it holds the quantised activation and,
 *                    for T > 128, the W16 rows of up to 256 outlier columns)
 * Two calls that share a workspace must not overlap on the GPU.
 * T <= 128 runs the decode-shaped kernel (weight streaming, split over K);
 * larger T runs the prefill kernel (tensor-core bound).
 * ------------------------------------------------------------------------- */
size_t int8_mixed_linear_workspace_size(int T, int K, int N);

i8r_status int8_mixed_linear(const void *X, int T, int K,
                             const int8_t *Wq, const float *sW, const void *W16, int N,
                             float alpha, void *Y,
                             void *workspace, size_t workspace_bytes,
                             cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * int8_mixed_linear_wq: the same layer with only Wq and sW resident.  The
 * fp16 weight need not be kept, which is the memory-halving use of the method
 * (LLM.int8() abstract).  The 16-bit part multiplies X[:,O] by the outlier
 * rows of W dequantised from the int8 codes:
 *   W~[k,n] = fp16_rn( Wq[k,n] * fl32(sW[n] / 127) )
 * (one fp32 division per column, one fp32 multiply, round to nearest even),
 * so Y = fp16( acc*sX[t]*sW[n]/127^2 + X[:,O] W~[O,:] ).
 * Arguments, layouts and workspace rules are those of int8_mixed_linear,
 * with workspace of at least int8_mixed_linear_wq_workspace_size(T, K, N)
 * bytes.  That workspace holds the dequantised rows of the first
 * int8_mixed_linear_wq_max_outliers(K) outlier columns (at least 256 and
 * 1/16 of K, rounded up to a multiple of 64, and not more than K rounded
 * up to 64), at every T; the GEMM dequantises the rows of any further
 * outlier columns itself, by index, with the same rounding (slower per row,
 * same result).
 * ------------------------------------------------------------------------- */
size_t int8_mixed_linear_wq_workspace_size(int T, int K, int N);

int int8_mixed_linear_wq_max_outliers(int K);

i8r_status int8_mixed_linear_wq(const void *X, int T, int K,
                                const int8_t *Wq, const float *sW, int N,
                                float alpha, void *Y,
                                void *workspace, size_t workspace_bytes,
                                cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * int8_mixed_linear_chain: several int8_mixed_linear layers run in order on one
 * stream with one shared workspace: the projections of a decoder layer (the
 * pages' unit of use: the Int8 multiplication of the feed-forward and
 * attention projection layers; LLM.int8() abstract).
 *
 *   layers  [n] host array of i8r_layer; each entry has the meaning of the
 *           int8_mixed_linear arguments of the same names (W16 may be null
 *           for the Wq-only variant, as in int8_mixed_linear_wq).  A layer's
 *           X may be an earlier layer's Y: the layers run one after the
 *           other in stream order, so each sees the Y of those before it.
 *   workspace  at least int8_mixed_linear_chain_workspace_size(n, layers)
 *           bytes (the largest layer's need), 256-byte aligned.
 * Every layer is checked on the host before anything is enqueued; a bad
 * layer returns its error and enqueues nothing.  n = 0 is a no-op.  The call
 * is asynchronous and graph-capturable, like int8_mixed_linear.
 * ------------------------------------------------------------------------- */
typedef struct {
    const void *X;            /* [T,K] fp16 */
    int T, K;
    const int8_t *Wq;         /* [K,N] int8 */
    const float *sW;          /* [N] fp32 */
    const void *W16;          /* [K,N] fp16, or null: outlier rows dequantised from Wq */
    int N;
    float alpha;
    void *Y;                  /* [T,N] fp16 */
} i8r_layer;

size_t int8_mixed_linear_chain_workspace_size(int n, const i8r_layer *layers);

i8r_status int8_mixed_linear_chain(int n, const i8r_layer *layers,
                                   void *workspace, size_t workspace_bytes,
                                   cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * int8_mixed_linear_noalloc: the same layer, with no workspace argument and no
 * device allocation of any kind.  The paper has no counterpart; this entry
 * point exists for callers that cannot allocate device memory where they call
 * the layer, such as a plugin inside an inference runtime that has reserved
 * the GPU's memory for its own pool and passes in only input and output
 * buffers, or a latency-critical path where cudaMalloc/cudaFree may not run
 * because they can block or synchronise the device.
 *
 * Its scratch is one fixed array of int8_mixed_linear_noalloc_max_workspace()
 * bytes (8 MiB) inside the library, which every GPU that runs the library
 * holds until the process exits.  Shapes whose
 * int8_mixed_linear_workspace_size(T, K, N) exceeds that are rejected with
 * I8R_ERANGE before anything is enqueued (T <= 16 fits every 175B-sized
 * projection).  The first call on a device looks up the array's address
 * there (cudaGetSymbolAddress, with that device current), so make that first
 * call before any stream capture; the address is looked up again when the
 * calling thread's current context is no longer the one it was found in
 * (after cudaDeviceReset, say), and that call too belongs outside a capture.
 * Every call on a device shares the one array: two calls that overlap on the
 * GPU (different streams, no ordering between them) race and corrupt each
 * other's results.
 * Arguments, layouts, result and errors are otherwise those of
 * int8_mixed_linear.
 * ------------------------------------------------------------------------- */
size_t int8_mixed_linear_noalloc_max_workspace(void);

i8r_status int8_mixed_linear_noalloc(const void *X, int T, int K,
                                     const int8_t *Wq, const float *sW, const void *W16, int N,
                                     float alpha, void *Y, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Group-wise 4-bit weight codec.  The FlexGen summary page (research.elamur.ai,
 * "sheng-2023-flexgen") states that FlexGen compresses weights (and the KV
 * cache) to 4 bits with group-wise quantization, without retraining or
 * calibration; it gives no formula.  The reading taken here, for weights:
 *   - a group is 64 consecutive rows k of one output column n of W [K,N];
 *   - its 16 levels are lo + q*s, q = 0..15, with lo the group's minimum and
 *     s = fp16_rn( fl32( fl32(hi - lo) / 15 ) ), hi the group's maximum;
 *   - code q = clamp(rhaz( fl32( fl32(w - lo) * fl32(1 / s) ) ), 0, 15), each
 *     step an IEEE fp32 operation (s = 0 gives q = 0);
 *   - the decoded weight is W~ = fp16_rn(q*s + lo), rounded once;
 *   - the product is Y = fp16( X W~ ) with fp32 accumulation; X stays fp16.
 * K must be a multiple of 256 (>= 256) and N a multiple of 16.
 *
 * The packed weight is two device buffers in the layout the product streams
 * (columns padded to a multiple of 256; KT = K / 256; both caller-owned):
 *   W4  int4_packed_code_bytes(K, N) bytes: 32 KB blocks, block (nt, kt) at
 *       byte (nt*KT + kt) * 32768 holds columns n = 256*nt + r (r < 256) and
 *       rows k = 256*kt .. 256*kt + 255; column r's 128 bytes start at r*128
 *       and hold eight 16-byte chunks, chunk c (codes k = 256*kt + 32c ..
 *       +31) at chunk position c ^ (r % 8); in a chunk, 32-bit word i holds
 *       codes 8i .. 8i+7, nibble j (bits 4j .. 4j+3) code 8i + 2j and nibble
 *       j + 4 code 8i + 2j + 1, for j = 0..3;
 *   S4  int4_packed_scale_bytes(K, N) bytes: 4 KB blocks, block (nt, kt) at
 *       byte (nt*KT + kt) * 4096; column r's 16 bytes at r*16 are the fp16
 *       pairs (s, lo) of groups 4*kt .. 4*kt + 3.
 * Padding columns have codes 0 and s = lo = 0.
 *
 * int4_quantize_weight_groupwise: W16 [K,N] fp16 -> W4, S4.
 * int4_dequantize_weight: W4, S4 -> W16d [K,N] fp16, the decoded weight W~
 *   (for checking the codec; the product decodes on the fly).
 * int4_linear: Y [T,N] fp16 = X [T,K] fp16 times W~, for 1 <= T <= 64 rows
 *   (T = 0 is a no-op; larger T returns I8R_ERANGE), with fp32 sums of the
 *   exact fp16 products.  The weight is streamed at 0.5625 bytes per weight
 *   and decoded on the fly: for T <= 2 on the CUDA cores (one mixed-precision
 *   fused multiply-add per weight and row), otherwise into the tensor cores'
 *   operand memory.  X 16-byte aligned.  Workspace of at least
 *   int4_linear_workspace_size(T, K, N)
 *   bytes, 256-byte aligned (fp32 partial sums of tiles split over the SMs);
 *   its contents on entry are ignored.  Two calls sharing a workspace must
 *   not overlap on the GPU.  Sizes out of these rules return 0 from the size
 *   queries and an error from the calls, before anything is enqueued.
 * ------------------------------------------------------------------------- */
size_t int4_packed_code_bytes(int K, int N);

size_t int4_packed_scale_bytes(int K, int N);

i8r_status int4_quantize_weight_groupwise(const void *W16, int K, int N, uint8_t *W4, void *S4,
                                          cudaStream_t stream);

i8r_status int4_dequantize_weight(const uint8_t *W4, const void *S4, int K, int N, void *W16d,
                                  cudaStream_t stream);

size_t int4_linear_workspace_size(int T, int K, int N);

i8r_status int4_linear(const void *X, int T, int K, const uint8_t *W4, const void *S4, int N, void *Y,
                       void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* int4_debug_set_product_path: 0 (the default) runs int4_linear's product on
 * the CUDA cores for T <= 2 and on the tensor cores otherwise, 1 always on the
 * tensor cores, 2 on the CUDA cores whenever T <= 4.  The two give the same
 * sums up to the order of fp32 additions; the switch (process-wide) exists so
 * that tests and measurements can compare them. */
void int4_debug_set_product_path(int mode);

/* ---------------------------------------------------------------------------
 * Outlier statistics: the outlier feature dimensions of X and the share of
 * values that go through the 8-bit product (the pages report that share as
 * above 99.9% on large models; LLM.int8() abstract).
 *
 *   num_outlier_cols [1] int32   |O|
 *   col_idx          [K] int32   O in ascending order in [0, |O|); the rest untouched
 *   col_hit_count    [K] int32   rows t with |X[t,k]| >= alpha, per column (nullable)
 *   frac_8bit        [1] fp32    1 - |O|/K, computed in double and rounded to fp32
 *   workspace        at least int8_outlier_stats_workspace_size(K) bytes
 * ------------------------------------------------------------------------- */
size_t int8_outlier_stats_workspace_size(int K);

i8r_status int8_outlier_stats(const void *X, int T, int K, float alpha,
                              int32_t *num_outlier_cols, int32_t *col_idx,
                              int32_t *col_hit_count, float *frac_8bit,
                              void *workspace, size_t workspace_bytes,
                              cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Intermediate results, for checking the pipeline stage by stage.
 *
 * int8_quantize_activation: the activation side of int8_mixed_linear
 *   mask  [ceil(K/32)] uint32   bit k%32 of word k/32 set when column k is an outlier
 *   idx   [K] int32             O ascending in [0, count)
 *   count [1] int32             |O|
 *   sX    [T] fp32              row absmax over the non-outlier columns
 *   Xq    [T,K] int8            row codes, 0 in outlier columns
 *   Xo    [T,K] fp16 (nullable) Xo[t,j] = X[t, idx[j]] for j < |O|, 0 for
 *                               |O| <= j < min(64*ceil(|O|/64), K); later columns untouched
 *   workspace  at least int8_quantize_activation_workspace_size(T, K) bytes
 *              (256: a counter for the one-kernel path), 16-byte aligned
 *
 * int8_debug_set_activation_path: 1 (the default) runs the activation side
 *   as one kernel wherever that pays: for batches of 1 to 7 rows with
 *   T*K <= 32768 the row quantiser finds the outlier mask itself (every block
 *   reads all of X), for 8 to 128 rows that fit in the SMs' shared memory one
 *   cooperative kernel holds X and finds the mask across a grid barrier.
 *   2 takes that cooperative kernel whenever the batch fits, 0 always the
 *   outlier scan followed by the row quantiser.  When the runtime
 *   refuses the cooperative launch (too few SMs or too little shared memory
 *   free to the context), the call takes the scan + quantiser pair instead;
 *   3 behaves as 1 with every cooperative launch treated as refused, so that
 *   fallback can be tested.  All give the same bits; the switch
 *   (process-wide) exists so that tests can compare them.
 *
 * int8_gemm_i8_s32: acc [T,N] int32 = Xq [T,K] int8 x Wq [K,N] int8, exact,
 *   by the same tensor-core kernels int8_mixed_linear uses (decode-shaped for
 *   T <= 128, prefill otherwise).  Needs workspace of at least
 *   int8_gemm_i8_s32_workspace_size(T, K, N) bytes (may be 0; pass NULL then).
 * ------------------------------------------------------------------------- */
size_t int8_quantize_activation_workspace_size(int T, int K);

i8r_status int8_quantize_activation(const void *X, int T, int K, float alpha,
                                    uint32_t *mask, int32_t *idx, int32_t *count,
                                    float *sX, int8_t *Xq, void *Xo,
                                    void *workspace, size_t workspace_bytes,
                                    cudaStream_t stream);

void int8_debug_set_activation_path(int mode);

size_t int8_gemm_i8_s32_workspace_size(int T, int K, int N);

i8r_status int8_gemm_i8_s32(const int8_t *Xq, int T, int K, const int8_t *Wq, int N,
                            int32_t *acc, void *workspace, size_t workspace_bytes,
                            cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Status, errors and measurement.
 * ------------------------------------------------------------------------- */

/* Synchronises `stream`, then returns in *code (HOST pointer) the current
 * device's status word (I8R_DEV_*) and resets it to I8R_DEV_OK. */
i8r_status int8_read_and_clear_device_status(int *code, cudaStream_t stream);

/* Failure-detection self-test: enqueues one kernel whose single thread waits
 * on a shared-memory barrier that nothing ever completes.  The bounded wait
 * gives up after limit_us microseconds (1 .. 1e6), records
 * I8R_DEV_PIPELINE_TIMEOUT in the device status word and returns, exactly as
 * a pipeline wait in the GEMM kernels would.  The GPU is not faulted and the
 * context stays usable; read the code with
 * int8_read_and_clear_device_status(). */
i8r_status int8_selftest_wait_timeout(int limit_us, cudaStream_t stream);

/* Static description of a status code. */
const char *int8_status_string(i8r_status status);

/* The last CUDA error seen by an entry point on this host thread (cudaError_t). */
int int8_last_cuda_error(void);

/* Measurement hook: the next int8_mixed_linear, int8_gemm_i8_s32 or int4_linear call made
 * by this host thread records `before` (a cudaEvent_t) on its stream right
 * before its tensor-core GEMM kernel and `after` right after it, then forgets
 * both.  Pass NULL, NULL to cancel. */
void int8_time_next_gemm(cudaEvent_t before, cudaEvent_t after);

/* Number of kernels this library has enqueued in this process (all threads,
 * all devices), for launch accounting. */
uint64_t int8_kernel_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* INT8ROW_H */
