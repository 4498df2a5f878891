// HBM-bound kernels of the LLM.int8() linear: weight conversion (column
// absmax + codes), outlier-column detection, the outlier index list, and the
// activation's row quantisation with the outlier gather.  All loads and stores
// are 16-byte vectors; every kernel owns its outputs (no zero-initialised
// accumulators, no atomics), so repeated runs are bit-identical.
#pragma once

#include "device_common.cuh"

namespace i8r {

constexpr int kStripCols = 64;        // columns owned by one block in the column scans
constexpr int kStripThreads = 256;    // 8 warps; a warp covers 4 rows x 64 columns per step

union Vec16 {
    uint4 u;
    __half2 h2[4];
    __half h[8];
};

// ---------------------------------------------------------------------------
// Weight conversion, pass 1: sW[n] = max_k |W16[k,n]| ("one normalisation
// constant per output column", LLM.int8() abstract).  Block b owns columns
// [64b, 64b+64) and scans every row; lane l reads the 16-byte group
// (l % 8) of row 4w + l/8 (+ 32 i).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kStripThreads) weight_absmax_kernel(const __half *__restrict__ W16, int K, int N,
                                                                     float *__restrict__ sW) {
    __shared__ float part[kStripThreads / 8][kStripCols];
    const int tid = threadIdx.x;
    const int grp = tid & 7, sub = tid >> 3;                // 8 column groups x 32 row slots
    const int col = blockIdx.x * kStripCols + grp * 8;
    float m[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (col < N) {
        for (int k = sub; k < K; k += kStripThreads / 8) {
            Vec16 v;
            v.u = __ldg(reinterpret_cast<const uint4 *>(W16 + static_cast<size_t>(k) * N + col));
#pragma unroll
            for (int i = 0; i < 8; ++i) m[i] = fmaxf(m[i], fabsf(__half2float(v.h[i])));
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) part[sub][grp * 8 + i] = m[i];
    __syncthreads();
    if (tid < kStripCols) {
        float r = 0.0f;
        for (int s = 0; s < kStripThreads / 8; ++s) r = fmaxf(r, part[s][tid]);
        const int c = blockIdx.x * kStripCols + tid;
        if (c < N) sW[c] = r;
    }
}

// Weight conversion, pass 2: Wq[k,n] = clamp(rhaz(W16[k,n] * fl32(127/sW[n])), +-127).
__global__ void __launch_bounds__(256) weight_codes_kernel(const __half *__restrict__ W16, int K, int N,
                                                          const float *__restrict__ sW, int8_t *__restrict__ Wq) {
    const size_t groups = static_cast<size_t>(K) * (N / 8);
    const int gpr = N / 8;
    for (size_t g = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; g < groups;
         g += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const size_t k = g / gpr;
        const int n = static_cast<int>(g - k * gpr) * 8;
        Vec16 v;
        v.u = __ldg(reinterpret_cast<const uint4 *>(W16 + k * N + n));
        const float4 s0 = __ldg(reinterpret_cast<const float4 *>(sW + n));
        const float4 s1 = __ldg(reinterpret_cast<const float4 *>(sW + n + 4));
        const float s[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t b = static_cast<uint32_t>(quant_code(__half2float(v.h[i]), recip127(s[i]))) & 0xFFu;
            if (i < 4) lo |= b << (8 * i); else hi |= b << (8 * (i - 4));
        }
        *reinterpret_cast<uint2 *>(Wq + k * N + n) = make_uint2(lo, hi);
    }
}

// ---------------------------------------------------------------------------
// Outlier feature dimensions: mask bit k set when any |X[t,k]| >= alpha
// (outliers defined by magnitude; "The LLM.int8() Methodology").
// Column-strip form, used by the outlier statistics: block (x, y) owns
// columns [64x, 64x+64) of rows [y*rows_per_part, (y+1)*rows_per_part) and
// writes the two partial mask words part_masks[y*words + 2x + {0,1}].  With
// one part (gridDim.y == 1) the partial words are the mask, and the optional
// per-column hit counts are exact.  A thread keeps 8 row loads in flight.
// ---------------------------------------------------------------------------

template <bool kHits>
__global__ void __launch_bounds__(kStripThreads) outlier_mask_kernel(const __half *__restrict__ X, int T, int K,
                                                                    float alpha, int rows_per_part,
                                                                    uint32_t *__restrict__ part_masks,
                                                                    int32_t *__restrict__ hits, int4 *__restrict__ zero,
                                                                    size_t zero16) {
    constexpr int kWarps = kStripThreads / 32;
    constexpr int kSlots = kStripThreads / 8;          // 32 row slots per step
    constexpr int kUnroll = 8;                         // row loads in flight per thread
    __shared__ uint32_t wflags[kWarps][8];
    __shared__ int32_t wcnt[kHits ? kWarps : 1][kHits ? kStripCols : 1];
    griddep_launch_dependents();       // the row quantiser may start loading its rows
    if (zero) {
        const size_t nthreads = static_cast<size_t>(gridDim.x) * gridDim.y * kStripThreads;
        for (size_t i = (static_cast<size_t>(blockIdx.y) * gridDim.x + blockIdx.x) * kStripThreads + threadIdx.x;
             i < zero16; i += nthreads)
            zero[i] = make_int4(0, 0, 0, 0);
    }
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int grp = tid & 7, sub = tid >> 3;           // column group (8 columns), row slot
    const int col = blockIdx.x * kStripCols + grp * 8;
    const int r0 = blockIdx.y * rows_per_part;
    const int r1 = min(T, r0 + rows_per_part);
    uint32_t f = 0;
    int32_t h[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (col < K) {
        for (int t = r0 + sub; t < r1; t += kUnroll * kSlots) {
            Vec16 v[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int tt = t + u * kSlots;
                v[u].u = tt < r1 ? __ldg(reinterpret_cast<const uint4 *>(X + static_cast<size_t>(tt) * K + col))
                                 : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const bool live = t + u * kSlots < r1;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const bool hit = live && fabsf(__half2float(v[u].h[i])) >= alpha;
                    f |= static_cast<uint32_t>(hit) << i;
                    if (kHits) h[i] += hit;
                }
            }
        }
    }
    // lanes l, l^8, l^16, l^24 share a column group: combine them, then the warps
    f |= __shfl_xor_sync(0xFFFFFFFFu, f, 8);
    f |= __shfl_xor_sync(0xFFFFFFFFu, f, 16);
    if (lane < 8) wflags[warp][lane] = f;
    if (kHits) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            h[i] += __shfl_xor_sync(0xFFFFFFFFu, h[i], 8);
            h[i] += __shfl_xor_sync(0xFFFFFFFFu, h[i], 16);
        }
        if (lane < 8) {
#pragma unroll
            for (int i = 0; i < 8; ++i) wcnt[warp][lane * 8 + i] = h[i];
        }
    }
    __syncthreads();
    const int words = (K + 31) / 32;
    if (tid < 2) {
        // word tid covers column groups 4*tid .. 4*tid+3
        uint32_t w = 0;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            uint32_t byte = 0;
#pragma unroll
            for (int ww = 0; ww < kWarps; ++ww) byte |= wflags[ww][tid * 4 + g];
            w |= byte << (8 * g);
        }
        const int word = blockIdx.x * 2 + tid;
        if (word < words) part_masks[static_cast<size_t>(blockIdx.y) * words + word] = w;
    }
    if (kHits && tid < kStripCols) {
        int32_t r = 0;
#pragma unroll
        for (int ww = 0; ww < kWarps; ++ww) r += wcnt[ww][tid];
        const int c = blockIdx.x * kStripCols + tid;
        if (c < K) hits[c] = r;
    }
}

// ---------------------------------------------------------------------------
// Outlier feature dimensions for int8_mixed_linear: the same mask bits as
// outlier_mask_kernel, scanned in row bands so that every warp load is 512
// contiguous bytes of one row.  Block (b, c) covers columns
// [2048b, 2048b + 2048) (8 per thread) of rows [c*rows_per_block, ...) and
// ORs its non-zero 32-column words into `mask` with atomics; clear_mask_kernel
// zeroes the mask first, and this kernel, its programmatic dependent, waits
// for that only after its row loads.  Optionally clears `zero` on the way.
// ---------------------------------------------------------------------------
constexpr int kScanThreads = 256;
constexpr int kBandCols = kScanThreads * 8;

__global__ void __launch_bounds__(256) clear_mask_kernel(uint32_t *__restrict__ mask, int nwords,
                                                         unsigned *__restrict__ grid_ctr) {
    griddep_launch_dependents();        // the scan may start loading rows
    for (int w = threadIdx.x; w < nwords; w += blockDim.x) mask[w] = 0u;
    if (grid_ctr && threadIdx.x == 0) {                   // the fused kernel's grid barrier
        grid_ctr[0] = 0u;                                 // arrivals
        grid_ctr[1] = 0u;                                 // some block's rows did not arrive
    }
}

__global__ void __launch_bounds__(kScanThreads) outlier_scan_kernel(const __half *__restrict__ X, int T, int K,
                                                                   float alpha, int rows_per_block,
                                                                   uint32_t *__restrict__ mask,
                                                                   int4 *__restrict__ zero, size_t zero16) {
    constexpr int kUnroll = 8;          // row loads in flight per thread
    griddep_launch_dependents();        // the row quantiser may start loading its rows
    if (zero) {
        const size_t nthreads = static_cast<size_t>(gridDim.x) * gridDim.y * kScanThreads;
        for (size_t i = (static_cast<size_t>(blockIdx.y) * gridDim.x + blockIdx.x) * kScanThreads + threadIdx.x;
             i < zero16; i += nthreads)
            zero[i] = make_int4(0, 0, 0, 0);
    }
    const int col = blockIdx.x * kBandCols + threadIdx.x * 8;
    const int r0 = blockIdx.y * rows_per_block;
    const int r1 = min(T, r0 + rows_per_block);
    uint32_t f = 0;
    if (col < K) {
        const __half *xc = X + col;
        for (int t = r0; t < r1; t += kUnroll) {
            Vec16 v[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u)
                v[u].u = t + u < r1 ? __ldg(reinterpret_cast<const uint4 *>(xc + static_cast<size_t>(t + u) * K))
                                    : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const bool live = t + u < r1;
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    f |= static_cast<uint32_t>(live && fabsf(__half2float(v[u].h[i])) >= alpha) << i;
            }
        }
    }
    // four neighbouring threads hold the four bytes of one 32-column word
    uint32_t w = f << (8 * (threadIdx.x & 3));
    w |= __shfl_xor_sync(0xFFFFFFFFu, w, 1);
    w |= __shfl_xor_sync(0xFFFFFFFFu, w, 2);
    griddep_wait();                     // the mask has been cleared
    if ((threadIdx.x & 3) == 0 && w != 0u) atomicOr(mask + col / 32, w);
}

// ---------------------------------------------------------------------------
// The outlier set O as an ascending index list, by prefix popcount of the
// mask (one block).  Also |O| and, when asked, 1 - |O|/K rounded from double.
// ---------------------------------------------------------------------------
constexpr int kIndexThreads = 1024;

// The mask is the OR of `nparts` partial masks (part p at part_masks + p*words);
// it is written to `mask` (which may alias the first part when nparts == 1).
__global__ void __launch_bounds__(kIndexThreads) outlier_index_kernel(const uint32_t *part_masks, int nparts, int K,
                                                                     uint32_t *mask, int32_t *__restrict__ idx,
                                                                     int32_t *__restrict__ count,
                                                                     float *__restrict__ frac_8bit) {
    __shared__ int32_t warp_sums[kIndexThreads / 32];
    const int nwords = (K + 31) / 32;
    const int per = (nwords + kIndexThreads - 1) / kIndexThreads;
    const int w0 = threadIdx.x * per;
    const int w1 = min(w0 + per, nwords);
    const bool copy = mask != part_masks;
    int local = 0;
    for (int w = w0; w < w1; ++w) {
        uint32_t m = part_masks[w];
        for (int p = 1; p < nparts; ++p) m |= part_masks[static_cast<size_t>(p) * nwords + w];
        if (copy) mask[w] = m;          // each thread re-reads only the words it wrote
        local += __popc(m);
    }
    // block-wide exclusive scan of `local`
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = local;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += y;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int s = warp_sums[lane];
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, s, d);
            if (lane >= d) s += y;
        }
        warp_sums[lane] = s;   // inclusive over warps
    }
    __syncthreads();
    int pos = incl - local + (warp > 0 ? warp_sums[warp - 1] : 0);
    for (int w = w0; w < w1; ++w) {
        uint32_t m = mask[w];
        while (m) {
            const int b = __ffs(m) - 1;
            idx[pos++] = w * 32 + b;
            m &= m - 1;
        }
    }
    if (threadIdx.x == kIndexThreads - 1) {
        const int total = warp_sums[kIndexThreads / 32 - 1];
        *count = total;
        if (frac_8bit) *frac_8bit = static_cast<float>(1.0 - static_cast<double>(total) / static_cast<double>(K));
    }
}

// ---------------------------------------------------------------------------
// Row quantisation of the non-outlier part plus the outlier gather (one
// block per row of X, after the G blocks that compact outlier weight rows for
// the GEMMs):
//   sX[t]   = max over k not in O of |X[t,k]|
//   Xq[t,k] = 0 for k in O, else clamp(rhaz(X[t,k] * fl32(127/sX[t])), +-127)
//   Xo[t,j] = X[t, O_j] for j < |O|, 0 up to the next multiple of 64 (or K)
// ("Vector-wise quantization" and "Mixed-precision decomposition").
// Every block ORs the partial masks of the outlier scan into shared memory
// and ranks the outlier columns itself (prefix counts of the mask words'
// population counts), so no index kernel runs in between; row 0's block also
// publishes the mask, the ascending index list and |O|.
// The kernel is launched as a programmatic dependent of the outlier scan: the
// row is loaded before the block waits for the scan to finish.
// ---------------------------------------------------------------------------
constexpr int kRowRegChunks = 8;     // 16-byte chunks kept in registers per thread

// Threads per row: enough that a row fits the register chunks, few enough
// that many rows are in flight per SM (the kernel is latency-bound per row).
inline int row_threads(int K) { return K <= 4096 ? 64 : (K <= 8192 ? 128 : 256); }

// Dynamic shared memory of quantize_rows_kernel: the mask words and the
// exclusive prefix of their population counts.
inline size_t quantize_smem_bytes(int K) { return static_cast<size_t>((K + 31) / 32) * 8; }

// The W16 rows of the first o_rows outlier columns, compacted for the
// prefill GEMM (its outlier stages then load two 64 x 64 boxes each instead
// of gathering rows):  W16o[j,:] = W16[O_j,:] for j < |O|, zero rows up to the
// next multiple of 16 (at most o_rows; the MMAs read no row past that, so the
// rest of a 64-row box may hold anything).  Without W16 (the Wq-only variant) the
// rows are dequantised instead, W16o[j,n] = fp16_rn(Wq[O_j,n] * fl32(sW[n]/127));
// the GEMMs dequantise any rows past o_rows themselves.
// Block e of the G compaction blocks copies rows e, e+G, ... with eight
// 16-byte stores in flight per thread, 256 ranks of the index list at a time
// (the window held in shared memory).
constexpr int kCompactOutlierRows = 256;

template <int kThreads>
__device__ __forceinline__ void gather_outlier_weight_rows(const uint32_t *smask, const int *spre, int w0, int w1,
                                                           int total, const __half *__restrict__ W16,
                                                           const int8_t *__restrict__ Wq, const float *__restrict__ sW,
                                                           int N, __half *__restrict__ W16o, int o_rows, int e, int G) {
    __shared__ int oidx[kCompactOutlierRows];
    const int rows = min((total + 15) / 16 * 16, o_rows);
    const int vec = N / 8;
    constexpr int kBatch = 8;
    // outlier ranks [cb, cb + 256) at a time: that window's column indices, then its rows
    for (int cb = 0; cb < rows; cb += kCompactOutlierRows) {
        const int ce = cb + kCompactOutlierRows;
        if (cb > 0) __syncthreads();                 // every row of the previous window is copied
        for (int w = w0; w < w1; ++w) {
            int j = spre[w];
            uint32_t m = smask[w];
            if (j >= ce || j + __popc(m) <= cb) continue;
            while (m && j < ce) {
                if (j >= cb) oidx[j - cb] = w * 32 + (__ffs(m) - 1);
                ++j;
                m &= m - 1;
            }
        }
        __syncthreads();
        int r0 = e;                                  // the first row of this window that block e copies
        if (r0 < cb) r0 += (cb - e + G - 1) / G * G;
        for (int r = r0; r < min(ce, rows); r += G) {
            uint4 *dst = reinterpret_cast<uint4 *>(W16o + static_cast<size_t>(r) * N);
            if (!W16) {
                // dequantised rows: 8 codes and 8 column scales per 16-byte store
                const uint2 *q8 = r < total ? reinterpret_cast<const uint2 *>(Wq + static_cast<size_t>(oidx[r - cb]) * N)
                                            : nullptr;
                for (int c = static_cast<int>(threadIdx.x); c < vec; c += kThreads) {
                    Vec16 v;
                    v.u = make_uint4(0u, 0u, 0u, 0u);
                    if (q8) {
                        const uint2 qq = __ldg(q8 + c);
                        const float4 s0 = __ldg(reinterpret_cast<const float4 *>(sW) + 2 * c);
                        const float4 s1 = __ldg(reinterpret_cast<const float4 *>(sW) + 2 * c + 1);
                        const float sc[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
    #pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int q = static_cast<int8_t>(((i < 4 ? qq.x : qq.y) >> (8 * (i & 3))) & 0xFFu);
                            v.h[i] = __float2half_rn(__fmul_rn(static_cast<float>(q), __fdiv_rn(sc[i], 127.0f)));
                        }
                    }
                    dst[c] = v.u;
                }
                continue;
            }
            const uint4 *src = r < total ? reinterpret_cast<const uint4 *>(W16 + static_cast<size_t>(oidx[r - cb]) * N)
                                         : nullptr;
            for (int c0 = static_cast<int>(threadIdx.x); c0 < vec; c0 += kThreads * kBatch) {
                uint4 v[kBatch];
    #pragma unroll
                for (int b = 0; b < kBatch; ++b) {
                    const int c = c0 + b * kThreads;
                    v[b] = (src && c < vec) ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
                }
    #pragma unroll
                for (int b = 0; b < kBatch; ++b) {
                    const int c = c0 + b * kThreads;
                    if (c < vec) dst[c] = v[b];
                }
            }
        }
    }
}

// Absolute value of eight fp16 lanes (sign bits cleared) folded into a
// running fp16x2 maximum; exact, since max and |.| are exact in fp16.
__device__ __forceinline__ __half2 habs_max8(__half2 m, const uint4 &u) {
    const uint32_t a[4] = {u.x & 0x7FFF7FFFu, u.y & 0x7FFF7FFFu, u.z & 0x7FFF7FFFu, u.w & 0x7FFF7FFFu};
#pragma unroll
    for (int k = 0; k < 4; ++k) m = __hmax2(m, *reinterpret_cast<const __half2 *>(&a[k]));
    return m;
}

// The int8 code of y = fl32(x * inv) with the rule of quant_code, in four
// steps: rhaz(y) = trunc(y + copysign(1/2, y)) for the exact sum, and the sum
// rounded toward zero truncates to the same integer (that integer lies
// between zero and the exact sum and is a float, so rounding toward zero
// cannot pass it).  |y| <= 127 * (1 + 2^-23) for x in the row's range, so
// no clamp is needed.
__device__ __forceinline__ int quant_code_fast(float x, float inv) {
    const float y = __fmul_rn(x, inv);
    return __float2int_rz(__fadd_rz(y, copysignf(0.5f, y)));
}

// Four codes in [-127, 127] as the bytes of a word, q0 lowest.
__device__ __forceinline__ uint32_t pack4_s8(int q0, int q1, int q2, int q3) {
    const uint32_t p01 = __byte_perm(static_cast<uint32_t>(q0), static_cast<uint32_t>(q1), 0x0040u);
    const uint32_t p23 = __byte_perm(static_cast<uint32_t>(q2), static_cast<uint32_t>(q3), 0x0040u);
    return __byte_perm(p01, p23, 0x5410u);
}

// |x| >= alpha on a pair of fp16 values, 0xFFFF per half where it holds:
// the magnitude bits (bits & 0x7FFF) at least those of the smallest fp16
// >= alpha (thr2, both halves) -- magnitude bit patterns order like the values
// -- and at most those of infinity, so that NaN, like the float compare
// fabsf(x) >= alpha, is no outlier.
__device__ __forceinline__ uint32_t outlier_pair(uint32_t u, uint32_t thr2) {
    const uint32_t a = u & 0x7FFF7FFFu;
    return __vcmpgeu2(a, thr2) & __vcmpleu2(a, 0x7C007C00u);
}

// The outlier bits of 32 columns (word w) over T rows (outlier_pair).
__device__ __forceinline__ uint32_t outlier_word(const __half *__restrict__ X, int T, int K, int w, uint32_t thr2) {
    uint32_t m = 0;
    for (int r = 0; r < T; ++r) {
        const uint4 *src = reinterpret_cast<const uint4 *>(X + static_cast<size_t>(r) * K + w * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (w * 32 + q * 8 >= K) break;                 // K % 32 == 16: the last word has two chunks
            const uint4 u = __ldg(src + q);
            const uint32_t h0 = outlier_pair(u.x, thr2), h1 = outlier_pair(u.y, thr2);
            const uint32_t h2 = outlier_pair(u.z, thr2), h3 = outlier_pair(u.w, thr2);
            const uint32_t f = (h0 & 1u) | ((h0 >> 15) & 2u) | ((h1 & 1u) << 2) | ((h1 >> 13) & 8u) |
                               ((h2 & 1u) << 4) | ((h2 >> 11) & 32u) | ((h3 & 1u) << 6) | ((h3 >> 9) & 128u);
            m |= f << (8 * q);
        }
    }
    return m;
}

// With parts == nullptr (batches of a few rows) every block finds the outlier
// mask itself from X (thr2, as outlier_word), so the call needs neither the
// mask clear nor the outlier scan: one launch, and it also clears `zero`
// (zero16 16-byte words, grid-strided) on the way.
template <int kRowThreads>
__global__ void __launch_bounds__(kRowThreads) quantize_rows_kernel(
    const __half *__restrict__ X, int T, int K, const uint32_t *__restrict__ parts, int nparts,
    float *__restrict__ sX, int8_t *__restrict__ Xq, __half *__restrict__ Xo, uint32_t *__restrict__ mask_out,
    int32_t *__restrict__ idx_out, int32_t *__restrict__ count_out, const __half *__restrict__ W16,
    const int8_t *__restrict__ Wq, const float *__restrict__ sW, int N, __half *__restrict__ W16o, int o_rows,
    int G, uint32_t thr2, int4 *__restrict__ zero, size_t zero16) {
    constexpr int kWarps = kRowThreads / 32;
    extern __shared__ uint32_t qs[];
    __shared__ float red[kWarps];
    __shared__ int wsum[kWarps];
    const int nwords = (K + 31) / 32;
    uint32_t *smask = qs;
    int *spre = reinterpret_cast<int *>(qs + nwords);
    const int t = static_cast<int>(blockIdx.x) - G;             // row; < 0: compaction block
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int chunks = K / 8;
    griddep_launch_dependents();        // the GEMM may start its prologue and weight loads

    // The row goes into registers first: X does not depend on the outlier scan.
    const __half *xrow = X + static_cast<size_t>(t < 0 ? 0 : t) * K;
    Vec16 keep[kRowRegChunks];
    if (t >= 0) {
#pragma unroll
        for (int c = 0; c < kRowRegChunks; ++c) {
            const int i = tid + c * kRowThreads;
            if (i < chunks) keep[c].u = __ldg(reinterpret_cast<const uint4 *>(xrow) + i);
        }
    }
    griddep_wait();                     // the outlier scan's partial masks are complete

    // the mask (OR of the parts, or found here), then each word's count of earlier outliers
    if (parts) {
        for (int w = tid; w < nwords; w += kRowThreads) {
            uint32_t m = parts[w];
            for (int q = 1; q < nparts; ++q) m |= parts[static_cast<size_t>(q) * nwords + w];
            smask[w] = m;
        }
    } else {
        for (int w = tid; w < nwords; w += kRowThreads) smask[w] = outlier_word(X, T, K, w, thr2);
        if (zero) {
            const size_t nthreads = static_cast<size_t>(gridDim.x) * kRowThreads;
            for (size_t i = static_cast<size_t>(blockIdx.x) * kRowThreads + tid; i < zero16; i += nthreads)
                zero[i] = make_int4(0, 0, 0, 0);
        }
    }
    __syncthreads();
    const int per = (nwords + kRowThreads - 1) / kRowThreads;
    const int w0 = min(tid * per, nwords), w1 = min(w0 + per, nwords);
    int local = 0;
    for (int w = w0; w < w1; ++w) local += __popc(smask[w]);
    int incl = local;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        if (w < warp) before += wsum[w];
        total += wsum[w];
    }
    {
        int run = before + incl - local;
        for (int w = w0; w < w1; ++w) {
            spre[w] = run;
            run += __popc(smask[w]);
        }
    }
    __syncthreads();
    if (t < 0) {
        gather_outlier_weight_rows<kRowThreads>(smask, spre, w0, w1, total, W16, Wq, sW, N, W16o, o_rows,
                                                static_cast<int>(blockIdx.x), G);
        return;
    }
    const uint8_t *mbytes = reinterpret_cast<const uint8_t *>(smask);

    // row absmax over the non-outlier columns
    __half2 hmax = __float2half2_rn(0.0f);
    float amax = 0.0f;
    auto scan = [&](int i, const Vec16 &v) {
        const uint32_t mb = mbytes[i];
        if (mb == 0) {
            hmax = habs_max8(hmax, v.u);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if (!((mb >> e) & 1u)) amax = fmaxf(amax, fabsf(__half2float(v.h[e])));
        }
    };
#pragma unroll
    for (int c = 0; c < kRowRegChunks; ++c) {
        const int i = tid + c * kRowThreads;
        if (i < chunks) scan(i, keep[c]);
    }
    for (int i = tid + kRowRegChunks * kRowThreads; i < chunks; i += kRowThreads) {
        Vec16 v;
        v.u = __ldg(reinterpret_cast<const uint4 *>(xrow) + i);
        scan(i, v);
    }
    amax = fmaxf(amax, fmaxf(__low2float(hmax), __high2float(hmax)));
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, d));
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s = fmaxf(s, red[w]);
    const float inv = recip127(s);
    if (tid == 0) sX[t] = s;

    int8_t *qrow = Xq + static_cast<size_t>(t) * K;
    __half *orow = Xo ? Xo + static_cast<size_t>(t) * K : nullptr;
    auto emit = [&](int i, const Vec16 &v) {
        const uint32_t mb = mbytes[i];
        int q[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) q[e] = quant_code_fast(__half2float(v.h[e]), inv);
        if (mb) {
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if ((mb >> e) & 1u) q[e] = 0;
        }
        reinterpret_cast<uint2 *>(qrow)[i] =
            make_uint2(pack4_s8(q[0], q[1], q[2], q[3]), pack4_s8(q[4], q[5], q[6], q[7]));
        if (orow && mb) {
            // this chunk's outliers go to their ranks in Xo
            const int w = i >> 2, sh = (i & 3) * 8;
            int j = spre[w] + __popc(smask[w] & ((1u << sh) - 1u));
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if ((mb >> e) & 1u) orow[j++] = v.h[e];
        }
    };
#pragma unroll
    for (int c = 0; c < kRowRegChunks; ++c) {
        const int i = tid + c * kRowThreads;
        if (i < chunks) emit(i, keep[c]);
    }
    for (int i = tid + kRowRegChunks * kRowThreads; i < chunks; i += kRowThreads) {
        Vec16 v;
        v.u = __ldg(reinterpret_cast<const uint4 *>(xrow) + i);
        emit(i, v);
    }
    if (orow) {
        const int padded = min((total + 63) / 64 * 64, K);   // past K the GEMMs' Xo boxes read zeros
        for (int jj = total + tid; jj < padded; jj += kRowThreads) orow[jj] = __float2half_rn(0.0f);
    }

    // row 0's block: the mask, the index list and its length
    if (t == 0 && idx_out) {
        if (mask_out)
            for (int w = tid; w < nwords; w += kRowThreads) mask_out[w] = smask[w];
        for (int w = w0; w < w1; ++w) {
            int j = spre[w];
            uint32_t m = smask[w];
            while (m) {
                idx_out[j++] = w * 32 + (__ffs(m) - 1);
                m &= m - 1;
            }
        }
        if (tid == 0) *count_out = total;
    }
}

}  // namespace i8r
