// The activation side of the layer (a1-a3) in one cooperative kernel, for
// batches whose X fits in the GPU's shared memory (148 SMs x ~200 KB: the
// 2048 x 5120 fp16 OPT-13B prefill batch and every decode batch do; by
// default the library uses it for batches of 8 to 128 rows, where it is the
// faster of the two paths):
//
//   1. each block copies its R rows of X into shared memory (one bulk copy
//      per row, issued before waiting for the kernel before it) and ORs the
//      columns' |x| >= alpha bits into the outlier mask (atomicOr per word);
//   2. a grid-wide barrier: every block has added its rows to the mask (the
//      launch is cooperative, so every block is resident and the barrier
//      can complete; the wait is bounded all the same);
//   3. each block reads the finished mask and quantises its rows from
//      shared memory: sX[t] = max over non-outlier k of |X[t,k]|, Xq, and Xo
//      at the outliers' ranks ("Vector-wise quantization" and "Mixed-
//      precision decomposition" of the LLM.int8() method).  Block 0 writes the
//      index list and |O|; with W16o the blocks share the compaction of the
//      outlier weight rows.
//
// X is read from memory once; the two-kernel path (scan, then quantiser)
// reads it twice and pays a kernel boundary in between.  The arithmetic is
// that of quantize_rows_kernel (same helpers), so the results are the same
// bits.  Rows are processed by groups of warps: a few warps per row when a
// block holds many rows, the whole block on one row when it holds one.
//
// The outlier test runs on packed fp16 pairs as an integer compare
// (outlier_pair): for alpha >= 0, |x| >= alpha holds exactly when the
// magnitude bits of x (bits & 0x7FFF) are at least those of the smallest fp16
// value >= alpha and x is not NaN, so two compares test two elements.  The
// host supplies that threshold.
#pragma once

#include "device_common.cuh"
#include "quant_kernels.cuh"

namespace i8r {

constexpr int kFusedThreads = 1024;
constexpr int kFusedMinRows = 8;    // fewer rows: the scan + quantiser pair is faster
// Fewer rows than kFusedMinRows and at most this many elements of X: the row
// quantiser finds the mask itself (every block reads all of X), no scan.
constexpr long long kSelfMaskElems = 1 << 15;
constexpr size_t kFusedSmemMax = 200 * 1024;

// Shared memory of activation_fused_kernel: R rows of X, the mask words and
// their ranks, and the row-copy barrier.
__host__ __device__ inline size_t fused_smem_bytes(int R, int K) {
    return static_cast<size_t>(R) * K * 2 + static_cast<size_t>((K + 31) / 32) * 8 + 16;
}

__global__ void __launch_bounds__(kFusedThreads, 1) activation_fused_kernel(
    const __half *__restrict__ X, int T, int K, uint32_t thr2, int R, uint32_t *__restrict__ mask,
    unsigned *__restrict__ grid_ctr, float *__restrict__ sX, int8_t *__restrict__ Xq, __half *__restrict__ Xo,
    int32_t *__restrict__ idx_out, int32_t *__restrict__ count_out, const __half *__restrict__ W16,
    const int8_t *__restrict__ Wq, const float *__restrict__ sW, int N, __half *__restrict__ W16o, int o_rows,
    int4 *__restrict__ zero, size_t zero16) {
    constexpr int kWarps = kFusedThreads / 32;
    extern __shared__ __align__(16) uint8_t fs[];
    __shared__ float red[kWarps];
    __shared__ int wsum[kWarps];
    __shared__ int ok_s;
    const int nwords = (K + 31) / 32;
    const int chunks = K / 8;
    const int row0 = static_cast<int>(blockIdx.x) * R;
    const int nrows = max(0, min(R, T - row0));
    __half *rows = reinterpret_cast<__half *>(fs);
    uint32_t *smask = reinterpret_cast<uint32_t *>(fs + static_cast<size_t>(R) * K * 2);
    int *spre = reinterpret_cast<int *>(smask + nwords);
    uint64_t *bar = reinterpret_cast<uint64_t *>(spre + nwords);
    const uint8_t *mbytes = reinterpret_cast<const uint8_t *>(smask);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    volatile int never = 0;

    // 1. this block's rows into shared memory (X does not depend on earlier kernels)
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
        if (nrows > 0) {
            mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nrows) * K * 2);
            for (int r = 0; r < nrows; ++r)
                bulk_load(rows + static_cast<size_t>(r) * K, X + static_cast<size_t>(row0 + r) * K,
                          static_cast<uint32_t>(K) * 2, bar);
        }
    }
    griddep_wait();                     // the mask and the grid counter are clear
    if (zero) {
        const size_t nthreads = static_cast<size_t>(gridDim.x) * kFusedThreads;
        for (size_t i = static_cast<size_t>(blockIdx.x) * kFusedThreads + tid; i < zero16; i += nthreads)
            zero[i] = make_int4(0, 0, 0, 0);
    }
    if (tid == 0) ok_s = nrows > 0 ? (mbar_wait(bar, 0, &never, I8R_DEV_PIPELINE_TIMEOUT) ? 1 : 0) : 1;
    __syncthreads();
    const bool rows_ok = ok_s != 0;
    if (rows_ok && nrows > 0) {
        // four neighbouring threads hold the four bytes of one 32-column word
        for (int c0 = 0; c0 < chunks; c0 += kFusedThreads) {
            const int c = c0 + tid;
            uint32_t h0 = 0, h1 = 0, h2 = 0, h3 = 0;   // per fp16 pair: 0xFFFF where some row hit
            if (c < chunks)
                for (int r = 0; r < nrows; ++r) {
                    const uint4 u = reinterpret_cast<const uint4 *>(rows + static_cast<size_t>(r) * K)[c];
                    h0 |= outlier_pair(u.x, thr2);
                    h1 |= outlier_pair(u.y, thr2);
                    h2 |= outlier_pair(u.z, thr2);
                    h3 |= outlier_pair(u.w, thr2);
                }
            // element 2i is the low half of word i, 2i+1 the high half
            const uint32_t f = (h0 & 1u) | ((h0 >> 15) & 2u) | ((h1 & 1u) << 2) | ((h1 >> 13) & 8u) |
                               ((h2 & 1u) << 4) | ((h2 >> 11) & 32u) | ((h3 & 1u) << 6) | ((h3 >> 9) & 128u);
            uint32_t w = f << (8 * (tid & 3));
            w |= __shfl_xor_sync(0xFFFFFFFFu, w, 1);
            w |= __shfl_xor_sync(0xFFFFFFFFu, w, 2);
            if ((tid & 3) == 0 && w != 0u) atomicOr(mask + c / 4, w);
        }
    }

    // 2. every block's rows are in the mask.  A block whose rows never arrived
    // says so (grid_ctr[1]) before it arrives, so no block goes on with a
    // mask that lacks its rows.
    __syncthreads();
    if (tid == 0) {
        if (!rows_ok) atomicOr(grid_ctr + 1, 1u);
        __threadfence();
        atomicAdd(grid_ctr, 1u);
        const uint64_t t0 = global_timer_ns();
        int done = 0;
        for (uint32_t it = 0; it < kWaitLimitIters; ++it) {
            if (*reinterpret_cast<volatile unsigned *>(grid_ctr) >= gridDim.x) {
                done = 1;
                break;
            }
            if ((it & 63u) == 0 && global_timer_ns() - t0 > kWaitLimitNs) break;
        }
        if (!done) report_status(I8R_DEV_PIPELINE_TIMEOUT);
        __threadfence();
        ok_s = done && rows_ok && *reinterpret_cast<volatile unsigned *>(grid_ctr + 1) == 0u;
    }
    __syncthreads();
    griddep_launch_dependents();        // every block of this grid is resident: the GEMM may come in
    if (!ok_s) {
        // reported above; |O| = 0 keeps the GEMM from reading an index list nobody wrote
        if (blockIdx.x == 0 && tid == 0) *count_out = 0;
        return;
    }

    // 3. the mask, then each word's count of earlier outliers
    for (int w = tid; w < nwords; w += kFusedThreads) smask[w] = __ldcg(mask + w);
    __syncthreads();
    const int per = (nwords + kFusedThreads - 1) / kFusedThreads;
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
    if (blockIdx.x == 0) {
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
    // the compaction rows go to the blocks from the last one down: they hold
    // the fewest rows of X (or none), so the copies stay off the longest path
    if (W16o)
        gather_outlier_weight_rows<kFusedThreads>(smask, spre, w0, w1, total, W16, Wq, sW, N, W16o, o_rows,
                                                  static_cast<int>(gridDim.x - 1 - blockIdx.x),
                                                  static_cast<int>(gridDim.x));

    // rows: gs warps per row (one when the block holds many rows), ng rows at a time
    int gs = kWarps / max(1, min(nrows, kWarps));
    while (gs & (gs - 1)) gs &= gs - 1;                 // a power of two
    const int ng = kWarps / gs;
    const int g = warp / gs, gt = gs * 32;
    const int li = (warp % gs) * 32 + lane;
    const int padded = min((total + 63) / 64 * 64, K);  // past K the GEMMs' Xo boxes read zeros
    for (int base = 0; base < nrows; base += ng) {
        const int r = base + g;
        const bool live = r < nrows;
        const __half *xs = rows + static_cast<size_t>(live ? r : 0) * K;
        // row absmax over the non-outlier columns
        __half2 hmax = __float2half2_rn(0.0f);
        float amax = 0.0f;
        if (live)
            for (int c = li; c < chunks; c += gt) {
                Vec16 v;
                v.u = reinterpret_cast<const uint4 *>(xs)[c];
                const uint32_t mb = mbytes[c];
                if (mb == 0) {
                    hmax = habs_max8(hmax, v.u);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        if (!((mb >> e) & 1u)) amax = fmaxf(amax, fabsf(__half2float(v.h[e])));
                }
            }
        amax = fmaxf(amax, fmaxf(__low2float(hmax), __high2float(hmax)));
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, d));
        float s = amax;
        if (gs > 1) {
            if (lane == 0) red[warp] = amax;
            __syncthreads();
            s = 0.0f;
            for (int q = 0; q < gs; ++q) s = fmaxf(s, red[g * gs + q]);
            __syncthreads();                            // red is rewritten by the next round
        }
        if (!live) continue;
        const int t = row0 + r;
        const float inv = recip127(s);
        if (li == 0) sX[t] = s;
        int8_t *qrow = Xq + static_cast<size_t>(t) * K;
        __half *orow = Xo ? Xo + static_cast<size_t>(t) * K : nullptr;
        for (int c = li; c < chunks; c += gt) {
            Vec16 v;
            v.u = reinterpret_cast<const uint4 *>(xs)[c];
            const uint32_t mb = mbytes[c];
            int q[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) q[e] = quant_code_fast(__half2float(v.h[e]), inv);
            if (mb) {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if ((mb >> e) & 1u) q[e] = 0;
            }
            reinterpret_cast<uint2 *>(qrow)[c] =
                make_uint2(pack4_s8(q[0], q[1], q[2], q[3]), pack4_s8(q[4], q[5], q[6], q[7]));
            if (orow && mb) {
                // this chunk's outliers go to their ranks in Xo
                const int w = c >> 2, sh = (c & 3) * 8;
                int j = spre[w] + __popc(smask[w] & ((1u << sh) - 1u));
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if ((mb >> e) & 1u) orow[j++] = v.h[e];
            }
        }
        if (orow)
            for (int jj = total + li; jj < padded; jj += gt) orow[jj] = __float2half_rn(0.0f);
    }
}

}  // namespace i8r
