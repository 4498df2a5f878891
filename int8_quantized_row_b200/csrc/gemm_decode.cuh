// Decode-shaped LLM.int8() GEMM: few rows of X (T <= 128), bound by streaming
// the int8 weight from HBM (the weight-read "memory wall" of token generation,
// FP6-LLM page, "Memory Wall Issues").
//
// Swap-AB: the MMA's M = 128 columns of W (A = Wq tile, MN-major), its N = T
// rounded up to 16 (B = Xq tile, K-major), so the weight fills the 128-lane
// tensor-core dimension.  Split-K, stream-K style: the (column tile, k-block)
// units are cut into gridDim.x equal contiguous ranges, one per CTA, so every
// SM streams the same number of weight bytes.  A CTA accumulates each run of
// k-blocks of one column tile in TMEM (double-buffered) and adds the exact
// int32 partial sums into acc32 [T,N] (zeroed beforehand) with red.add.  A
// second kernel applies the scales and the 16-bit outlier part.  No CTA
// ever waits on another.
#pragma once

#include "device_common.cuh"

namespace i8r {
namespace decode {

constexpr int BM = 128;            // columns of W per tile (MMA M)
constexpr int BK = 128;            // int8 K per stage (bytes)
constexpr int A_BYTES = BM * BK;   // 16 KB
constexpr int THREADS = 192;
constexpr int MAX_T = 128;
constexpr int MAX_STAGES = 12;
constexpr size_t SMEM_BUDGET = 200 * 1024;

struct Params {
    int T, TP, K, N;
    int KB, num_tiles;
    long long total_units;
    int stages, stage_bytes;
    uint32_t tmem_cols;            // allocation (power of two >= 2*TP, >= 32); buffer b at b*tmem_cols/2
    int32_t *acc32;                // [T,N] int32, zero on entry
};

struct Barriers {
    uint64_t full[MAX_STAGES];
    uint64_t empty[MAX_STAGES];
    uint64_t tmem_full[2];
    uint64_t tmem_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

__host__ __device__ inline size_t smem_bytes(int stages, int stage_bytes) {
    return 1024 + static_cast<size_t>(stages) * stage_bytes + sizeof(Barriers);
}

// The run of units [u0, u1) of CTA `cta` out of `ctas`.
__device__ __forceinline__ void cta_range(long long total, int cta, int ctas, long long &u0, long long &u1) {
    u0 = total * cta / ctas;
    u1 = total * (cta + 1) / ctas;
}

__global__ void __launch_bounds__(THREADS, 1)
    gemm_decode_kernel(const __grid_constant__ CUtensorMap map_wq, const __grid_constant__ CUtensorMap map_xq,
                       const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Barriers *bars = reinterpret_cast<Barriers *>(smem + static_cast<size_t>(p.stages) * p.stage_bytes);
    volatile int *abort = &bars->abort;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->tmem_full[b], 1);
            mbar_init(&bars->tmem_empty[b], 4);
        }
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        fence_mbar_init();
        tma_prefetch_map(&map_wq);
        tma_prefetch_map(&map_xq);
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, p.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = bars->tmem_base;

    long long u0, u1;
    cta_range(p.total_units, blockIdx.x, gridDim.x, u0, u1);

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        int stage = 0;
        uint32_t phase = 0;
        int pending[MAX_STAGES];
        for (int s = 0; s < MAX_STAGES; ++s) pending[s] = -1;
        const uint32_t tx = static_cast<uint32_t>(p.stage_bytes);
        for (long long u = u0; u < u1; ++u) {
            const int tile = static_cast<int>(u / p.KB);
            const int kb = static_cast<int>(u - static_cast<long long>(tile) * p.KB);
            if (!warp_wait(&bars->empty[stage], phase ^ 1u, abort, I8R_DEV_PIPELINE_TIMEOUT)) break;
            if (lane == 0) {
                uint8_t *a = smem + static_cast<size_t>(stage) * p.stage_bytes;
                mbar_arrive_expect_tx(&bars->full[stage], tx);
                tma_load_2d(a, &map_wq, &bars->full[stage], tile * BM, kb * BK);
                tma_load_2d(a + A_BYTES, &map_xq, &bars->full[stage], kb * BK, 0);
                pending[stage] = static_cast<int>(phase);
            }
            __syncwarp();
            if (++stage == p.stages) { stage = 0; phase ^= 1u; }
        }
        if (*abort && lane == 0) {
            volatile int never = 0;
            for (int s = 0; s < p.stages; ++s)
                if (pending[s] >= 0) mbar_wait(&bars->full[s], static_cast<uint32_t>(pending[s]), &never, 0);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t id = idesc_i8(BM, p.TP, true, false);
        int stage = 0;
        uint32_t phase = 0;
        uint32_t tph[2] = {0, 0};
        int seg = 0;
        bool ok = true;
        for (long long u = u0; ok && u < u1;) {
            const int tile = static_cast<int>(u / p.KB);
            const long long seg_end = min(u1, static_cast<long long>(tile + 1) * p.KB);
            const int buf = seg & 1;
            if (!warp_wait(&bars->tmem_empty[buf], tph[buf] ^ 1u, abort, I8R_DEV_TMEM_TIMEOUT)) break;
            tc_fence_after_sync();
            const uint32_t d = tmem + static_cast<uint32_t>(buf) * (p.tmem_cols / 2);
            for (long long v = u; v < seg_end; ++v) {
                if (!warp_wait(&bars->full[stage], phase, abort, I8R_DEV_PIPELINE_TIMEOUT)) { ok = false; break; }
                tc_fence_after_sync();
                if (lane == 0) {
                    const uint32_t a = smem_u32(smem + static_cast<size_t>(stage) * p.stage_bytes);
                    const uint32_t b = a + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 32; ++kk) {
                        const uint64_t ad = smem_desc_sw128(a + kk * 32 * 128, A_BYTES, 1024);
                        const uint64_t bd = smem_desc_sw128(b + kk * 32, 16, 1024);
                        mma_i8(d, ad, bd, id, (v != u || kk != 0) ? 1u : 0u);
                    }
                    mma_commit(&bars->empty[stage]);
                }
                __syncwarp();
                if (++stage == p.stages) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
            if (lane == 0) mma_commit(&bars->tmem_full[buf]);
            __syncwarp();
            tph[buf] ^= 1u;
            ++seg;
            u = seg_end;
        }
        if (lane == 0) {
            volatile int never = 0;
            mma_commit(&bars->drain);
            mbar_wait(&bars->drain, 0, &never, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int quad = warp & 3;
        uint32_t tph[2] = {0, 0};
        int seg = 0;
        for (long long u = u0; u < u1;) {
            const int tile = static_cast<int>(u / p.KB);
            const long long seg_end = min(u1, static_cast<long long>(tile + 1) * p.KB);
            const int buf = seg & 1;
            if (!warp_wait(&bars->tmem_full[buf], tph[buf], abort, I8R_DEV_TMEM_TIMEOUT)) break;
            tc_fence_after_sync();
            const int n = tile * BM + quad * 32 + lane;       // this thread's column of W / Y
            const uint32_t taddr = tmem + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(buf) * (p.tmem_cols / 2);
            for (int c = 0; c < p.TP; c += 16) {
                uint32_t r[16];
                tmem_ld16(taddr + c, r);
                tmem_wait_ld();
                if (n < p.N) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int t = c + i;
                        if (t < p.T && r[i] != 0u)
                            atomicAdd(p.acc32 + static_cast<size_t>(t) * p.N + n, static_cast<int>(r[i]));
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->tmem_empty[buf]);
            tph[buf] ^= 1u;
            ++seg;
            u = seg_end;
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, p.tmem_cols);
    }
}

// ---------------------------------------------------------------------------
// Finaliser: Y[t,n] = fp16( acc32[t,n] * sX[t] * sW[n] / 127^2
//                           + sum_j Xo[t,j] * W16[O_j, n] )
// Thread = 8 consecutive columns x 8 rows; the 16-bit outlier part runs on
// CUDA cores (|O| is small; W16's outlier rows stay in L2).
// ---------------------------------------------------------------------------
constexpr int FIN_THREADS = 128;
constexpr int FIN_ROWS = 8;

__global__ void __launch_bounds__(FIN_THREADS) finalize_kernel(const int32_t *__restrict__ acc32, int T, int K, int N,
                                                              const float *__restrict__ sX,
                                                              const float *__restrict__ sW,
                                                              const __half *__restrict__ Xo,
                                                              const int32_t *__restrict__ idx,
                                                              const int32_t *__restrict__ count_ptr,
                                                              const __half *__restrict__ W16, __half *__restrict__ Y) {
    const int n = (blockIdx.x * FIN_THREADS + threadIdx.x) * 8;
    const int t0 = blockIdx.y * FIN_ROWS;
    if (n >= N) return;
    const int rows = min(FIN_ROWS, T - t0);
    const int count = *count_ptr;
    float o[FIN_ROWS][8];
#pragma unroll
    for (int r = 0; r < FIN_ROWS; ++r)
#pragma unroll
        for (int e = 0; e < 8; ++e) o[r][e] = 0.0f;
    for (int j = 0; j < count; ++j) {
        Vec16 w;
        w.u = __ldg(reinterpret_cast<const uint4 *>(W16 + static_cast<size_t>(idx[j]) * N + n));
        float wf[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) wf[e] = __half2float(w.h[e]);
#pragma unroll
        for (int r = 0; r < FIN_ROWS; ++r) {
            if (r < rows) {
                const float x = __half2float(Xo[static_cast<size_t>(t0 + r) * K + j]);
#pragma unroll
                for (int e = 0; e < 8; ++e) o[r][e] = fmaf(x, wf[e], o[r][e]);
            }
        }
    }
    const float4 s0 = __ldg(reinterpret_cast<const float4 *>(sW + n));
    const float4 s1 = __ldg(reinterpret_cast<const float4 *>(sW + n + 4));
    const float sw[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
    for (int r = 0; r < FIN_ROWS; ++r) {
        if (r < rows) {
            const int t = t0 + r;
            const float rs = sX[t] * (1.0f / 16129.0f);
            const int4 a0 = *reinterpret_cast<const int4 *>(acc32 + static_cast<size_t>(t) * N + n);
            const int4 a1 = *reinterpret_cast<const int4 *>(acc32 + static_cast<size_t>(t) * N + n + 4);
            const int a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            Vec16 out;
#pragma unroll
            for (int e = 0; e < 4; ++e)
                out.h2[e] = __floats2half2_rn(fmaf(static_cast<float>(a[2 * e]), rs * sw[2 * e], o[r][2 * e]),
                                              fmaf(static_cast<float>(a[2 * e + 1]), rs * sw[2 * e + 1],
                                                   o[r][2 * e + 1]));
            *reinterpret_cast<uint4 *>(Y + static_cast<size_t>(t) * N + n) = out.u;
        }
    }
}

}  // namespace decode
}  // namespace i8r
