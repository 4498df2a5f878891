// Decode-shaped LLM.int8() GEMM: few rows of X (T <= 128), bound by streaming
// the int8 weight from HBM (the weight-read "memory wall" of token generation,
// FP6-LLM page, "Memory Wall Issues").
//
// Swap-AB: the MMA's M = 128 columns of W (A = Wq tile, MN-major), its N = T
// rounded up to 16 (B = Xq tile, K-major), so the weight fills the 128-lane
// tensor-core dimension.  A tile is 256 columns: two 128-column MMAs per
// k-step share one Xq tile, and every 256-byte weight line a stage touches is
// used whole.  Split-K, stream-K style: the (tile, k-block) units are cut
// into gridDim.x equal contiguous ranges, one per CTA, so every SM streams the
// same number of weight bytes.  A CTA accumulates each run of k-blocks of one
// tile in TMEM (double-buffered) and adds the exact int32 partial sums into
// acc32 [T,N] (zeroed beforehand) with red.add.
//
// The 16-bit outlier part Yo[t,n] = sum_j X[t,O_j] W16[O_j,n] (fp32) comes
// from the row quantiser's launch (its outlier-product blocks), which this
// kernel waits for with griddepcontrol.wait like the rest of the activation.
//
// Finalisation: after adding its partial sums, each epilogue warp bumps a
// counter for its (tile, 32-lane quadrant).  The warp that brings the counter
// to the number of CTAs covering the tile knows every partial sum has landed;
// it writes
//   Y[t,n] = fp16( acc32[t,n] * sX[t] * sW[n] / 127^2 + Yo[t,n] )
// for its 64 columns.  No CTA ever waits on another.  (Stream-K leaves most
// tiles split between the end of one CTA's range and the start of the next,
// so these finalisations run in the kernel's tail, which is why they do no
// more than combine two loaded values per output.)
//
// Launched as a programmatic dependent of the activation kernels: the weight
// tiles of the first stages are requested before griddepcontrol.wait, since
// they do not depend on the activation.
#pragma once

#include "device_common.cuh"

namespace i8r {
namespace decode {

constexpr int BMH = 128;           // columns per MMA (MMA M)
constexpr int BM = 2 * BMH;        // columns per tile
constexpr int BK = 128;            // int8 K per stage (bytes)
constexpr int A_HALF = BMH * BK;   // 16 KB
constexpr int A_BYTES = 2 * A_HALF;
constexpr int THREADS = 192;
constexpr int MAX_T = 128;
constexpr int MAX_STAGES = 8;
constexpr size_t SMEM_BUDGET = 200 * 1024;

struct Params {
    int T, TP, K, N;
    int KB, num_tiles;
    long long total_units;
    int stages, stage_bytes;
    uint32_t tmem_cols;            // power of two >= 4*TP, >= 32; buffer b at b*tmem_cols/2
    int32_t *acc32;                // [T,N] int32, zero on entry
    // finalisation (finalize != 0): Y from acc32 once a tile is complete
    int finalize;
    int32_t *counters;             // [num_tiles * 4], zero on entry
    const float *sX, *sW;
    const int32_t *count;
    __half *Y;
    const float *Yo;               // [T,N] fp32: the 16-bit outlier part (read when |O| > 0)
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

// CTA c of `ctas` owns units [floor(c*U/ctas), floor((c+1)*U/ctas)).
__device__ __forceinline__ long long unit_begin(long long total, int c, int ctas) {
    return total * c / ctas;
}
// The CTA whose range holds unit u.
__device__ __forceinline__ int unit_owner(long long total, long long u, int ctas) {
    return static_cast<int>(((u + 1) * ctas - 1) / total);
}

constexpr int FIN_ROWS = 16;

// Y for the columns of one finished (tile, quadrant), from the int32 sums and
// (with outliers) Yo; 16 rows at a time with all loads of a group in flight.
__device__ __forceinline__ void finalize_columns(const Params &p, int tile, int quad, int lane, int count) {
    const int nbase = tile * BM + quad * 32 + lane;
    for (int t0 = 0; t0 < p.T; t0 += FIN_ROWS) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int n = nbase + h * BMH;
            if (n >= p.N) continue;
            const float sw = p.sW[n];
            int a[FIN_ROWS];
            float yo[FIN_ROWS];
#pragma unroll
            for (int r = 0; r < FIN_ROWS; ++r) {
                const bool ok = t0 + r < p.T;
                const size_t at = static_cast<size_t>(t0 + r) * p.N + n;
                a[r] = ok ? __ldcg(p.acc32 + at) : 0;
                yo[r] = (ok && count > 0) ? __ldcg(p.Yo + at) : 0.0f;
            }
#pragma unroll
            for (int r = 0; r < FIN_ROWS; ++r) {
                const int t = t0 + r;
                if (t < p.T) {
                    const float rs = p.sX[t] * (1.0f / 16129.0f);
                    p.Y[static_cast<size_t>(t) * p.N + n] =
                        __float2half_rn(fmaf(static_cast<float>(a[r]), rs * sw, yo[r]));
                }
            }
        }
    }
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
    const uint32_t half_cols = p.tmem_cols / 2;

    const long long u0 = unit_begin(p.total_units, blockIdx.x, gridDim.x);
    const long long u1 = unit_begin(p.total_units, blockIdx.x + 1, gridDim.x);

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        const uint32_t tx = static_cast<uint32_t>(p.stage_bytes);
        int pending[MAX_STAGES];
        for (int s = 0; s < MAX_STAGES; ++s) pending[s] = -1;
        // Weight tiles of the first stages: they do not depend on the
        // activation kernels, so they are requested before waiting on them.
        const int pre = static_cast<int>(min(static_cast<long long>(p.stages), u1 - u0));
        if (lane == 0) {
            for (int i = 0; i < pre; ++i) {
                const long long u = u0 + i;
                const int tile = static_cast<int>(u / p.KB);
                const int kb = static_cast<int>(u - static_cast<long long>(tile) * p.KB);
                uint8_t *a = smem + static_cast<size_t>(i) * p.stage_bytes;
                mbar_arrive_expect_tx(&bars->full[i], tx);   // fresh barrier: the slot is free
                tma_load_2d(a, &map_wq, &bars->full[i], tile * BM, kb * BK);
                tma_load_2d(a + A_HALF, &map_wq, &bars->full[i], tile * BM + BMH, kb * BK);
                pending[i] = 0;
            }
        }
        griddep_wait();
        if (lane == 0) {
            for (int i = 0; i < pre; ++i) {
                const long long u = u0 + i;
                const int kb = static_cast<int>(u % p.KB);
                tma_load_2d(smem + static_cast<size_t>(i) * p.stage_bytes + A_BYTES, &map_xq, &bars->full[i],
                            kb * BK, 0);
            }
        }
        __syncwarp();
        int stage = pre % p.stages;
        uint32_t phase = (pre == p.stages) ? 1u : 0u;
        for (long long u = u0 + pre; u < u1; ++u) {
            const int tile = static_cast<int>(u / p.KB);
            const int kb = static_cast<int>(u - static_cast<long long>(tile) * p.KB);
            if (!warp_wait(&bars->empty[stage], phase ^ 1u, abort, I8R_DEV_PIPELINE_TIMEOUT)) break;
            if (lane == 0) {
                uint8_t *a = smem + static_cast<size_t>(stage) * p.stage_bytes;
                mbar_arrive_expect_tx(&bars->full[stage], tx);
                tma_load_2d(a, &map_wq, &bars->full[stage], tile * BM, kb * BK);
                tma_load_2d(a + A_HALF, &map_wq, &bars->full[stage], tile * BM + BMH, kb * BK);
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
        const uint32_t id = idesc_i8(BMH, p.TP, true, false);
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
            const uint32_t d0 = tmem + static_cast<uint32_t>(buf) * half_cols;
            const uint32_t d1 = d0 + static_cast<uint32_t>(p.TP);
            for (long long v = u; v < seg_end; ++v) {
                if (!warp_wait(&bars->full[stage], phase, abort, I8R_DEV_PIPELINE_TIMEOUT)) { ok = false; break; }
                tc_fence_after_sync();
                if (lane == 0) {
                    const uint32_t a = smem_u32(smem + static_cast<size_t>(stage) * p.stage_bytes);
                    const uint32_t b = a + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 32; ++kk) {
                        const uint32_t acc = (v != u || kk != 0) ? 1u : 0u;
                        const uint64_t bd = smem_desc_sw128(b + kk * 32, 16, 1024);
                        mma_i8(d0, smem_desc_sw128(a + kk * 32 * 128, A_HALF, 1024), bd, id, acc);
                        mma_i8(d1, smem_desc_sw128(a + A_HALF + kk * 32 * 128, A_HALF, 1024), bd, id, acc);
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
        griddep_wait();                                   // acc32 / counters zeroed, activation ready
        const int count = p.finalize ? *p.count : 0;
        uint32_t tph[2] = {0, 0};
        int seg = 0;
        for (long long u = u0; u < u1;) {
            const int tile = static_cast<int>(u / p.KB);
            const long long tile_u0 = static_cast<long long>(tile) * p.KB;
            const long long seg_end = min(u1, tile_u0 + p.KB);
            const int buf = seg & 1;
            if (!warp_wait(&bars->tmem_full[buf], tph[buf], abort, I8R_DEV_TMEM_TIMEOUT)) break;
            tc_fence_after_sync();
            const uint32_t taddr = tmem + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(buf) * half_cols;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int n = tile * BM + h * BMH + quad * 32 + lane;   // this thread's column
                for (int c = 0; c < p.TP; c += 16) {
                    uint32_t r[16];
                    tmem_ld16(taddr + h * p.TP + c, r);
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
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->tmem_empty[buf]);
            if (p.finalize) {
                // publish this warp's partial sums, then count the contribution
                __threadfence();
                __syncwarp();
                int last = 0;
                if (lane == 0) {
                    const int contributors = unit_owner(p.total_units, tile_u0 + p.KB - 1, gridDim.x) -
                                             unit_owner(p.total_units, tile_u0, gridDim.x) + 1;
                    const int before = atomicAdd(p.counters + tile * 4 + quad, 1);
                    last = before == contributors - 1;
                }
                last = __shfl_sync(0xFFFFFFFFu, last, 0);
                if (last) {
                    __threadfence();
                    finalize_columns(p, tile, quad, lane, count);
                }
            }
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

}  // namespace decode
}  // namespace i8r
