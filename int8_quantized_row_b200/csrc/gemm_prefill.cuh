// Prefill-shaped LLM.int8() GEMM on sm_100a tensor cores.
//
// One persistent CTA per SM walks 128 x 256 output tiles (rows of X x columns
// of W).  Per tile (vector-wise scales + mixed-precision decomposition:
// LLM.int8() abstract; "The LLM.int8() Methodology"):
//   8-bit part:  acc = sum_k Xq[t,k] Wq[k,n] in int32 in TMEM,
//                tcgen05.mma kind::i8, A = Xq tile K-major, B = Wq tile MN-major
//   dequantise:  the epilogue rewrites the accumulator in place as fp32
//                acc * sX[t] * sW[n] / 127^2 (tcgen05.ld -> scale -> tcgen05.st)
//   16-bit part: tcgen05.mma kind::f16 over ceil(|O|/16) K-steps of Xo and the
//                W16 outlier rows accumulates onto that fp32 value
//   output:      fp16(Y) staged in shared memory, TMA bulk stores
// |O| is read from device memory, so there is no host round trip.  With no
// outliers the epilogue writes Y straight from the int32 accumulator.
//
// The accumulator is double-buffered (2 x 256 TMEM columns), so the epilogue
// of one tile overlaps the MMAs of the next.  The 16-bit MMAs of a tile need
// the epilogue's in-place dequantisation first, so they are issued a few
// k-blocks into the NEXT tile (kDefer), by which time that conversion is done.
// Producer and MMA warp walk the same schedule of stages:
//   tile 0 k-blocks ..., tile 1 k-blocks 0..kDefer-1, tile 0 outlier blocks,
//   tile 1 k-blocks kDefer.., tile 2 k-blocks 0..kDefer-1, tile 1 outlier ...
//
// Warp roles (192 threads):
//   warp 0    producer: TMA loads of Xq / Wq / Xo tiles into a 4-stage ring;
//             W16 outlier rows fetched by index with cp.async (all 32 lanes),
//             then fenced into the async proxy before the stage is published
//   warp 1    TMEM allocation + MMA issue (one lane)
//   warps 2-5 epilogue: one 32-lane TMEM quadrant each; sX and the tile's sW
//             are fetched while the MMAs still run; Y leaves in 32 x 32 fp16
//             blocks (rows/columns past T/N are clipped by TMA)
// Stage: A 128 rows x 128 B (16 KB) + B 256 x 128 B (32 KB).  An outlier
// stage reuses the bytes: A = 128 rows x 64 fp16, B = 64 outlier rows x 256
// fp16 (4 MN-major chunks of 64 columns).
//
// Launched as a programmatic dependent of the activation kernels: the weight
// tiles of the first stages are requested before griddepcontrol.wait.
#pragma once

#include "device_common.cuh"

namespace i8r {
namespace prefill {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;                    // int8 K per stage (bytes)
constexpr int OBK = 64;                    // fp16 K (outlier columns) per outlier stage
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK;           // 16 KB
constexpr int B_BYTES = BN * BK;           // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int B_CHUNK_I8 = 128 * BK;       // 128 columns x 128 k-rows
constexpr int B_CHUNK_F16 = 64 * OBK * 2;  // 64 columns x 64 rows of fp16 = 8 KB
constexpr int THREADS = 192;
constexpr int TMEM_COLS = 512;             // two 256-column accumulators
constexpr int kDefer = 4;                  // k-blocks of the next tile before a tile's outlier MMAs

// Per epilogue warp: a copy of the tile's 256 column scales and two 32 x 32
// fp16 staging blocks for the bulk stores.
constexpr int EPI_SW_BYTES = BN * 4;                     // 1 KB
constexpr int EPI_STAGE_BYTES = 32 * 32 * 2;             // 2 KB
constexpr int EPI_WARP_BYTES = EPI_SW_BYTES + 2 * EPI_STAGE_BYTES;
constexpr int EPI_BYTES = 4 * EPI_WARP_BYTES;            // 20 KB
constexpr size_t SMEM_BYTES = 1024 /*alignment slack*/ + STAGES * STAGE_BYTES + EPI_BYTES + 256 /*barriers*/;

struct Params {
    int T, K, N;
    int num_m, num_tiles, KB;
    const int32_t *count;      // |O| (device); nullptr => no 16-bit part
    const int32_t *idx;        // O, ascending
    const __half *W16;         // [K,N] fp16, rows read by index
    const float *sX;           // [T]
    const float *sW;           // [N]
    __half *Y;                 // [T,N] fp16 (mode Y)
    int32_t *acc_out;          // [T,N] int32 (mode S32)
};

struct Barriers {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t acc_int_full[2];      // MMA -> epilogue: the int8 k-blocks of the tile are done
    uint64_t acc_conv[2];          // epilogue -> MMA: accumulator rewritten as scaled fp32
    uint64_t acc_final_full[2];    // MMA -> epilogue: the 16-bit MMAs are done
    uint64_t acc_empty[2];         // epilogue -> MMA: accumulator drained
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

// The order in which the producer fills and the MMA warp consumes stages.
// visit(kind, tile, local_tile_index, block): kind 0 = int8 k-block, 1 = outlier
// block.  Returns false as soon as a visit does (abort).
template <typename Visit>
__device__ __forceinline__ bool walk_schedule(const Params &p, int nob, Visit &&visit) {
    const int defer = p.KB < kDefer ? p.KB : kDefer;
    int prev_tile = -1, prev_it = -1;
    int it = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++it) {
        for (int kb = 0; kb < p.KB; ++kb) {
            if (!visit(0, tile, it, kb)) return false;
            if (kb + 1 == defer && prev_tile >= 0) {
                for (int ob = 0; ob < nob; ++ob)
                    if (!visit(1, prev_tile, prev_it, ob)) return false;
                prev_tile = -1;
            }
        }
        prev_tile = tile;
        prev_it = it;
    }
    if (prev_tile >= 0)
        for (int ob = 0; ob < nob; ++ob)
            if (!visit(1, prev_tile, prev_it, ob)) return false;
    return true;
}

template <bool kS32>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_prefill_kernel(const __grid_constant__ CUtensorMap map_xq, const __grid_constant__ CUtensorMap map_wq,
                        const __grid_constant__ CUtensorMap map_xo, const __grid_constant__ CUtensorMap map_y,
                        const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *epi = smem + STAGES * STAGE_BYTES;
    Barriers *bars = reinterpret_cast<Barriers *>(epi + EPI_BYTES);
    volatile int *abort = &bars->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->acc_int_full[b], 1);
            mbar_init(&bars->acc_conv[b], 4);
            mbar_init(&bars->acc_final_full[b], 1);
            mbar_init(&bars->acc_empty[b], 4);
        }
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        fence_mbar_init();
        tma_prefetch_map(&map_xq);
        tma_prefetch_map(&map_wq);
        if (!kS32) {
            tma_prefetch_map(&map_xo);
            tma_prefetch_map(&map_y);
        }
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = bars->tmem_base;

    // Weight tiles of this CTA's first stages do not depend on the activation
    // kernels: request them before waiting on those kernels.
    const int pre = p.KB < STAGES ? p.KB : STAGES;
    if (warp == 0 && lane == 0) {
        const int n0 = (blockIdx.x / p.num_m) * BN;
        for (int i = 0; i < pre; ++i) {
            uint8_t *b = smem + i * STAGE_BYTES + A_BYTES;
            mbar_arrive_expect_tx(&bars->full[i], STAGE_BYTES);   // fresh barrier: the slot is free
            tma_load_2d(b, &map_wq, &bars->full[i], n0, i * BK);
            tma_load_2d(b + B_CHUNK_I8, &map_wq, &bars->full[i], n0 + 128, i * BK);
        }
    }
    griddep_wait();
    const int count = (!kS32 && p.count) ? *p.count : 0;
    const int nob = (count + OBK - 1) / OBK;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        int stage = 0;
        uint32_t phase = 0;
        int pending[STAGES];
#pragma unroll
        for (int s = 0; s < STAGES; ++s) pending[s] = -1;
        int issued = 0;
        const bool ok = walk_schedule(p, nob, [&](int kind, int tile, int, int blk) -> bool {
            const int m0 = (tile % p.num_m) * BM;
            const int n0 = (tile / p.num_m) * BN;
            uint8_t *a = smem + stage * STAGE_BYTES;
            if (kind == 0 && issued < pre) {
                // weight half already requested: add the activation tile
                if (lane == 0) tma_load_2d(a, &map_xq, &bars->full[stage], blk * BK, m0);
            } else {
                if (!warp_wait(&bars->empty[stage], phase ^ 1u, abort, I8R_DEV_PIPELINE_TIMEOUT)) return false;
                if (kind == 0) {
                    if (lane == 0) {
                        uint8_t *b = a + A_BYTES;
                        mbar_arrive_expect_tx(&bars->full[stage], STAGE_BYTES);
                        tma_load_2d(a, &map_xq, &bars->full[stage], blk * BK, m0);
                        tma_load_2d(b, &map_wq, &bars->full[stage], n0, blk * BK);
                        tma_load_2d(b + B_CHUNK_I8, &map_wq, &bars->full[stage], n0 + 128, blk * BK);
                    }
                } else {
                    // W16 rows of outliers blk*64 .. blk*64+63, zero past |O| (rounded to 16)
                    const uint32_t b = smem_u32(a + A_BYTES);
                    const int rows = min(OBK, (count - blk * OBK + 15) / 16 * 16);
                    const int g0 = blk * OBK + lane, g1 = blk * OBK + 32 + lane;
                    const int k0 = g0 < count ? p.idx[g0] : -1;
                    const int k1 = g1 < count ? p.idx[g1] : -1;
                    const int n = n0 + lane * 8;       // this lane's 8 columns
                    const uint32_t chunk = b + (lane >> 3) * B_CHUNK_F16;
                    const uint32_t unit = lane & 7;
                    for (int j = 0; j < rows; ++j) {
                        const int k = __shfl_sync(0xFFFFFFFFu, j < 32 ? k0 : k1, j & 31);
                        const bool have = (k >= 0) && (n < p.N);
                        const __half *src = have ? p.W16 + static_cast<size_t>(k) * p.N + n : p.W16;
                        const uint32_t dst = chunk + j * 128 + ((unit ^ (j & 7)) << 4);   // 128-B swizzle
                        cp_async_16(dst, src, have ? 16u : 0u);
                    }
                    // make the rows visible to the tensor core (async proxy) before
                    // the stage is published
                    cp_async_wait_all();
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&bars->full[stage], A_BYTES);
                        tma_load_2d(a, &map_xo, &bars->full[stage], blk * OBK, m0);
                    }
                }
            }
            __syncwarp();
            if (kind == 0) ++issued;
#pragma unroll
            for (int s = 0; s < STAGES; ++s) if (s == stage) pending[s] = static_cast<int>(phase);
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            return true;
        });
        // Before leaving, make sure nothing this warp issued is still landing in
        // shared memory (only matters after an abort).
        if (!ok && lane == 0) {
            volatile int never = 0;
#pragma unroll
            for (int s = 0; s < STAGES; ++s)
                if (pending[s] >= 0) mbar_wait(&bars->full[s], static_cast<uint32_t>(pending[s]), &never, 0);
        }
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------------------ MMA issuer
        // One thread: anything between two MMA bursts (a warp-wide shuffle, a
        // reconvergence) delays the next burst and idles the tensor pipe.
        const uint32_t id_i8 = idesc_i8(BM, BN, false, true);
        const uint32_t id_f16 = idesc_f16(BM, BN, false, true);
        int stage = 0;
        uint32_t phase = 0;
        walk_schedule(p, nob, [&](int kind, int, int it, int blk) -> bool {
            const int buf = it & 1;
            const uint32_t use = static_cast<uint32_t>(it >> 1) & 1u;   // parity of this buffer's use
            const uint32_t d = tmem + static_cast<uint32_t>(buf * BN);
            if (kind == 0 && blk == 0) {
                if (!mbar_wait(&bars->acc_empty[buf], use ^ 1u, abort, I8R_DEV_TMEM_TIMEOUT)) return false;
                tc_fence_after_sync();
            }
            if (kind == 1 && blk == 0) {
                if (!mbar_wait(&bars->acc_conv[buf], use, abort, I8R_DEV_TMEM_TIMEOUT)) return false;
                tc_fence_after_sync();
            }
            if (!mbar_wait(&bars->full[stage], phase, abort, I8R_DEV_PIPELINE_TIMEOUT)) return false;
            tc_fence_after_sync();
            if (kind == 1) fence_proxy_async_smem();   // cp.async rows -> tensor core reads
            {
                const uint32_t a = smem_u32(smem + stage * STAGE_BYTES);
                const uint32_t b = a + A_BYTES;
                if (kind == 0) {
#pragma unroll
                    for (int kk = 0; kk < BK / 32; ++kk) {
                        const uint64_t ad = smem_desc_sw128(a + kk * 32, 16, 1024);
                        const uint64_t bd = smem_desc_sw128(b + kk * 32 * 128, B_CHUNK_I8, 1024);
                        mma_i8(d, ad, bd, id_i8, (blk | kk) != 0);
                    }
                } else {
                    const int nk = min(OBK / 16, (count - blk * OBK + 15) / 16);
                    for (int kk = 0; kk < nk; ++kk) {
                        const uint64_t ad = smem_desc_sw128(a + kk * 32, 16, 1024);
                        const uint64_t bd = smem_desc_sw128(b + kk * 16 * 128, B_CHUNK_F16, 1024);
                        mma_f16(d, ad, bd, id_f16, 1u);     // onto the dequantised fp32 values
                    }
                }
                mma_commit(&bars->empty[stage]);
                if (kind == 0 && blk == p.KB - 1) mma_commit(&bars->acc_int_full[buf]);
                if (kind == 1 && blk == nob - 1) mma_commit(&bars->acc_final_full[buf]);
            }
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            return true;
        });
        // Drain: every MMA this thread issued has completed before TMEM is freed.
        volatile int never = 0;
        mma_commit(&bars->drain);
        mbar_wait(&bars->drain, 0, &never, 0);
    } else if (warp >= 2) {
        // ------------------------------------------------------------ epilogue
        const int quad = warp & 3;                 // TMEM lanes 32*quad .. 32*quad+31
        const int row = quad * 32 + lane;
        uint8_t *mine = epi + (warp - 2) * EPI_WARP_BYTES;
        float *sw_s = reinterpret_cast<float *>(mine);
        uint8_t *stage_s = mine + EPI_SW_BYTES;
        int chunk_seq = 0;                         // staging block = chunk_seq & 1
        int it = 0;
        for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++it) {
            const int buf = it & 1;
            const uint32_t use = static_cast<uint32_t>(it >> 1) & 1u;
            const int m0 = (tile % p.num_m) * BM;
            const int n0 = (tile / p.num_m) * BN;
            const int t = m0 + row;
            const bool row_ok = t < p.T;
            // fetched while this tile's MMAs still run
            float rs = 0.0f;
            if (!kS32) {
                rs = row_ok ? p.sX[t] * (1.0f / 16129.0f) : 0.0f;
                const int nl = n0 + lane * 8;
                float4 s0 = make_float4(0.f, 0.f, 0.f, 0.f), s1 = s0;
                if (nl < p.N) {
                    s0 = __ldg(reinterpret_cast<const float4 *>(p.sW + nl));
                    s1 = __ldg(reinterpret_cast<const float4 *>(p.sW + nl + 4));
                }
                __syncwarp();                      // previous tile's readers are done
                reinterpret_cast<float4 *>(sw_s)[lane * 2] = s0;
                reinterpret_cast<float4 *>(sw_s)[lane * 2 + 1] = s1;
                __syncwarp();
            }
            if (!warp_wait(&bars->acc_int_full[buf], use, abort, I8R_DEV_TMEM_TIMEOUT)) break;
            tc_fence_after_sync();
            const uint32_t taddr = tmem + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(buf * BN);

            if (kS32) {
#pragma unroll 1
                for (int c = 0; c < BN / 32; ++c) {
                    const int nc = n0 + c * 32;
                    uint32_t r[32];
                    tmem_ld32(taddr + c * 32, r);
                    tmem_wait_ld();
                    if (row_ok) {
                        int4 *dst = reinterpret_cast<int4 *>(p.acc_out + static_cast<size_t>(t) * p.N + nc);
#pragma unroll
                        for (int g = 0; g < 8; ++g)
                            if (nc + g * 4 < p.N)
                                dst[g] = make_int4(static_cast<int>(r[4 * g]), static_cast<int>(r[4 * g + 1]),
                                                   static_cast<int>(r[4 * g + 2]), static_cast<int>(r[4 * g + 3]));
                    }
                }
            } else {
                if (nob) {
                    // pass 1: rewrite the int32 accumulator as fp32 acc * sX * sW / 127^2,
                    // then hand it back to the MMA warp for the 16-bit part
#pragma unroll 1
                    for (int c = 0; c < BN / 32; ++c) {
                        uint32_t r[32];
                        tmem_ld32(taddr + c * 32, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            r[i] = __float_as_uint(static_cast<float>(static_cast<int>(r[i])) * (rs * sw_s[c * 32 + i]));
                        tmem_st32(taddr + c * 32, r);
                    }
                    tmem_wait_st();
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->acc_conv[buf]);
                    if (!warp_wait(&bars->acc_final_full[buf], use, abort, I8R_DEV_TMEM_TIMEOUT)) break;
                    tc_fence_after_sync();
                }
                // pass 2 (or the only pass): fp16 Y through the staging blocks
#pragma unroll 1
                for (int c = 0; c < BN / 32; ++c) {
                    const int nc = n0 + c * 32;
                    uint32_t r[32];
                    tmem_ld32(taddr + c * 32, r);
                    tmem_wait_ld();
                    uint4 out[4];
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        __half2 h[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int i0 = g * 8 + 2 * e, i1 = i0 + 1;
                            float y0, y1;
                            if (nob) {
                                y0 = __uint_as_float(r[i0]);
                                y1 = __uint_as_float(r[i1]);
                            } else {
                                y0 = static_cast<float>(static_cast<int>(r[i0])) * (rs * sw_s[c * 32 + i0]);
                                y1 = static_cast<float>(static_cast<int>(r[i1])) * (rs * sw_s[c * 32 + i1]);
                            }
                            h[e] = __floats2half2_rn(y0, y1);
                        }
                        out[g] = *reinterpret_cast<uint4 *>(h);
                    }
                    // the staging block this chunk reuses must have been read out by its bulk store
                    uint8_t *blk = stage_s + (chunk_seq & 1) * EPI_STAGE_BYTES;
                    if (lane == 0) bulk_wait_group_read<1>();
                    __syncwarp();
                    // row `lane` of the 32 x 32 block; the 16-byte pieces are written in an
                    // order rotated by lane/2 so that no two lanes of a quarter-warp hit the
                    // same banks
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int g = (j + (lane >> 1)) & 3;
                        uint4 v = out[0];
                        if (g == 1) v = out[1];
                        if (g == 2) v = out[2];
                        if (g == 3) v = out[3];
                        *reinterpret_cast<uint4 *>(blk + lane * 64 + g * 16) = v;
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&map_y, blk, nc, m0 + quad * 32);
                        bulk_commit_group();
                    }
                    ++chunk_seq;
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->acc_empty[buf]);
        }
        if (!kS32 && lane == 0) bulk_wait_group_all();
        __syncwarp();
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();                                  // lane 0 issued the MMAs alone
        tc_fence_after_sync();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace prefill
}  // namespace i8r
