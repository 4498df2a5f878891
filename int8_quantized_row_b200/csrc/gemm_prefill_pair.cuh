// Prefill-shaped LLM.int8() GEMM on sm_100a tensor cores, CTA-pair version.
//
// A cluster of two CTAs (one per SM) computes 256 x 256 output tiles with
// cta_group::2 MMAs (M = 256, N = 256): CTA r holds rows 128r..128r+127 of the
// A tile and columns 128r..128r+127 of the B tile in its own shared memory,
// the tensor cores read both halves, and CTA r's TMEM receives its 128 rows.
// Each SM therefore loads half the weight bytes per MMA that a single-CTA
// 128 x 256 tile needs.  A stage holds 256 of K (64 KB per CTA, 3 stages), so
// the issuing thread sends 8 MMAs per stage: the tensor pipe keeps only a
// short queue of issued MMAs, and per-stage bookkeeping (barrier wait, commits,
// schedule) between bursts of 4 left it idle for a third of the time.
//
// Per tile (vector-wise scales + mixed-precision decomposition: LLM.int8()
// abstract; "The LLM.int8() Methodology"):
//   8-bit part:  acc = sum_k Xq[t,k] Wq[k,n], int32 in TMEM (kind::i8,
//                A = Xq K-major, B = Wq MN-major)
//   dequantise:  each CTA's epilogue rewrites its accumulator rows in place
//                as fp32 acc * sX[t] * sW[n] / 127^2 (tcgen05.ld/st)
//   16-bit part: kind::f16 MMAs over Xo and the W16 outlier rows accumulate
//                onto that value, issued kDefer k-blocks into the next tile
//   output:      fp16 Y in 32 x 32 blocks through shared memory, TMA stores
// The accumulator is double-buffered (2 x 256 TMEM columns per CTA).
//
// Synchronisation (the even CTA is the leader and issues every MMA):
//   full[s]        leader's, one arrival per use: the leader's, which declares
//                  the bytes of both CTAs' stage; both CTAs' TMA loads complete
//                  on it.  Every stage use goes through full[s], so its phase
//                  flips exactly once per trip round the ring.  (The peer's
//                  bytes need no arrival of their own, so the hot path has no
//                  cluster-scope fence.)  Outlier stages are all TMA as well:
//                  the W16 rows of the outlier columns arrive as one-row loads.
//   empty[s]       each CTA's own; the leader's MMA commit arrives on both
//   acc_int_full, acc_final_full  each CTA's own; committed to both
//   acc_conv, acc_empty           leader's, 8 arrivals (4 epilogue warps x 2)
// Every wait is bounded (timeout -> device status word, abort flag); both
// CTAs always reach the final cluster barrier.
#pragma once

#include "device_common.cuh"

namespace i8r {
namespace prefill2 {

constexpr int BM = 256;                    // rows per pair tile (128 per CTA)
constexpr int BN = 256;                    // columns per pair tile (B: 128 per CTA)
constexpr int BK = 256;                    // int8 K per stage (bytes)
constexpr int A_BOX_K = 128;               // K bytes per A load (128-byte swizzle span)
constexpr int OBK = 64;                    // fp16 outlier columns per outlier stage
constexpr int STAGES = 3;
constexpr int A_BYTES = 128 * BK;          // 32 KB: this CTA's 128 rows, two 16 KB K halves
constexpr int A_HALF_BYTES = 128 * A_BOX_K;
constexpr int B_BYTES = 128 * BK;          // 32 KB: this CTA's 128 columns
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int XO_BYTES = 128 * OBK * 2;    // 16 KB: an outlier stage's Xo rows
constexpr int B_CHUNK_F16 = 64 * OBK * 2;  // 64 columns x 64 outlier rows, fp16
constexpr int THREADS = 192;
constexpr int TMEM_COLS = 512;
constexpr int kDefer = 4;

constexpr int EPI_SW_BYTES = BN * 4;
constexpr int EPI_STAGE_BYTES = 32 * 32 * 2;
constexpr int EPI_WARP_BYTES = EPI_SW_BYTES + 2 * EPI_STAGE_BYTES;
constexpr int EPI_BYTES = 4 * EPI_WARP_BYTES;
constexpr size_t SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + 512;

struct Params {
    int T, K, N;
    int num_m, num_tiles, KB;      // tiles of 256 x 256
    const int32_t *count;
    const int32_t *idx;
    const float *sX;
    const float *sW;
    __half *Y;
    int32_t *acc_out;
    int o_rows;                    // outlier rows compacted into the W16o map (multiple of 64)
    int wq_only;                   // no W16 map: blocks past o_rows are dequantised from Wq by index
    const int8_t *Wq;              // [K,N] int8 (the Wq-only variant's rows past the compacted ones)
};

struct Barriers {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t acc_int_full[2];
    uint64_t acc_conv[2];
    uint64_t acc_final_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint64_t wq_ready[STAGES];     // leader's: both CTAs wrote their dequantised outlier rows (Wq-only)
    uint32_t tmem_base;
    int abort;
    int orow[OBK];                 // W16 row of each outlier of the stage being loaded
};
static_assert(sizeof(Barriers) <= 512, "barrier block outgrew its shared-memory reserve");

// Same stage order for the producer (both CTAs) and the MMA warp (leader).
template <typename Visit>
__device__ __forceinline__ bool walk_schedule(const Params &p, int nob, int cluster_id, int clusters, Visit &&visit) {
    const int defer = p.KB < kDefer ? p.KB : kDefer;
    int prev_tile = -1, prev_it = -1;
    int it = 0;
    for (int tile = cluster_id; tile < p.num_tiles; tile += clusters, ++it) {
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
    gemm_prefill_pair_kernel(const __grid_constant__ CUtensorMap map_xq, const __grid_constant__ CUtensorMap map_wq,
                             const __grid_constant__ CUtensorMap map_xo, const __grid_constant__ CUtensorMap map_w16,
                             const __grid_constant__ CUtensorMap map_w16x4, const __grid_constant__ CUtensorMap map_w16o,
                             const __grid_constant__ CUtensorMap map_y, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *epi = smem + STAGES * STAGE_BYTES;
    Barriers *bars = reinterpret_cast<Barriers *>(epi + EPI_BYTES);
    volatile int *abort = &bars->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();         // 0: leader, 1: peer
    const bool leader = rank == 0;
    const int cluster_id = blockIdx.x >> 1;
    const int clusters = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->acc_int_full[b], 1);
            mbar_init(&bars->acc_conv[b], 8);
            mbar_init(&bars->acc_final_full[b], 1);
            mbar_init(&bars->acc_empty[b], 8);
        }
        mbar_init(&bars->drain, 1);
        for (int s = 0; s < STAGES; ++s) mbar_init(&bars->wq_ready[s], 2);
        bars->abort = 0;
        fence_mbar_init();
        tma_prefetch_map(&map_xq);
        tma_prefetch_map(&map_wq);
        if (!kS32) {
            tma_prefetch_map(&map_xo);
            tma_prefetch_map(&map_w16);
            tma_prefetch_map(&map_w16x4);
            tma_prefetch_map(&map_w16o);
            tma_prefetch_map(&map_y);
        }
    }
    if (warp == 1) {
        tmem_alloc_pair(&bars->tmem_base, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before_sync();
    cluster_sync_all();                               // both CTAs' barriers exist from here on
    tc_fence_after_sync();
    const uint32_t tmem = bars->tmem_base;

    // shared::cluster addresses of the leader's barriers
    const uint32_t lead_full = mapa_shared(smem_u32(&bars->full[0]), 0);
    const uint32_t lead_acc_conv = mapa_shared(smem_u32(&bars->acc_conv[0]), 0);
    const uint32_t lead_acc_empty = mapa_shared(smem_u32(&bars->acc_empty[0]), 0);
    const uint32_t lead_wq_ready = mapa_shared(smem_u32(&bars->wq_ready[0]), 0);

    // Weight halves of this CTA's first stages do not depend on the activation
    // kernels: request them first.
    const int pre = p.KB < STAGES ? p.KB : STAGES;
    if (warp == 0 && lane == 0 && cluster_id < p.num_tiles) {
        const int n0 = (cluster_id / p.num_m) * BN + 128 * static_cast<int>(rank);
        for (int i = 0; i < pre; ++i) {
            if (leader) mbar_arrive_expect_tx(&bars->full[i], 2 * STAGE_BYTES);   // fresh barrier
            tma_load_2d_pair(smem + i * STAGE_BYTES + A_BYTES, &map_wq, lead_full + 8u * i, n0, i * BK);
        }
    }
    griddep_wait();
    const int count = (!kS32 && p.count) ? *p.count : 0;
    const int nob = (count + OBK - 1) / OBK;

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        int stage = 0;
        uint32_t phase = 0;
        int pending[STAGES];
#pragma unroll
        for (int s = 0; s < STAGES; ++s) pending[s] = -1;
        int issued = 0;
        const bool ok = walk_schedule(p, nob, cluster_id, clusters, [&](int kind, int tile, int, int blk) -> bool {
            const int m0 = (tile % p.num_m) * BM + 128 * static_cast<int>(rank);   // this CTA's rows
            const int n0 = (tile / p.num_m) * BN + 128 * static_cast<int>(rank);   // this CTA's columns
            uint8_t *a = smem + stage * STAGE_BYTES;
            if (kind == 0 && issued < pre) {
                if (lane == 0) {
                    tma_load_2d_pair(a, &map_xq, lead_full + 8u * stage, blk * BK, m0);
                    tma_load_2d_pair(a + A_HALF_BYTES, &map_xq, lead_full + 8u * stage, blk * BK + A_BOX_K, m0);
                }
            } else {
                if (!warp_wait(&bars->empty[stage], phase ^ 1u, abort, I8R_DEV_PIPELINE_TIMEOUT)) return false;
                if (kind == 0) {
                    if (lane == 0) {
                        if (leader) mbar_arrive_expect_tx(&bars->full[stage], 2 * STAGE_BYTES);
                        tma_load_2d_pair(a, &map_xq, lead_full + 8u * stage, blk * BK, m0);
                        tma_load_2d_pair(a + A_HALF_BYTES, &map_xq, lead_full + 8u * stage, blk * BK + A_BOX_K, m0);
                        tma_load_2d_pair(a + A_BYTES, &map_wq, lead_full + 8u * stage, n0, blk * BK);
                    }
                } else {
                    // The Xo tile, then this CTA's 128 columns (two 64-column
                    // pieces) of the W16 rows of outliers blk*64 .. .  Blocks
                    // inside the compacted rows (W16o, zero past |O|) are two
                    // 64 x 64 boxes.  Past them, the MMAs read round16(rows left)
                    // rows, in groups of four:
                    //   four outliers     one gather of the four rows
                    //   no outlier        a four-row box at row K: out of range,
                    //                     so the TMA writes zeros
                    //   some outliers     one-row loads, row K for the padding
                    // The lanes fetch the row indices together; one lane issues
                    // the loads (a TMA load takes its operands from uniform
                    // registers, so per-lane operands are issued a lane at a time,
                    // and each load has a fixed cost: the fewer, the better).
                    const int left = count - blk * OBK;
                    const bool compact = blk * OBK + OBK <= p.o_rows;
                    const int rows = compact ? OBK : min(OBK, (left + 15) / 16 * 16);
                    if (!compact && !p.wq_only)
                        for (int j = lane; j < rows; j += 32) bars->orow[j] = j < left ? p.idx[blk * OBK + j] : p.K;
                    __syncwarp();
                    if (!compact && p.wq_only) {
                        // Wq-only past the compacted rows: the Xo tile by TMA, and this
                        // CTA's 128 columns of the outlier rows dequantised from Wq by
                        // index, W~ = fp16_rn(q * fl32(sW/127)) as the quantiser's
                        // compaction does (zero past |O|), written with generic stores
                        // into the 128-byte-swizzled chunks a box load would fill: 16
                        // bytes per lane, two rows per pass.  Each CTA then arrives on
                        // the leader's wq_ready, which the MMA issuer also waits for.
                        if (lane == 0) {
                            if (leader) mbar_arrive_expect_tx(&bars->full[stage], 2u * static_cast<uint32_t>(XO_BYTES));
                            tma_load_2d_pair(a, &map_xo, lead_full + 8u * stage, blk * OBK, m0);
                        }
                        const int u16 = lane & 15;
                        const int col = n0 + 8 * u16;
                        const bool col_ok = col < p.N;
                        float dq[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) dq[e] = col_ok ? __fdiv_rn(p.sW[col + e], 127.0f) : 0.0f;
                        uint8_t *chunk = a + A_BYTES + (u16 >> 3) * B_CHUNK_F16;
                        const int unit = u16 & 7;
                        for (int r = lane >> 4; r < rows; r += 2) {
                            const int k = r < left ? p.idx[blk * OBK + r] : -1;
                            uint2 q8 = make_uint2(0u, 0u);
                            if (k >= 0 && col_ok)
                                q8 = __ldg(reinterpret_cast<const uint2 *>(p.Wq + static_cast<size_t>(k) * p.N + col));
                            __align__(16) __half v[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const int q = static_cast<int8_t>(((e < 4 ? q8.x : q8.y) >> (8 * (e & 3))) & 0xFFu);
                                v[e] = __float2half_rn(__fmul_rn(static_cast<float>(q), dq[e]));
                            }
                            *reinterpret_cast<uint4 *>(chunk + r * 128 + ((unit ^ (r & 7)) << 4)) =
                                *reinterpret_cast<const uint4 *>(v);
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster(lead_wq_ready + 8u * stage);
                    } else if (lane == 0 && compact) {
                        if (leader)
                            mbar_arrive_expect_tx(&bars->full[stage], 2u * static_cast<uint32_t>(XO_BYTES + OBK * 256));
                        const uint32_t fb = lead_full + 8u * stage;
                        tma_load_2d_pair(a, &map_xo, fb, blk * OBK, m0);
                        tma_load_2d_pair(a + A_BYTES, &map_w16o, fb, n0, blk * OBK);
                        tma_load_2d_pair(a + A_BYTES + B_CHUNK_F16, &map_w16o, fb, n0 + 64, blk * OBK);
                    } else if (lane == 0) {
                        if (leader)
                            mbar_arrive_expect_tx(&bars->full[stage], 2u * static_cast<uint32_t>(XO_BYTES + rows * 256));
                        const uint32_t fb = lead_full + 8u * stage;
                        tma_load_2d_pair(a, &map_xo, fb, blk * OBK, m0);
                        uint8_t *b = a + A_BYTES;
                        for (int j = 0; j < rows; j += 4) {
                            for (int c = 0; c < 2; ++c) {
                                uint8_t *dst = b + c * B_CHUNK_F16 + j * 128;
                                const int x = n0 + 64 * c;
                                if (j + 4 <= left) {
                                    tma_gather4_pair(dst, &map_w16, fb, x, bars->orow[j], bars->orow[j + 1],
                                                     bars->orow[j + 2], bars->orow[j + 3]);
                                } else if (j >= left) {
                                    tma_load_2d_pair(dst, &map_w16x4, fb, x, p.K);
                                } else {
                                    for (int e = 0; e < 4; ++e)
                                        tma_load_2d_pair(dst + e * 128, &map_w16, fb, x, bars->orow[j + e]);
                                }
                            }
                        }
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
        if (!ok && lane == 0 && leader) {
            // let loads already issued land before the CTAs leave (abort only)
            volatile int never = 0;
#pragma unroll
            for (int s = 0; s < STAGES; ++s)
                if (pending[s] >= 0) mbar_wait(&bars->full[s], static_cast<uint32_t>(pending[s]), &never, 0);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader)
        // One thread: anything between two MMA bursts (a warp-wide shuffle, a
        // reconvergence) delays the next burst and idles the tensor pipe.
        if (leader && lane == 0) {
            const uint32_t id_i8 = idesc_i8(BM, BN, false, true);
            const uint32_t id_f16 = idesc_f16(BM, BN, false, true);
            const uint32_t own_empty = smem_u32(&bars->empty[0]);
            const uint32_t peer_empty = mapa_shared(own_empty, 1);
            const uint32_t own_int = smem_u32(&bars->acc_int_full[0]);
            const uint32_t peer_int = mapa_shared(own_int, 1);
            const uint32_t own_final = smem_u32(&bars->acc_final_full[0]);
            const uint32_t peer_final = mapa_shared(own_final, 1);
            const uint32_t own_empty_c = mapa_shared(own_empty, 0);
            const uint32_t own_int_c = mapa_shared(own_int, 0);
            const uint32_t own_final_c = mapa_shared(own_final, 0);
            int stage = 0;
            uint32_t phase = 0;
            uint32_t wq_phase = 0;                       // bit s: parity of wq_ready[s]'s next phase
            walk_schedule(p, nob, cluster_id, clusters, [&](int kind, int, int it, int blk) -> bool {
                const int buf = it & 1;
                const uint32_t use = static_cast<uint32_t>(it >> 1) & 1u;
                const uint32_t d = tmem + static_cast<uint32_t>(buf * BN);
                if (kind == 0 && blk == 0) {
                    if (!mbar_wait_cluster(&bars->acc_empty[buf], use ^ 1u, abort, I8R_DEV_TMEM_TIMEOUT)) return false;
                    tc_fence_after_sync();
                }
                if (kind == 1 && blk == 0) {
                    if (!mbar_wait_cluster(&bars->acc_conv[buf], use, abort, I8R_DEV_TMEM_TIMEOUT)) return false;
                    tc_fence_after_sync();
                }
                if (!mbar_wait(&bars->full[stage], phase, abort, I8R_DEV_PIPELINE_TIMEOUT)) return false;
                if (kind == 1 && p.wq_only && blk * OBK + OBK > p.o_rows) {
                    // the dequantised rows both CTAs wrote with generic stores
                    if (!mbar_wait_cluster(&bars->wq_ready[stage], (wq_phase >> stage) & 1u, abort,
                                           I8R_DEV_PIPELINE_TIMEOUT))
                        return false;
                    wq_phase ^= 1u << stage;
                    fence_proxy_async_smem();
                }
                tc_fence_after_sync();
                {
                    const uint32_t a = smem_u32(smem + stage * STAGE_BYTES);
                    const uint32_t b = a + A_BYTES;
                    if (kind == 0) {
#pragma unroll
                        for (int kk = 0; kk < BK / 32; ++kk) {
                            const uint64_t ad = smem_desc_sw128(a + (kk >> 2) * A_HALF_BYTES + (kk & 3) * 32, 16, 1024);
                            const uint64_t bd = smem_desc_sw128(b + kk * 32 * 128, B_BYTES, 1024);
                            mma_i8_pair(d, ad, bd, id_i8, (blk | kk) != 0);
                        }
                    } else {
                        const int nk = min(OBK / 16, (count - blk * OBK + 15) / 16);
                        for (int kk = 0; kk < nk; ++kk) {
                            const uint64_t ad = smem_desc_sw128(a + kk * 32, 16, 1024);
                            const uint64_t bd = smem_desc_sw128(b + kk * 16 * 128, B_CHUNK_F16, 1024);
                            mma_f16_pair(d, ad, bd, id_f16, 1u);
                        }
                    }
                    mma_commit_pair(own_empty_c + 8u * stage);
                    mma_commit_pair(peer_empty + 8u * stage);
                    if (kind == 0 && blk == p.KB - 1) {
                        mma_commit_pair(own_int_c + 8u * buf);
                        mma_commit_pair(peer_int + 8u * buf);
                    }
                    if (kind == 1 && blk == nob - 1) {
                        mma_commit_pair(own_final_c + 8u * buf);
                        mma_commit_pair(peer_final + 8u * buf);
                    }
                }
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                return true;
            });
            volatile int never = 0;
            mma_commit_pair(mapa_shared(smem_u32(&bars->drain), 0));
            mbar_wait(&bars->drain, 0, &never, 0);
        }
    } else if (warp >= 2) {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        uint8_t *mine = epi + (warp - 2) * EPI_WARP_BYTES;
        float *sw_s = reinterpret_cast<float *>(mine);
        uint8_t *stage_s = mine + EPI_SW_BYTES;
        int chunk_seq = 0;
        int it = 0;
        for (int tile = cluster_id; tile < p.num_tiles; tile += clusters, ++it) {
            const int buf = it & 1;
            const uint32_t use = static_cast<uint32_t>(it >> 1) & 1u;
            const int m0 = (tile % p.num_m) * BM + 128 * static_cast<int>(rank);
            const int n0 = (tile / p.num_m) * BN;
            const int t = m0 + row;
            const bool row_ok = t < p.T;
            float rs = 0.0f;
            if (!kS32) {
                rs = row_ok ? p.sX[t] * (1.0f / 16129.0f) : 0.0f;
                const int nl = n0 + lane * 8;
                float4 s0 = make_float4(0.f, 0.f, 0.f, 0.f), s1 = s0;
                if (nl < p.N) {
                    s0 = __ldg(reinterpret_cast<const float4 *>(p.sW + nl));
                    s1 = __ldg(reinterpret_cast<const float4 *>(p.sW + nl + 4));
                }
                __syncwarp();
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
                    if (lane == 0) mbar_arrive_cluster(lead_acc_conv + 8u * buf);
                    if (!warp_wait(&bars->acc_final_full[buf], use, abort, I8R_DEV_TMEM_TIMEOUT)) break;
                    tc_fence_after_sync();
                }
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
                    uint8_t *blk = stage_s + (chunk_seq & 1) * EPI_STAGE_BYTES;
                    if (lane == 0) bulk_wait_group_read<1>();
                    __syncwarp();
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
            if (lane == 0) mbar_arrive_cluster(lead_acc_empty + 8u * buf);
        }
        if (!kS32 && lane == 0) bulk_wait_group_all();
        __syncwarp();
    }

    // Neither CTA leaves while the other may still touch its shared memory or
    // TMEM (remote arrivals, the leader's MMAs reading the peer's tiles).
    tc_fence_before_sync();
    __syncthreads();
    cluster_sync_all();
    if (warp == 1) {
        __syncwarp();                                  // lane 0 issued the MMAs alone
        tc_fence_after_sync();
        tmem_dealloc_pair(tmem, TMEM_COLS);
    }
}

}  // namespace prefill2
}  // namespace i8r
