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
// tile in TMEM (up to four buffers, so the MMAs run ahead of the epilogue) and
// adds the exact int32 partial sums into acc32 [T,N] (zeroed beforehand) with
// bulk tensor reduce-adds from shared memory, done in L2.
//
// The 16-bit outlier part (LLM.int8() abstract: the outlier feature
// dimensions go through a 16-bit matrix multiplication) runs on the same
// tensor cores: the CTA that owns k-block 0 of a tile also runs an outlier
// segment for it, ceil(|O|/64) stages of kind::f16 MMAs
//   Yo[t,n] = sum_j Xo[t,j] * W16[O_j,n]      (fp32 in TMEM)
// with A = the W16 rows of the outliers (MN-major) and B = Xo (K-major), and
// stores it to Yo [T,N] with bulk tensor stores.  The rows of the first
// o_rows outliers come compacted by the activation side (W16o: W16 rows, or
// the Wq-only variant's dequantised rows) and load as four 64 x 64 boxes; any
// further rows are copied in place by the lanes with cp.async, 16 bytes
// each.  Those stages go through the same ring as the weight stages, filled
// by the same (only) producer warp: a parity wait cannot tell a phase from
// the one two uses later, so every slot has one producer that waits on each
// of its uses.  The row copies do not stall that warp: each lane hands its
// cp.async copies to the stage's barrier (cp.async.mbarrier.arrive), so
// several outlier stages can be in flight at once.
//
// Y is written by decode_finalize_kernel, a programmatic dependent of this
// kernel, over the whole grid:
//   Y[t,n] = fp16( acc32[t,n] * sX[t] * sW[n] / 127^2 + Yo[t,n] )
// so no CTA waits on another at the end of its range.
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
constexpr int OBK = 64;            // outliers per outlier stage: 64 W16 rows x 256 columns = A_BYTES,
                                   // and T x 64 fp16 of Xo = the bytes of a T x 128 Xq tile
constexpr int O_CHUNK = 64 * OBK * 2;   // 64 columns x 64 W16 rows (one 128-byte swizzle span)
constexpr int THREADS = 192;       // warp 0 producer, 1 MMA, 2-5 epilogue
constexpr int MAX_T = 128;
constexpr int MAX_STAGES = 8;
constexpr int MAX_BUF = 4;         // TMEM accumulator buffers: the MMA runs up to three segments
                                   // ahead of a finalising epilogue
static_assert(4 * O_CHUNK == A_BYTES, "an outlier stage's W16 rows fill the weight slot");
// Every piece of a tile hands its int32 partial sums to acc32 as bulk tensor
// reduce-adds (done in L2) and decode_finalize_kernel writes Y afterwards:
// no CTA waits on another at the end (measured faster than finalising in the
// tile's last piece at every batch size).
constexpr int RED_ROWS = 32;                       // rows per bulk reduce (a 32 x 32 int32 box, 4 KB)
constexpr int RED_BYTES = RED_ROWS * 32 * 4;
constexpr int RED_SMEM = 4 * 2 * RED_BYTES;        // two staging boxes per epilogue warp
constexpr size_t SMEM_MAX = 227 * 1024;

struct Params {
    int T, TP, K, N;
    int KB, num_tiles;
    long long total_units;
    int stages, stage_bytes;
    uint32_t tmem_cols;            // nbuf * buf_cols (a power of two, <= 512)
    uint32_t buf_cols;             // columns of one accumulator buffer: a power of two >= 2*TP, >= 32
    int nbuf;                      // accumulator buffers (2 or 4), used in turn by the segments
    int32_t *acc32;                // [T,N] int32, zero on entry
    // the layer (finalize != 0): the outlier segments, and Y by decode_finalize_kernel
    int finalize;
    const float *sX, *sW;
    const int32_t *count;          // |O|
    const int32_t *idx;            // the outlier columns, ascending
    const __half *W16;             // [K,N] fp16 (null for the Wq-only variant)
    const int8_t *Wq;              // [K,N] int8 (the Wq-only variant's rows past the compacted ones)
    int o_rows;                    // rows of the compacted outlier rows W16o (W16 rows, or dequantised Wq rows)
    int wq_only;                   // no W16: outlier rows from W16o, dequantised from Wq past o_rows
    int may_outlier;               // alpha < +inf: a tile's first stage may be an outlier stage
    __half *Y;
    float *Yo;                     // [T,N] fp32: the 16-bit outlier part (written when |O| > 0)
};

struct Barriers {
    uint64_t full[MAX_STAGES];
    uint64_t empty[MAX_STAGES];
    uint64_t tmem_full[MAX_BUF];
    uint64_t tmem_empty[MAX_BUF];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

// The ring (stages x stage_bytes; an outlier stage, 64 W16 rows of a tile and
// T x 64 fp16 of Xo, has the size of a weight stage), then the barriers, then
// (bulk mode) the epilogue warps' reduce staging boxes; 1024 bytes for aligning
// the base to the 128-byte swizzle's 1024-byte period.
__host__ __device__ inline size_t staging_offset(int stages, int stage_bytes) {      // from the aligned base
    return static_cast<size_t>(stages) * stage_bytes + (sizeof(Barriers) + 127) / 128 * 128;
}
__host__ __device__ inline size_t smem_bytes(int stages, int stage_bytes) {
    return 1024 + staging_offset(stages, stage_bytes) + RED_SMEM;
}

// CTA c of `ctas` owns units [floor(c*U/ctas), floor((c+1)*U/ctas)).
__device__ __forceinline__ long long unit_begin(long long total, int c, int ctas) {
    return total * c / ctas;
}
// The CTA whose range holds unit u.
__device__ __forceinline__ int unit_owner(long long total, long long u, int ctas) {
    return static_cast<int>(((u + 1) * ctas - 1) / total);
}

// The stages of one CTA in order, the same for all its warps: for each tile
// its range [u0, u1) touches, first (if the range holds the tile's k-block 0)
// the tile's nob outlier blocks (kind 1, j = outlier block), then the int8
// k-blocks of that tile in the range (kind 0, j = k-block).  The CTA holding a
// tile's k-block 0 reaches that tile last, so its int8 piece is usually the
// tile's last one, and its outlier piece is stored just before.
// A run of one kind for one tile is a segment: one TMEM accumulator buffer.
// visit(kind, tile, j, first_of_segment, last_of_segment) returns false to stop.
template <typename Visit>
__device__ __forceinline__ bool walk_stages(const Params &p, long long u0, long long u1, int nob, Visit &&visit) {
    for (long long u = u0; u < u1;) {
        const int tile = static_cast<int>(u / p.KB);
        const long long tile_u0 = static_cast<long long>(tile) * p.KB;
        const long long end = min(u1, tile_u0 + p.KB);
        if (u == tile_u0)
            for (int b = 0; b < nob; ++b)
                if (!visit(1, tile, b, b == 0, b == nob - 1)) return false;
        for (long long v = u; v < end; ++v)
            if (!visit(0, tile, static_cast<int>(v - tile_u0), v == u, v == end - 1)) return false;
        u = end;
    }
    return true;
}

// Y from the reduced int32 sums: one thread per 8 columns of a row,
//   Y[t,n] = fp16( acc32[t,n] * (sX[t] / 127^2) * sW[n] + Yo[t,n] )
// (one fp32 fma after the scale product); a programmatic dependent of the GEMM.
__global__ void __launch_bounds__(256) decode_finalize_kernel(const int32_t *__restrict__ acc32,
                                                              const float *__restrict__ Yo,
                                                              const int32_t *__restrict__ count,
                                                              const float *__restrict__ sX, const float *__restrict__ sW,
                                                              int T, int N, __half *__restrict__ Y) {
    griddep_wait();
    const int groups = N / 8;
    const long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (g >= static_cast<long long>(T) * groups) return;
    const int t = static_cast<int>(g / groups), n = static_cast<int>(g % groups) * 8;
    const bool yo = Yo && *count > 0;
    const size_t at = static_cast<size_t>(t) * N + n;
    const int4 a0 = __ldcg(reinterpret_cast<const int4 *>(acc32 + at));
    const int4 a1 = __ldcg(reinterpret_cast<const int4 *>(acc32 + at + 4));
    const float4 w0 = __ldg(reinterpret_cast<const float4 *>(sW + n));
    const float4 w1 = __ldg(reinterpret_cast<const float4 *>(sW + n + 4));
    float4 o0 = make_float4(0.f, 0.f, 0.f, 0.f), o1 = o0;
    if (yo) {
        o0 = __ldcg(reinterpret_cast<const float4 *>(Yo + at));
        o1 = __ldcg(reinterpret_cast<const float4 *>(Yo + at + 4));
    }
    const float rs = sX[t] * (1.0f / 16129.0f);
    const int av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    const float ov[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
    __align__(16) __half y[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] = __float2half_rn(fmaf(static_cast<float>(av[e]), rs * wv[e], ov[e]));
    *reinterpret_cast<uint4 *>(Y + at) = *reinterpret_cast<const uint4 *>(y);
}

__global__ void __launch_bounds__(THREADS, 1)
    gemm_decode_kernel(const __grid_constant__ CUtensorMap map_wq, const __grid_constant__ CUtensorMap map_xq,
                       const __grid_constant__ CUtensorMap map_xo, const __grid_constant__ CUtensorMap map_w16o,
                       const __grid_constant__ CUtensorMap map_acc, const __grid_constant__ CUtensorMap map_yo,
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
        for (int b = 0; b < MAX_BUF; ++b) {
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
    const uint32_t buf_cols = p.buf_cols;

    const long long u0 = unit_begin(p.total_units, blockIdx.x, gridDim.x);
    const long long u1 = unit_begin(p.total_units, blockIdx.x + 1, gridDim.x);
    const uint32_t tx = static_cast<uint32_t>(p.stage_bytes);

    // Weight tiles of the first stages do not depend on the activation kernels:
    // request them first.  Only the first segment's, and none when the range
    // starts a tile that may open with outlier stages (|O| is not known yet).
    const long long first_seg = min(u1, (u0 / p.KB + 1) * p.KB) - u0;
    const int pre = (p.may_outlier && u0 % p.KB == 0) ? 0 : static_cast<int>(min(static_cast<long long>(p.stages), first_seg));
    if (warp == 0 && lane == 0) {
        for (int i = 0; i < pre; ++i) {
            const long long u = u0 + i;
            const int tile = static_cast<int>(u / p.KB);
            const int kb = static_cast<int>(u - static_cast<long long>(tile) * p.KB);
            uint8_t *a = smem + static_cast<size_t>(i) * p.stage_bytes;
            mbar_arrive_expect_tx(&bars->full[i], tx);   // fresh barrier: the slot is free
            tma_load_2d(a, &map_wq, &bars->full[i], tile * BM, kb * BK);
            tma_load_2d(a + A_HALF, &map_wq, &bars->full[i], tile * BM + BMH, kb * BK);
        }
    }
    griddep_wait();                               // activation, |O|, acc32 zeroed
    const int count = p.finalize ? *p.count : 0;
    const int nob = p.may_outlier ? (count + OBK - 1) / OBK : 0;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (nob > 0 && lane == 0) {
            if (p.o_rows > 0) tma_prefetch_map(&map_w16o);
            tma_prefetch_map(&map_xo);
        }
        int pending[MAX_STAGES];
        for (int s = 0; s < MAX_STAGES; ++s) pending[s] = -1;
        int stage = 0, n = 0;
        uint32_t phase = 0;
        const bool ok = walk_stages(p, u0, u1, nob, [&](int kind, int tile, int j, bool, bool) -> bool {
            uint8_t *a = smem + static_cast<size_t>(stage) * p.stage_bytes;
            uint64_t *fb = &bars->full[stage];
            if (kind == 0 && n < pre) {
                if (lane == 0) tma_load_2d(a + A_BYTES, &map_xq, fb, j * BK, 0);
            } else {
                if (!warp_wait(&bars->empty[stage], phase ^ 1u, abort, I8R_DEV_PIPELINE_TIMEOUT)) return false;
                if (kind == 0) {
                    if (lane == 0) {
                        mbar_arrive_expect_tx(fb, tx);
                        tma_load_2d(a, &map_wq, fb, tile * BM, j * BK);
                        tma_load_2d(a + A_HALF, &map_wq, fb, tile * BM + BMH, j * BK);
                        tma_load_2d(a + A_BYTES, &map_xq, fb, j * BK, 0);
                    }
                } else if ((j + 1) * OBK <= p.o_rows) {
                    // compacted rows (W16 rows, or dequantised Wq rows): four 64 x 64 boxes
                    if (lane == 0) {
                        mbar_arrive_expect_tx(fb, tx);
                        tma_load_2d(a + A_BYTES, &map_xo, fb, j * OBK, 0);
                        for (int c = 0; c < 4; ++c)
                            tma_load_2d(a + c * O_CHUNK, &map_w16o, fb, tile * BM + 64 * c, j * OBK);
                    }
                } else if (p.wq_only) {
                    // Wq-only variant past the compacted rows: the lanes dequantise the
                    // Wq rows of outliers j*64 .. by index, W~ = fp16_rn(q * fl32(sW/127))
                    // as the quantiser's compaction does, zero past |O| rounded up to 16;
                    // lane l writes columns 8l .. 8l+7 of every row into the
                    // 128-byte-swizzled chunk l/8.  Generic stores: fenced to the async
                    // proxy before the arrive (the MMA warp fences again before reading).
                    const int rows = min(OBK, (count - j * OBK + 15) / 16 * 16);
                    const int g0 = j * OBK + lane, g1 = j * OBK + 32 + lane;
                    const int k0 = g0 < count ? p.idx[g0] : -1;
                    const int k1 = g1 < count ? p.idx[g1] : -1;
                    const int col = tile * BM + lane * 8;
                    const bool col_ok = col < p.N;
                    float d[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) d[e] = col_ok ? __fdiv_rn(p.sW[col + e], 127.0f) : 0.0f;
                    uint8_t *chunk = a + (lane >> 3) * O_CHUNK;
                    const int unit = lane & 7;
                    for (int r = 0; r < rows; ++r) {
                        const int k = __shfl_sync(0xFFFFFFFFu, r < 32 ? k0 : k1, r & 31);
                        uint2 q8 = make_uint2(0u, 0u);
                        if (k >= 0 && col_ok) q8 = __ldg(reinterpret_cast<const uint2 *>(p.Wq + static_cast<size_t>(k) * p.N + col));
                        __align__(16) __half v[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int q = static_cast<int8_t>(((e < 4 ? q8.x : q8.y) >> (8 * (e & 3))) & 0xFFu);
                            v[e] = __float2half_rn(__fmul_rn(static_cast<float>(q), d[e]));
                        }
                        *reinterpret_cast<uint4 *>(chunk + r * 128 + ((unit ^ (r & 7)) << 4)) =
                            *reinterpret_cast<const uint4 *>(v);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive_expect_tx(fb, static_cast<uint32_t>(p.TP * OBK * 2));
                        tma_load_2d(a + A_BYTES, &map_xo, fb, j * OBK, 0);
                    }
                } else {
                    // The W16 rows of outliers j*64 .., zero past |O| rounded up to 16
                    // (the MMAs read no further): lane l copies columns 8l .. 8l+7 of
                    // every row into the 128-byte-swizzled chunk l/8 and hands the
                    // copies to the stage's barrier; lane 0 then adds the Xo tile.
                    // (The MMA warp fences to the async proxy before reading.)
                    const int rows = min(OBK, (count - j * OBK + 15) / 16 * 16);
                    const int g0 = j * OBK + lane, g1 = j * OBK + 32 + lane;
                    const int k0 = g0 < count ? p.idx[g0] : -1;
                    const int k1 = g1 < count ? p.idx[g1] : -1;
                    const int col = tile * BM + lane * 8;
                    const uint32_t chunk = smem_u32(a) + static_cast<uint32_t>((lane >> 3) * O_CHUNK);
                    const uint32_t unit = static_cast<uint32_t>(lane & 7);
                    for (int r = 0; r < rows; ++r) {
                        const int k = __shfl_sync(0xFFFFFFFFu, r < 32 ? k0 : k1, r & 31);
                        const bool have = k >= 0 && col < p.N;
                        const __half *src = have ? p.W16 + static_cast<size_t>(k) * p.N + col : p.W16;
                        cp_async_16(chunk + static_cast<uint32_t>(r * 128) + ((unit ^ static_cast<uint32_t>(r & 7)) << 4),
                                    src, have ? 16u : 0u);
                    }
                    cp_async_mbar_arrive(fb);
                    __syncwarp();                          // every lane's copies tracked before the arrive
                    if (lane == 0) {
                        mbar_arrive_expect_tx(fb, static_cast<uint32_t>(p.TP * OBK * 2));
                        tma_load_2d(a + A_BYTES, &map_xo, fb, j * OBK, 0);
                    }
                }
            }
            if (lane == 0) pending[stage] = static_cast<int>(phase);
            if (kind == 0) ++n;
            __syncwarp();
            if (++stage == p.stages) { stage = 0; phase ^= 1u; }
            return true;
        });
        if (!ok && lane == 0) {
            // let the loads and copies already issued land before the CTA leaves (abort only)
            volatile int never = 0;
            for (int s = 0; s < p.stages; ++s)
                if (pending[s] >= 0) mbar_wait(&bars->full[s], static_cast<uint32_t>(pending[s]), &never, 0);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t id_i8 = idesc_i8(BMH, p.TP, true, false);
        const uint32_t id_f16 = idesc_f16(BMH, p.TP, true, false);
        int stage = 0, seg = 0;
        uint32_t phase = 0;
        uint32_t tph = 0;                                 // bit b: phase of buffer b
        walk_stages(p, u0, u1, nob, [&](int kind, int, int j, bool first, bool last) -> bool {
            const int buf = seg % p.nbuf;
            if (first) {
                if (!warp_wait(&bars->tmem_empty[buf], ((tph >> buf) & 1u) ^ 1u, abort, I8R_DEV_TMEM_TIMEOUT)) return false;
                tc_fence_after_sync();
            }
            if (!warp_wait(&bars->full[stage], phase, abort, I8R_DEV_PIPELINE_TIMEOUT)) return false;
            tc_fence_after_sync();
            if (kind == 1) fence_proxy_async_smem();      // cp.async rows -> tensor core reads
            if (lane == 0) {
                const uint32_t d0 = tmem + static_cast<uint32_t>(buf) * buf_cols;
                const uint32_t d1 = d0 + static_cast<uint32_t>(p.TP);
                const uint32_t a = smem_u32(smem + static_cast<size_t>(stage) * p.stage_bytes);
                const uint32_t b = a + A_BYTES;
                if (kind == 0) {
#pragma unroll
                    for (int kk = 0; kk < BK / 32; ++kk) {
                        const uint32_t acc = (!first || kk != 0) ? 1u : 0u;
                        const uint64_t bd = smem_desc_sw128(b + kk * 32, 16, 1024);
                        mma_i8(d0, smem_desc_sw128(a + kk * 32 * 128, A_HALF, 1024), bd, id_i8, acc);
                        mma_i8(d1, smem_desc_sw128(a + A_HALF + kk * 32 * 128, A_HALF, 1024), bd, id_i8, acc);
                    }
                } else {
                    // 16 outliers per MMA: A = 16 W16 rows (2 KB of each 64-column
                    // chunk), B = 16 fp16 of each Xo row (32 bytes)
                    const int nk = min(OBK / 16, (count - j * OBK + 15) / 16);
                    for (int kk = 0; kk < nk; ++kk) {
                        const uint32_t acc = (!first || kk != 0) ? 1u : 0u;
                        const uint64_t bd = smem_desc_sw128(b + kk * 32, 16, 1024);
                        mma_f16(d0, smem_desc_sw128(a + kk * 16 * 128, O_CHUNK, 1024), bd, id_f16, acc);
                        mma_f16(d1, smem_desc_sw128(a + A_HALF + kk * 16 * 128, O_CHUNK, 1024), bd, id_f16, acc);
                    }
                }
                mma_commit(&bars->empty[stage]);
                if (last) mma_commit(&bars->tmem_full[buf]);
            }
            __syncwarp();
            if (last) {
                tph ^= 1u << buf;
                ++seg;
            }
            if (++stage == p.stages) { stage = 0; phase ^= 1u; }
            return true;
        });
        if (lane == 0) {
            volatile int never = 0;
            mma_commit(&bars->drain);
            mbar_wait(&bars->drain, 0, &never, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int quad = warp & 3;
        uint32_t tph = 0;
        int seg = 0;
        int red_n = 0;                                    // bulk reduces issued by this warp
        walk_stages(p, u0, u1, nob, [&](int kind, int tile, int, bool, bool last) -> bool {
            if (!last) return true;
            const int buf = seg % p.nbuf;
            if (!warp_wait(&bars->tmem_full[buf], (tph >> buf) & 1u, abort, I8R_DEV_TMEM_TIMEOUT)) return false;
            tc_fence_after_sync();
            const uint32_t taddr = tmem + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(buf) * buf_cols;
            // This piece's int32 sums go into acc32 (32 x 32 boxes staged in shared
            // memory, added in L2 by bulk tensor reduce-adds; exact and order-free),
            // or the tile's outlier part into Yo (the same boxes, bulk tensor
            // stores).  Box rows past T are not written by the bulk operations,
            // and tensor-memory rows past TP are not read.
            uint8_t *stg = smem + staging_offset(p.stages, p.stage_bytes) + static_cast<size_t>(quad) * 2 * RED_BYTES;
            for (int h = 0; h < 2; ++h) {
                const int n0 = tile * BM + h * BMH + quad * 32;
                for (int t0 = 0; t0 < p.T; t0 += RED_ROWS) {
                    int32_t *box = reinterpret_cast<int32_t *>(stg + (red_n & 1) * RED_BYTES);
                    if (red_n >= 2) {
                        if (lane == 0) bulk_wait_group_read<1>();   // the box written two bulk ops ago is free
                        __syncwarp();
                    }
                    uint32_t r0[16], r1[16];
                    const bool second = t0 + 16 < p.TP;
                    tmem_ld16(taddr + h * p.TP + t0, r0);
                    if (second) tmem_ld16(taddr + h * p.TP + t0 + 16, r1);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) box[i * 32 + lane] = static_cast<int32_t>(r0[i]);
                    if (second) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) box[(i + 16) * 32 + lane] = static_cast<int32_t>(r1[i]);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        if (kind == 0)
                            tma_reduce_add_2d(&map_acc, box, n0, t0);
                        else
                            tma_store_2d(&map_yo, box, n0, t0);
                        bulk_commit_group();
                    }
                    ++red_n;
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->tmem_empty[buf]);
            tph ^= 1u << buf;
            ++seg;
            return true;
        });
        if (lane == 0 && red_n > 0) bulk_wait_group_all();     // every reduce has landed in acc32
        __syncwarp();
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
