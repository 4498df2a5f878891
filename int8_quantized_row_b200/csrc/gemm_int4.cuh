// Group-wise 4-bit weight codec and its decode-shaped product (the FlexGen
// summary page: weights compressed to 4 bits group-wise, with no retraining
// or calibration).  The page gives no formula; the readings taken are those of
// the header's int4_* entry points:
//   a group is 64 consecutive rows k of one output column n; its 16 levels are
//   lo + q*s, q in 0..15, lo the group's minimum and s = half(fl32(fl32(hi-lo)/15));
//   q = clamp(rhaz(fl32(fl32(w - lo) * fl32(1/s))), 0, 15);
//   the decoded weight is half_rn(q*s + lo) (one fused multiply-add in fp16);
//   Y = half( sum_k X[t,k] * W~[k,n] ) with fp32 accumulation.
//
// Packed layout (int4_quantize_weight_groupwise writes it, everything here
// reads it).  Columns are padded to NP = 256*ceil(N/256); KT = K/256.
//   W4: blocks of 256 columns x 256 rows of K, 32 KB each, block (nt, kt) at
//       byte (nt*KT + kt) * 32768; column r of the block (n = 256*nt + r) has
//       128 bytes at r*128 holding codes k = 256*kt + 0..255 as eight 16-byte
//       chunks, chunk c (codes 32c .. 32c+31) stored at chunk position
//       c ^ (r & 7); in a chunk, 32-bit word i holds codes 8i .. 8i+7 with
//       nibble j (bits 4j..4j+3) = code 8i+2j and nibble j+4 = code 8i+2j+1
//       for j < 4.
//   S4: blocks of 256 columns x 4 groups, 4 KB each, block (nt, kt) at byte
//       (nt*KT + kt) * 4096; column r has 16 bytes at r*16: four (s, lo) fp16
//       pairs for groups 4*kt .. 4*kt+3.
// One block of each is what a pipeline stage of the product consumes, so a
// stage is two contiguous bulk copies (32 KB + 4 KB) that stream through DRAM
// in order, and the chunk order is the 128-byte swizzle that keeps the
// decoding threads' shared-memory reads free of bank conflicts.  The nibble
// order turns one shift and one mask into two fp16 codes: (w >> 4j) & 0x000F000F
// puts codes 8i+2j and 8i+2j+1 in the low and high halves of a 32-bit word.
//
// The product (gemm_int4_decode_kernel), for T <= 64 rows of X:
//   swap-AB: the MMA's M = 128 columns of W, its N = T rounded up to 16, so the
//   weight fills the tensor core's 128 rows; a tile is 256 columns (two MMAs
//   share the X tile).  Split over K stream-K style, as the int8 decode GEMM.
//   A stage is 256 of K: the packed codes and scales of the tile (36 KB) and
//   the X tile (T x 256 fp16, TMA), filled by one producer warp.  Eight
//   decoder warps turn the codes into fp16 and store them with tcgen05.st into
//   tensor memory, 128 of K at a time, into a ring of three (two for T > 32)
//   A sub-buffers; two MMA warps, one per 128-column half, issue tcgen05.mma
//   kind::f16 with A read from tensor memory and B (X) from shared memory,
//   fp32 accumulators in tensor memory (two buffers).
//   What bounds it: each kind::f16 MMA of M = 128, K = 16 occupies the tensor
//   pipe for about as long at N = 16 as at N = 64 (measured: the issuing warp
//   spends about 80 cycles per MMA), so with the weight on the M axis the
//   pipe takes at most about 128*16 weights per 80 cycles per SM, near 0.6 of
//   the rate at which HBM delivers 4-bit codes; the int8 product (K = 32 per
//   MMA, one byte per weight) is not bound this way.  Four epilogue
//   warps write Y for tiles a CTA holds whole; for a tile split over CTAs each
//   piece stores its fp32 partial sums in the CTA's slot and the last piece to
//   finish adds every piece's sums in CTA order (the same order whichever
//   finishes last, so the result is deterministic) and writes Y.
#pragma once

#include "device_common.cuh"

namespace i8r {
namespace w4 {

constexpr int G = 64;                       // rows of K per group
constexpr int BN = 256;                     // columns per tile
constexpr int BMH = 128;                    // columns per MMA (MMA M)
constexpr int BK = 256;                     // K per stage
constexpr int CODE_BYTES = BN * BK / 2;     // 32 KB of packed codes per stage
constexpr int SCALE_BYTES = BN * 16;        // 4 KB: four (s, lo) pairs per column
constexpr int MAX_T = 64;
constexpr int MAX_CTAS = 256;               // partial-sum slots are sized for up to this many CTAs
constexpr int COUNTERS_PER_TILE = 8;        // split-tile counters: the tensor kernel uses 4 (one per quadrant),
                                            // the CUDA-core kernel 8 (one per 32-column group)
constexpr int MAX_STAGES = 6;
constexpr int SUB = 2;                      // tensor-memory hand-offs of A per stage
constexpr int KSUB = BK / SUB;              // K per hand-off
constexpr int DECODERS = 8;                 // decoder warps 3..10: 4 lane quadrants x 2 column halves x PARTS
constexpr int PARTS = DECODERS / 8;         // decoder warps sharing one column's chunks of a hand-off
constexpr int CPW = KSUB / 32 / PARTS;      // 32-code chunks per decoder warp per hand-off
constexpr int ISSUERS = 2;                  // MMA-issuing warps 1 and 2, one per column half
constexpr int FIRST_DEC = 1 + ISSUERS;      // first decoder warp
constexpr int THREADS = 32 * (1 + ISSUERS + DECODERS + 4);
static_assert(ISSUERS == 1 || ISSUERS == 2, "one or two MMA-issuing warps");
static_assert(SUB * KSUB == BK && KSUB % 64 == 0 && DECODERS % 8 == 0 && CPW >= 1, "hand-off split");
constexpr size_t SMEM_BUDGET = 200 * 1024;
constexpr int MAX_NA = 3;                   // A sub-buffers in tensor memory (a ring over the hand-offs)
constexpr uint32_t TMEM_COLS = 512;         // A: NA x KSUB columns (KSUB/2 per column half);
                                            // D: 2 buffers x 2 halves x TP; NA = 3 for TP <= 32, else 2

__host__ __device__ inline int padded_n(int N) { return (N + BN - 1) / BN * BN; }
__host__ __device__ inline size_t code_bytes(int K, int N) { return static_cast<size_t>(padded_n(N)) * K / 2; }
__host__ __device__ inline size_t scale_bytes(int K, int N) { return static_cast<size_t>(padded_n(N)) * (K / G) * 4; }

struct Params {
    int T, TP, K, N;
    int KB, num_tiles;                      // stages per tile, tiles of 256 columns
    long long total_units;
    int stages, stage_bytes;
    int na;                                 // A sub-buffers (2 or 3)
    const uint8_t *W4;
    const uint8_t *S4;
    __half *Y;
    float *part;                            // [MAX_CTAS][2][TP][256] fp32 partial sums
    int *counters;                          // [num_tiles * 4], zero on entry
};

struct Barriers {
    uint64_t full[MAX_STAGES];
    uint64_t empty[MAX_STAGES];
    uint64_t a_full[MAX_NA];
    uint64_t a_empty[MAX_NA];
    uint64_t tmem_full[2];
    uint64_t tmem_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

__host__ __device__ inline size_t smem_bytes(int stages, int stage_bytes) {
    return 1024 + static_cast<size_t>(stages) * stage_bytes + sizeof(Barriers);
}

// ------------------------------------------------------------------ codec

__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<const __half2 *>(&u); }
__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<const uint32_t *>(&h); }

// The four decoded fp16 pairs of one 32-bit word of codes (pair j = codes 2j and
// 2j+1, i.e. nibbles j and j+4): half_rn(q*s + lo), one fp16x2 fused
// multiply-add each.  The codes become exact fp16 integers first: masking
// nibbles 0 and 4 (1 and 5) into the mantissa under the exponent of 1024 gives
// 1024 + q (1024 + 16q), and 1024 + q - 1024, (1024 + 16q)/16 - 64 are exact.
__device__ __forceinline__ void decode_word(uint32_t w, __half2 s2, __half2 lo2, uint32_t *out) {
    const __half2 k1024 = u32_as_h2(0x64006400u), k1_16 = u32_as_h2(0x2C002C00u), km64 = u32_as_h2(0xD400D400u);
    const uint32_t w8 = w >> 8;
    const __half2 q0 = __hsub2(u32_as_h2((w & 0x000F000Fu) | 0x64006400u), k1024);
    const __half2 q1 = __hfma2(u32_as_h2((w & 0x00F000F0u) | 0x64006400u), k1_16, km64);
    const __half2 q2 = __hsub2(u32_as_h2((w8 & 0x000F000Fu) | 0x64006400u), k1024);
    const __half2 q3 = __hfma2(u32_as_h2((w8 & 0x00F000F0u) | 0x64006400u), k1_16, km64);
    out[0] = h2_as_u32(__hfma2(q0, s2, lo2));
    out[1] = h2_as_u32(__hfma2(q1, s2, lo2));
    out[2] = h2_as_u32(__hfma2(q2, s2, lo2));
    out[3] = h2_as_u32(__hfma2(q3, s2, lo2));
}

// One thread per (column, group): the group's levels, its 64 codes and its
// (s, lo), written into the packed blocks.  Columns past N are padding: codes
// 0 and s = lo = 0.
__global__ void __launch_bounds__(256) int4_pack_kernel(const __half *__restrict__ W16, int K, int N,
                                                         uint8_t *__restrict__ W4, uint8_t *__restrict__ S4) {
    const int NP = padded_n(N);
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    const int g = blockIdx.y;
    if (n >= NP) return;
    const int KT = K / BK;
    const int nt = n / BN, r = n % BN, kt = g / 4, gs = g % 4;
    uint8_t *cblk = W4 + (static_cast<size_t>(nt) * KT + kt) * CODE_BYTES + static_cast<size_t>(r) * 128;
    uint8_t *sblk = S4 + (static_cast<size_t>(nt) * KT + kt) * SCALE_BYTES + static_cast<size_t>(r) * 16 + gs * 4;
    uint32_t words[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    __half s16 = __float2half_rn(0.0f), lo16 = __float2half_rn(0.0f);
    if (n < N) {
        float lo = INFINITY, hi = -INFINITY;
        for (int k = g * G; k < (g + 1) * G; ++k) {
            const float w = __half2float(W16[static_cast<size_t>(k) * N + n]);
            if (w < lo) lo = w;                         // first of equal values kept (signed zeros)
            if (w > hi) hi = w;
        }
        s16 = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 15.0f));
        lo16 = __float2half_rn(lo);
        const float s = __half2float(s16);
        const float inv = s > 0.0f ? __fdiv_rn(1.0f, s) : 0.0f;
        for (int e = 0; e < G; ++e) {
            const float w = __half2float(W16[static_cast<size_t>(g * G + e) * N + n]);
            float q = round_half_away(__fmul_rn(__fsub_rn(w, lo), inv));
            q = fminf(fmaxf(q, 0.0f), 15.0f);
            const uint32_t code = static_cast<uint32_t>(q);
            const int i = e / 8, within = e % 8;             // word, code in word
            const int nib = (within & 1) ? 4 + within / 2 : within / 2;
            words[i] |= code << (4 * nib);
        }
    }
    // this group's 64 codes are chunks 2*gs and 2*gs+1 of the column's 128 bytes
    for (int h = 0; h < 2; ++h) {
        const int c = 2 * gs + h;
        *reinterpret_cast<uint4 *>(cblk + ((c ^ (r & 7)) * 16)) =
            make_uint4(words[4 * h], words[4 * h + 1], words[4 * h + 2], words[4 * h + 3]);
    }
    __half2 sl = __halves2half2(s16, lo16);
    *reinterpret_cast<__half2 *>(sblk) = sl;
}

// The decoded weight W~ [K,N] fp16 (for checking the codec): one thread per
// (column, group), with the product kernel's decode.
__global__ void __launch_bounds__(256) int4_unpack_kernel(const uint8_t *__restrict__ W4, const uint8_t *__restrict__ S4,
                                                           int K, int N, __half *__restrict__ Wd) {
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    const int g = blockIdx.y;
    if (n >= N) return;
    const int KT = K / BK;
    const int nt = n / BN, r = n % BN, kt = g / 4, gs = g % 4;
    const uint8_t *cblk = W4 + (static_cast<size_t>(nt) * KT + kt) * CODE_BYTES + static_cast<size_t>(r) * 128;
    const __half2 sl = *reinterpret_cast<const __half2 *>(S4 + (static_cast<size_t>(nt) * KT + kt) * SCALE_BYTES +
                                                          static_cast<size_t>(r) * 16 + gs * 4);
    const __half2 s2 = __half2half2(__low2half(sl)), lo2 = __half2half2(__high2half(sl));
    for (int h = 0; h < 2; ++h) {
        const int c = 2 * gs + h;
        const uint4 u = *reinterpret_cast<const uint4 *>(cblk + ((c ^ (r & 7)) * 16));
        const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
        for (int i = 0; i < 4; ++i) {
            uint32_t pr[4];
            decode_word(wv[i], s2, lo2, pr);
            for (int j = 0; j < 4; ++j) {
                const int k = g * G + 32 * h + 8 * i + 2 * j;
                Wd[static_cast<size_t>(k) * N + n] = __ushort_as_half(static_cast<unsigned short>(pr[j] & 0xFFFFu));
                Wd[static_cast<size_t>(k + 1) * N + n] = __ushort_as_half(static_cast<unsigned short>(pr[j] >> 16));
            }
        }
    }
}

__global__ void int4_clear_kernel(int *__restrict__ counters, int n) {
    griddep_launch_dependents();            // the product may start streaming weights
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) counters[i] = 0;
}

// ------------------------------------------------------------------ product

__device__ __forceinline__ long long unit_begin(long long total, int c, int ctas) { return total * c / ctas; }
__device__ __forceinline__ int unit_owner(long long total, long long u, int ctas) {
    return static_cast<int>(((u + 1) * ctas - 1) / total);
}

// The runs of units of one tile in [u0, u1): visit(tile, kb, first, last).
template <typename Visit>
__device__ __forceinline__ bool walk(const Params &p, long long u0, long long u1, Visit &&visit) {
    for (long long u = u0; u < u1;) {
        const int tile = static_cast<int>(u / p.KB);
        const long long tile_u0 = static_cast<long long>(tile) * p.KB;
        const long long end = min(u1, tile_u0 + p.KB);
        for (long long v = u; v < end; ++v)
            if (!visit(tile, static_cast<int>(v - tile_u0), v == u, v == end - 1)) return false;
        u = end;
    }
    return true;
}

__global__ void __launch_bounds__(THREADS, 1)
    gemm_int4_decode_kernel(const __grid_constant__ CUtensorMap map_x, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Barriers *bars = reinterpret_cast<Barriers *>(smem + static_cast<size_t>(p.stages) * p.stage_bytes);
    volatile int *abort = &bars->abort;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], DECODERS + ISSUERS);   // the decoders' reads, the MMAs' reads of X
        }
        for (int b = 0; b < MAX_NA; ++b) {
            mbar_init(&bars->a_full[b], DECODERS);
            mbar_init(&bars->a_empty[b], ISSUERS);
        }
        for (int d = 0; d < 2; ++d) {
            mbar_init(&bars->tmem_full[d], ISSUERS);
            mbar_init(&bars->tmem_empty[d], 4);
        }
        mbar_init(&bars->drain, ISSUERS);
        bars->abort = 0;
        fence_mbar_init();
        tma_prefetch_map(&map_x);
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = bars->tmem_base;
    // A sub-buffer a: columns KSUB*a .. +KSUB-1 (column half h at +KSUB/2*h; two fp16 of K per column);
    // sub-stage j of the CTA (SUB per stage) uses sub-buffer j % NA.
    // D buffer d, column half h: NA*KSUB + (2d + h)*TP.
    const uint32_t a_base = tmem;
    const uint32_t d_base = tmem + static_cast<uint32_t>(p.na * KSUB);
    auto d_col = [&](int d, int h) { return static_cast<uint32_t>((2 * d + h) * p.TP); };

    const long long u0 = unit_begin(p.total_units, blockIdx.x, gridDim.x);
    const long long u1 = unit_begin(p.total_units, blockIdx.x + 1, gridDim.x);
    const int KT = p.KB;
    auto code_src = [&](int tile, int kb) {
        return p.W4 + (static_cast<size_t>(tile) * KT + kb) * CODE_BYTES;
    };
    auto scale_src = [&](int tile, int kb) {
        return p.S4 + (static_cast<size_t>(tile) * KT + kb) * SCALE_BYTES;
    };
    const uint32_t tx = static_cast<uint32_t>(p.stage_bytes);
    const int x_box_bytes = p.TP * 128;

    // the weight blocks of the first stages do not depend on earlier kernels
    const int pre = static_cast<int>(min(static_cast<long long>(p.stages), u1 - u0));
    if (warp == 0 && lane == 0) {
        for (int i = 0; i < pre; ++i) {
            const long long u = u0 + i;
            const int tile = static_cast<int>(u / p.KB), kb = static_cast<int>(u % p.KB);
            uint8_t *st = smem + static_cast<size_t>(i) * p.stage_bytes;
            mbar_arrive_expect_tx(&bars->full[i], tx);
            bulk_load(st, code_src(tile, kb), CODE_BYTES, &bars->full[i]);
            bulk_load(st + CODE_BYTES, scale_src(tile, kb), SCALE_BYTES, &bars->full[i]);
        }
    }
    griddep_wait();                                         // X and the cleared counters

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        int pending[MAX_STAGES];
        for (int s = 0; s < MAX_STAGES; ++s) pending[s] = -1;
        int stage = 0, n = 0;
        uint32_t phase = 0;
        const bool ok = walk(p, u0, u1, [&](int tile, int kb, bool, bool) -> bool {
            uint8_t *st = smem + static_cast<size_t>(stage) * p.stage_bytes;
            uint64_t *fb = &bars->full[stage];
            if (n >= pre) {
                if (!warp_wait(&bars->empty[stage], phase ^ 1u, abort, I8R_DEV_PIPELINE_TIMEOUT)) return false;
                if (lane == 0) {
                    mbar_arrive_expect_tx(fb, tx);
                    bulk_load(st, code_src(tile, kb), CODE_BYTES, fb);
                    bulk_load(st + CODE_BYTES, scale_src(tile, kb), SCALE_BYTES, fb);
                }
            }
            if (lane == 0) {
                uint8_t *xs = st + CODE_BYTES + SCALE_BYTES;
                for (int a = 0; a < 4; ++a) tma_load_2d(xs + a * x_box_bytes, &map_x, fb, kb * BK + 64 * a, 0);
                pending[stage] = static_cast<int>(phase);
            }
            ++n;
            __syncwarp();
            if (++stage == p.stages) { stage = 0; phase ^= 1u; }
            return true;
        });
        if (!ok && lane == 0) {
            volatile int never = 0;
            for (int s = 0; s < p.stages; ++s)
                if (pending[s] >= 0) mbar_wait(&bars->full[s], static_cast<uint32_t>(pending[s]), &never, 0);
        }
    } else if (warp <= ISSUERS) {
        // ------------------------------------------------------------ MMA issuers
        // one warp issues both column halves' MMAs, or each of two warps one half
        // (a single thread's tcgen05.mma issue rate, not the tensor pipe, limits
        // these small MMAs); each commits its own MMAs to the same barriers
        const uint32_t idesc = idesc_f16(BMH, p.TP, false, false);
        int stage = 0, seg = 0;
        uint32_t phase = 0, tph = 0;
        int a = 0;                                          // A sub-buffer of the next sub-stage
        uint32_t aph = 0;                                   // its phase parity (flips each lap of the ring)
        walk(p, u0, u1, [&](int, int, bool first, bool last) -> bool {
            const int d = seg & 1;
            if (first) {
                if (!warp_wait(&bars->tmem_empty[d], ((tph >> d) & 1u) ^ 1u, abort, I8R_DEV_TMEM_TIMEOUT)) return false;
                tc_fence_after_sync();
            }
            if (!warp_wait(&bars->full[stage], phase, abort, I8R_DEV_PIPELINE_TIMEOUT)) return false;
            const uint32_t xs = smem_u32(smem + static_cast<size_t>(stage) * p.stage_bytes + CODE_BYTES + SCALE_BYTES);
            const uint64_t xdesc = smem_desc_sw128(xs, 16, 1024);   // the start address is its low 14 bits (16-byte units)
            const uint32_t dd0 = d_base + d_col(d, 0), dd1 = d_base + d_col(d, 1);
            const bool do0 = ISSUERS == 1 || warp == 1, do1 = ISSUERS == 1 || warp == 2;
            for (int b = 0; b < SUB; ++b) {
                if (!warp_wait(&bars->a_full[a], aph, abort, I8R_DEV_TMEM_TIMEOUT)) return false;
                tc_fence_after_sync();
                if (lane == 0) {
                    const uint32_t ab = a_base + static_cast<uint32_t>(KSUB * a);
#pragma unroll
                    for (int kk = 0; kk < KSUB / 16; ++kk) {               // 16 of K per MMA
                        const uint32_t acc = (first && b == 0 && kk == 0) ? 0u : 1u;
                        const int k0 = KSUB * b + 16 * kk;                 // in the stage; X atoms are 64 of K
                        const uint64_t bd = xdesc + static_cast<uint64_t>(((k0 / 64) * x_box_bytes + (k0 % 64) * 2) >> 4);
                        if (do0) mma_f16_tmem_a(dd0, ab + static_cast<uint32_t>(8 * kk), bd, idesc, acc);
                        if (do1) mma_f16_tmem_a(dd1, ab + static_cast<uint32_t>(KSUB / 2 + 8 * kk), bd, idesc, acc);
                    }
                    mma_commit(&bars->a_empty[a]);
                }
                __syncwarp();
                if (++a == p.na) { a = 0; aph ^= 1u; }
            }
            if (lane == 0) {
                mma_commit(&bars->empty[stage]);
                if (last) mma_commit(&bars->tmem_full[d]);
            }
            __syncwarp();
            if (last) {
                tph ^= 1u << d;
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
    } else if (warp < FIRST_DEC + DECODERS) {
        // ------------------------------------------------------------ decoders
        // warp -> TMEM lane quadrant q = warp % 4 (the lanes it may access),
        // column half h and part: tile column r = 128h + 32q + lane, and in
        // sub-buffer b the chunks (32 codes each) (KSUB/32)*b + CPW*part .. +CPW-1
        const int q = warp & 3, gi = (warp - FIRST_DEC) >> 2;
        const int h = gi & 1, part = gi >> 1;
        const int r = h * BMH + q * 32 + lane;
        const uint32_t lane_bits = static_cast<uint32_t>(q * 32) << 16;
        int stage = 0;
        uint32_t phase = 0;
        int a = 0;
        uint32_t aph = 0;
        walk(p, u0, u1, [&](int, int, bool, bool) -> bool {
            if (!warp_wait(&bars->full[stage], phase, abort, I8R_DEV_PIPELINE_TIMEOUT)) return false;
            const uint8_t *st = smem + static_cast<size_t>(stage) * p.stage_bytes;
            const uint4 sl = *reinterpret_cast<const uint4 *>(st + CODE_BYTES + r * 16);   // (s, lo) of the 4 groups
            const uint32_t slw[4] = {sl.x, sl.y, sl.z, sl.w};
            uint4 code[SUB * CPW];
#pragma unroll
            for (int b = 0; b < SUB; ++b)
#pragma unroll
                for (int j = 0; j < CPW; ++j) {
                    const int c = KSUB / 32 * b + CPW * part + j;
                    code[b * CPW + j] = *reinterpret_cast<const uint4 *>(st + r * 128 + ((c ^ (r & 7)) * 16));
                }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->empty[stage]);    // this warp's shared-memory reads are done
#pragma unroll
            for (int b = 0; b < SUB; ++b) {
                if (!warp_wait(&bars->a_empty[a], aph ^ 1u, abort, I8R_DEV_TMEM_TIMEOUT)) return false;
                tc_fence_after_sync();
#pragma unroll
                for (int j = 0; j < CPW; ++j) {
                    const int c = KSUB / 32 * b + CPW * part + j;     // chunk of the stage: group c / 2
                    const __half2 sl2 = u32_as_h2(slw[c / 2]);
                    const __half2 s2 = __half2half2(__low2half(sl2)), lo2 = __half2half2(__high2half(sl2));
                    const uint4 cw = code[b * CPW + j];
                    uint32_t v[16];
                    decode_word(cw.x, s2, lo2, v);
                    decode_word(cw.y, s2, lo2, v + 4);
                    decode_word(cw.z, s2, lo2, v + 8);
                    decode_word(cw.w, s2, lo2, v + 12);
                    tmem_st16(a_base + lane_bits + static_cast<uint32_t>(KSUB * a + KSUB / 2 * h + 16 * (CPW * part + j)), v);
                }
                tmem_wait_st();
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->a_full[a]);
                if (++a == p.na) { a = 0; aph ^= 1u; }
            }
            if (++stage == p.stages) { stage = 0; phase ^= 1u; }
            return true;
        });
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;
        const uint32_t lane_bits = static_cast<uint32_t>(q * 32) << 16;
        uint32_t tph = 0;
        int seg = 0;
        walk(p, u0, u1, [&](int tile, int, bool, bool last) -> bool {
            if (!last) return true;
            const int d = seg & 1;
            if (!warp_wait(&bars->tmem_full[d], (tph >> d) & 1u, abort, I8R_DEV_TMEM_TIMEOUT)) return false;
            tc_fence_after_sync();
            const long long tile_u0 = static_cast<long long>(tile) * p.KB;
            const int c0 = unit_owner(p.total_units, tile_u0, gridDim.x);
            const int c1 = unit_owner(p.total_units, tile_u0 + p.KB - 1, gridDim.x);
            const int me = blockIdx.x;
            auto slot_of = [&](int c) { return (c == c0) ? 1 : 0; };    // the tile is c0's last run, the others' first
            auto part_at = [&](int c, int t, int hh) {
                return p.part + ((static_cast<size_t>(c) * 2 + slot_of(c)) * p.TP + t) * BN + hh * BMH + q * 32 + lane;
            };
            int mode = 0;                                   // 0: whole tile, 1: last piece, 2: store partial
            int *counter = p.counters + tile * COUNTERS_PER_TILE + q;
            if (c1 > c0) {
                int last_piece = 0;
                if (lane == 0) last_piece = atomicAdd(counter, 0) == c1 - c0;
                mode = __shfl_sync(0xFFFFFFFFu, last_piece, 0) ? 1 : 2;
            }
            if (mode == 1) __threadfence();
            for (int hh = 0; hh < 2; ++hh) {
                const int n = tile * BN + hh * BMH + q * 32 + lane;
                for (int t0 = 0; t0 < p.TP; t0 += 16) {
                    uint32_t v[16];
                    tmem_ld16(d_base + lane_bits + d_col(d, hh) + static_cast<uint32_t>(t0), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int t = t0 + e;
                        if (t >= p.T) continue;
                        const float own = __uint_as_float(v[e]);
                        if (mode == 2) {
                            __stcg(part_at(me, t, hh), own);
                        } else {
                            float y = own;
                            if (mode == 1) {
                                y = 0.0f;
                                for (int c = c0; c <= c1; ++c) y += (c == me) ? own : __ldcg(part_at(c, t, hh));
                            }
                            if (n < p.N) p.Y[static_cast<size_t>(t) * p.N + n] = __float2half_rn(y);
                        }
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->tmem_empty[d]);
            if (mode == 2) {
                // publish this piece, then count it; the piece that completes the
                // count adds every piece (CTA order) and writes Y
                __threadfence();
                __syncwarp();
                int done = 0;
                if (lane == 0) done = atomicAdd(counter, 1) == c1 - c0;     // every other piece counted
                if (__shfl_sync(0xFFFFFFFFu, done, 0)) {
                    __threadfence();
                    for (int hh = 0; hh < 2; ++hh) {
                        const int n = tile * BN + hh * BMH + q * 32 + lane;
                        for (int t = 0; t < p.T; ++t) {
                            float y = 0.0f;
                            for (int c = c0; c <= c1; ++c) y += __ldcg(part_at(c, t, hh));
                            if (n < p.N) p.Y[static_cast<size_t>(t) * p.N + n] = __float2half_rn(y);
                        }
                    }
                }
            }
            tph ^= 1u << d;
            ++seg;
            return true;
        });
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------------------------ product, few rows
// For one or two rows of X the CUDA cores do better than the tensor path
// above: per weight the work is the decode (13 instructions per 8 codes, the
// same decode_word, so the same fp16 W~) and one mixed-precision fused
// multiply-add per row (fma.rn.f32.f16: the fp16 product is exact in fp32,
// one rounding per add, as in the tensor core's fp32 accumulation), where the
// tensor path is bound by issuing MMAs.  The kernel is bound by instruction
// issue (about 140 warp instructions per 1024 weights at T = 1), so each
// further row costs about a third more; the host takes it for T <= 2.
//   A stage is one (tile, 256 of K) unit as above: its packed codes and
//   scales and the T rows of X over those 256 of K (bulk copies of 512 bytes),
//   filled by one producer warp.  Sixteen compute warps: warp group g (0..7)
//   takes columns 32g .. 32g+31 of the tile, one per lane, and half h of the
//   stage's K (chunks 4h .. 4h+3, groups 2h and 2h+1).  Each lane keeps four
//   fp32 sums per row (by pair parity and position, a fixed order).  At the
//   end of a tile's run the h = 1 warps hand their sums to the h = 0 warps
//   through shared memory (mbarriers, bounded waits), which add them and
//   write Y, or for a tile split over CTAs store the piece in the CTA's slot
//   and count it; the piece that completes the count adds the pieces in CTA
//   order.
constexpr int SMALL_T = 4;                  // instances exist for T = 1 .. SMALL_T
constexpr int SMALL_WARPS = 16;
constexpr int SMALL_THREADS = 32 * (1 + SMALL_WARPS);
constexpr int SMALL_MAX_STAGES = 6;
constexpr int SMALL_SMEM_BUDGET = 220 * 1024;
constexpr int X_SLICE_BYTES = BK * 2;       // one row of X over a stage's K

struct SmallBarriers {
    uint64_t full[SMALL_MAX_STAGES];
    uint64_t empty[SMALL_MAX_STAGES];
    uint64_t red_full;
    uint64_t red_empty;
    int abort;
};

__host__ __device__ inline int small_stage_bytes(int T) { return CODE_BYTES + SCALE_BYTES + T * X_SLICE_BYTES; }
__host__ __device__ inline size_t small_fixed_bytes(int T) {
    return 128 + static_cast<size_t>(T) * BN * 4 + sizeof(SmallBarriers);
}
__host__ __device__ inline int small_stages(int T) {
    const int s = static_cast<int>((SMALL_SMEM_BUDGET - small_fixed_bytes(T)) / small_stage_bytes(T));
    return s < SMALL_MAX_STAGES ? s : SMALL_MAX_STAGES;
}
__host__ __device__ inline size_t small_smem_bytes(int T) {
    return small_fixed_bytes(T) + static_cast<size_t>(small_stages(T)) * small_stage_bytes(T);
}

// c0 += lo(w) * lo(x), c1 += hi(w) * hi(x): fp16 operands, fp32 sums.
__device__ __forceinline__ void fma_f16x2_f32(uint32_t w, uint32_t x, float &c0, float &c1) {
    asm("{\n\t.reg .b16 wl, wh, xl, xh;\n\t"
        "mov.b32 {wl, wh}, %2;\n\t"
        "mov.b32 {xl, xh}, %3;\n\t"
        "fma.rn.f32.f16 %0, wl, xl, %0;\n\t"
        "fma.rn.f32.f16 %1, wh, xh, %1;\n\t}"
        : "+f"(c0), "+f"(c1)
        : "r"(w), "r"(x));
}

// One compute warp's share of a stage: column r of the tile, chunks 4H .. 4H+3
// (groups 2H and 2H+1), every row of X; H is a constant so that the chunk,
// scale and X offsets are immediates.
template <int TT, int H>
__device__ __forceinline__ void small_stage_math(const uint8_t *st, int r, float (&acc)[TT][4]) {
    constexpr int XOFF = CODE_BYTES + SCALE_BYTES;
    const uint2 sl = *reinterpret_cast<const uint2 *>(st + CODE_BYTES + r * 16 + H * 8);   // groups 2H, 2H+1
    const uint8_t *col = st + r * 128;
    const int sw = r & 7;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
        const int c = 4 * H + cc;                           // chunk of the stage: codes 32c .. 32c+31
        const __half2 sl2 = u32_as_h2(cc < 2 ? sl.x : sl.y);
        const __half2 s2 = __half2half2(__low2half(sl2)), lo2 = __half2half2(__high2half(sl2));
        const uint4 cw4 = *reinterpret_cast<const uint4 *>(col + ((c ^ sw) << 4));
        uint32_t v[16];                                     // v[4i+j]: codes 8i+2j, 8i+2j+1 of the chunk
        decode_word(cw4.x, s2, lo2, v);
        decode_word(cw4.y, s2, lo2, v + 4);
        decode_word(cw4.z, s2, lo2, v + 8);
        decode_word(cw4.w, s2, lo2, v + 12);
#pragma unroll
        for (int t = 0; t < TT; ++t) {
            // x over the chunk's 32 codes: 64 bytes of row t's slice
            const uint4 *xp = reinterpret_cast<const uint4 *>(st + XOFF + t * X_SLICE_BYTES + c * 64);
            const uint4 x0 = xp[0], x1 = xp[1], x2 = xp[2], x3 = xp[3];
            const uint32_t xv[16] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w,
                                     x2.x, x2.y, x2.z, x2.w, x3.x, x3.y, x3.z, x3.w};
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
                fma_f16x2_f32(v[e], xv[e], acc[t][0], acc[t][1]);
                fma_f16x2_f32(v[e + 1], xv[e + 1], acc[t][2], acc[t][3]);
            }
        }
    }
}

template <int TT>
__global__ void __launch_bounds__(SMALL_THREADS, 1)
    gemm_int4_small_kernel(const __half *__restrict__ X, const Params p) {
    constexpr int XOFF = CODE_BYTES + SCALE_BYTES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    float *red = reinterpret_cast<float *>(smem + static_cast<size_t>(p.stages) * p.stage_bytes);   // [TT][BN]
    SmallBarriers *bars = reinterpret_cast<SmallBarriers *>(red + TT * BN);
    volatile int *abort = &bars->abort;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], SMALL_WARPS);
        }
        mbar_init(&bars->red_full, SMALL_WARPS / 2);     // the h = 1 warps have stored their sums
        mbar_init(&bars->red_empty, SMALL_WARPS / 2);    // the h = 0 warps have read them
        bars->abort = 0;
        fence_mbar_init();
    }
    __syncthreads();

    const long long u0 = unit_begin(p.total_units, blockIdx.x, gridDim.x);
    const long long u1 = unit_begin(p.total_units, blockIdx.x + 1, gridDim.x);
    const int KT = p.KB;
    const uint32_t tx = static_cast<uint32_t>(p.stage_bytes);

    // the weight blocks of the first stages do not depend on earlier kernels
    const int pre = static_cast<int>(min(static_cast<long long>(p.stages), u1 - u0));
    if (warp == 0 && lane == 0) {
        for (int i = 0; i < pre; ++i) {
            const long long u = u0 + i;
            const size_t blk = static_cast<size_t>(u / KT) * KT + static_cast<size_t>(u % KT);
            uint8_t *st = smem + static_cast<size_t>(i) * p.stage_bytes;
            mbar_arrive_expect_tx(&bars->full[i], tx);
            bulk_load(st, p.W4 + blk * CODE_BYTES, CODE_BYTES, &bars->full[i]);
            bulk_load(st + CODE_BYTES, p.S4 + blk * SCALE_BYTES, SCALE_BYTES, &bars->full[i]);
        }
    }
    griddep_wait();                                         // X and the cleared counters

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        int pending[SMALL_MAX_STAGES];
        for (int s = 0; s < SMALL_MAX_STAGES; ++s) pending[s] = -1;
        int stage = 0, n = 0;
        uint32_t phase = 0;
        const bool ok = walk(p, u0, u1, [&](int tile, int kb, bool, bool) -> bool {
            uint8_t *st = smem + static_cast<size_t>(stage) * p.stage_bytes;
            uint64_t *fb = &bars->full[stage];
            if (n >= pre) {
                if (!warp_wait(&bars->empty[stage], phase ^ 1u, abort, I8R_DEV_PIPELINE_TIMEOUT)) return false;
                if (lane == 0) {
                    const size_t blk = static_cast<size_t>(tile) * KT + kb;
                    mbar_arrive_expect_tx(fb, tx);
                    bulk_load(st, p.W4 + blk * CODE_BYTES, CODE_BYTES, fb);
                    bulk_load(st + CODE_BYTES, p.S4 + blk * SCALE_BYTES, SCALE_BYTES, fb);
                }
            }
            if (lane == 0) {
#pragma unroll
                for (int t = 0; t < TT; ++t)
                    bulk_load(st + XOFF + t * X_SLICE_BYTES, X + static_cast<size_t>(t) * p.K + static_cast<size_t>(kb) * BK,
                              X_SLICE_BYTES, fb);
                pending[stage] = static_cast<int>(phase);
            }
            ++n;
            __syncwarp();
            if (++stage == p.stages) { stage = 0; phase ^= 1u; }
            return true;
        });
        if (!ok && lane == 0) {
            volatile int never = 0;
            for (int s = 0; s < p.stages; ++s)
                if (pending[s] >= 0) mbar_wait(&bars->full[s], static_cast<uint32_t>(pending[s]), &never, 0);
        }
        return;
    }

    // ---------------------------------------------------------------- compute
    const int cw = warp - 1;
    const int h = cw >> 3, grp = cw & 7;
    const int r = grp * 32 + lane;                          // column of the tile
    float acc[TT][4];
    int stage = 0, seg = 0;
    uint32_t phase = 0;
    walk(p, u0, u1, [&](int tile, int, bool first, bool last) -> bool {
        if (first) {
#pragma unroll
            for (int t = 0; t < TT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.0f;
        }
        if (!warp_wait(&bars->full[stage], phase, abort, I8R_DEV_PIPELINE_TIMEOUT)) return false;
        const uint8_t *st = smem + static_cast<size_t>(stage) * p.stage_bytes;
        if (h == 0)
            small_stage_math<TT, 0>(st, r, acc);
        else
            small_stage_math<TT, 1>(st, r, acc);
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->empty[stage]);    // this warp's shared-memory reads are done
        if (++stage == p.stages) { stage = 0; phase ^= 1u; }
        if (!last) return true;

        // the end of this CTA's run of the tile: the two halves of K meet
        float y[TT];
#pragma unroll
        for (int t = 0; t < TT; ++t) y[t] = (acc[t][0] + acc[t][1]) + (acc[t][2] + acc[t][3]);
        const uint32_t rph = static_cast<uint32_t>(seg & 1);
        ++seg;
        if (h == 1) {
            if (!warp_wait(&bars->red_empty, rph ^ 1u, abort, I8R_DEV_PIPELINE_TIMEOUT)) return false;
#pragma unroll
            for (int t = 0; t < TT; ++t) red[t * BN + r] = y[t];
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->red_full);
            return true;
        }
        if (!warp_wait(&bars->red_full, rph, abort, I8R_DEV_PIPELINE_TIMEOUT)) return false;
#pragma unroll
        for (int t = 0; t < TT; ++t) y[t] += red[t * BN + r];
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->red_empty);

        const long long tile_u0 = static_cast<long long>(tile) * p.KB;
        const int c0 = unit_owner(p.total_units, tile_u0, gridDim.x);
        const int c1 = unit_owner(p.total_units, tile_u0 + p.KB - 1, gridDim.x);
        const int col = tile * BN + r;
        if (c1 == c0) {
            if (col < p.N)
#pragma unroll
                for (int t = 0; t < TT; ++t) p.Y[static_cast<size_t>(t) * p.N + col] = __float2half_rn(y[t]);
            return true;
        }
        // the tile is c0's last run and the first of the others: slots 1 and 0
        auto part_at = [&](int c, int t) {
            return p.part + ((static_cast<size_t>(c) * 2 + (c == c0 ? 1 : 0)) * p.TP + t) * BN + r;
        };
#pragma unroll
        for (int t = 0; t < TT; ++t) __stcg(part_at(blockIdx.x, t), y[t]);
        __threadfence();
        __syncwarp();
        int done = 0;
        if (lane == 0) done = atomicAdd(p.counters + tile * COUNTERS_PER_TILE + grp, 1) == c1 - c0;
        if (__shfl_sync(0xFFFFFFFFu, done, 0)) {
            __threadfence();
            if (col < p.N)
#pragma unroll
                for (int t = 0; t < TT; ++t) {
                    float sum = 0.0f;
                    for (int c = c0; c <= c1; ++c) sum += __ldcg(part_at(c, t));
                    p.Y[static_cast<size_t>(t) * p.N + col] = __float2half_rn(sum);
                }
        }
        return true;
    });
}

}  // namespace w4
}  // namespace i8r
