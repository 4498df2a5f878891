// int8row C ABI: argument checks, workspace layout, tensor maps, launches.
// The declarations and their contracts are in include/int8row.h.
//
// Pipeline of int8_mixed_linear (all on the caller's stream, no host sync):
//   clear_mask_kernel       zeroes the outlier column bitmask
//   outlier_scan_kernel     X -> outlier column bitmask, atomic OR per word   (a1)
//   quantize_rows_kernel    X -> sX, Xq (outliers zeroed), Xo gather, the
//                           index list; for T > 128 (and for the Wq-only
//                           variant at every T) it also compacts the
//                           outliers' W16 rows (dequantised Wq rows)        (a1-a3)
// The scan and the quantiser are programmatic dependents of the kernel
// before them, so each loads its rows of X before waiting for it.
//   T > 128:  gemm_prefill_pair_kernel (CTA pairs, 256 x 256 tiles): int8 +
//             fp16 tensor-core MMA, epilogue -> Y
//   T <= 128: gemm_decode_kernel   split-K int8 MMA -> int32 partial sums, one
//             fp16 MMA segment per tile for the outlier part; the last
//             contributor of each tile applies the scales and adds the two
// The GEMMs are launched as programmatic dependents of the quantiser, so their
// prologue and first weight tiles overlap the activation kernels.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "int8row.h"
#include "device_common.cuh"
#include "quant_kernels.cuh"
#include "activation_fused.cuh"
#include "gemm_prefill_pair.cuh"
#include "gemm_decode.cuh"
#include "gemm_int4.cuh"

namespace {

using namespace i8r;

constexpr int kMaxK = 133144;          // K * 127^2 < 2^31
constexpr int kMaxDevices = 64;
constexpr size_t kAlign = 256;

std::atomic<uint64_t> g_launches{0};
thread_local int tl_last_cuda_error = 0;
thread_local cudaEvent_t tl_ev_before = nullptr;
thread_local cudaEvent_t tl_ev_after = nullptr;

struct DeviceInfo {
    bool ready = false;
    CUcontext ctx = nullptr;   // the context the setup below was done in
    bool sm100 = false;
    int sms = 0;
    int pair_clusters = 0;     // CTA pairs of the prefill GEMM that fit the GPU at once
    bool fused_ok = false;     // the one-kernel activation path can be launched (cooperative)
    void *noalloc_scratch = nullptr;   // device address of the no-alloc scratch in `ctx`
};
// Which activation path runs (int8_debug_set_activation_path): 1 (default) the
// one cooperative kernel for 8 <= T <= 128 when X fits in shared memory, 2 that
// kernel whenever X fits, 0 always the scan + quantiser pair, 3 as 1 but with
// the cooperative launch treated as refused (the fallback to the pair runs).
std::atomic<int> g_activation_fused{1};
// Which 4-bit product runs (int4_debug_set_product_path): 0 (default) the
// CUDA-core kernel for T <= kInt4SmallRows, the tensor-core kernel above;
// 1 always the tensor-core kernel; 2 the CUDA-core kernel whenever
// T <= w4::SMALL_T.
std::atomic<int> g_int4_path{0};
constexpr int kInt4SmallRows = 2;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mutex;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;

#define I8R_CUDA(call)                                             \
    do {                                                           \
        cudaError_t e_ = (call);                                   \
        if (e_ != cudaSuccess) {                                   \
            tl_last_cuda_error = static_cast<int>(e_);             \
            return I8R_ECUDA;                                      \
        }                                                          \
    } while (0)

#define I8R_TRY(expr)                         \
    do {                                      \
        i8r_status s_ = (expr);               \
        if (s_ != I8R_OK) return s_;          \
    } while (0)

inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Driver entry points the library uses (fetched once, under g_dev_mutex).
i8r_status driver_entry_points() {
    if (g_encode && g_ctx_current) return I8R_OK;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    I8R_CUDA(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
    if (q != cudaDriverEntryPointSuccess || !fn) return I8R_ECUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    fn = nullptr;
    I8R_CUDA(cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q));
    if (q != cudaDriverEntryPointSuccess || !fn) return I8R_ECUDA;
    g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
    return I8R_OK;
}

CUcontext current_context() {
    CUcontext c = nullptr;
    if (g_ctx_current && g_ctx_current(&c) != CUDA_SUCCESS) c = nullptr;
    return c;
}

// Per-device setup: architecture check, SM count, kernel attributes, the
// driver's entry points.  Kernel attributes and symbol addresses belong to a
// context, so the setup is done again whenever the calling thread's current
// context is not the one it was done in (after cudaDeviceReset, or under a
// context the caller made current).
template <int TT>
cudaError_t set_int4_small_attribute() {
    return cudaFuncSetAttribute(w4::gemm_int4_small_kernel<TT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(w4::small_smem_bytes(TT)));
}

// Shared memory beyond 48 KB for every instance of the CUDA-core 4-bit product.
i8r_status set_int4_small_attributes() {
    I8R_CUDA(set_int4_small_attribute<1>());
    I8R_CUDA(set_int4_small_attribute<2>());
    I8R_CUDA(set_int4_small_attribute<3>());
    I8R_CUDA(set_int4_small_attribute<4>());
    return I8R_OK;
}

i8r_status device_setup(const DeviceInfo **out) {
    int dev = 0;
    I8R_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return I8R_ERANGE;
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    I8R_TRY(driver_entry_points());
    DeviceInfo &d = g_dev[dev];
    if (!d.ready || current_context() != d.ctx) {
        d.ready = false;
        d.noalloc_scratch = nullptr;
        int major = 0, minor = 0;
        I8R_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
        I8R_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
        I8R_CUDA(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
        d.sm100 = (major == 10 && minor == 0);
        if (d.sm100) {
            I8R_CUDA(cudaFuncSetAttribute(prefill2::gemm_prefill_pair_kernel<false>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          static_cast<int>(prefill2::SMEM_BYTES)));
            I8R_CUDA(cudaFuncSetAttribute(prefill2::gemm_prefill_pair_kernel<true>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          static_cast<int>(prefill2::SMEM_BYTES)));
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(2 * (d.sms / 2));
            cfg.blockDim = dim3(prefill2::THREADS);
            cfg.dynamicSmemBytes = prefill2::SMEM_BYTES;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 2;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            I8R_CUDA(cudaOccupancyMaxActiveClusters(&d.pair_clusters, prefill2::gemm_prefill_pair_kernel<false>, &cfg));
            if (d.pair_clusters < 1) return I8R_EARCH;
            I8R_CUDA(cudaFuncSetAttribute(decode::gemm_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          static_cast<int>(decode::SMEM_MAX)));
            I8R_CUDA(cudaFuncSetAttribute(w4::gemm_int4_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          static_cast<int>(w4::SMEM_BUDGET + 4096)));
            I8R_TRY(set_int4_small_attributes());
            I8R_CUDA(cudaFuncSetAttribute(activation_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          static_cast<int>(kFusedSmemMax)));
            int per_sm = 0;
            I8R_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, activation_fused_kernel, kFusedThreads,
                                                                   kFusedSmemMax));
            d.fused_ok = per_sm >= 1;
        }
        // the runtime calls above made the device's context current if it was not
        d.ctx = current_context();
        d.ready = true;
    }
    if (!d.sm100) return I8R_EARCH;
    *out = &d;
    return I8R_OK;
}

// 2-D row-major tensor [rows, cols] of `elem` bytes, box [box_rows, box_cols],
// 128-byte swizzle unless asked otherwise, zero fill out of bounds on loads.
// `promote` widens the L2 fetch of each box row (256 B helps when the next
// 128 B are read soon by the same CTA; it doubles DRAM reads when they are not).
i8r_status make_map(CUtensorMap *map, const void *base, CUtensorMapDataType type, int elem, uint64_t rows,
                    uint64_t cols, uint32_t box_rows, uint32_t box_cols,
                    CUtensorMapL2promotion promote = CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * static_cast<uint64_t>(elem)};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, type, 2, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, promote,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        tl_last_cuda_error = static_cast<int>(r);
        return I8R_ECUDA;
    }
    return I8R_OK;
}

i8r_status check_launch() {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        tl_last_cuda_error = static_cast<int>(e);
        return I8R_ECUDA;
    }
    return I8R_OK;
}

#define I8R_LAUNCHED()                        \
    do {                                      \
        i8r_status s_ = check_launch();       \
        if (s_ != I8R_OK) return s_;          \
    } while (0)

i8r_status check_shape(int T, int K, int N, bool need_n) {
    if (T < 0 || K < 0 || (need_n && N < 0)) return I8R_EINVAL;
    if (K < 16 || K > kMaxK) return I8R_ERANGE;
    if (K % 16) return I8R_EALIGN;
    if (need_n) {
        if (N < 16) return I8R_ERANGE;
        if (N % 16) return I8R_EALIGN;
    }
    return I8R_OK;
}

i8r_status check_ptr(const void *p) {
    if (!p) return I8R_EINVAL;
    if (!aligned16(p)) return I8R_EALIGN;
    return I8R_OK;
}


// Workspace of int8_mixed_linear.
struct Workspace {
    size_t count, ctr, mask, idx, sX, Xq, Xo, W16o, Yo, acc32, total;
};

// Rows of the compacted outlier weight rows kept for the prefill GEMM: 256
// with W16 (past them the GEMM gathers W16 rows itself); for the Wq-only
// variant, which has no other source, at least 256 and K/16 (rounded up to
// 64), at most K rounded up to 64.
inline int compact_rows(int K, bool wq_only = false) {
    const int all = (K + 63) / 64 * 64;
    if (!wq_only) return std::min(all, kCompactOutlierRows);
    return std::min(all, std::max(kCompactOutlierRows, ((K + 15) / 16 + 63) / 64 * 64));
}

// Rows of compacted outlier rows a call uses: the Wq-only variant's (above);
// the prefill GEMM's 256; and at decode sizes at least 256 and K/64 (rounded
// up to 64; 1.6 % of the columns), since there every row the GEMM gathers
// itself costs the tile's first CTA a slow stage.
inline int outlier_rows(int T, int K, bool wq_only) {
    if (wq_only || T > decode::MAX_T) return compact_rows(K, wq_only);
    const int all = (K + 63) / 64 * 64;
    return std::min(all, std::max(kCompactOutlierRows, ((K + 63) / 64 + 63) / 64 * 64));
}

// compact_decode: decode-sized calls with W16 also compact the first
// outlier_rows(T, K) outlier rows of W16 (the GEMM then loads them as tiles);
// without it (the allocation-free entry point's smaller scratch) the decode
// GEMM gathers every outlier row from W16 itself.
Workspace ws_layout(int T, int K, int N, bool wq_only = false, bool compact_decode = true) {
    Workspace w{};
    size_t off = 0;
    w.count = off; off = align_up(off + sizeof(int32_t));
    w.ctr = off;   off = align_up(off + 2 * sizeof(uint32_t));    // the fused activation kernel's grid barrier
    w.mask = off;  off = align_up(off + static_cast<size_t>((K + 31) / 32) * 4);
    w.idx = off;   off = align_up(off + static_cast<size_t>(K) * 4);
    w.sX = off;    off = align_up(off + static_cast<size_t>(T) * 4);
    w.Xq = off;    off = align_up(off + static_cast<size_t>(T) * K);
    w.Xo = off;    off = align_up(off + static_cast<size_t>(T) * K * 2);
    w.W16o = off;
    if (T > decode::MAX_T || wq_only || compact_decode)
        off = align_up(off + static_cast<size_t>(outlier_rows(T, K, wq_only)) * N * 2);
    w.Yo = off;
    if (T <= decode::MAX_T) off = align_up(off + static_cast<size_t>(T) * N * 4);   // fp32 outlier part
    w.acc32 = off;
    if (T <= decode::MAX_T) off = align_up(off + static_cast<size_t>(T) * N * 4);   // split-K accumulator
    w.total = off;
    return w;
}

// Magnitude bits of the smallest fp16 value >= alpha (alpha >= 0, not NaN);
// 0x7C00 (infinity) when no finite fp16 reaches it.  fp16 magnitudes order
// like their bit patterns, so |x| >= alpha <=> (bits(x) & 0x7FFF) >= this,
// for every finite x.
uint32_t half_threshold_bits(float alpha) {
    auto value = [](uint32_t b) -> double {                 // exact value of a finite fp16 magnitude
        const uint32_t e = (b >> 10) & 0x1Fu, m = b & 0x3FFu;
        return e == 0 ? std::ldexp(static_cast<double>(m), -24) : std::ldexp(static_cast<double>(m | 0x400u), static_cast<int>(e) - 25);
    };
    if (!(static_cast<double>(alpha) <= value(0x7BFFu))) return 0x7C00u;
    uint32_t lo = 0, hi = 0x7BFFu;                          // value(hi) >= alpha
    while (lo < hi) {
        const uint32_t mid = (lo + hi) / 2;
        if (value(mid) >= static_cast<double>(alpha)) hi = mid; else lo = mid + 1;
    }
    return lo;
}

// Launch a kernel as a programmatic dependent of the previous kernel on
// the stream (its prologue may overlap that kernel; it waits with
// griddepcontrol.wait before touching the previous kernel's outputs).
// `cluster_x` > 1 launches clusters of that many CTAs along x.
template <typename... Params, typename... Args>
cudaError_t launch_dependent(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             int cluster_x, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.numAttrs = 1;
    if (cluster_x > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = static_cast<unsigned>(cluster_x);
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
    }
    cfg.attrs = attr;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// The row quantiser: G compaction blocks, then one block per row, launched as
// a programmatic dependent of the outlier scan (or, finding the mask itself,
// as the call's first kernel: an ordinary launch).
template <int kThreads, typename... Args>
cudaError_t launch_rows(cudaStream_t s, int T, int G, size_t smem, bool dependent, Args &&...args) {
    if (dependent)
        return launch_dependent(quantize_rows_kernel<kThreads>, dim3(G + T), dim3(kThreads), smem, s, 1,
                                std::forward<Args>(args)...);
    quantize_rows_kernel<kThreads><<<dim3(G + T), dim3(kThreads), smem, s>>>(std::forward<Args>(args)...);
    return cudaGetLastError();
}

// Grid of the row-band outlier scan: bands of 2048 columns, row blocks of at
// least 8 rows, about four blocks per SM.
dim3 scan_grid(int T, int K, int sms, int *rows_per_block) {
    const int bands = (K + kBandCols - 1) / kBandCols;
    const int want = std::max(1, (4 * sms + bands - 1) / bands);
    const int chunks = std::max(1, std::min((T + 7) / 8, want));
    *rows_per_block = std::max(1, (T + chunks - 1) / chunks);
    return dim3(bands, (T + *rows_per_block - 1) / *rows_per_block);
}

// a1-a3 on the stream: mask, row quantisation, index list and gather.
// `zero` / `zero_bytes`: a region the scan clears on the way (may be null).
// With W16o, the quantiser's launch also compacts the W16 rows of the first
// outlier_rows(T, K) outlier columns into W16o ([outlier_rows(T, K), N]); with
// W16 null (the Wq-only variant) it dequantises those rows of Wq instead.
i8r_status launch_activation(const DeviceInfo *dev, const __half *X, int T, int K, float alpha, uint32_t *mask,
                             int32_t *idx, int32_t *count, float *sX, int8_t *Xq, __half *Xo, void *zero,
                             size_t zero_bytes, cudaStream_t s, const __half *W16 = nullptr, int N = 0,
                             __half *W16o = nullptr, const int8_t *Wq = nullptr, const float *sW = nullptr,
                             unsigned *grid_ctr = nullptr) {
    const int nwords = (K + 31) / 32;
    // One cooperative kernel when this batch of X fits in the blocks' shared
    // memory: one block per SM (blocks past the last row still clear their
    // share of `zero` and take part in the barrier).  By default only for
    // decode-sized batches of at least 8 rows: below that the grid-wide barrier
    // costs more than the two small kernels it replaces, and at prefill sizes
    // (OPT-13B fc1, 2048 rows) the two paths measured level.
    const int fG = std::max(1, dev->sms);
    const int fR = (T + fG - 1) / fG;
    const int mode = g_activation_fused.load(std::memory_order_relaxed);
    const bool size_ok = mode == 2 ? T >= 1 : ((mode == 1 || mode == 3) && T >= kFusedMinRows && T <= decode::MAX_T);
    const bool fused = grid_ctr && size_ok && dev->fused_ok && fused_smem_bytes(fR, K) <= kFusedSmemMax;
    // Below kFusedMinRows rows (modes 1 and 3) the row quantiser finds the mask
    // itself: every block reads the few rows of X (at most kSelfMaskElems
    // elements, from L2 after the first), one launch in all.
    const bool self_mask = !fused && (mode == 1 || mode == 3) && T >= 1 && T < kFusedMinRows &&
                           static_cast<long long>(T) * K <= kSelfMaskElems;
    if (self_mask) {
        const int rt = row_threads(K);
        const int o_rows = W16o ? outlier_rows(T, K, W16 == nullptr) : 0;
        const int G = W16o ? std::min(o_rows, 128) : 0;
        const size_t smem = quantize_smem_bytes(K);
        const uint32_t thr = half_threshold_bits(alpha);
        const uint32_t thr2 = thr | (thr << 16);
        const uint32_t *no_parts = nullptr;
        cudaError_t e;
        if (rt == 64)
            e = launch_rows<64>(s, T, G, smem, false, X, T, K, no_parts, 0, sX, Xq, Xo, mask, idx, count, W16, Wq,
                                sW, N, W16o, o_rows, G, thr2, static_cast<int4 *>(zero), zero_bytes / 16);
        else if (rt == 128)
            e = launch_rows<128>(s, T, G, smem, false, X, T, K, no_parts, 0, sX, Xq, Xo, mask, idx, count, W16, Wq,
                                 sW, N, W16o, o_rows, G, thr2, static_cast<int4 *>(zero), zero_bytes / 16);
        else
            e = launch_rows<256>(s, T, G, smem, false, X, T, K, no_parts, 0, sX, Xq, Xo, mask, idx, count, W16, Wq,
                                 sW, N, W16o, o_rows, G, thr2, static_cast<int4 *>(zero), zero_bytes / 16);
        if (e != cudaSuccess) {
            tl_last_cuda_error = static_cast<int>(e);
            return I8R_ECUDA;
        }
        I8R_LAUNCHED();
        return I8R_OK;
    }
    clear_mask_kernel<<<1, 256, 0, s>>>(mask, nwords, fused ? grid_ctr : nullptr);
    I8R_LAUNCHED();
    if (fused) {
        const int o_rows = W16o ? outlier_rows(T, K, W16 == nullptr) : 0;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(fG));
        cfg.blockDim = dim3(kFusedThreads);
        cfg.dynamicSmemBytes = fused_smem_bytes(fR, K);
        cfg.stream = s;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        attr[1].id = cudaLaunchAttributeCooperative;       // every block resident: the grid barrier completes
        attr[1].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        const uint32_t thr = half_threshold_bits(alpha);
        // mode 3 (a test switch) takes the refusal path below without asking
        const cudaError_t e =
            mode == 3 ? cudaErrorCooperativeLaunchTooLarge
                      : cudaLaunchKernelEx(&cfg, activation_fused_kernel, X, T, K, thr | (thr << 16), fR, mask,
                                           grid_ctr, sX, Xq, Xo, idx, count, W16, Wq, sW, N, W16o, o_rows,
                                           static_cast<int4 *>(zero), zero_bytes / 16);
        if (e == cudaSuccess) {
            I8R_LAUNCHED();
            return I8R_OK;
        }
        // The cooperative launch can be refused when the context has fewer SMs
        // or less shared memory free than at setup (another green context, MPS
        // limits).  Nothing was enqueued; the mask is clear, so the two-kernel
        // path below gives the same bits.  Any other error is the caller's.
        if (e != cudaErrorCooperativeLaunchTooLarge && e != cudaErrorLaunchOutOfResources) {
            tl_last_cuda_error = static_cast<int>(e);
            return I8R_ECUDA;
        }
        (void)cudaGetLastError();       // the refusal is not sticky: clear it
    }
    if (T == 0) {
        // no rows: an empty outlier set still has to be published
        outlier_index_kernel<<<1, kIndexThreads, 0, s>>>(mask, 1, K, mask, idx, count, nullptr);
        I8R_LAUNCHED();
        return I8R_OK;
    }
    int rows_per_block = 0;
    const dim3 grid = scan_grid(T, K, dev->sms, &rows_per_block);
    cudaError_t e = launch_dependent(outlier_scan_kernel, grid, dim3(kScanThreads), 0, s, 1, X, T, K, alpha,
                                     rows_per_block, mask, static_cast<int4 *>(zero), zero_bytes / 16);
    if (e != cudaSuccess) {
        tl_last_cuda_error = static_cast<int>(e);
        return I8R_ECUDA;
    }
    I8R_LAUNCHED();
    // row 0's block of the quantiser publishes the index list and |O|
    const int rt = row_threads(K);
    const int o_rows = W16o ? outlier_rows(T, K, W16 == nullptr) : 0;
    const int G = W16o ? std::min(o_rows, 128) : 0;     // compaction blocks
    const size_t smem = quantize_smem_bytes(K);
    const uint32_t *m = mask;
    uint32_t *no_mask_out = nullptr;
    int4 *no_zero = nullptr;
    if (rt == 64)
        e = launch_rows<64>(s, T, G, smem, true, X, T, K, m, 1, sX, Xq, Xo, no_mask_out, idx, count, W16, Wq, sW, N,
                            W16o, o_rows, G, 0u, no_zero, size_t{0});
    else if (rt == 128)
        e = launch_rows<128>(s, T, G, smem, true, X, T, K, m, 1, sX, Xq, Xo, no_mask_out, idx, count, W16, Wq, sW,
                             N, W16o, o_rows, G, 0u, no_zero, size_t{0});
    else
        e = launch_rows<256>(s, T, G, smem, true, X, T, K, m, 1, sX, Xq, Xo, no_mask_out, idx, count, W16, Wq, sW,
                             N, W16o, o_rows, G, 0u, no_zero, size_t{0});
    if (e != cudaSuccess) {
        tl_last_cuda_error = static_cast<int>(e);
        return I8R_ECUDA;
    }
    I8R_LAUNCHED();
    return I8R_OK;
}


void record_before(cudaStream_t s) {
    if (tl_ev_before) cudaEventRecord(tl_ev_before, s);
}
void record_after(cudaStream_t s) {
    if (tl_ev_after) cudaEventRecord(tl_ev_after, s);
    tl_ev_before = nullptr;
    tl_ev_after = nullptr;
}

// Prefill GEMM (T > 128): Y mode when Y != nullptr, else int32 accumulators.
// CTA pairs (clusters of 2) compute 256 x 256 tiles with cta_group::2 MMAs,
// persistent over the tiles.
i8r_status launch_prefill(const DeviceInfo *dev, const int8_t *Xq, const __half *Xo, int T, int K,
                          const int8_t *Wq, const float *sW, const __half *W16, int N, const int32_t *count,
                          const int32_t *idx, const float *sX, __half *Y, int32_t *acc_out, cudaStream_t s,
                          const __half *W16o = nullptr) {
    CUtensorMap map_xq, map_wq, map_xo, map_w16, map_w16x4, map_w16o, map_y;
    I8R_TRY(make_map(&map_xq, Xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, T, K, 128, prefill2::A_BOX_K));
    I8R_TRY(make_map(&map_wq, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, N, prefill2::BK, 128));
    const bool wq_only = Xo && !W16;
    if (Xo) {
        I8R_TRY(make_map(&map_xo, Xo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, T, K, 128, prefill2::OBK));
    } else {
        map_xo = map_xq;   // unused: no 16-bit part
    }
    if (Xo && W16) {
        // 64-column pieces of W16 rows: one-row box (also the gather map), and
        // a four-row box for the zero padding
        I8R_TRY(make_map(&map_w16, W16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, K, N, 1, 64));
        I8R_TRY(make_map(&map_w16x4, W16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, K, N, 4, 64));
    } else {
        map_w16 = map_xq;  // unused: no W16 (int32 output mode, or the Wq-only variant)
        map_w16x4 = map_xq;
    }
    // compacted outlier rows: 64 x 64 boxes
    const int o_rows = (Xo && W16o) ? compact_rows(K, wq_only) : 0;
    if (o_rows > 0) {
        I8R_TRY(make_map(&map_w16o, W16o, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, o_rows, N, 64, 64));
    } else {
        map_w16o = map_xq;
    }
    if (Y) {
        // 32 x 32 output blocks, unswizzled 64-byte rows
        I8R_TRY(make_map(&map_y, Y, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, T, N, 32, 32,
                         CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_SWIZZLE_NONE));
    } else {
        map_y = map_xq;    // unused: int32 output mode
    }
    prefill2::Params p{};
    p.T = T;
    p.K = K;
    p.N = N;
    p.num_m = (T + prefill2::BM - 1) / prefill2::BM;
    const int num_n = (N + prefill2::BN - 1) / prefill2::BN;
    p.num_tiles = p.num_m * num_n;
    p.KB = (K + prefill2::BK - 1) / prefill2::BK;
    p.count = Y ? count : nullptr;
    p.idx = idx;
    p.sX = sX;
    p.sW = sW;
    p.Y = Y;
    p.acc_out = acc_out;
    p.o_rows = o_rows;
    p.wq_only = wq_only ? 1 : 0;
    p.Wq = Wq;
    const int clusters = p.num_tiles < dev->pair_clusters ? p.num_tiles : dev->pair_clusters;
    record_before(s);
    cudaError_t e;
    if (Y)
        e = launch_dependent(prefill2::gemm_prefill_pair_kernel<false>, dim3(2 * clusters), dim3(prefill2::THREADS),
                             prefill2::SMEM_BYTES, s, 2, map_xq, map_wq, map_xo, map_w16, map_w16x4, map_w16o, map_y, p);
    else
        e = launch_dependent(prefill2::gemm_prefill_pair_kernel<true>, dim3(2 * clusters), dim3(prefill2::THREADS),
                             prefill2::SMEM_BYTES, s, 2, map_xq, map_wq, map_xo, map_w16, map_w16x4, map_w16o, map_y, p);
    if (e != cudaSuccess) {
        tl_last_cuda_error = static_cast<int>(e);
        return I8R_ECUDA;
    }
    I8R_LAUNCHED();
    record_after(s);
    return I8R_OK;
}

// Decode GEMM (T <= 128): int32 partial sums added into acc32, which must be
// zero on entry.  With `fin` (non-null) it also runs the 16-bit part (|O| > 0:
// Xo times the rows of the first fin->o_rows outliers from W16o, the rest from
// W16 by fin->idx) into fin->Yo, and decode_finalize_kernel then writes Y.
i8r_status launch_decode(const DeviceInfo *dev, const int8_t *Xq, int T, int K, const int8_t *Wq, int N,
                         int32_t *acc32, const decode::Params *fin, cudaStream_t s, const __half *Xo = nullptr,
                         const __half *W16 = nullptr, const __half *W16o = nullptr) {
    decode::Params p = fin ? *fin : decode::Params{};
    p.finalize = fin ? 1 : 0;
    p.T = T;
    p.TP = (T + 15) / 16 * 16;
    p.K = K;
    p.N = N;
    p.KB = (K + decode::BK - 1) / decode::BK;
    p.num_tiles = (N + decode::BM - 1) / decode::BM;
    p.total_units = static_cast<long long>(p.num_tiles) * p.KB;
    p.stage_bytes = decode::A_BYTES + p.TP * decode::BK;
    // the ring takes what shared memory the reduce staging boxes leave
    p.stages = static_cast<int>((decode::SMEM_MAX - decode::smem_bytes(0, 0)) / p.stage_bytes);
    if (p.stages > decode::MAX_STAGES) p.stages = decode::MAX_STAGES;
    p.may_outlier = (fin && fin->may_outlier) ? 1 : 0;
    uint32_t cols = 32;
    while (cols < static_cast<uint32_t>(2 * p.TP)) cols <<= 1;
    p.buf_cols = cols;
    p.nbuf = cols * decode::MAX_BUF <= 512 ? decode::MAX_BUF : 2;
    p.tmem_cols = cols * static_cast<uint32_t>(p.nbuf);
    p.acc32 = acc32;
    CUtensorMap map_wq, map_xq, map_xo, map_w16o, map_acc, map_yo;
    // Two 128-column boxes per stage cover 256 contiguous bytes of every weight
    // row, so the 256-byte L2 line is used whole.
    I8R_TRY(make_map(&map_wq, Wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, N, decode::BK, decode::BMH));
    I8R_TRY(make_map(&map_xq, Xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, T, K, p.TP, decode::BK));
    map_xo = map_w16o = map_yo = map_xq;   // unused without a 16-bit part
    // acc32 (and Yo) [T, N] in 32 x 32 boxes, unswizzled 128-byte rows
    I8R_TRY(make_map(&map_acc, acc32, CU_TENSOR_MAP_DATA_TYPE_INT32, 4, T, N, decode::RED_ROWS, 32,
                     CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_SWIZZLE_NONE));
    if (fin && fin->Yo)
        I8R_TRY(make_map(&map_yo, fin->Yo, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, T, N, decode::RED_ROWS, 32,
                         CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_SWIZZLE_NONE));
    p.W16 = W16;
    p.Wq = Wq;
    if (fin && Xo) {
        I8R_TRY(make_map(&map_xo, Xo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, T, K, p.TP, decode::OBK));
        if (W16o) I8R_TRY(make_map(&map_w16o, W16o, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, p.o_rows, N, 64, 64));
    }
    const long long g = p.total_units < dev->sms ? p.total_units : dev->sms;
    const size_t smem = decode::smem_bytes(p.stages, p.stage_bytes);
    record_before(s);
    cudaError_t e = launch_dependent(decode::gemm_decode_kernel, dim3(static_cast<unsigned>(g)),
                                     dim3(decode::THREADS), smem, s, 1, map_wq, map_xq, map_xo, map_w16o, map_acc, map_yo,
                                     p);
    if (e != cudaSuccess) {
        tl_last_cuda_error = static_cast<int>(e);
        return I8R_ECUDA;
    }
    I8R_LAUNCHED();
    record_after(s);
    if (fin) {
        const long long items = static_cast<long long>(T) * (N / 8);
        e = launch_dependent(decode::decode_finalize_kernel, dim3(static_cast<unsigned>((items + 255) / 256)), dim3(256),
                             0, s, 1, static_cast<const int32_t *>(acc32), static_cast<const float *>(fin->Yo),
                             fin->count, fin->sX, fin->sW, T, N, fin->Y);
        if (e != cudaSuccess) {
            tl_last_cuda_error = static_cast<int>(e);
            return I8R_ECUDA;
        }
        I8R_LAUNCHED();
    }
    return I8R_OK;
}

// The CUDA-core 4-bit product's instances, T = 1 .. w4::SMALL_T rows.
cudaError_t launch_int4_small(int T, unsigned grid, const __half *X, const w4::Params &p, cudaStream_t s) {
    const dim3 g(grid), b(w4::SMALL_THREADS);
    switch (T) {
        case 1: return launch_dependent(w4::gemm_int4_small_kernel<1>, g, b, w4::small_smem_bytes(1), s, 1, X, p);
        case 2: return launch_dependent(w4::gemm_int4_small_kernel<2>, g, b, w4::small_smem_bytes(2), s, 1, X, p);
        case 3: return launch_dependent(w4::gemm_int4_small_kernel<3>, g, b, w4::small_smem_bytes(3), s, 1, X, p);
        default: return launch_dependent(w4::gemm_int4_small_kernel<4>, g, b, w4::small_smem_bytes(4), s, 1, X, p);
    }
}

// The group-wise 4-bit codec: shape rules and the product's workspace.
i8r_status check_int4_shape(int K, int N) {
    if (K < 0 || N < 0) return I8R_EINVAL;
    if (K < w4::BK || N < 16) return I8R_ERANGE;
    if (K % w4::BK || N % 16) return I8R_EALIGN;
    return I8R_OK;
}

struct Int4Workspace {
    size_t part, counters, total;
};

Int4Workspace int4_ws_layout(int T, int N) {
    Int4Workspace w{};
    const int TP = (T + 15) / 16 * 16;
    w.part = 0;
    w.counters = align_up(static_cast<size_t>(w4::MAX_CTAS) * 2 * TP * w4::BN * 4);
    w.total = align_up(w.counters + static_cast<size_t>(w4::padded_n(N) / w4::BN) * w4::COUNTERS_PER_TILE * 4);
    return w;
}

__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    mbar_wait(&bar, 0, &abort_flag, I8R_DEV_PIPELINE_TIMEOUT, limit_ns);
}

__global__ void zero_kernel(int4 *p, size_t n16) {
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n16;
         i += static_cast<size_t>(gridDim.x) * blockDim.x)
        p[i] = make_int4(0, 0, 0, 0);
}

}  // namespace

// ---------------------------------------------------------------------------
// Scratch for int8_mixed_linear_noalloc.  Some callers cannot allocate device
// memory where they call this layer: a plugin inside an inference runtime that
// has reserved the GPU's memory for its own pool and hands the plugin only its
// input and output buffers, or a latency-critical path where cudaMalloc and
// cudaFree are not allowed because they can block or synchronise the device.
// For them the workspace is this fixed array, reserved once per GPU when the
// library's device code is loaded there and held until the process exits.
// In host code `g_noalloc_scratch` names the symbol, not a device address:
// the address each device uses is looked up with cudaGetSymbolAddress.
// ---------------------------------------------------------------------------
static constexpr size_t kNoAllocScratchBytes = 8u << 20;   // 8 MiB per GPU
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device, looked up with
// that device current the first time the device is used in its current
// context (device_setup forgets the address when the context changes, e.g.
// after cudaDeviceReset, where the array is placed afresh).
static i8r_status noalloc_scratch_address(void **out) {
    const DeviceInfo *info = nullptr;
    I8R_TRY(device_setup(&info));
    int dev = 0;
    I8R_CUDA(cudaGetDevice(&dev));
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    DeviceInfo &d = g_dev[dev];
    if (!d.noalloc_scratch) {
        void *p = nullptr;
        I8R_CUDA(cudaGetSymbolAddress(&p, g_noalloc_scratch));
        if (!p) return I8R_ECUDA;
        d.noalloc_scratch = p;
    }
    *out = d.noalloc_scratch;
    return I8R_OK;
}

extern "C" {

i8r_status int8_quantize_weight_colwise(const void *W16, int K, int N, int8_t *Wq, float *sW, cudaStream_t stream) {
    I8R_TRY(check_shape(0, K, N, true));
    I8R_TRY(check_ptr(W16));
    I8R_TRY(check_ptr(Wq));
    I8R_TRY(check_ptr(sW));
    const DeviceInfo *dev = nullptr;
    I8R_TRY(device_setup(&dev));
    const __half *w = static_cast<const __half *>(W16);
    weight_absmax_kernel<<<(N + kStripCols - 1) / kStripCols, kStripThreads, 0, stream>>>(w, K, N, sW);
    I8R_LAUNCHED();
    const size_t groups = static_cast<size_t>(K) * (N / 8);
    size_t blocks = (groups + 255) / 256;
    const size_t cap = static_cast<size_t>(dev->sms) * 16;
    if (blocks > cap) blocks = cap;
    weight_codes_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(w, K, N, sW, Wq);
    I8R_LAUNCHED();
    return I8R_OK;
}

size_t int8_mixed_linear_workspace_size(int T, int K, int N) {
    if (T < 0 || K < 0 || N < 0) return 0;
    return ws_layout(T, K, N).total;
}

namespace {

// int8_mixed_linear and its Wq-only variant (W16 null).
i8r_status mixed_linear_impl(const void *X, int T, int K, const int8_t *Wq, const float *sW, const void *W16, int N,
                             float alpha, void *Y, void *workspace, size_t workspace_bytes, cudaStream_t stream,
                             bool compact_decode = true) {
    const bool wq_only = W16 == nullptr;
    I8R_TRY(check_shape(T, K, N, true));
    if (std::isnan(alpha) || alpha < 0.0f) return I8R_EINVAL;
    if (T == 0) return I8R_OK;
    I8R_TRY(check_ptr(X));
    I8R_TRY(check_ptr(Wq));
    I8R_TRY(check_ptr(sW));
    if (!wq_only) I8R_TRY(check_ptr(W16));
    I8R_TRY(check_ptr(Y));
    const Workspace w = ws_layout(T, K, N, wq_only, compact_decode);
    if (!workspace || workspace_bytes < w.total) return I8R_EWORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return I8R_EALIGN;
    const DeviceInfo *dev = nullptr;
    I8R_TRY(device_setup(&dev));

    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int32_t *count = reinterpret_cast<int32_t *>(ws + w.count);
    uint32_t *mask = reinterpret_cast<uint32_t *>(ws + w.mask);
    int32_t *idx = reinterpret_cast<int32_t *>(ws + w.idx);
    float *sX = reinterpret_cast<float *>(ws + w.sX);
    int8_t *Xq = reinterpret_cast<int8_t *>(ws + w.Xq);
    __half *Xo = reinterpret_cast<__half *>(ws + w.Xo);
    const bool small_t = T <= decode::MAX_T;
    int32_t *acc32 = small_t ? reinterpret_cast<int32_t *>(ws + w.acc32) : nullptr;
    float *Yo = small_t ? reinterpret_cast<float *>(ws + w.Yo) : nullptr;
    const __half *x = static_cast<const __half *>(X);
    const __half *w16 = static_cast<const __half *>(W16);
    __half *y = static_cast<__half *>(Y);

    // decode: the activation side clears the split-K accumulator
    const size_t zero_bytes = small_t ? w.total - w.acc32 : 0;
    // compacted outlier rows: the first outlier_rows(T, K) rows of W16 (the GEMMs
    // gather any further rows from W16 themselves), or the Wq-only variant's
    // dequantised rows
    __half *W16o = (small_t && !wq_only && !compact_decode) ? nullptr : reinterpret_cast<__half *>(ws + w.W16o);
    I8R_TRY(launch_activation(dev, x, T, K, alpha, mask, idx, count, sX, Xq, Xo, small_t ? acc32 : nullptr,
                              zero_bytes, stream, w16, N, W16o, Wq, sW, reinterpret_cast<unsigned *>(ws + w.ctr)));
    if (!small_t)
        return launch_prefill(dev, Xq, Xo, T, K, Wq, sW, w16, N, count, idx, sX, y, nullptr, stream, W16o);

    decode::Params fin{};
    fin.sX = sX;
    fin.sW = sW;
    fin.count = count;
    fin.idx = idx;
    fin.o_rows = (wq_only || compact_decode) ? outlier_rows(T, K, wq_only) : 0;
    fin.wq_only = wq_only ? 1 : 0;
    fin.may_outlier = std::isinf(alpha) ? 0 : 1;   // alpha = +inf: no finite input is an outlier
    fin.Y = y;
    fin.Yo = Yo;
    return launch_decode(dev, Xq, T, K, Wq, N, acc32, &fin, stream, Xo, w16, W16o);
}

}  // namespace

i8r_status int8_mixed_linear(const void *X, int T, int K, const int8_t *Wq, const float *sW, const void *W16, int N,
                             float alpha, void *Y, void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (!W16) return I8R_EINVAL;
    return mixed_linear_impl(X, T, K, Wq, sW, W16, N, alpha, Y, workspace, workspace_bytes, stream);
}

size_t int8_mixed_linear_wq_workspace_size(int T, int K, int N) {
    if (T < 0 || K < 0 || N < 0) return 0;
    return ws_layout(T, K, N, true).total;
}

int int8_mixed_linear_wq_max_outliers(int K) { return K < 0 ? 0 : compact_rows(K, true); }

i8r_status int8_mixed_linear_wq(const void *X, int T, int K, const int8_t *Wq, const float *sW, int N, float alpha,
                                void *Y, void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    return mixed_linear_impl(X, T, K, Wq, sW, nullptr, N, alpha, Y, workspace, workspace_bytes, stream);
}

size_t int8_mixed_linear_chain_workspace_size(int n, const i8r_layer *layers) {
    if (n < 0 || (n > 0 && !layers)) return 0;
    size_t need = 0;
    for (int i = 0; i < n; ++i) {
        const i8r_layer &l = layers[i];
        if (l.T < 0 || l.K < 0 || l.N < 0) return 0;
        need = std::max(need, ws_layout(l.T, l.K, l.N, l.W16 == nullptr).total);
    }
    return need;
}

i8r_status int8_mixed_linear_chain(int n, const i8r_layer *layers, void *workspace, size_t workspace_bytes,
                                   cudaStream_t stream) {
    if (n < 0 || (n > 0 && !layers)) return I8R_EINVAL;
    // every layer is checked before anything is enqueued
    for (int i = 0; i < n; ++i) {
        const i8r_layer &l = layers[i];
        I8R_TRY(check_shape(l.T, l.K, l.N, true));
        if (std::isnan(l.alpha) || l.alpha < 0.0f) return I8R_EINVAL;
        if (l.T == 0) continue;
        I8R_TRY(check_ptr(l.X));
        I8R_TRY(check_ptr(l.Wq));
        I8R_TRY(check_ptr(l.sW));
        if (l.W16) I8R_TRY(check_ptr(l.W16));
        I8R_TRY(check_ptr(l.Y));
        if (!workspace || workspace_bytes < ws_layout(l.T, l.K, l.N, l.W16 == nullptr).total) return I8R_EWORKSPACE;
    }
    if (n > 0 && reinterpret_cast<uintptr_t>(workspace) % kAlign) return I8R_EALIGN;
    for (int i = 0; i < n; ++i) {
        const i8r_layer &l = layers[i];
        I8R_TRY(mixed_linear_impl(l.X, l.T, l.K, l.Wq, l.sW, l.W16, l.N, l.alpha, l.Y, workspace, workspace_bytes,
                                  stream));
    }
    return I8R_OK;
}

size_t int8_mixed_linear_noalloc_max_workspace(void) { return kNoAllocScratchBytes; }

void int8_debug_set_activation_path(int mode) { g_activation_fused.store(mode < 0 ? 0 : (mode > 3 ? 3 : mode)); }

void int4_debug_set_product_path(int mode) { g_int4_path.store(mode < 0 ? 0 : (mode > 2 ? 2 : mode)); }

i8r_status int8_mixed_linear_noalloc(const void *X, int T, int K, const int8_t *Wq, const float *sW,
                                     const void *W16, int N, float alpha, void *Y, cudaStream_t stream) {
    I8R_TRY(check_shape(T, K, N, true));
    // the fixed scratch holds no compacted outlier rows at decode sizes: the
    // GEMM gathers them from W16 (same results, and more shapes fit)
    if (ws_layout(T, K, N, false, false).total > kNoAllocScratchBytes) return I8R_ERANGE;
    if (!W16) return I8R_EINVAL;
    void *scratch = nullptr;
    I8R_TRY(noalloc_scratch_address(&scratch));
    // Nothing in the scratch has to start at zero: int8_mixed_linear writes
    // every region before it reads it.
    return mixed_linear_impl(X, T, K, Wq, sW, W16, N, alpha, Y, scratch, kNoAllocScratchBytes, stream, false);
}

size_t int8_outlier_stats_workspace_size(int K) {
    if (K < 0) return 0;
    return align_up(static_cast<size_t>((K + 31) / 32) * 4);
}

i8r_status int8_outlier_stats(const void *X, int T, int K, float alpha, int32_t *num_outlier_cols, int32_t *col_idx,
                              int32_t *col_hit_count, float *frac_8bit, void *workspace, size_t workspace_bytes,
                              cudaStream_t stream) {
    I8R_TRY(check_shape(T, K, 0, false));
    if (std::isnan(alpha) || alpha < 0.0f) return I8R_EINVAL;
    if (T > 0) I8R_TRY(check_ptr(X));
    if (!num_outlier_cols || !col_idx || !frac_8bit) return I8R_EINVAL;
    if (col_hit_count && !aligned16(col_hit_count)) return I8R_EALIGN;
    if (!workspace || workspace_bytes < int8_outlier_stats_workspace_size(K)) return I8R_EWORKSPACE;
    if (!aligned16(workspace)) return I8R_EALIGN;
    const DeviceInfo *dev = nullptr;
    I8R_TRY(device_setup(&dev));
    uint32_t *mask = static_cast<uint32_t *>(workspace);
    const int blocks = (K + kStripCols - 1) / kStripCols;
    const __half *x = static_cast<const __half *>(X);
    // one row part: every block scans all rows of its columns, so the hit counts are complete
    const int rows = T > 0 ? T : 1;
    if (col_hit_count)
        outlier_mask_kernel<true><<<blocks, kStripThreads, 0, stream>>>(x, T, K, alpha, rows, mask, col_hit_count,
                                                                        nullptr, 0);
    else
        outlier_mask_kernel<false><<<blocks, kStripThreads, 0, stream>>>(x, T, K, alpha, rows, mask, nullptr,
                                                                         nullptr, 0);
    I8R_LAUNCHED();
    outlier_index_kernel<<<1, kIndexThreads, 0, stream>>>(mask, 1, K, mask, col_idx, num_outlier_cols, frac_8bit);
    I8R_LAUNCHED();
    return I8R_OK;
}

size_t int8_quantize_activation_workspace_size(int T, int K) {
    (void)T;
    (void)K;
    return kAlign;                 // the one-kernel path's grid-barrier counter
}

i8r_status int8_quantize_activation(const void *X, int T, int K, float alpha, uint32_t *mask, int32_t *idx,
                                    int32_t *count, float *sX, int8_t *Xq, void *Xo, void *workspace,
                                    size_t workspace_bytes, cudaStream_t stream) {
    I8R_TRY(check_shape(T, K, 0, false));
    if (std::isnan(alpha) || alpha < 0.0f) return I8R_EINVAL;
    if (T > 0) {
        I8R_TRY(check_ptr(X));
        I8R_TRY(check_ptr(sX));
        I8R_TRY(check_ptr(Xq));
        if (Xo) I8R_TRY(check_ptr(Xo));
    }
    I8R_TRY(check_ptr(mask));
    I8R_TRY(check_ptr(idx));
    if (!count) return I8R_EINVAL;
    if (!workspace || workspace_bytes < kAlign) return I8R_EWORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) % 16) return I8R_EALIGN;
    const DeviceInfo *dev = nullptr;
    I8R_TRY(device_setup(&dev));
    return launch_activation(dev, static_cast<const __half *>(X), T, K, alpha, mask, idx, count, sX, Xq,
                             static_cast<__half *>(Xo), nullptr, 0, stream, nullptr, 0, nullptr, nullptr, nullptr,
                             static_cast<unsigned *>(workspace));
}

size_t int8_gemm_i8_s32_workspace_size(int T, int K, int N) {
    (void)T;
    (void)K;
    (void)N;
    return 0;
}

i8r_status int8_gemm_i8_s32(const int8_t *Xq, int T, int K, const int8_t *Wq, int N, int32_t *acc, void *workspace,
                            size_t workspace_bytes, cudaStream_t stream) {
    (void)workspace;
    (void)workspace_bytes;
    I8R_TRY(check_shape(T, K, N, true));
    if (T == 0) return I8R_OK;
    I8R_TRY(check_ptr(Xq));
    I8R_TRY(check_ptr(Wq));
    I8R_TRY(check_ptr(acc));
    const DeviceInfo *dev = nullptr;
    I8R_TRY(device_setup(&dev));
    if (T > decode::MAX_T)
        return launch_prefill(dev, Xq, nullptr, T, K, Wq, nullptr, nullptr, N, nullptr, nullptr, nullptr, nullptr,
                              acc, stream);
    const size_t n16 = static_cast<size_t>(T) * N / 4;
    zero_kernel<<<dev->sms * 4, 256, 0, stream>>>(reinterpret_cast<int4 *>(acc), n16);
    I8R_LAUNCHED();
    return launch_decode(dev, Xq, T, K, Wq, N, acc, nullptr, stream);
}

size_t int4_packed_code_bytes(int K, int N) {
    if (check_int4_shape(K, N) != I8R_OK) return 0;
    return w4::code_bytes(K, N);
}

size_t int4_packed_scale_bytes(int K, int N) {
    if (check_int4_shape(K, N) != I8R_OK) return 0;
    return w4::scale_bytes(K, N);
}

i8r_status int4_quantize_weight_groupwise(const void *W16, int K, int N, uint8_t *W4, void *S4, cudaStream_t stream) {
    I8R_TRY(check_int4_shape(K, N));
    I8R_TRY(check_ptr(W16));
    I8R_TRY(check_ptr(W4));
    I8R_TRY(check_ptr(S4));
    const DeviceInfo *dev = nullptr;
    I8R_TRY(device_setup(&dev));
    const dim3 grid(static_cast<unsigned>(w4::padded_n(N) / 256), static_cast<unsigned>(K / w4::G));
    w4::int4_pack_kernel<<<grid, 256, 0, stream>>>(static_cast<const __half *>(W16), K, N, W4,
                                                     static_cast<uint8_t *>(S4));
    I8R_LAUNCHED();
    return I8R_OK;
}

i8r_status int4_dequantize_weight(const uint8_t *W4, const void *S4, int K, int N, void *W16d, cudaStream_t stream) {
    I8R_TRY(check_int4_shape(K, N));
    I8R_TRY(check_ptr(W4));
    I8R_TRY(check_ptr(S4));
    I8R_TRY(check_ptr(W16d));
    const DeviceInfo *dev = nullptr;
    I8R_TRY(device_setup(&dev));
    const dim3 grid(static_cast<unsigned>((N + 255) / 256), static_cast<unsigned>(K / w4::G));
    w4::int4_unpack_kernel<<<grid, 256, 0, stream>>>(W4, static_cast<const uint8_t *>(S4), K, N,
                                                       static_cast<__half *>(W16d));
    I8R_LAUNCHED();
    return I8R_OK;
}

size_t int4_linear_workspace_size(int T, int K, int N) {
    if (T < 0 || T > w4::MAX_T || check_int4_shape(K, N) != I8R_OK) return 0;
    return int4_ws_layout(T, N).total;
}

i8r_status int4_linear(const void *X, int T, int K, const uint8_t *W4, const void *S4, int N, void *Y,
                       void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    I8R_TRY(check_int4_shape(K, N));
    if (T < 0) return I8R_EINVAL;
    if (T > w4::MAX_T) return I8R_ERANGE;
    if (T == 0) return I8R_OK;
    I8R_TRY(check_ptr(X));
    I8R_TRY(check_ptr(W4));
    I8R_TRY(check_ptr(S4));
    I8R_TRY(check_ptr(Y));
    const Int4Workspace w = int4_ws_layout(T, N);
    if (!workspace || workspace_bytes < w.total) return I8R_EWORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return I8R_EALIGN;
    const DeviceInfo *dev = nullptr;
    I8R_TRY(device_setup(&dev));

    w4::Params p{};
    p.T = T;
    p.TP = (T + 15) / 16 * 16;
    p.K = K;
    p.N = N;
    p.KB = K / w4::BK;
    p.num_tiles = w4::padded_n(N) / w4::BN;
    p.total_units = static_cast<long long>(p.num_tiles) * p.KB;
    p.stage_bytes = w4::CODE_BYTES + w4::SCALE_BYTES + 4 * p.TP * 128;
    p.stages = static_cast<int>(w4::SMEM_BUDGET / p.stage_bytes);
    if (p.stages > w4::MAX_STAGES) p.stages = w4::MAX_STAGES;
    p.na = (w4::MAX_NA * w4::KSUB + 4 * p.TP <= static_cast<int>(w4::TMEM_COLS)) ? w4::MAX_NA : 2;
    p.W4 = W4;
    p.S4 = static_cast<const uint8_t *>(S4);
    p.Y = static_cast<__half *>(Y);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    p.part = reinterpret_cast<float *>(ws + w.part);
    p.counters = reinterpret_cast<int *>(ws + w.counters);
    const int ncount = p.num_tiles * w4::COUNTERS_PER_TILE;
    const long long g = std::min<long long>(p.total_units, std::min(dev->sms, w4::MAX_CTAS));
    const int path = g_int4_path.load(std::memory_order_relaxed);
    const bool small = path == 2 ? T <= w4::SMALL_T : (path == 0 && T <= kInt4SmallRows);
    cudaError_t e;
    if (small) {
        // the CUDA-core product: a stage is the codes, the scales and T slices of X
        p.stage_bytes = w4::small_stage_bytes(T);
        p.stages = w4::small_stages(T);
        w4::int4_clear_kernel<<<(ncount + 255) / 256, 256, 0, stream>>>(p.counters, ncount);
        I8R_LAUNCHED();
        record_before(stream);
        e = launch_int4_small(T, static_cast<unsigned>(g), static_cast<const __half *>(X), p, stream);
    } else {
        CUtensorMap map_x;
        I8R_TRY(make_map(&map_x, X, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, T, K, p.TP, 64));
        w4::int4_clear_kernel<<<(ncount + 255) / 256, 256, 0, stream>>>(p.counters, ncount);
        I8R_LAUNCHED();
        record_before(stream);
        e = launch_dependent(w4::gemm_int4_decode_kernel, dim3(static_cast<unsigned>(g)), dim3(w4::THREADS),
                             w4::smem_bytes(p.stages, p.stage_bytes), stream, 1, map_x, p);
    }
    if (e != cudaSuccess) {
        tl_last_cuda_error = static_cast<int>(e);
        return I8R_ECUDA;
    }
    I8R_LAUNCHED();
    record_after(stream);
    return I8R_OK;
}

i8r_status int8_read_and_clear_device_status(int *code, cudaStream_t stream) {
    if (!code) return I8R_EINVAL;
    I8R_CUDA(cudaStreamSynchronize(stream));
    int v = 0;
    I8R_CUDA(cudaMemcpyFromSymbol(&v, i8r::g_device_status, sizeof(int)));
    const int zero = 0;
    I8R_CUDA(cudaMemcpyToSymbol(i8r::g_device_status, &zero, sizeof(int)));
    *code = v;
    return I8R_OK;
}

const char *int8_status_string(i8r_status status) {
    switch (status) {
        case I8R_OK: return "ok";
        case I8R_EINVAL: return "invalid argument (null pointer, negative size, NaN or negative alpha)";
        case I8R_EALIGN: return "misaligned pointer, or K / N not a multiple of 16";
        case I8R_ERANGE: return "size out of range (16 <= K <= 133144, N >= 16)";
        case I8R_EWORKSPACE: return "workspace missing or too small";
        case I8R_ECUDA: return "CUDA error (see int8_last_cuda_error)";
        case I8R_EDEVICE: return "a kernel reported an anomaly in the device status word";
        case I8R_EARCH: return "current device is not sm_100 (B200)";
    }
    return "unknown status";
}

i8r_status int8_selftest_wait_timeout(int limit_us, cudaStream_t stream) {
    if (limit_us < 1 || limit_us > 1000000) return I8R_ERANGE;
    const DeviceInfo *dev = nullptr;
    I8R_TRY(device_setup(&dev));
    wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(static_cast<uint64_t>(limit_us) * 1000u);
    I8R_LAUNCHED();
    return I8R_OK;
}

int int8_last_cuda_error(void) { return tl_last_cuda_error; }

void int8_time_next_gemm(cudaEvent_t before, cudaEvent_t after) {
    tl_ev_before = before;
    tl_ev_after = after;
}

uint64_t int8_kernel_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
