// libw8a16.so: the C ABI declared in include/w8a16.h.  Host code only
// validates arguments, builds TMA tensor maps and launches the kernels in
// quantize.cuh, prepack.cuh, decode.cuh and prefill2.cuh on the caller's
// stream.  Nothing here allocates device memory or synchronizes (except the
// w8_device_status diagnostic).
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <climits>
#include <map>
#include <mutex>
#include <utility>

#include "../../include/w8a16.h"
#include "common.cuh"
#include "decode.cuh"
#include "prefill2.cuh"
#include "prepack.cuh"
#include "quantize.cuh"
#include "clip.cuh"

namespace {

using namespace w8;

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool ready = false;
    int status = W8_OK;   // W8_ERR_DEVICE if not sm_100
    int sms = 0;
    int pairs = 0;   // resident prefill CTA pairs (0 = not yet queried)
    // resident quantize clusters per cluster size (0 = not yet queried)
    int qclusters_f32[quant::kMaxCluster + 1] = {};
    int qclusters_f16[quant::kMaxCluster + 1] = {};
    int qclusters_asym_f32[quant::kMaxCluster + 1] = {};
    int qclusters_asym_f16[quant::kMaxCluster + 1] = {};
    // resident clusters of the decode kernel's cluster form, by (kernel,
    // cluster size) (0 = not yet queried)
    std::map<std::pair<const void *, int>, int> dclusters;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

// A failed runtime call: clear the pending (non-sticky) error so that the
// caller's next, unrelated CUDA call does not report it, and say so.
inline int cuda_fail() {
    cudaGetLastError();
    return W8_ERR_CUDA;
}

// Per-device one-time setup: architecture check, SM count, kernel attributes.
int device_info(DeviceInfo **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cuda_fail();
    if (dev < 0 || dev >= kMaxDevices) return W8_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceInfo &d = g_dev[dev];
    if (!d.ready) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return cuda_fail();
        d.sms = sms;
        d.status = (major == 10 && minor == 0) ? W8_OK : W8_ERR_DEVICE;
        if (d.status == W8_OK) {
            cudaError_t e = cudaSuccess;
            auto smem = [&e](const void *fn, int bytes) {
                if (e == cudaSuccess) e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
            };
            smem((const void *)decode::decode_kernel<1, false>, decode::Cfg<1>::kSmemBytes);
            smem((const void *)decode::decode_kernel<2, false>, decode::Cfg<2>::kSmemBytes);
            smem((const void *)decode::decode_kernel<4, false>, decode::Cfg<4>::kSmemBytes);
            smem((const void *)decode::decode_kernel<8, false>, decode::Cfg<8>::kSmemBytes);
            smem((const void *)decode::decode_kernel<1, true>, decode::Cfg<1>::kSmemBytes);
            smem((const void *)decode::decode_kernel<1, false, true>, decode::Cfg<1>::kSmemBytesCluster);
            smem((const void *)decode::decode_kernel<2, false, true>, decode::Cfg<2>::kSmemBytesCluster);
            smem((const void *)decode::decode_kernel<1, true, true>, decode::Cfg<1>::kSmemBytesCluster);
            smem((const void *)decode::decode_kernel<2, true, true>, decode::Cfg<2>::kSmemBytesCluster);
            smem((const void *)decode::decode_kernel<2, true>, decode::Cfg<2>::kSmemBytes);
            smem((const void *)decode::decode_kernel<4, true>, decode::Cfg<4>::kSmemBytes);
            smem((const void *)decode::decode_kernel<8, true>, decode::Cfg<8>::kSmemBytes);
            smem((const void *)prefill2::prefill2_kernel<false, prefill2::kSym>, prefill2::kSmemBytes);
            smem((const void *)prefill2::prefill2_kernel<true, prefill2::kSym>, prefill2::kSmemBytes);
            smem((const void *)prefill2::prefill2_kernel<false, prefill2::kZeroPoint>, prefill2::kSmemBytes);
            smem((const void *)prefill2::prefill2_kernel<true, prefill2::kZeroPoint>, prefill2::kSmemBytes);
            smem((const void *)prefill2::prefill2_kernel<false, prefill2::kOutliers>, prefill2::kSmemBytes);
#define W8_Q_SMEM(T, A, CAP)                                                                                  \
    smem((const void *)quant::quantize_kernel<T, A, CAP, true>, quant::kSmemBytes);                          \
    smem((const void *)quant::quantize_kernel<T, A, CAP, false>, quant::kSmemBytes);
            W8_Q_SMEM(float, false, 1)
            W8_Q_SMEM(__half, false, 1)
            W8_Q_SMEM(float, true, 1)
            W8_Q_SMEM(__half, true, 1)
            W8_Q_SMEM(float, false, quant::kMaxBatch)
            W8_Q_SMEM(__half, false, quant::kMaxBatch)
#undef W8_Q_SMEM
            smem((const void *)clip::percentile_quantize_kernel<float, false>, clip::kSmemBytes);
            smem((const void *)clip::percentile_quantize_kernel<__half, false>, clip::kSmemBytes);
            smem((const void *)clip::percentile_quantize_kernel<float, true>, clip::kSmemBytes);
            smem((const void *)clip::percentile_quantize_kernel<__half, true>, clip::kSmemBytes);
            if (e != cudaSuccess) return cuda_fail();
        }
        d.ready = true;
    }
    *out = &d;
    return d.status;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}

// 2-D row-major tensor [rows, cols] of `elem`-byte elements.
int make_map_2d(CUtensorMap *map, const void *ptr, CUtensorMapDataType dtype, int elem, uint64_t cols,
                uint64_t rows, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
    auto fn = encode_fn();
    if (!fn) return W8_ERR_CUDA;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * (uint64_t)elem};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dtype, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? W8_OK : W8_ERR_CUDA;
}

// X [M, K] fp16 viewed as [K/64][M][64] (K % 64 == 0): dims {64, M, K/64},
// strides {2K, 128} bytes, box {64, rows, 4}, 128-byte swizzle.  The image
// of a box is four consecutive [rows][64] slices, each swizzled as a 2-D
// box of one slice would be.  Returns false if the driver declines it.
bool make_map_x3(CUtensorMap *map, const void *X, uint64_t M, uint64_t K, uint32_t rows) {
    auto fn = encode_fn();
    if (!fn || K % 64 != 0) return false;
    cuuint64_t dims[3] = {64, M, K / 64};
    cuuint64_t strides[2] = {K * 2, 128};
    cuuint32_t box[3] = {64, rows, 4};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void *>(X), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool overlap(const void *a, size_t an, const void *b, size_t bn) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return an && bn && x < y + bn && y < x + an;
}

inline int launch_status() {
    return cudaGetLastError() == cudaSuccess ? W8_OK : W8_ERR_CUDA;
}

inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ---------------------------------------------------------------- quantize
// Cluster size for K rows: the K range is split C ways so that the rows all
// CTAs hold between their two passes (two slices of K/C rows x 128 B per
// SM) stay well inside L2, so that small matrices still spread over the
// SMs, and -- clusters of 8 leave a sixth of the SMs idle on this part --
// preferring 4 where that suffices.
inline int quantize_cluster(int64_t K, int rows_per_box) {
    if (K > 8192) return quant::kMaxCluster;
    return (int)std::max<int64_t>(1, std::min<int64_t>(4, cdiv(K, 2 * rows_per_box)));
}

// A batch of up to quant::kMaxBatch weights in one launch (one weight is a
// batch of one).  The cluster size follows the largest K.
template <typename T, bool kAsym, int kCap>
int launch_quantize(DeviceInfo *d, int count, const void *const *W, CUtensorMapDataType dt, const int64_t *K,
                    const int64_t *N, int8_t *const *q, uint16_t *const *scales, int8_t *const *zeros,
                    float clip_bound, cudaStream_t st) {
    constexpr int rows = quant::Box<T>::kRows;
    int64_t kmax = 1;
    for (int i = 0; i < count; ++i) kmax = std::max(kmax, K[i]);
    const int C = quantize_cluster(kmax, rows);
    static thread_local quant::Params<kCap> p;   // up to about 12 KB: not on the stack
    if (count > kCap) return W8_ERR_SHAPE;
    memset(&p, 0, sizeof(p));
    int64_t panels = 0;
    for (int i = 0; i < count; ++i) {
        const int64_t kc = cdiv(cdiv(K[i], C), rows) * rows;
        if (kc > INT32_MAX) return W8_ERR_SHAPE;
        int rc = make_map_2d(&p.maps[i], W[i], dt, (int)sizeof(T), (uint64_t)N[i], (uint64_t)K[i], quant::kPanel,
                             quant::Box<T>::kTmaRows, CU_TENSOR_MAP_SWIZZLE_NONE);
        if (rc != W8_OK) return rc;
        p.mats[i].q = q[i];
        p.mats[i].scales = scales[i];
        p.mats[i].zeros = zeros ? zeros[i] : nullptr;
        p.mats[i].K = K[i];
        p.mats[i].N = N[i];
        p.mats[i].kc = (int)kc;
        p.mats[i].panel0 = (int)panels;
        panels += cdiv(N[i], quant::kPanel);
        if (panels > INT32_MAX) return W8_ERR_SHAPE;
    }
    p.count = count;
    p.panels = (int)panels;
    p.clip = clip_bound;
    if (panels == 0) return W8_OK;

    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(quant::kThreads, 1, 1);
    cfg.dynamicSmemBytes = quant::kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // persistent clusters: as many as can be resident at once
    int resident = 0;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        int &cached = kAsym ? (sizeof(T) == 4 ? d->qclusters_asym_f32[C] : d->qclusters_asym_f16[C])
                            : (sizeof(T) == 4 ? d->qclusters_f32[C] : d->qclusters_f16[C]);
        if (cached == 0) {
            cfg.gridDim = dim3((unsigned)(C * d->sms), 1, 1);
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, quant::quantize_kernel<T, kAsym, kCap, true>, &cfg) !=
                    cudaSuccess ||
                n < 1) {
                cudaGetLastError();
                n = std::max(1, d->sms / C);
            }
            cached = n;
        }
        resident = cached;
    }
    p.clusters = (int)std::min<int64_t>(panels, resident);
    cfg.gridDim = dim3((unsigned)(p.clusters * C), 1, 1);
    // clusters of 8 (tall weights): each panel's passes back to back
    const cudaError_t le = C == quant::kMaxCluster ? cudaLaunchKernelEx(&cfg, quant::quantize_kernel<T, kAsym, kCap, false>, p)
                                                   : cudaLaunchKernelEx(&cfg, quant::quantize_kernel<T, kAsym, kCap, true>, p);
    if (le != cudaSuccess) {
        cudaGetLastError();
        return W8_ERR_CUDA;
    }
    return launch_status();
}

// Programmatic dependent launch: this kernel's prologue and an L2 prefetch
// of its first weight tiles overlap the previous kernel in the stream.
// csz > 0: the cluster form, p.G CTAs in clusters of csz.
template <int MT, bool kZp, bool kCl>
int launch_decode(const CUtensorMap &map, const decode::Params &p, cudaStream_t st, int csz) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.G, 1, 1);
    cfg.blockDim = dim3(decode::kThreads, 1, 1);
    cfg.dynamicSmemBytes = kCl ? decode::Cfg<MT>::kSmemBytesCluster : decode::Cfg<MT>::kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = kCl ? csz : 1;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = kCl ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, decode::decode_kernel<MT, kZp, kCl>, map, p) != cudaSuccess) return cuda_fail();
    return launch_status();
}

// Clusters of `csz` CTAs of the decode kernel's cluster form that can be
// resident at once (cached per device).
template <int MT, bool kZp>
int decode_resident_clusters(DeviceInfo *d, int csz) {
    const void *fn = (const void *)decode::decode_kernel<MT, kZp, true>;
    std::lock_guard<std::mutex> lock(g_mu);
    int &cached = d->dclusters[{fn, csz}];
    if (cached == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(csz * d->sms), 1, 1);
        cfg.blockDim = dim3(decode::kThreads, 1, 1);
        cfg.dynamicSmemBytes = decode::Cfg<MT>::kSmemBytesCluster;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = csz;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, decode::decode_kernel<MT, kZp, true>, &cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
        cached = n > 0 ? n : -1;
    }
    return cached;
}

// Cluster size for the cluster form of the decode kernel, 0 for the
// stream-K form.  The cluster form pays off when the channel blocks are
// few: one cluster per block, as many CTAs per block as keep every cluster
// resident at once (one wave), each with at least one K block, and enough
// CTAs in all to keep HBM busy.
#ifndef W8_DECODE_CLUSTER_MIN_FILL
#define W8_DECODE_CLUSTER_MIN_FILL 0.7
#endif
template <int MT, bool kZp>
int decode_cluster_size(DeviceInfo *d, int64_t NB, int64_t KB) {
    if constexpr (MT > 2) {
        return 0;
    } else {
        for (int c = (int)std::min<int64_t>(decode::kMaxClusterDec, d->sms / std::max<int64_t>(NB, 1)); c >= 2;
             --c) {
            if (c > KB) continue;
            if (decode_resident_clusters<MT, kZp>(d, c) < NB) continue;
            return (double)(NB * c) >= W8_DECODE_CLUSTER_MIN_FILL * d->sms ? c : 0;
        }
        return 0;
    }
}

// The decode path of both entry points (w8a16_linear with a workspace,
// w8a16_linear_decode_static with the static scratch): the same kernel and
// split for the same shape, so the two give the same bits.  p holds
// everything but the split (T, G) and the scratch pointers' use.
template <int MT, bool kZp>
int launch_decode_any(DeviceInfo *d, const CUtensorMap &map, decode::Params p, int64_t NB, cudaStream_t st) {
    const int csz = decode_cluster_size<MT, kZp>(d, NB, p.KB);
    const int64_t T = NB * p.KB;
    if (csz > 0) {
        if constexpr (MT <= 2) {
            p.T = (uint32_t)T;
            p.G = (uint32_t)(NB * csz);
            return launch_decode<MT, kZp, true>(map, p, st, csz);
        }
    }
    const int G = (int)std::max<int64_t>(1, std::min<int64_t>(T, d->sms));
    if ((uint64_t)T * (uint64_t)(G + 1) >= (1ull << 32)) return W8_ERR_SHAPE;
    p.T = (uint32_t)T;
    p.G = (uint32_t)G;
    return launch_decode<MT, kZp, false>(map, p, st, 0);
}

// Percentile clip (clip.cuh): one persistent CTA per SM, panels of 32
// columns; t = K - r + 1 with r = clamp(ceil(p K), 1, K) in IEEE double.
int64_t percentile_rank(int64_t K, double pct) {
    const double rr = std::ceil(pct * (double)K);
    return rr < 1.0 ? 1 : (rr > (double)K ? K : (int64_t)rr);
}

template <typename T, bool kOut>
int launch_percentile(DeviceInfo *d, const void *W, CUtensorMapDataType dt, int64_t K, int64_t N, double pct,
                      int8_t *q, uint16_t *scales, int32_t *o_count, int32_t *o_rows, uint16_t *o_vals,
                      cudaStream_t st) {
    const int64_t r = percentile_rank(K, pct);
    const int64_t panels = cdiv(N, clip::kPanel);
    if (panels > INT32_MAX || K > INT32_MAX) return W8_ERR_SHAPE;
    CUtensorMap map;
    int rc = make_map_2d(&map, W, dt, (int)sizeof(T), (uint64_t)N, (uint64_t)K, clip::kPanel,
                         clip::Geo<T>::kRows, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc != W8_OK) return rc;
    clip::Params p;
    p.q = q;
    p.scales = scales;
    p.K = K;
    p.N = N;
    p.t = (int)(K - r + 1);
    p.panels = (int)panels;
    p.o_count = o_count;
    p.o_rows = o_rows;
    p.o_vals = o_vals;
    p.cap = (int)(K - r);
    const int grid = (int)std::min<int64_t>(panels, d->sms);
    clip::percentile_quantize_kernel<T, kOut><<<grid, clip::kThreads, clip::kSmemBytes, st>>>(map, p);
    return launch_status();
}

// Tensor-core linear for M > 64 on CTA pairs (prefill2.cuh).
// Outlier side list of a linear call (all null when there is none).
struct Outliers {
    const int32_t *count = nullptr;
    const int32_t *rows = nullptr;
    const uint16_t *vals = nullptr;
    int64_t cap = 0;
    uint16_t *xt = nullptr;   // workspace for X^T (tensor-core path)
};

int launch_prefill2(DeviceInfo *d, const uint16_t *X, const uint8_t *packed, const uint16_t *scales,
                    const int8_t *zeros, const uint16_t *bias, uint16_t *Y, int64_t M, int64_t K, int64_t N,
                    float *partials, int *counters, const Outliers &o, cudaStream_t st) {
    CUtensorMap map;
    int rc = make_map_2d(&map, X, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)K, (uint64_t)M, 64,
                         prefill2::kBTc, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != W8_OK) return rc;
    prefill2::Params p;
    p.packed = packed;
    p.scales = scales;
    p.zeros = zeros;
    p.bias = bias;
    p.Y = Y;
    p.partials = partials;
    p.counters = counters;
    p.M = (int)M;
    p.N = N;
    p.NB = (int)cdiv(N, 128);
    p.KB = (int)cdiv(K, 64);
    p.KS = (int)cdiv(p.KB, prefill2::kKStep);
    p.TT = (int)cdiv(M, prefill2::kBT);
    const int64_t tiles = cdiv(p.NB, 2) * p.TT;
    // 32-bit work counts (a 2^31-tile output would not fit in device memory)
    if (tiles >= INT32_MAX / 2 || (int64_t)p.KS * 2 * d->sms >= INT32_MAX) return W8_ERR_SHAPE;
    p.tiles = (int)tiles;
    p.XT = o.xt;
    p.Mp = cdiv(M, prefill2::kBT) * prefill2::kBT;
    p.o_count = o.count;
    p.o_rows = o.rows;
    p.o_vals = o.vals;
    p.o_cap = (int)o.cap;
    p.o_extra = partials;   // no K split with outliers: the partial-sum area is free
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(prefill2::kThreads, 1, 1);
    cfg.dynamicSmemBytes = prefill2::kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // programmatic dependent launch: the prologue overlaps the previous
    // kernel's tail (the kernel waits before every global access)
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;   // the occupancy query takes the cluster shape only
    int resident = 0;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (d->pairs == 0) {
            cfg.gridDim = dim3((unsigned)d->sms, 1, 1);
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, prefill2::prefill2_kernel<false, prefill2::kSym>, &cfg) !=
                    cudaSuccess ||
                n < 1) {
                cudaGetLastError();
                n = d->sms / 2;
            }
            d->pairs = n;
        }
        resident = d->pairs;
    }
    // Schedule (prefill2.cuh).  Whole tiles round robin over the pairs,
    // unless splitting the last waves' K steps over all pairs saves at least
    // kSplitMinSteps 256-wide K steps per pair: a split tile's fix-up
    // (partial sums written, counted, read back and added) costs 20-40 us
    // on the critical path, measured, against about 1.65 us per K step.
    // That holds for long K with few tiles (e.g. 13696 x 4096 with M up to
    // 512).  The pair count never exceeds half the SMs (the workspace's
    // partial-sum slots).
    constexpr int64_t kSplitMinSteps = 24;
    const int P = std::max(1, std::min(resident, d->sms / 2));
    int pairs = std::min(P, p.tiles), sk_tiles = 0, split_pairs = P;
    if (p.tiles >= P) {
        if (p.tiles % P != 0 && p.KS > 1) sk_tiles = P + p.tiles % P;
    } else if (p.KS > 1) {
        sk_tiles = p.tiles;
        split_pairs = (int)std::min<int64_t>(P, (int64_t)p.tiles * p.KS);   // at least one K step each
    }
    bool split = false;
    if (sk_tiles > 0 && !o.count) {
        const int64_t whole_steps = cdiv(p.tiles, P) * p.KS;
        const int64_t split_steps =
            (int64_t)((p.tiles - sk_tiles) / P) * p.KS + cdiv((int64_t)sk_tiles * p.KS, split_pairs);
        split = whole_steps - split_steps >= kSplitMinSteps;
    }
    if (split) {
        pairs = split_pairs;
        p.dp_tiles = p.tiles - sk_tiles;
        p.sk_iters = sk_tiles * p.KS;   // < 2 P KS
    } else {
        p.dp_tiles = p.tiles;
        p.sk_iters = 0;
    }
    cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
    cfg.numAttrs = 2;
    using namespace prefill2;
    cudaError_t e;
    if (o.count) {
        // X^T for the epilogue's outlier term, on the same stream first
        const dim3 tgrid((unsigned)cdiv(K, 32), (unsigned)(p.Mp / 32), 1);
        transpose_x_kernel<<<tgrid, dim3(32, 8, 1), 0, st>>>(X, o.xt, (int)M, K, p.Mp);
        e = cudaGetLastError();
        if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, prefill2_kernel<false, kOutliers>, map, p);
    } else if (zeros) {
        e = split ? cudaLaunchKernelEx(&cfg, prefill2_kernel<true, kZeroPoint>, map, p)
                  : cudaLaunchKernelEx(&cfg, prefill2_kernel<false, kZeroPoint>, map, p);
    } else {
        e = split ? cudaLaunchKernelEx(&cfg, prefill2_kernel<true, kSym>, map, p)
                  : cudaLaunchKernelEx(&cfg, prefill2_kernel<false, kSym>, map, p);
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        return W8_ERR_CUDA;
    }
    return launch_status();
}

}  // namespace

extern "C" {

int w8_version(void) { return 100; }

const char *w8_error_string(int status) {
    switch (status) {
        case W8_OK: return "ok";
        case W8_ERR_NULL: return "a required pointer is NULL";
        case W8_ERR_SHAPE: return "a size is out of range or not a multiple of 8";
        case W8_ERR_ALIGN: return "a device pointer is not 16-byte aligned";
        case W8_ERR_DTYPE: return "unknown weight dtype";
        case W8_ERR_WORKSPACE: return "workspace missing or too small";
        case W8_ERR_CUDA: return "CUDA runtime call or kernel launch failed";
        case W8_ERR_TIMEOUT: return "a bounded device wait ran out";
        case W8_ERR_ALIAS: return "output overlaps an input";
        case W8_ERR_DEVICE: return "current device is not sm_100 (B200)";
        case W8_ERR_LIMIT:
            return "size beyond the fixed scratch of w8a16_linear_decode_static "
                   "(needs 1 <= M <= 16, N <= 2^20, at most 160 SMs)";
        default: return "unknown status";
    }
}

// Both quantization forms: zeros == nullptr selects the symmetric one.
static int quantize_common(const void *W, int w_dtype, int64_t K, int64_t N, int8_t *q, uint16_t *scales,
                           int8_t *zeros, bool asym, void *stream, float clip_bound = INFINITY,
                           double percentile = 0.0) {
    if (w_dtype != W8_F32 && w_dtype != W8_F16) return W8_ERR_DTYPE;
    if (K < 1 || N < 0 || N % 8 != 0 || K > (int64_t)INT32_MAX || N > (int64_t)INT32_MAX * 8)
        return W8_ERR_SHAPE;
    if (N == 0) return W8_OK;   // nothing to read or write: pointers may be NULL
    if (!W || !q || !scales || (asym && !zeros)) return W8_ERR_NULL;
    if (!aligned16(W) || !aligned16(q) || !aligned16(scales)) return W8_ERR_ALIGN;
    const size_t welem = w_dtype == W8_F32 ? 4 : 2;
    if (overlap(W, (size_t)K * N * welem, q, (size_t)K * N) ||
        overlap(W, (size_t)K * N * welem, scales, (size_t)N * 2) ||
        overlap(q, (size_t)K * N, scales, (size_t)N * 2))
        return W8_ERR_ALIAS;
    if (asym && (overlap(zeros, (size_t)N, W, (size_t)K * N * welem) || overlap(zeros, (size_t)N, q, (size_t)K * N) ||
                 overlap(zeros, (size_t)N, scales, (size_t)N * 2)))
        return W8_ERR_ALIAS;
    DeviceInfo *d = nullptr;
    int rc = device_info(&d);
    if (rc != W8_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (percentile > 0.0) {
        if (w_dtype == W8_F32)
            return launch_percentile<float, false>(d, W, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, K, N, percentile, q,
                                                   scales, nullptr, nullptr, nullptr, st);
        return launch_percentile<__half, false>(d, W, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, K, N, percentile, q,
                                                scales, nullptr, nullptr, nullptr, st);
    }
    if (asym) {
        if (w_dtype == W8_F32)
            return launch_quantize<float, true, 1>(d, 1, &W, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, &K, &N, &q, &scales,
                                                &zeros, INFINITY, st);
        return launch_quantize<__half, true, 1>(d, 1, &W, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, &K, &N, &q, &scales,
                                             &zeros, INFINITY, st);
    }
    if (w_dtype == W8_F32)
        return launch_quantize<float, false, 1>(d, 1, &W, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, &K, &N, &q, &scales,
                                             nullptr, clip_bound, st);
    return launch_quantize<__half, false, 1>(d, 1, &W, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, &K, &N, &q, &scales,
                                          nullptr, clip_bound, st);
}

int w8_quantize_per_channel(const void *W, int w_dtype, int64_t K, int64_t N, int8_t *q,
                            uint16_t *scales, void *stream) {
    return quantize_common(W, w_dtype, K, N, q, scales, nullptr, false, stream);
}

int w8_quantize_per_channel_asym(const void *W, int w_dtype, int64_t K, int64_t N, int8_t *q,
                                 uint16_t *scales, int8_t *zeros, void *stream) {
    return quantize_common(W, w_dtype, K, N, q, scales, zeros, true, stream);
}

int w8_quantize_per_channel_batched(int count, const void *const *W, int w_dtype, const int64_t *K,
                                    const int64_t *N, int8_t *const *q, uint16_t *const *scales, void *stream) {
    if (count < 0) return W8_ERR_SHAPE;
    if (count == 0) return W8_OK;
    if (!W || !K || !N || !q || !scales) return W8_ERR_NULL;
    if (w_dtype != W8_F32 && w_dtype != W8_F16) return W8_ERR_DTYPE;
    const size_t welem = w_dtype == W8_F32 ? 4 : 2;
    for (int i = 0; i < count; ++i) {
        if (K[i] < 1 || N[i] < 0 || N[i] % 8 != 0 || K[i] > (int64_t)INT32_MAX || N[i] > (int64_t)INT32_MAX * 8)
            return W8_ERR_SHAPE;
        if (N[i] == 0) continue;
        if (!W[i] || !q[i] || !scales[i]) return W8_ERR_NULL;
        if (!aligned16(W[i]) || !aligned16(q[i]) || !aligned16(scales[i])) return W8_ERR_ALIGN;
    }
    // no output overlaps any weight or any other output
    for (int i = 0; i < count; ++i) {
        if (N[i] == 0) continue;
        const size_t qb = (size_t)K[i] * N[i], sb = (size_t)N[i] * 2;
        if (overlap(q[i], qb, scales[i], sb)) return W8_ERR_ALIAS;
        for (int j = 0; j < count; ++j) {
            if (N[j] == 0) continue;
            const size_t wb = (size_t)K[j] * N[j] * welem;
            if (overlap(q[i], qb, W[j], wb) || overlap(scales[i], sb, W[j], wb)) return W8_ERR_ALIAS;
            if (j != i && (overlap(q[i], qb, q[j], (size_t)K[j] * N[j]) ||
                           overlap(scales[i], sb, scales[j], (size_t)N[j] * 2) ||
                           overlap(q[i], qb, scales[j], (size_t)N[j] * 2)))
                return W8_ERR_ALIAS;
        }
    }
    DeviceInfo *d = nullptr;
    int rc = device_info(&d);
    if (rc != W8_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    for (int i0 = 0; i0 < count; i0 += quant::kMaxBatch) {
        // the weights with N > 0 of this chunk, in order
        const void *w[quant::kMaxBatch];
        int64_t k[quant::kMaxBatch], n[quant::kMaxBatch];
        int8_t *qq[quant::kMaxBatch];
        uint16_t *ss[quant::kMaxBatch];
        int cnt = 0;
        for (int i = i0; i < count && i < i0 + quant::kMaxBatch; ++i) {
            if (N[i] == 0) continue;
            w[cnt] = W[i];
            k[cnt] = K[i];
            n[cnt] = N[i];
            qq[cnt] = q[i];
            ss[cnt] = scales[i];
            ++cnt;
        }
        if (cnt == 0) continue;
        rc = w_dtype == W8_F32
                 ? launch_quantize<float, false, quant::kMaxBatch>(d, cnt, w, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, k, n, qq, ss, nullptr,
                                                 INFINITY, st)
                 : launch_quantize<__half, false, quant::kMaxBatch>(d, cnt, w, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, k, n, qq, ss, nullptr,
                                                  INFINITY, st);
        if (rc != W8_OK) return rc;
    }
    return W8_OK;
}

size_t w8_outlier_capacity(int64_t K, double p) {
    if (K < 1 || !(p > 0.0 && p <= 1.0)) return 0;
    return (size_t)(K - percentile_rank(K, p));
}

int w8_quantize_per_channel_outliers(const void *W, int w_dtype, int64_t K, int64_t N, double p, int8_t *q,
                                     uint16_t *scales, int32_t *o_count, int32_t *o_rows, uint16_t *o_vals,
                                     void *stream) {
    if (w_dtype != W8_F32 && w_dtype != W8_F16) return W8_ERR_DTYPE;
    if (K < 1 || N < 0 || N % 8 != 0 || K > (int64_t)INT32_MAX || N > (int64_t)INT32_MAX * 8 ||
        !(p > 0.0 && p <= 1.0))
        return W8_ERR_SHAPE;
    const int64_t cap = K - percentile_rank(K, p);
    if (cap > clip::kMaxOutliers) return W8_ERR_LIMIT;
    if (N == 0) return W8_OK;
    if (!W || !q || !scales || !o_count || (cap > 0 && (!o_rows || !o_vals))) return W8_ERR_NULL;
    if (!aligned16(W) || !aligned16(q) || !aligned16(scales)) return W8_ERR_ALIGN;
    const size_t welem = w_dtype == W8_F32 ? 4 : 2;
    const size_t wb = (size_t)K * N * welem, qb = (size_t)K * N, cb = (size_t)N * 4,
                 rb = (size_t)N * cap * 4, vb = (size_t)N * cap * 2;
    if (overlap(W, wb, q, qb) || overlap(W, wb, scales, (size_t)N * 2) || overlap(q, qb, scales, (size_t)N * 2) ||
        overlap(o_count, cb, W, wb) || overlap(o_count, cb, q, qb) || overlap(o_rows, rb, W, wb) ||
        overlap(o_rows, rb, q, qb) || overlap(o_vals, vb, W, wb) || overlap(o_vals, vb, q, qb) ||
        overlap(o_rows, rb, o_vals, vb) || overlap(o_count, cb, o_rows, rb) || overlap(o_count, cb, o_vals, vb))
        return W8_ERR_ALIAS;
    DeviceInfo *d = nullptr;
    int rc = device_info(&d);
    if (rc != W8_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (w_dtype == W8_F32)
        return launch_percentile<float, true>(d, W, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, K, N, p, q, scales, o_count,
                                              o_rows, o_vals, st);
    return launch_percentile<__half, true>(d, W, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, K, N, p, q, scales, o_count,
                                           o_rows, o_vals, st);
}

int w8_quantize_per_channel_clip(const void *W, int w_dtype, int64_t K, int64_t N, int clip_mode,
                                 double clip_param, int8_t *q, uint16_t *scales, void *stream) {
    if (clip_mode == W8_CLIP_FIXED) {
        const float c = (float)clip_param;
        if (!(c >= 0.0f)) return W8_ERR_SHAPE;   // negative or NaN
        return quantize_common(W, w_dtype, K, N, q, scales, nullptr, false, stream, c);
    }
    if (clip_mode == W8_CLIP_PERCENTILE) {
        if (!(clip_param > 0.0 && clip_param <= 1.0)) return W8_ERR_SHAPE;
        return quantize_common(W, w_dtype, K, N, q, scales, nullptr, false, stream, INFINITY, clip_param);
    }
    return W8_ERR_DTYPE;
}

size_t w8_prepacked_bytes(int64_t K, int64_t N) {
    if (K < 1 || N < 1) return 0;
    return (size_t)cdiv(N, W8_TILE_N) * (size_t)cdiv(K, W8_TILE_K) * W8_TILE_BYTES;
}

// q is the [K, N] code matrix (K*N bytes), packed the tiled copy
// (w8_prepacked_bytes(K, N) bytes, larger than K*N for ragged shapes).
static int pack_args(const void *q, const void *packed, int64_t K, int64_t N) {
    if (!q || !packed) return W8_ERR_NULL;
    if (K < 1 || N < 1 || N % 8 != 0 || cdiv(K, 64) > 65535 * 1024LL || cdiv(N, 128) > 65535)
        return W8_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(packed)) return W8_ERR_ALIGN;
    if (overlap(q, (size_t)K * (size_t)N, packed, w8_prepacked_bytes(K, N))) return W8_ERR_ALIAS;
    return W8_OK;
}

int w8_prepack(const int8_t *q, int64_t K, int64_t N, uint8_t *packed, void *stream) {
    int rc = pack_args(q, packed, K, N);
    if (rc != W8_OK) return rc;
    DeviceInfo *d = nullptr;
    if ((rc = device_info(&d)) != W8_OK) return rc;
    const int KB = (int)cdiv(K, 64);
    dim3 grid((unsigned)KB, (unsigned)cdiv(N, 128));
    pack::prepack_kernel<<<grid, pack::kThreads, 0, static_cast<cudaStream_t>(stream)>>>(q, K, N, KB,
                                                                                        packed);
    return launch_status();
}

int w8_unpack(const uint8_t *packed, int64_t K, int64_t N, int8_t *q, void *stream) {
    int rc = pack_args(q, packed, K, N);
    if (rc != W8_OK) return rc;
    DeviceInfo *d = nullptr;
    if ((rc = device_info(&d)) != W8_OK) return rc;
    const int KB = (int)cdiv(K, 64);
    dim3 grid((unsigned)KB, (unsigned)cdiv(N, 128));
    pack::unpack_kernel<<<grid, pack::kThreads, 0, static_cast<cudaStream_t>(stream)>>>(packed, K, N, KB,
                                                                                       q);
    return launch_status();
}


// Workspace: [fp32 partial sums][int32 counters].  The partial area is the
// larger of the two kernels' needs -- decode: 2 slots per SM; prefill: 2
// slots per CTA pair, each a 256-token x 256-channel tile -- and has the
// same size for every shape on a device, so the counters always start at
// the same offset: a workspace that served one shape (and was left with
// zero counters) serves any other.  Counters: one per 128 channels
// (decode) or two per stream-K tile, fewer than 2 x SMs (prefill).
static size_t decode_partials_bytes(int sms) {
    return (size_t)2 * sms * decode::kMaxPartialFloats * sizeof(float);
}

static size_t partial_area_bytes(int sms) {
    const size_t pre = (size_t)(sms / 2) * 4 * prefill2::kPartFloats * sizeof(float);
    return std::max(decode_partials_bytes(sms), pre);
}

static size_t workspace_total(int sms, int64_t N) {
    const int64_t counters = std::max<int64_t>(cdiv(N, 128), 2 * (int64_t)sms);
    return partial_area_bytes(sms) + (size_t)cdiv(counters * 4, 256) * 256;
}

// X^T for the outlier term of the tensor-core path: K rows of M rounded up
// to the 256-token tile, fp16.
static size_t xt_bytes(int64_t M, int64_t K) {
    if (M <= decode::kMaxTokens) return 0;
    return (size_t)cdiv((int64_t)K * cdiv(M, prefill2::kBT) * prefill2::kBT * 2, 256) * 256;
}

size_t w8a16_linear_outliers_workspace_bytes(int64_t M, int64_t K, int64_t N) {
    if (M < 1 || K < 1 || N < 1) return 0;
    DeviceInfo *d = nullptr;
    if (device_info(&d) != W8_OK) return 0;
    return workspace_total(d->sms, N) + xt_bytes(M, K);
}

size_t w8a16_workspace_bytes(int64_t M, int64_t K, int64_t N) {
    if (M < 1 || K < 1 || N < 1) return 0;
    DeviceInfo *d = nullptr;
    if (device_info(&d) != W8_OK) return 0;
    return workspace_total(d->sms, N);
}

// Both code forms: zeros == nullptr selects the symmetric one.
static int linear_common(const uint16_t *X, const uint8_t *packed, const uint16_t *scales, const int8_t *zeros,
                         bool asym, const uint16_t *bias, uint16_t *Y, int64_t M, int64_t K, int64_t N,
                         void *workspace, size_t workspace_bytes, void *stream, Outliers o = Outliers()) {
    if (M < 0 || K < 1 || N < 1 || K % 8 != 0 || N % 8 != 0 || M > (int64_t)INT32_MAX ||
        K > (int64_t)INT32_MAX || cdiv(K, 64) > INT32_MAX)
        return W8_ERR_SHAPE;
    if (!packed || !scales || (asym && !zeros)) return W8_ERR_NULL;
    if (M == 0) return W8_OK;   // empty batch: X and Y may be NULL
    if (!X || !Y) return W8_ERR_NULL;
    if (!aligned16(X) || !aligned16(packed) || !aligned16(scales) || !aligned16(Y) ||
        (bias && !aligned16(bias)) || (workspace && !aligned16(workspace)))
        return W8_ERR_ALIGN;
    const size_t ybytes = (size_t)M * N * 2;
    if (overlap(Y, ybytes, X, (size_t)M * K * 2) ||
        overlap(Y, ybytes, packed, w8_prepacked_bytes(K, N)) ||
        overlap(Y, ybytes, scales, (size_t)N * 2) || (bias && overlap(Y, ybytes, bias, (size_t)N * 2)) ||
        (asym && overlap(Y, ybytes, zeros, (size_t)N)))
        return W8_ERR_ALIAS;
    DeviceInfo *d = nullptr;
    int rc = device_info(&d);
    if (rc != W8_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int KB = (int)cdiv(K, 64);
    const int64_t NB = cdiv(N, 128);

    const size_t base_need = workspace_total(d->sms, N);
    const size_t need = o.count ? base_need + xt_bytes(M, K) : base_need;
    if (!workspace || workspace_bytes < need) return W8_ERR_WORKSPACE;
    if (o.count && M > decode::kMaxTokens) o.xt = reinterpret_cast<uint16_t *>(static_cast<uint8_t *>(workspace) + base_need);
    if (overlap(workspace, need, Y, ybytes) || overlap(workspace, need, X, (size_t)M * K * 2))
        return W8_ERR_ALIAS;
    float *partials = static_cast<float *>(workspace);
    int *counters = reinterpret_cast<int *>(static_cast<uint8_t *>(workspace) + partial_area_bytes(d->sms));

    if (M <= decode::kMaxTokens) {
        const int MT = M <= 8 ? 1 : M <= 16 ? 2 : M <= 32 ? 4 : 8;
        CUtensorMap map;
        const bool x3 = make_map_x3(&map, X, (uint64_t)M, (uint64_t)K, 8 * MT);
        if (!x3) {
            rc = make_map_2d(&map, X, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)K, (uint64_t)M, 64,
                             8 * MT, CU_TENSOR_MAP_SWIZZLE_128B);
            if (rc != W8_OK) return rc;
        }
        decode::Params p;
        p.packed = packed;
        p.scales = scales;
        p.zeros = zeros;
        p.bias = bias;
        p.Y = Y;
        p.partials = partials;
        p.counters = counters;
        p.X = X;
        p.K = K;
        p.x3 = x3 ? 1 : 0;
        p.o_count = o.count;
        p.o_rows = o.rows;
        p.o_vals = o.vals;
        p.o_cap = (int)o.cap;
        p.M = (int)M;
        p.N = N;
        p.KB = KB;
        if (asym) {
            switch (MT) {
                case 1: return launch_decode_any<1, true>(d, map, p, NB, st);
                case 2: return launch_decode_any<2, true>(d, map, p, NB, st);
                case 4: return launch_decode_any<4, true>(d, map, p, NB, st);
                default: return launch_decode_any<8, true>(d, map, p, NB, st);
            }
        }
        switch (MT) {
            case 1: return launch_decode_any<1, false>(d, map, p, NB, st);
            case 2: return launch_decode_any<2, false>(d, map, p, NB, st);
            case 4: return launch_decode_any<4, false>(d, map, p, NB, st);
            default: return launch_decode_any<8, false>(d, map, p, NB, st);
        }
    }

    return launch_prefill2(d, X, packed, scales, asym ? zeros : nullptr, bias, Y, M, K, N, partials, counters, o,
                           st);
}

int w8a16_linear(const uint16_t *X, const uint8_t *packed, const uint16_t *scales,
                 const uint16_t *bias, uint16_t *Y, int64_t M, int64_t K, int64_t N,
                 void *workspace, size_t workspace_bytes, void *stream) {
    return linear_common(X, packed, scales, nullptr, false, bias, Y, M, K, N, workspace, workspace_bytes,
                         stream);
}

int w8a16_linear_outliers(const uint16_t *X, const uint8_t *packed, const uint16_t *scales,
                          const int32_t *o_count, const int32_t *o_rows, const uint16_t *o_vals, int64_t o_cap,
                          const uint16_t *bias, uint16_t *Y, int64_t M, int64_t K, int64_t N, void *workspace,
                          size_t workspace_bytes, void *stream) {
    if (!o_count || (o_cap > 0 && (!o_rows || !o_vals))) return W8_ERR_NULL;
    if (o_cap < 0 || o_cap > clip::kMaxOutliers) return W8_ERR_LIMIT;
    if (M > 0 && Y && (overlap(Y, (size_t)M * N * 2, o_count, (size_t)N * 4) ||
                       overlap(Y, (size_t)M * N * 2, o_rows, (size_t)N * o_cap * 4) ||
                       overlap(Y, (size_t)M * N * 2, o_vals, (size_t)N * o_cap * 2)))
        return W8_ERR_ALIAS;
    Outliers o;
    o.count = o_count;
    o.rows = o_rows;
    o.vals = o_vals;
    o.cap = o_cap;
    return linear_common(X, packed, scales, nullptr, false, bias, Y, M, K, N, workspace, workspace_bytes, stream, o);
}

int w8a16_linear_asym(const uint16_t *X, const uint8_t *packed, const uint16_t *scales, const int8_t *zeros,
                      const uint16_t *bias, uint16_t *Y, int64_t M, int64_t K, int64_t N, void *workspace,
                      size_t workspace_bytes, void *stream) {
    return linear_common(X, packed, scales, zeros, true, bias, Y, M, K, N, workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------- diagnostics
namespace {
__global__ void bounded_wait_selftest_kernel(unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
        // nothing ever arrives on `bar`: the wait must give up by itself
        mbar_wait(&bar, 0, SITE_SELFTEST, limit_ns);
    }
}
}  // namespace

int w8_test_bounded_wait(uint64_t limit_ns, void *stream) {
    if (limit_ns < 1000 || limit_ns > 5000000000ull) return W8_ERR_SHAPE;
    DeviceInfo *d = nullptr;
    int rc = device_info(&d);
    if (rc != W8_OK) return rc;
    bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
    return launch_status();
}

int w8_test_set_decode_helper_delay(uint64_t delay_ns) {
    if (delay_ns > 1000000ull) return W8_ERR_SHAPE;
    const unsigned long long v = delay_ns;
    if (cudaMemcpyToSymbol(decode::g_helper_delay_ns, &v, sizeof v) != cudaSuccess) return cuda_fail();
    return W8_OK;
}

int w8_device_status(void *stream, uint32_t *out) {
    if (!out) return W8_ERR_NULL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned int v = 0, zero = 0;
    if (cudaStreamSynchronize(st) != cudaSuccess) return cuda_fail();
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof v) != cudaSuccess) return cuda_fail();
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof zero) != cudaSuccess) return cuda_fail();
    *out = v;
    return W8_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- allocation-free decode
// w8a16_linear_decode_static: the decode kernel with its split-K scratch in
// a fixed array of static device memory instead of a caller workspace, for
// callers that cannot allocate device memory.  Layout of the array:
// [fp32 partials: 2 slots x up to W8_STATIC_MAX_SMS CTAs][int32 counters:
// one per 128-channel block, up to W8_STATIC_MAX_N / 128].
namespace {
constexpr size_t kStaticPartialBytes =
    (size_t)2 * W8_STATIC_MAX_SMS * decode::kPartialFloats16 * sizeof(float);
constexpr size_t kStaticCounterBytes = (size_t)(W8_STATIC_MAX_N / 128) * sizeof(int);
static_assert(kStaticPartialBytes + kStaticCounterBytes == (size_t)W8_STATIC_SCRATCH_BYTES,
              "header size of the static scratch");
}  // namespace

// One copy per device that loads this library, zero at load, kept until exit.
static __device__ __align__(256) uint8_t g_decode_scratch[W8_STATIC_SCRATCH_BYTES];

namespace {
// Device address of g_decode_scratch, looked up once per device.  In host
// code the array's name is only a host-side stand-in, never a device
// address, so kernels get this pointer instead.
void *g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

int static_scratch(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return W8_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return W8_ERR_CUDA;
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return W8_OK;
}
}  // namespace

extern "C" int w8a16_linear_decode_static(const uint16_t *X, const uint8_t *packed,
                                          const uint16_t *scales, const uint16_t *bias, uint16_t *Y,
                                          int64_t M, int64_t K, int64_t N, void *stream) {
    if (M < 0 || K < 1 || N < 1 || K % 8 != 0 || N % 8 != 0 || K > (int64_t)INT32_MAX ||
        cdiv(K, 64) > INT32_MAX)
        return W8_ERR_SHAPE;
    if (M > 16 || N > (int64_t)W8_STATIC_MAX_N) return W8_ERR_LIMIT;
    if (!packed || !scales) return W8_ERR_NULL;
    if (M == 0) return W8_OK;
    if (!X || !Y) return W8_ERR_NULL;
    if (!aligned16(X) || !aligned16(packed) || !aligned16(scales) || !aligned16(Y) ||
        (bias && !aligned16(bias)))
        return W8_ERR_ALIGN;
    const size_t ybytes = (size_t)M * N * 2;
    if (overlap(Y, ybytes, X, (size_t)M * K * 2) ||
        overlap(Y, ybytes, packed, w8_prepacked_bytes(K, N)) ||
        overlap(Y, ybytes, scales, (size_t)N * 2) || (bias && overlap(Y, ybytes, bias, (size_t)N * 2)))
        return W8_ERR_ALIAS;
    DeviceInfo *d = nullptr;
    int rc = device_info(&d);
    if (rc != W8_OK) return rc;
    if (d->sms > W8_STATIC_MAX_SMS) return W8_ERR_LIMIT;
    void *scratch = nullptr;
    if ((rc = static_scratch(&scratch)) != W8_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int KB = (int)cdiv(K, 64);
    const int64_t NB = cdiv(N, 128);
    int *counters = reinterpret_cast<int *>(static_cast<uint8_t *>(scratch) + kStaticPartialBytes);
    // the counters must start at zero; an earlier call that gave up a wait
    // may have left some set
    if (cudaMemsetAsync(counters, 0, (size_t)NB * sizeof(int), st) != cudaSuccess) {
        cudaGetLastError();
        return W8_ERR_CUDA;
    }
    const int MT = M <= 8 ? 1 : 2;
    // the same X maps as w8a16_linear: one 3-D load per stage when K % 64 == 0
    CUtensorMap map;
    const bool x3 = make_map_x3(&map, X, (uint64_t)M, (uint64_t)K, 8 * MT);
    if (!x3) {
        rc = make_map_2d(&map, X, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)K, (uint64_t)M, 64, 8 * MT,
                         CU_TENSOR_MAP_SWIZZLE_128B);
        if (rc != W8_OK) return rc;
    }
    decode::Params p;
    p.packed = packed;
    p.scales = scales;
    p.zeros = nullptr;
    p.X = X;
    p.K = K;
    p.o_count = nullptr;
    p.o_rows = nullptr;
    p.o_vals = nullptr;
    p.o_cap = 0;
    p.x3 = x3 ? 1 : 0;
    p.bias = bias;
    p.Y = Y;
    p.partials = static_cast<float *>(scratch);
    p.counters = counters;
    p.M = (int)M;
    p.N = N;
    p.KB = KB;
    {
        const int64_t T = NB * KB;
        if ((uint64_t)T * (uint64_t)(std::min<int64_t>(T, d->sms) + 1) >= (1ull << 32)) return W8_ERR_LIMIT;
    }
    return MT == 1 ? launch_decode_any<1, false>(d, map, p, NB, st) : launch_decode_any<2, false>(d, map, p, NB, st);
}
