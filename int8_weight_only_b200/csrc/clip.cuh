// Percentile-clipped symmetric int8 quantization: the "percentage clip"
// calibration of the LightSeq 2020 slides (slide "quantization: clipping +
// symmetric").  Per output channel n the bound put on level 127 is the
// r-th smallest |W[k,n]| -- the t-th largest, t = K - r + 1 -- instead of
// the maximum, and then, as in the symmetric quantizer,
//   s_n = fp16_rne( fp32(bound_n) / 127 ),  q = clamp( rne(W / s_n), -127, 127 ).
//
// The order statistic is found by radix selection on the bit pattern of
// |w| (for non-negative floats the pattern orders as the value): four
// passes over the channel, each a 256-bin histogram of one byte of the
// pattern among the values whose higher bytes equal those already chosen;
// the bin holding the t-th largest fixes that byte.  A fifth pass writes
// the codes.
//
// Work unit: a panel of 32 columns over all K rows, one CTA per panel
// (persistent CTAs walk the panels).  A producer thread streams the panel
// five times through a ring of 2-D TMA boxes (32 columns x 16 KB of rows);
// pass 1 loads keep the panel in L2 (evict-last) for the four passes that
// follow.  Consumer lane = column: each warp takes every 16th row of a box.
#pragma once

#include "common.cuh"
#include "quantize.cuh"

namespace w8 {
namespace clip {

constexpr int kConsumerWarps = 16;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kPanel = 32;
constexpr int kStages = 8;
constexpr int kBoxBytes = 16384;
constexpr int kBins = 256;
constexpr int kBinStride = kBins + 1;   // per-column rows offset by one bank
constexpr int kPasses = 5;              // four selection passes, then the codes
constexpr int kSmemBytes = kStages * kBoxBytes + 1024;

template <typename T>
struct Geo {
    static constexpr int kRowBytes = kPanel * (int)sizeof(T);
    static constexpr int kRows = kBoxBytes / kRowBytes;   // 128 fp32 or 256 fp16 rows
};

// Outlier split (the GOBO page's observation applied here): the weights
// strictly above the bound are kept apart as (row, fp16 value) in a side
// list of `cap` slots per channel, rows increasing, unused slots 0, and get
// the code 0.  At most t - 1 = cap weights of a channel exceed the bound.
constexpr int kMaxOutliers = 64;

struct Params {
    int8_t *q;
    uint16_t *scales;
    int64_t K;
    int64_t N;
    int t;         // rank from the top: the bound is the t-th largest |w|
    int panels;    // ceil(N / 32)
    // outlier split only
    int32_t *o_count;    // [N]
    int32_t *o_rows;     // [N][cap]
    uint16_t *o_vals;    // [N][cap] fp16
    int cap;             // t - 1 <= kMaxOutliers
};

__device__ __forceinline__ uint32_t abs_bits(float v) { return __float_as_uint(v) & 0x7FFFFFFFu; }

template <typename T>
__device__ __forceinline__ float load_elem(const uint8_t *p);
template <>
__device__ __forceinline__ float load_elem<float>(const uint8_t *p) {
    return *reinterpret_cast<const float *>(p);
}
template <>
__device__ __forceinline__ float load_elem<__half>(const uint8_t *p) {
    return __half2float(*reinterpret_cast<const __half *>(p));
}

// grid = persistent CTAs, kThreads threads, kSmemBytes dynamic shared
// memory.  tmap_w: W [K, N], box 32 columns x Geo<T>::kRows rows, no swizzle.
template <typename T, bool kOut>
__global__ void __launch_bounds__(kThreads, 1)
percentile_quantize_kernel(const __grid_constant__ CUtensorMap tmap_w, const Params p) {
    using G = Geo<T>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *ring = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    __shared__ uint64_t full[kStages], empty[kStages];
    __shared__ uint32_t hist[kPanel * kBinStride];
    __shared__ uint32_t col_prefix[kPanel];   // chosen high bytes of the bound's pattern
    __shared__ int col_rem[kPanel];           // rank still to find within them
    __shared__ float col_scale[kPanel], col_inv[kPanel];
    // outlier split: this panel's side lists, filled in the code pass
    __shared__ int o_n[kOut ? kPanel : 1];
    __shared__ int32_t o_row[kOut ? kPanel : 1][kOut ? kMaxOutliers : 1];
    __shared__ uint16_t o_val[kOut ? kPanel : 1][kOut ? kMaxOutliers : 1];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nbox = (int)((p.K + G::kRows - 1) / G::kRows);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kConsumerWarps);
        }
        fence_barrier_init();
        prefetch_tensormap(&tmap_w);
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t keep = policy_evict_last(), drop = policy_evict_first();
            int s = 0;
            uint32_t ph = 0;
            int issued = 0;
            bool ok = true;
            for (int panel = blockIdx.x; panel < p.panels && ok; panel += gridDim.x) {
                for (int pass = 0; pass < kPasses && ok; ++pass) {
                    for (int i = 0; i < nbox; ++i) {
                        if (!mbar_wait_parked(&empty[s], ph ^ 1u, SITE_CLIP_EMPTY)) { ok = false; break; }
                        mbar_arrive_expect_tx(&full[s], kBoxBytes);
                        tma_load_2d_hint(ring + s * kBoxBytes, &tmap_w, panel * kPanel, i * G::kRows, &full[s],
                                         pass + 1 < kPasses ? keep : drop);
                        ++issued;
                        if (++s == kStages) { s = 0; ph ^= 1u; }
                    }
                }
            }
            // every issued copy lands before the CTA may leave
            for (int i = 0; i < kStages && i < issued; ++i) {
                if (--s < 0) { s = kStages - 1; ph ^= 1u; }
                mbar_wait(&full[s], ph, SITE_CLIP_DRAIN, 10000000ull);
            }
        }
        return;
    }

    // ---------------------------------------------------------- consumers
    // (warp-uniform `ok`; every consumer reaches every barrier below, and a
    // wait that ran out in any warp ends the work of all of them together)
    const int c = threadIdx.x;
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int panel = blockIdx.x; panel < p.panels && ok; panel += gridDim.x) {
        if (c < kPanel) {
            col_prefix[c] = 0;
            col_rem[c] = p.t;
            if constexpr (kOut) o_n[c] = 0;
        }
        for (int i = c; i < kPanel * kBinStride; i += kConsumers) hist[i] = 0;
        for (int pass = 0; pass < kPasses; ++pass) {
            // the histogram is zero and the column state of the last scan
            // is visible
            if (!named_bar_all(1, kConsumers, ok)) { ok = false; break; }
            const int shift = 24 - 8 * pass;   // byte of the pattern this pass histograms
            const uint32_t hi_mask = pass == 0 ? 0u : ~((1u << (shift + 8)) - 1u);
            // pass 4: col_prefix holds the bound's pattern
            const uint32_t prefix = col_prefix[lane];
            const float sc = pass == 4 ? col_scale[lane] : 0.0f;
            const float inv = pass == 4 ? col_inv[lane] : 0.0f;
            const int64_t n = (int64_t)panel * kPanel + lane;
            for (int i = 0; i < nbox; ++i) {
                if (ok && !warp_all(mbar_wait_parked(&full[s], ph, SITE_CLIP_LOAD))) ok = false;
                if (ok) {
                    const uint8_t *box = ring + s * kBoxBytes;
                    for (int rloc = warp; rloc < G::kRows; rloc += kConsumerWarps) {
                        const int64_t k = (int64_t)i * G::kRows + rloc;
                        if (k >= p.K) break;
                        const float v = load_elem<T>(box + rloc * G::kRowBytes + lane * (int)sizeof(T));
                        if (pass < 4) {
                            const uint32_t bits = abs_bits(v);
                            if ((bits & hi_mask) == prefix)
                                atomicAdd(&hist[lane * kBinStride + ((bits >> shift) & 0xFFu)], 1u);
                        } else if (n < p.N) {
                            bool sure;
                            int code = quant::quantize_fast(v, inv, sure);
                            if (!sure) code = quant::quantize_exact(v, sc);
                            if constexpr (kOut) {
                                if (abs_bits(v) > prefix) {   // |w| above the bound
                                    const int j = atomicAdd(&o_n[lane], 1);
                                    if (j < kMaxOutliers) {
                                        o_row[lane][j] = (int32_t)k;
                                        o_val[lane][j] = __half_as_ushort(__float2half_rn(v));
                                    }
                                    code = 0;
                                }
                            }
                            p.q[k * p.N + n] = (int8_t)code;
                        }
                    }
                }
                __syncwarp();
                if (ok && lane == 0) mbar_arrive(&empty[s]);
                if (++s == kStages) { s = 0; ph ^= 1u; }
            }
            if (pass == 4) {
                if constexpr (kOut) {
                    // every outlier of the panel is listed: sort each column's
                    // list by row (the order the warps met them varies) and
                    // store it, unused slots 0
                    if (!named_bar_all(1, kConsumers, ok)) { ok = false; break; }
                    const int64_t nn = (int64_t)panel * kPanel + c;
                    if (c < kPanel && nn < p.N) {
                        const int cnt = min(o_n[c], p.cap);
                        for (int a = 1; a < cnt; ++a) {
                            const int32_t r0 = o_row[c][a];
                            const uint16_t v0 = o_val[c][a];
                            int b2 = a - 1;
                            for (; b2 >= 0 && o_row[c][b2] > r0; --b2) {
                                o_row[c][b2 + 1] = o_row[c][b2];
                                o_val[c][b2 + 1] = o_val[c][b2];
                            }
                            o_row[c][b2 + 1] = r0;
                            o_val[c][b2 + 1] = v0;
                        }
                        p.o_count[nn] = cnt;
                        for (int j = 0; j < p.cap; ++j) {
                            p.o_rows[nn * p.cap + j] = j < cnt ? o_row[c][j] : 0;
                            p.o_vals[nn * p.cap + j] = j < cnt ? o_val[c][j] : (uint16_t)0;
                        }
                    }
                    // the lists are read before the next panel resets them
                    if (!named_bar_all(1, kConsumers, ok)) { ok = false; break; }
                }
                break;
            }
            // the histogram is complete
            if (!named_bar_all(1, kConsumers, ok)) { ok = false; break; }
            if (c < kPanel) {
                // the bin that holds the rem-th largest of the matching values
                const int rem = col_rem[c];
                uint32_t cum = 0;
                int b = kBins - 1;
                for (; b > 0; --b) {
                    const uint32_t h = hist[c * kBinStride + b];
                    if (cum + h >= (uint32_t)rem) break;
                    cum += h;
                }
                col_rem[c] = rem - (int)cum;
                const uint32_t pre = col_prefix[c] | ((uint32_t)b << shift);
                col_prefix[c] = pre;
                if (pass == 3) {
                    const float bound = __uint_as_float(pre);
                    const __half s16 = __float2half_rn(__fdiv_rn(bound, 127.0f));
                    const float sf = __half2float(s16);
                    col_scale[c] = sf;
                    col_inv[c] = sf != 0.0f ? __frcp_rn(sf) : 0.0f;
                    const int64_t nn = (int64_t)panel * kPanel + c;
                    if (nn < p.N) p.scales[nn] = __half_as_ushort(s16);
                }
            }
            // the scan has read the histogram: clear it for the next pass
            if (!named_bar_all(1, kConsumers, ok)) { ok = false; break; }
            for (int i = c; i < kPanel * kBinStride; i += kConsumers) hist[i] = 0;
        }
    }
}

}  // namespace clip
}  // namespace w8
