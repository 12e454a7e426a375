// Percentile-clipped symmetric int8 quantization: the "percentage clip"
// calibration of the LightSeq 2020 slides (slide "quantization: clipping +
// symmetric").  Per output channel n the bound put on level 127 is the
// r-th smallest |W[k,n]| -- the t-th largest, t = K - r + 1 -- instead of
// the maximum, and then, as in the symmetric quantizer,
//   s_n = fp16_rne( fp32(bound_n) / 127 ),  q = clamp( rne(W / s_n), -127, 127 ).
//
// The order statistic is found by radix selection on the bit pattern of
// |w| (for non-negative floats the pattern orders as the value, and the
// sign bit is clear, so a pattern has 31 bits).  A column's selection goes
// digit by digit from the top -- digits of 9, 8, 7 and 7 bits -- keeping
// the prefix of the bound's pattern found so far and the rank still to
// find among the values that carry that prefix.  A pass over the column
// does one of two things for it:
//  - histogram: count the values with the prefix by their next digit; the
//    bin that holds the wanted rank extends the prefix;
//  - collect: once at most kCap values carry the prefix, copy their
//    patterns into shared memory, and finish the selection there within
//    one warp, with no further pass over W (up to 32 patterns: one per
//    lane, ranked by a count over warp shuffles; more: digit by digit).
// On the usual weights the first pass (a 512-bin histogram) leaves a few
// values in the chosen bin, the second collects them and the third writes
// the codes: three passes over W instead of the five a byte-wise radix
// select takes.  A column whose values crowd into one bin at every digit
// (all equal, say) takes at most four selection passes.
//
// Work unit: a panel of 32 columns over all K rows, one CTA per panel
// (persistent CTAs walk the panels).  A producer thread streams the panel
// once per pass through a ring of 2-D TMA boxes (32 columns x 16 KB of
// rows) with the L2 evict-last hint, so that passes after the first read
// L2.  How many passes a panel takes is known only once its columns are
// resolved, so before each pass after the second the producer waits for
// the consumers' verdict on the pass two before it (the panel needs pass j
// exactly when pass j - 1 is still a selection pass).  In the selection
// passes consumer lane = column and each warp takes every 16th row of a
// box; the code pass uses the plain quantizer's layout (a thread per
// 16-byte row segment).
#pragma once

#include "common.cuh"
#include "quantize.cuh"

namespace w8 {
namespace clip {

constexpr int kConsumerWarps = 16;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kPanel = 32;
constexpr int kStages = 7;
constexpr int kBoxBytes = 16384;
constexpr int kCap = 768;                // values a column collects
constexpr int kFirstBits = 9;            // width of the first digit (512 bins)
constexpr int kRegion = kCap + 1;        // words per column (rows offset by one bank)
constexpr int kRegionBytes = kPanel * kRegion * 4;
constexpr int kScratch = 128;            // words of a warp's histogram in a collected column's selection
constexpr int kSmemBytes = kStages * kBoxBytes + 1024 + kRegionBytes + kConsumerWarps * kScratch * 4;
constexpr unsigned SITE_CLIP_DECIDE = 0x53;   // producer: the consumers' verdict on a pass

// Column modes of a selection pass.
constexpr int kDone = 0, kHist = 1, kCollect = 2;

// Width of the digit after `lvl` resolved top bits: 10 first, then 7.
__host__ __device__ constexpr int digit_width(int lvl) {
    return lvl == 0 ? kFirstBits : (lvl == kFirstBits ? 8 : (31 - lvl < 7 ? 31 - lvl : 7));
}
// Width of a digit in a collected column's selection (its histogram is a warp's 128-word scratch).
__host__ __device__ constexpr int collect_width(int lvl) { return 31 - lvl < 7 ? 31 - lvl : 7; }
// Mask of the top `lvl` bits of a 31-bit pattern.
__device__ __forceinline__ uint32_t prefix_mask(int lvl) { return lvl == 0 ? 0u : ~((1u << (31 - lvl)) - 1u); }

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

// Shared-memory atomics named as such (the histogram and the lists live in
// a dynamic shared-memory region the compiler would address generically).
__device__ __forceinline__ void red_add_shared(uint32_t *p, uint32_t v) {
    asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v));
}
__device__ __forceinline__ int atom_add_shared(int *p, int v) {
    int r;
    asm volatile("atom.shared.add.u32 %0, [%1], %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(v));
    return r;
}

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

// One warp: the bin of histogram hb[0, nb) (bins ordered by value, nb a
// power of two from 8 to 1024) that holds the rem-th largest of the counted
// values.  rem becomes the rank within that bin and grp the bin's count.
// Lane l sums bins [l cs, l cs + cs), cs = max(1, nb / 32) (the 32-bin
// chunks read in a rotated order, so the lanes hit distinct banks); the
// suffix sums over the lanes locate the chunk, and a second suffix scan
// within the chunk the bin.
__device__ __forceinline__ int select_bin(const uint32_t *hb, int nb, int lane, uint32_t &rem, uint32_t &grp) {
    const int cs = nb >= 32 ? nb / 32 : 1;
    uint32_t sum = 0;
    if (nb >= 32) {
#pragma unroll 4
        for (int i = 0; i < cs; ++i) sum += hb[lane * cs + ((i + lane) & (cs - 1))];
    } else if (lane < nb) {
        sum = hb[lane];
    }
    uint32_t s = sum;   // values in the chunks of this lane and above
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, s, off);
        if (lane + off < 32) s += y;
    }
    const uint32_t ball = __ballot_sync(0xffffffffu, s >= rem);
    const int lc = ball ? 31 - __clz(ball) : 0;   // the total is at least rem: lane 0 is set
    const uint32_t above = __shfl_sync(0xffffffffu, s - sum, lc);
    const int b0 = lc * cs;
    const uint32_t h = (lane < cs && b0 + lane < nb) ? hb[b0 + lane] : 0u;
    uint32_t s2 = h;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, s2, off);
        if (lane + off < 32) s2 += y;
    }
    const uint32_t ball2 = __ballot_sync(0xffffffffu, lane < cs && above + s2 >= rem);
    const int lb = ball2 ? 31 - __clz(ball2) : 0;
    const uint32_t above_b = above + __shfl_sync(0xffffffffu, s2 - h, lb);
    grp = __shfl_sync(0xffffffffu, h, lb);
    rem -= above_b;
    return b0 + lb;
}

// What a selection pass does with a warp's rows of one box (lane = column):
//  kScanHist0     first pass, K > kCap: count every value by its first digit
//  kScanCollect0  first pass, K <= kCap: keep every pattern (slot = row)
//  kScanSelect    later passes, each column by its own mode
// (kScanCode, the code pass, is code_box below.)  kCheck: the box holds
// rows past K (only the last one can).
constexpr int kScanHist0 = 0, kScanCollect0 = 1, kScanSelect = 2, kScanCode = 3;

struct LaneScan {
    uint32_t mask, prefix, dmask;   // the column's prefix test and digit
    int shift;
    bool hist;                      // histogram (else collect)
};

template <typename T, int kKind, bool kCheck, bool kOut>
__device__ __forceinline__ void scan_box(const uint8_t *box, int k0, int K, int warp, int lane, const LaneScan &ls,
                                         uint32_t *hb, int *cnt) {
    using G = Geo<T>;
    constexpr int kPer = G::kRows / kConsumerWarps;
    // the warp's rows, loaded before any shared memory update (atomics and
    // stores to the same memory would otherwise order every load after the
    // last update)
    float vals[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u)
        vals[u] = load_elem<T>(box + (warp + u * kConsumerWarps) * G::kRowBytes + lane * (int)sizeof(T));
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int k = k0 + warp + u * kConsumerWarps;
        if (kCheck && k >= K) break;
        const uint32_t bits = abs_bits(vals[u]);
        if constexpr (kKind == kScanHist0) {
            red_add_shared(&hb[bits >> (31 - kFirstBits)], 1u);
        } else if constexpr (kKind == kScanCollect0) {
            hb[k] = bits;
        } else {
            if ((bits & ls.mask) == ls.prefix) {
                if (ls.hist) {
                    red_add_shared(&hb[(bits >> ls.shift) & ls.dmask], 1u);
                } else {
                    const int j = atom_add_shared(cnt, 1);
                    if (j < kCap) hb[j] = bits;
                }
            }
        }
    }
}

// The code pass over one box, with the plain quantizer's thread layout: a
// thread owns one 16-byte segment of a row (4 fp32 or 8 fp16 columns) of
// kSweeps rows, loads each with one 16-byte read, forms the codes with one
// exactness decision per segment and stores them as one 4- or 8-byte word.
// Outlier split: a weight above its column's bound gets code 0 and is
// listed (row, fp16 value) in the column's region.
template <typename T>
struct CodeSeg {
    static constexpr int kCols = 16 / (int)sizeof(T);
    static constexpr int kThreadsPerRow = kPanel / kCols;              // 8 fp32, 4 fp16
    static constexpr int kSweep = kConsumers / kThreadsPerRow;          // 64 or 128 rows
    static constexpr int kSweeps = Geo<T>::kRows / kSweep;              // 2
};

template <typename T, bool kCheck, bool kOut>
__device__ __forceinline__ void code_box(const uint8_t *box, int k0, int K, int t, int rsub,
                                         const float (&sc)[CodeSeg<T>::kCols], const float (&inv)[CodeSeg<T>::kCols],
                                         const uint32_t (&bnd)[CodeSeg<T>::kCols], uint32_t *region, int *o_n,
                                         int8_t *qseg, int64_t N) {
    using S = CodeSeg<T>;
    using G = Geo<T>;
    float v[S::kSweeps][S::kCols];
#pragma unroll
    for (int w = 0; w < S::kSweeps; ++w) quant::load_seg<T>(box + (rsub + w * S::kSweep) * G::kRowBytes + 16 * t, v[w]);
#pragma unroll
    for (int w = 0; w < S::kSweeps; ++w) {
        const int k = k0 + rsub + w * S::kSweep;
        if (kCheck && k >= K) break;
        int code[S::kCols];   // codes in the low bytes
        if (!quant::quantize_fast_seg<S::kCols>(v[w], inv, code)) {
#pragma unroll
            for (int e = 0; e < S::kCols; ++e) code[e] = quant::quantize_exact(v[w][e], sc[e]);
        }
        if constexpr (kOut) {
#pragma unroll
            for (int e = 0; e < S::kCols; ++e) {
                if (abs_bits(v[w][e]) > bnd[e]) {   // |w| above the bound
                    const int col = t * S::kCols + e;
                    const int j = atom_add_shared(&o_n[col], 1);
                    if (j < kMaxOutliers) {
                        uint32_t *cr = region + col * kRegion;
                        reinterpret_cast<int32_t *>(cr)[j] = k;
                        reinterpret_cast<uint16_t *>(cr + kMaxOutliers)[j] = __half_as_ushort(__float2half_rn(v[w][e]));
                    }
                    code[e] = 0;
                }
            }
        }
        uint32_t packed[S::kCols / 4];
#pragma unroll
        for (int g = 0; g < S::kCols / 4; ++g) {
            const uint32_t lo = __byte_perm((uint32_t)code[4 * g], (uint32_t)code[4 * g + 1], 0x0040);
            const uint32_t hi = __byte_perm((uint32_t)code[4 * g + 2], (uint32_t)code[4 * g + 3], 0x0040);
            packed[g] = __byte_perm(lo, hi, 0x5410);
        }
        int8_t *dst = qseg + (int64_t)k * N;
        if constexpr (S::kCols == 4)
            *reinterpret_cast<uint32_t *>(dst) = packed[0];
        else
            *reinterpret_cast<uint2 *>(dst) = make_uint2(packed[0], packed[S::kCols / 4 - 1]);
    }
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
    // per column: the histogram or the collected patterns of a selection
    // pass; the outlier lists during the code pass
    uint32_t *region = reinterpret_cast<uint32_t *>(ring + kStages * kBoxBytes);
    uint32_t *scratch = region + kPanel * kRegion;
    __shared__ uint64_t full[kStages], empty[kStages];
    __shared__ uint64_t decide[2];            // the verdicts, alternating
    __shared__ int verdict[2];                // 1: the pass after the next one is needed
    __shared__ uint32_t col_prefix[kPanel];   // top bits of the bound's pattern found so far
    __shared__ int col_lvl[kPanel];           // how many of its 31 bits
    __shared__ uint32_t col_rem[kPanel];      // rank still to find among the values with the prefix
    __shared__ uint32_t col_grp[kPanel];      // how many values carry the prefix
    __shared__ int col_mode[kPanel];
    __shared__ int col_cnt[kPanel];           // collected so far
    __shared__ float col_scale[kPanel], col_inv[kPanel];
    __shared__ int o_n[kPanel];               // outlier split: listed so far

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int K = (int)p.K;
    const int nbox = (K + G::kRows - 1) / G::kRows;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kConsumerWarps);
        }
        mbar_init(&decide[0], 1);
        mbar_init(&decide[1], 1);
        fence_barrier_init();
        prefetch_tensormap(&tmap_w);
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t keep = policy_evict_last();
            int s = 0;
            uint32_t ph = 0;
            int issued = 0;
            uint32_t nd = 0;   // verdicts read
            bool ok = true;
            for (int panel = blockIdx.x; panel < p.panels && ok; panel += gridDim.x) {
                for (int pass = 0; ok; ++pass) {
                    if (pass >= 2) {
                        // pass `pass` exists when pass - 1 is a selection pass
                        if (!mbar_wait_parked(&decide[nd & 1], (nd >> 1) & 1, SITE_CLIP_DECIDE)) { ok = false; break; }
                        const int more = *reinterpret_cast<volatile int *>(&verdict[nd & 1]);
                        ++nd;
                        if (!more) break;
                    }
                    for (int i = 0; i < nbox; ++i) {
                        if (!mbar_wait_parked(&empty[s], ph ^ 1u, SITE_CLIP_EMPTY)) { ok = false; break; }
                        mbar_arrive_expect_tx(&full[s], kBoxBytes);
                        tma_load_2d_hint(ring + s * kBoxBytes, &tmap_w, panel * kPanel, i * G::kRows, &full[s], keep);
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
    uint32_t nd = 0;   // verdicts given
    bool ok = true;
    for (int panel = blockIdx.x; panel < p.panels && ok; panel += gridDim.x) {
        if (c < kPanel) {
            const bool in = (int64_t)panel * kPanel + c < p.N;
            col_prefix[c] = 0;
            col_lvl[c] = 0;
            col_rem[c] = (uint32_t)p.t;
            col_grp[c] = (uint32_t)K;
            col_mode[c] = !in ? kDone : (K <= kCap ? kCollect : kHist);
            col_cnt[c] = K <= kCap ? K : 0;   // the first pass keeps every row's pattern, in slot = row
        }
        bool code_pass = false;
        for (int pass = 0; ok; ++pass) {
            // the column state of the last resolution is visible
            if (!named_bar_all(1, kConsumers, ok)) { ok = false; break; }
            const int mode = col_mode[lane];
            if (!code_pass) {
                // clear the histograms of this pass: warp w, columns w and w + 16
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int col = warp + h * kConsumerWarps;
                    if (col_mode[col] == kHist) {
                        const int nb = 1 << digit_width(col_lvl[col]);
                        for (int b = lane; b < nb; b += 32) region[col * kRegion + b] = 0u;
                    }
                }
                if (!named_bar_all(1, kConsumers, ok)) { ok = false; break; }
            }
            // this lane's column: what to match and where to count it
            LaneScan ls;
            {
                const int lvl = col_lvl[lane];
                ls.mask = mode == kDone ? 0u : prefix_mask(lvl);
                ls.prefix = mode == kDone ? 0xFFFFFFFFu : col_prefix[lane];   // no pattern matches
                ls.shift = 31 - lvl - digit_width(lvl);
                ls.dmask = (1u << digit_width(lvl)) - 1u;
                ls.hist = mode == kHist;
            }
            uint32_t *const hb = region + lane * kRegion;
            // the code pass: this thread's segment and its columns' constants
            using S = CodeSeg<T>;
            const int st = c % S::kThreadsPerRow, srow = c / S::kThreadsPerRow;
            float ssc[S::kCols], sinv[S::kCols];
            uint32_t sbnd[S::kCols];
#pragma unroll
            for (int e = 0; e < S::kCols; ++e) {
                ssc[e] = code_pass ? col_scale[st * S::kCols + e] : 0.0f;
                sinv[e] = code_pass ? col_inv[st * S::kCols + e] : 0.0f;
                sbnd[e] = col_prefix[st * S::kCols + e];
            }
            // N % 8 == 0: a segment is all inside the weight or all outside
            const bool seg_ok = (int64_t)panel * kPanel + st * S::kCols < p.N;
            int8_t *const qseg = p.q + (int64_t)panel * kPanel + st * S::kCols;
            // which form this pass takes (the same in every warp)
            const int kind = code_pass ? kScanCode : (pass > 0 ? kScanSelect : (K > kCap ? kScanHist0 : kScanCollect0));
            for (int i = 0; i < nbox; ++i) {
                if (ok && !warp_all(mbar_wait_parked(&full[s], ph, SITE_CLIP_LOAD))) ok = false;
                if (ok) {
                    const uint8_t *box = ring + s * kBoxBytes;
                    const int k0 = i * G::kRows;
                    const bool chk = k0 + G::kRows > K;
#define W8_SCAN(KIND)                                                                       \
    (chk ? scan_box<T, KIND, true, kOut>(box, k0, K, warp, lane, ls, hb, &col_cnt[lane]) \
         : scan_box<T, KIND, false, kOut>(box, k0, K, warp, lane, ls, hb, &col_cnt[lane]))
                    if (kind == kScanCode) {
                        if (seg_ok) {
                            if (chk)
                                code_box<T, true, kOut>(box, k0, K, st, srow, ssc, sinv, sbnd, region, o_n, qseg, p.N);
                            else
                                code_box<T, false, kOut>(box, k0, K, st, srow, ssc, sinv, sbnd, region, o_n, qseg, p.N);
                        }
                    } else if (kind == kScanSelect)
                        W8_SCAN(kScanSelect);
                    else if (kind == kScanHist0)
                        W8_SCAN(kScanHist0);
                    else
                        W8_SCAN(kScanCollect0);
#undef W8_SCAN
                }
                __syncwarp();
                if (ok && lane == 0) mbar_arrive(&empty[s]);
                if (++s == kStages) { s = 0; ph ^= 1u; }
            }
            if (code_pass) {
                if constexpr (kOut) {
                    // every outlier of the panel is listed: sort each column's
                    // list by row (the order the warps met them varies) and
                    // store it, unused slots 0
                    if (!named_bar_all(1, kConsumers, ok)) { ok = false; break; }
                    const int64_t nn = (int64_t)panel * kPanel + c;
                    if (c < kPanel && nn < p.N) {
                        int32_t *orow = reinterpret_cast<int32_t *>(region + c * kRegion);
                        uint16_t *oval = reinterpret_cast<uint16_t *>(region + c * kRegion + kMaxOutliers);
                        const int cnt = min(o_n[c], p.cap);
                        for (int a = 1; a < cnt; ++a) {
                            const int32_t r0 = orow[a];
                            const uint16_t v0 = oval[a];
                            int b2 = a - 1;
                            for (; b2 >= 0 && orow[b2] > r0; --b2) {
                                orow[b2 + 1] = orow[b2];
                                oval[b2 + 1] = oval[b2];
                            }
                            orow[b2 + 1] = r0;
                            oval[b2 + 1] = v0;
                        }
                        p.o_count[nn] = cnt;
                        for (int j = 0; j < p.cap; ++j) {
                            p.o_rows[nn * p.cap + j] = j < cnt ? orow[j] : 0;
                            p.o_vals[nn * p.cap + j] = j < cnt ? oval[j] : (uint16_t)0;
                        }
                    }
                }
                // the next panel's state is written after every read of this one
                if (!named_bar_all(1, kConsumers, ok)) { ok = false; break; }
                break;
            }
            // ------------------------------------------------ resolution
            // every count and pattern of the pass is in shared memory
            if (!named_bar_all(1, kConsumers, ok)) { ok = false; break; }
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
                const int col = warp + h * kConsumerWarps;
                const int cmode = col_mode[col];
                if (cmode == kDone) continue;
                uint32_t *const cb = region + col * kRegion;
                int clvl = col_lvl[col];
                uint32_t pre = col_prefix[col];
                uint32_t rem = col_rem[col];
                uint32_t grp = col_grp[col];
                int nmode;
                if (cmode == kHist) {
                    const int w = digit_width(clvl);
                    const int b = select_bin(cb, 1 << w, lane, rem, grp);
                    pre |= (uint32_t)b << (31 - clvl - w);
                    clvl += w;
                    nmode = clvl == 31 ? kDone : (grp <= (uint32_t)kCap ? kCollect : kHist);
                } else {
                    // the collected patterns stay where they are; each digit's
                    // histogram goes to the warp's scratch
                    const int cnt = min(col_cnt[col], kCap);
                    uint32_t *const sb = scratch + warp * kScratch;
                    if (cnt <= 32) {
                        // one pattern per lane: the wanted one has fewer than rem
                        // patterns above it and at least rem at or above it
                        const uint32_t x = lane < cnt ? cb[lane] : 0u;
                        uint32_t above = 0, same = 0;
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const uint32_t y = __shfl_sync(0xffffffffu, x, j);
                            if (j < cnt) {
                                above += y > x;
                                same += y == x;
                            }
                        }
                        const uint32_t hit = __ballot_sync(0xffffffffu, lane < cnt && above < rem && rem <= above + same);
                        const int src = hit ? __ffs(hit) - 1 : 0;
                        pre = __shfl_sync(0xffffffffu, x, src);
                        rem -= __shfl_sync(0xffffffffu, above, src);
                        grp = __shfl_sync(0xffffffffu, same, src);
                        clvl = 31;
                    }
#pragma unroll 1
                    while (clvl < 31) {
                        const int w = collect_width(clvl);
                        const int sh = 31 - clvl - w;
                        const uint32_t m = prefix_mask(clvl);
                        for (int b = lane; b < (1 << w); b += 32) sb[b] = 0u;
                        __syncwarp();
                        for (int j = lane; j < cnt; j += 32) {
                            const uint32_t x = cb[j];
                            if ((x & m) == pre) atomicAdd(&sb[(x >> sh) & ((1u << w) - 1u)], 1u);
                        }
                        __syncwarp();
                        const int b = select_bin(sb, 1 << w, lane, rem, grp);
                        pre |= (uint32_t)b << sh;
                        clvl += w;
                        __syncwarp();
                    }
                    nmode = kDone;
                }
                if (lane == 0) {
                    col_prefix[col] = pre;
                    col_lvl[col] = clvl;
                    col_rem[col] = rem;
                    col_grp[col] = grp;
                    col_mode[col] = nmode;
                    col_cnt[col] = 0;
                }
            }
            if (!named_bar_all(1, kConsumers, ok)) { ok = false; break; }
            code_pass = __all_sync(0xffffffffu, col_mode[lane] == kDone);
            if (c == 0) {
                // the producer loads the pass after the next one only if the
                // next one selects
                verdict[nd & 1] = code_pass ? 0 : 1;
                mbar_arrive(&decide[nd & 1]);
            }
            ++nd;
            if (code_pass && c < kPanel) {
                const float bound = __uint_as_float(col_prefix[c]);
                const __half s16 = __float2half_rn(__fdiv_rn(bound, 127.0f));
                const float sf = __half2float(s16);
                col_scale[c] = sf;
                col_inv[c] = sf != 0.0f ? __frcp_rn(sf) : 0.0f;
                o_n[c] = 0;
                const int64_t nn = (int64_t)panel * kPanel + c;
                if (nn < p.N) p.scales[nn] = __half_as_ushort(s16);
            }
        }
    }
}

}  // namespace clip
}  // namespace w8
