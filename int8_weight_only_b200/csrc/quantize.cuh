// Per-output-channel symmetric int8 quantization (TPU-MLIR ChatGLM2 W8A16
// article, sections 2-3; LightSeq 2020 slides "clipping + symmetric").
//
//   s_n = fp16_rne( fp32(max_k |W[k,n]|) / 127 )
//   q[k,n] = clamp( rne( W[k,n] / float(s_n) ), -127, 127 ),  q = 0 if s_n == 0
//
// HBM-bound: the algorithmic traffic is one read of W (4 or 2 bytes per
// weight) plus one write of q (1 byte per weight).  Design:
//  - Work unit: a panel of 32 columns over all K rows.  A thread-block
//    cluster of C CTAs owns a panel; CTA r of the cluster takes rows
//    [r kc, (r+1) kc).  Clusters are persistent (as many as fit at once)
//    and walk the panels.
//  - One producer thread per CTA streams each panel's rows twice through
//    one 3-stage ring of 32 KB slots (two CTAs per SM) with 2-D TMA loads
//    (one per slot, two for fp16, whose 512-row slot exceeds the 256-row
//    box limit): pass 1 (L2 evict-last) for the column |max|, pass 2
//    (evict-first) to quantize.  32 KB slots halve the waits and releases
//    per byte against 16 KB ones (measured: 171 -> 151 us on fp32
//    4096 x 27392).
//    The passes are interleaved one panel apart -- P1(0) P1(1) P2(0) P1(2)
//    P2(1) ... -- so pass 1 of the next panel streams from HBM while this
//    panel's maxima are combined, and pass 2 reads L2: the rows held between
//    the passes are two slices per CTA, a few tens of MB in all.
//  - The C partial maxima of a panel are combined over distributed shared
//    memory: each CTA publishes its 32 partial maxima, arrives on every
//    peer's exchange barrier, and before pass 2 reads all peers' values.
//  - q = rne(w / s) is computed as rne(w * fl(1/s)) where that product is
//    provably on the same side of every rounding boundary as the correctly
//    rounded quotient, and with the IEEE division otherwise (see
//    quantize_fast), so the codes are those of the exact definition.
#pragma once

#include "common.cuh"

namespace w8 {
namespace quant {

constexpr int kConsumerWarps = 16;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kPanel = 32;          // columns per panel
constexpr int kStages = 3;
constexpr int kBoxBytes = 32768;    // one ring slot
constexpr int kSmemBytes = kStages * kBoxBytes + 1024;
constexpr int kMaxCluster = 8;
constexpr int kPartBufs = 3;        // partial-maxima buffers (see the exchange)

// Box geometry: 256 fp32 rows or 512 fp16 rows of 32 columns (32 KB),
// loaded as kLoads TMA boxes of kTmaRows rows (a box has at most 256).  A
// consumer thread owns one 16-byte segment of a row: 4 fp32 or 8 fp16
// columns; kThreadsPerRow threads cover a row, kSweep rows per sweep of all
// consumers, kSweeps sweeps per box.
template <typename T>
struct Box {
    static constexpr int kCols = 16 / (int)sizeof(T);
    static constexpr int kThreadsPerRow = kPanel / kCols;
    static constexpr int kRowBytes = kPanel * (int)sizeof(T);
    static constexpr int kRows = kBoxBytes / kRowBytes;
    static constexpr int kTmaRows = kRows < 256 ? kRows : 256;
    static constexpr int kLoads = kRows / kTmaRows;
    static constexpr int kSweep = kConsumers / kThreadsPerRow;
    static constexpr int kSweeps = kRows / kSweep;
};

// rne(w / s) clamped to [-127, 127], equal to the correctly rounded quotient
// rounded to the nearest integer (ties to even), with inv_s = fl(1/s).
//
// r = fl(w * inv_s) differs from the exact w/s by at most 2^-23 |w/s|
// (two roundings of relative size 2^-24), and the correctly rounded
// quotient fl(w/s) differs from w/s by at most 2^-24 |w/s|.  For |r| < 126
// both are within 2^-15 of each other, so when r is more than 2^-13 away
// from every half-integer both round to the same integer (and no clamp
// applies).  Otherwise the quotient is formed with the IEEE division.
//
// Split in two so a row segment takes one branch, not one per element:
// quantize_fast returns rne(r) and whether r was unambiguous; for s == 0
// the caller passes inv_s = 0, so r = 0 and the code is 0 as defined.
// It stays off the special-function unit (no floor, no float-to-int
// conversion): adding 1.5 * 2^23 rounds |r| < 2^22 to the nearest integer,
// ties to even (the sum's unit in the last place is 1), and that integer
// is the sum's low mantissa bits, i.e. its bit pattern minus 0x4B400000.
// The distance from r to the nearest integer then decides whether r is
// more than 2^-13 away from every half-integer.
__device__ __forceinline__ int quantize_fast(float w, float inv_s, bool &sure) {
    constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23
    const float r = w * inv_s;
    const float t = r + kMagic;
    const float d = fabsf(r - (t - kMagic));
    sure = (fabsf(r) < 126.0f) & (d < 0.5f - 0x1p-13f);
    return __float_as_int(t) - 0x4B400000;
}
// The same for a whole row segment, with one decision for all of it: every
// product is unambiguous exactly when the largest |r| and the largest
// distance to the nearest integer pass the two tests.  code[e] is the
// rounding sum's bit pattern, 0x4B400000 + rne(r): its low byte, the only
// part the packing keeps, is already the code's two's-complement byte
// (0x4B400000 has a zero low byte).
template <int kN>
__device__ __forceinline__ bool quantize_fast_seg(const float (&w)[kN], const float (&inv_s)[kN], int (&code)[kN]) {
    constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23
    float rmax = 0.0f, dmax = 0.0f;
#pragma unroll
    for (int e = 0; e < kN; ++e) {
        const float r = w[e] * inv_s[e];
        const float t = r + kMagic;
        dmax = fmaxf(dmax, fabsf(r - (t - kMagic)));
        rmax = fmaxf(rmax, fabsf(r));
        code[e] = __float_as_int(t);
    }
    return (rmax < 126.0f) & (dmax < 0.5f - 0x1p-13f);
}

__device__ __forceinline__ int quantize_exact(float w, float s) {
    if (s == 0.0f) return 0;
    const int v = __float2int_rn(__fdiv_rn(w, s));
    return max(-127, min(127, v));
}

// The asymmetric form: clamp(rne(w / s) + z, -128, 127).  There |w / s|
// stays below about 255.2 (|w| is at most the range hi - lo, and s is that
// range over 255 up to the fp16 rounding of s), so the same argument holds
// with 256 in place of 126: r and fl(w/s) are within 2^-15 + 2^-16 of each
// other, and r more than 2^-13 from every half-integer decides the code.
__device__ __forceinline__ int quantize_fast_asym(float w, float inv_s, int z, bool &sure) {
    constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23
    const float r = w * inv_s;
    const float t = r + kMagic;
    const float d = fabsf(r - (t - kMagic));
    sure = (fabsf(r) < 256.0f) & (d < 0.5f - 0x1p-13f);
    return max(-128, min(127, (__float_as_int(t) - 0x4B400000) + z));
}
__device__ __forceinline__ int quantize_exact_asym(float w, float s, int z) {
    if (s == 0.0f) return 0;
    // |w / s| < 2^20 whenever s is non-zero (s >= the smallest fp16 subnormal)
    const float r = fminf(fmaxf(__fdiv_rn(w, s), -1048576.0f), 1048576.0f);
    return max(-128, min(127, __float2int_rn(r) + z));
}

// Scale and zero point of a channel from its range [lo, hi] (lo <= 0 <= hi):
// s = fp16_rne(fp32(hi - lo) / 255), z = clamp(rne(-128 - lo / s), -128, 127).
__device__ __forceinline__ void asym_params(float lo, float hi, __half &s16, int &z) {
    s16 = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 255.0f));
    const float s = __half2float(s16);
    z = 0;
    if (s != 0.0f) z = max(-128, min(127, __float2int_rn(__fsub_rn(-128.0f, __fdiv_rn(lo, s)))));
}

// The 16-byte row segment of a thread, widened to fp32.
template <typename T>
__device__ __forceinline__ void load_seg(const uint8_t *p, float (&v)[Box<T>::kCols]);
template <>
__device__ __forceinline__ void load_seg<float>(const uint8_t *p, float (&v)[4]) {
    const float4 a = *reinterpret_cast<const float4 *>(p);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}
template <>
__device__ __forceinline__ void load_seg<__half>(const uint8_t *p, float (&v)[8]) {
    const uint4 a = *reinterpret_cast<const uint4 *>(p);
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __half2 h = *reinterpret_cast<const __half2 *>(&w[i]);
        v[2 * i] = __low2float(h);
        v[2 * i + 1] = __high2float(h);
    }
}

// A launch quantizes a batch of up to kMaxBatch weights (one weight is a
// batch of one): the clusters walk one global panel index over all of
// them, and each panel finds its weight in the table.
constexpr int kMaxBatch = 64;

struct Mat {
    int8_t *q;
    uint16_t *scales;
    int8_t *zeros;     // asymmetric form only: [N] zero points
    int64_t K;
    int64_t N;
    int kc;            // rows per cluster rank (multiple of the box height)
    int panel0;        // this weight's first global panel
};

// kCap: the table's capacity (1 for a single weight, whose lookups then
// fold away; kMaxBatch for a batch).
template <int kCap>
struct Params {
    CUtensorMap maps[kCap];   // per weight: W [K, N], box 32 columns x Box<T>::kTmaRows rows
    Mat mats[kCap];
    int count;
    int panels;        // all weights' panels, ceil(N / 32) each
    int clusters;      // clusters in the grid
    float clip;        // symmetric form: bound = min(max|W|, clip); +inf: no clip
};

// Global panel g: its weight, its panel within the weight, and this
// cluster rank's rows of it.
struct PanelRef {
    int m;
    int local;
    int64_t k_begin, k_end;
    int nbox;
};

template <int kRows, int kCap>
__device__ __forceinline__ PanelRef panel_ref(const Params<kCap> &p, int g, uint32_t rank) {
    int m = 0;
    if constexpr (kCap > 1)
        while (m + 1 < p.count && p.mats[m + 1].panel0 <= g) ++m;
    PanelRef r;
    r.m = m;
    r.local = g - p.mats[m].panel0;
    r.k_begin = (int64_t)rank * p.mats[m].kc;
    r.k_end = min64(p.mats[m].K, r.k_begin + p.mats[m].kc);
    r.nbox = (int)((max64(0, r.k_end - r.k_begin) + kRows - 1) / kRows);
    return r;
}

// grid = clusters * C CTAs, cluster dims (C, 1, 1), kThreads threads,
// kSmemBytes dynamic shared memory.  The tensor map covers W [K, N] with
// a box of 32 columns x Box<T>::kTmaRows rows, no swizzle.
//
// Step j of a CTA (panels P_j = cid + j * clusters):
//   (a) pass 1 over P_j, partial maxima into part[j % 3];
//   (b) wait until every peer published P_{j-1}, read the peers' partial
//       maxima of P_{j-1}, form its scales;
//   (c) arrive on every peer's exchange barrier for P_j (this also tells
//       the peers that P_{j-1}'s values have been read here);
//   (d) pass 2 over P_{j-1}.
// A CTA overwrites part[j % 3] in (a) only after its own (b) of step j-1,
// which waited for the peers' (c) of step j-1, issued after their reads of
// P_{j-2} -- the values part[j % 3] held before -- so three buffers never
// race.  The exchange barriers alternate by panel parity.
//
// kAsym: the asymmetric form -- pass 1 keeps the column minimum and maximum
// (both start at 0: the range always holds 0), the exchange combines both,
// and pass 2 writes clamp(rne(w / s) + z, -128, 127).
// kLag: pass 2 of a panel runs after pass 1 of the next (the order above,
// which hides the exchange behind the next panel's stream); without it a
// panel's two passes run back to back, which holds half as many rows in
// L2 between them.  Clusters of 8 (the tall weights) do better without:
// 13696 x 4096 fp32 95.7 -> 83.4 us, while 4096 x 27392 (clusters of 4)
// goes 148.8 -> 152.9 us.
template <typename T, bool kAsym, int kCap, bool kLag = true>
__global__ void __launch_bounds__(kThreads, 2)
quantize_kernel(const __grid_constant__ Params<kCap> p) {
    using B = Box<T>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *ring = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    __shared__ uint64_t full[kStages], empty[kStages];
    __shared__ uint64_t xbar[2];                    // exchange barriers, by panel parity
    __shared__ uint64_t cbar;                       // consumer-only barrier
    __shared__ float part[kPartBufs][kPanel];       // this CTA's partial maxima
    __shared__ float red[kConsumerWarps][kPanel];
    __shared__ float col_scale[kPanel];
    __shared__ float col_inv[kPanel];
    // asymmetric form: partial minima, and the zero points
    __shared__ float part_lo[kAsym ? kPartBufs : 1][kPanel];
    __shared__ float red_lo[kAsym ? kConsumerWarps : 1][kPanel];
    __shared__ int col_zero[kPanel];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const uint32_t csize = cluster_size();
    const int cid = blockIdx.x / csize;
    const int npan = cid < p.panels ? (p.panels - cid + p.clusters - 1) / p.clusters : 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kConsumerWarps);
        }
        mbar_init(&xbar[0], csize);
        mbar_init(&xbar[1], csize);
        mbar_init(&cbar, kConsumers);
        fence_barrier_init();
        if (cid < p.panels) prefetch_tensormap(&p.maps[panel_ref<B::kRows, kCap>(p, cid, rank).m]);
    }
    // barrier initialisation is visible to the whole cluster before any
    // remote arrive
    cluster_sync_all();

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t keep = policy_evict_last(), drop = policy_evict_first();
            int s = 0;
            uint32_t ph = 0;
            int issued = 0;
            bool ok = true;
            for (int j = 0; j <= npan && ok; ++j) {
                for (int pass = 0; pass < 2 && ok; ++pass) {
                    // pass 0: P1 of panel j; pass 1: P2 of panel j - 1
                    // (kLag) or of panel j
                    const int pj = (pass == 0 || !kLag) ? j : j - 1;
                    if (pj < 0 || pj >= npan) continue;
                    const PanelRef pr = panel_ref<B::kRows, kCap>(p, cid + pj * p.clusters, rank);
                    for (int i = 0; i < pr.nbox; ++i) {
                        if (!mbar_wait_parked(&empty[s], ph ^ 1u, SITE_Q_EMPTY)) { ok = false; break; }
                        mbar_arrive_expect_tx(&full[s], kBoxBytes);
#pragma unroll
                        for (int l = 0; l < B::kLoads; ++l)
                            tma_load_2d_hint(ring + s * kBoxBytes + l * B::kTmaRows * B::kRowBytes, &p.maps[pr.m],
                                             pr.local * kPanel,
                                             (int32_t)(pr.k_begin + (int64_t)i * B::kRows + l * B::kTmaRows),
                                             &full[s], pass == 0 ? keep : drop);
                        ++issued;
                        if (++s == kStages) { s = 0; ph ^= 1u; }
                    }
                }
            }
            // every issued copy has landed before the CTA can leave
            for (int i = 0; i < kStages && i < issued; ++i) {
                if (--s < 0) { s = kStages - 1; ph ^= 1u; }
                mbar_wait(&full[s], ph, SITE_Q_LOAD, 10000000ull);
            }
        }
    } else {
        // ------------------------------------------------------ consumers
        const int c = threadIdx.x;                  // 0 .. kConsumers - 1
        const int t = c % B::kThreadsPerRow;        // column segment
        const int rsub = c / B::kThreadsPerRow;     // row within a sweep
        const int col0 = t * B::kCols;              // first panel column of the segment
        int s = 0;
        uint32_t ph = 0;
        uint32_t cph = 0;
        bool ok = true;
        auto csync = [&]() -> bool {
            mbar_arrive(&cbar);
            const bool r = warp_all(mbar_wait_parked(&cbar, cph, SITE_Q_SYNC));
            cph ^= 1u;
            return r;
        };
        for (int j = 0; j <= npan && ok; ++j) {
            // ---------------- (a) pass 1 over panel j: column |max|
            if (j < npan) {
                const PanelRef pr1 = panel_ref<B::kRows, kCap>(p, cid + j * p.clusters, rank);
                float amax[B::kCols], amin[B::kCols];   // amin: asymmetric form only
#pragma unroll
                for (int e = 0; e < B::kCols; ++e) amax[e] = amin[e] = 0.0f;
                for (int i = 0; i < pr1.nbox; ++i) {
                    if (!warp_all(mbar_wait_parked(&full[s], ph, SITE_Q_LOAD))) { ok = false; break; }
                    const uint8_t *box = ring + s * kBoxBytes;
#pragma unroll
                    for (int w = 0; w < B::kSweeps; ++w) {
                        float v[B::kCols];
                        load_seg<T>(box + (rsub + w * B::kSweep) * B::kRowBytes + 16 * t, v);
                        if constexpr (kAsym) {
#pragma unroll
                            for (int e = 0; e < B::kCols; ++e) {
                                amax[e] = fmaxf(amax[e], v[e]);
                                amin[e] = fminf(amin[e], v[e]);
                            }
                        } else {
#pragma unroll
                            for (int e = 0; e < B::kCols; ++e) amax[e] = fmaxf(amax[e], fabsf(v[e]));
                        }
                    }
                    // the slot's values are in registers before it is released
                    // (arithmetic alone could be scheduled after the arrive,
                    // with a load still reading the slot the next copy fills)
#pragma unroll
                    for (int e = 0; e < B::kCols; ++e) {
                        asm volatile("" ::"f"(amax[e]));
                        if constexpr (kAsym) asm volatile("" ::"f"(amin[e]));
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[s]);
                    if (++s == kStages) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
                // lanes with the same t hold the same columns
#pragma unroll
                for (int off = B::kThreadsPerRow; off < 32; off <<= 1)
#pragma unroll
                    for (int e = 0; e < B::kCols; ++e) {
                        amax[e] = fmaxf(amax[e], __shfl_xor_sync(0xffffffffu, amax[e], off));
                        if constexpr (kAsym) amin[e] = fminf(amin[e], __shfl_xor_sync(0xffffffffu, amin[e], off));
                    }
                if (lane < B::kThreadsPerRow) {
#pragma unroll
                    for (int e = 0; e < B::kCols; ++e) {
                        red[warp][col0 + e] = amax[e];
                        if constexpr (kAsym) red_lo[warp][col0 + e] = amin[e];
                    }
                }
                if (!csync()) { ok = false; break; }
                if (c < kPanel) {
                    float m = 0.0f;
#pragma unroll
                    for (int w = 0; w < kConsumerWarps; ++w) m = fmaxf(m, red[w][c]);
                    part[j % kPartBufs][c] = m;
                    if constexpr (kAsym) {
                        float lo = 0.0f;
#pragma unroll
                        for (int w = 0; w < kConsumerWarps; ++w) lo = fminf(lo, red_lo[w][c]);
                        part_lo[j % kPartBufs][c] = lo;
                    }
                }
            }
            if constexpr (kLag) {
                if (j == 0) {
                    // (c) for panel 0; nothing to read yet
                    if (!csync()) { ok = false; break; }
                    if (c < (int)csize) mbar_arrive_cluster(mapa_shared(smem_u32(&xbar[0]), (uint32_t)c));
                    continue;
                }
            } else {
                // (c) publish panel j before combining it
                if (j >= npan) break;
                if (!csync()) { ok = false; break; }
                if (c < (int)csize) mbar_arrive_cluster(mapa_shared(smem_u32(&xbar[j & 1]), (uint32_t)c));
            }
            // ---------------- (b) combine the maxima of panel j - 1 (kLag) or j
            const int pj = kLag ? j - 1 : j;
            const PanelRef pr = panel_ref<B::kRows, kCap>(p, cid + pj * p.clusters, rank);
            // this weight's outputs, read from the parameter table once
            const int64_t mN = p.mats[pr.m].N;
            int8_t *const mq = p.mats[pr.m].q;
            uint16_t *const ms = p.mats[pr.m].scales;
            int8_t *const mz = p.mats[pr.m].zeros;
            if (!warp_all(mbar_wait_cluster(&xbar[pj & 1], (pj >> 1) & 1, SITE_Q_XCHG))) { ok = false; break; }
            if (c < kPanel) {
                float m = 0.0f;
                const uint32_t local = smem_u32(&part[pj % kPartBufs][c]);
                for (uint32_t r = 0; r < csize; ++r) m = fmaxf(m, ld_dsmem_f32(mapa_shared(local, r)));
                __half s16;
                int z = 0;
                if constexpr (kAsym) {
                    float lo = 0.0f;
                    const uint32_t local_lo = smem_u32(&part_lo[pj % kPartBufs][c]);
                    for (uint32_t r = 0; r < csize; ++r) lo = fminf(lo, ld_dsmem_f32(mapa_shared(local_lo, r)));
                    asym_params(lo, m, s16, z);
                } else {
                    s16 = __float2half_rn(__fdiv_rn(fminf(m, p.clip), 127.0f));
                }
                const float sf = __half2float(s16);
                col_scale[c] = sf;
                col_inv[c] = sf != 0.0f ? __frcp_rn(sf) : 0.0f;
                col_zero[c] = z;
                const int64_t n = (int64_t)pr.local * kPanel + c;
                if (rank == 0 && n < mN) {
                    ms[n] = __half_as_ushort(s16);
                    if constexpr (kAsym) mz[n] = (int8_t)z;
                }
            }
            // every consumer's partial maxima of panel j are in part[] and
            // every read of panel j - 1's values is done
            if (!csync()) { ok = false; break; }
            // ---------------- (c) publish panel j
            if (kLag && j < npan && c < (int)csize)
                mbar_arrive_cluster(mapa_shared(smem_u32(&xbar[j & 1]), (uint32_t)c));
            // ---------------- (d) pass 2 over panel j - 1 (from L2)
            float sc[B::kCols], inv[B::kCols];
            int zp[B::kCols];   // asymmetric form only
#pragma unroll
            for (int e = 0; e < B::kCols; ++e) {
                sc[e] = col_scale[col0 + e];
                inv[e] = col_inv[col0 + e];
                zp[e] = col_zero[col0 + e];
            }
            const int64_t n0 = (int64_t)pr.local * kPanel + col0;
            const bool cols_ok = n0 < mN;   // N % 8 == 0: a segment is all in or all out
            for (int i = 0; i < pr.nbox; ++i) {
                if (!warp_all(mbar_wait_parked(&full[s], ph, SITE_Q_LOAD))) { ok = false; break; }
                const uint8_t *box = ring + s * kBoxBytes;
#pragma unroll
                for (int w = 0; w < B::kSweeps; ++w) {
                    const int rloc = rsub + w * B::kSweep;
                    float v[B::kCols];
                    load_seg<T>(box + rloc * B::kRowBytes + 16 * t, v);
                    int code[B::kCols];   // codes in the low bytes
                    bool sure = true;
                    if constexpr (kAsym) {
#pragma unroll
                        for (int e = 0; e < B::kCols; ++e) {
                            bool se;
                            code[e] = quantize_fast_asym(v[e], inv[e], zp[e], se);
                            sure &= se;
                        }
                    } else {
                        sure = quantize_fast_seg<B::kCols>(v, inv, code);
                    }
                    if (!sure) {   // rare: some product lies near a rounding boundary
#pragma unroll
                        for (int e = 0; e < B::kCols; ++e) {
                            if constexpr (kAsym)
                                code[e] = quantize_exact_asym(v[e], sc[e], zp[e]);
                            else
                                code[e] = quantize_exact(v[e], sc[e]);
                        }
                    }
                    uint32_t packed[B::kCols / 4];
#pragma unroll
                    for (int g = 0; g < B::kCols / 4; ++g) {
                        // low bytes of four codes into one word
                        const uint32_t lo = __byte_perm((uint32_t)code[4 * g], (uint32_t)code[4 * g + 1], 0x0040);
                        const uint32_t hi = __byte_perm((uint32_t)code[4 * g + 2], (uint32_t)code[4 * g + 3], 0x0040);
                        packed[g] = __byte_perm(lo, hi, 0x5410);
                    }
                    const int64_t k = pr.k_begin + (int64_t)i * B::kRows + rloc;
                    if (k < pr.k_end && cols_ok) {
                        int8_t *dst = mq + k * mN + n0;
                        if (B::kCols == 4)
                            *reinterpret_cast<uint32_t *>(dst) = packed[0];
                        else
                            *reinterpret_cast<uint2 *>(dst) = make_uint2(packed[0], packed[B::kCols / 4 - 1]);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
                if (++s == kStages) { s = 0; ph ^= 1u; }
            }
        }
    }
    // no CTA leaves while a peer may still read its shared memory or arrive
    // on its barriers; every thread reaches this point on every path
    cluster_sync_all();
}

}  // namespace quant
}  // namespace w8
