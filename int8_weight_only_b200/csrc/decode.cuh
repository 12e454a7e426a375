// Decode-regime W8A16 linear (M <= 64 tokens): Y = X . dequant(q) (+ bias).
//
// For few tokens the cost is streaming the int8 weight from HBM once
// (TPU-MLIR ChatGLM2 W8A16 article, section 4: when the left matrix is
// small, loading the right matrix dominates, int8 halves that load, and the
// cast and scale hide under it).  Design:
//  - The packed weight is a sequence of T = ceil(N/128) * ceil(K/64) tiles
//    of 8 KB, channel-block major.  A single wave of G CTAs (one per SM)
//    splits that sequence into G equal contiguous ranges (stream-K split),
//    so every SM streams the same number of bytes and no tail wave exists.
//  - One producer warp per CTA moves each stage (up to 4 tiles = 32 KB, plus
//    the matching 64-wide slices of X) into a 4-stage shared-memory ring
//    with one 1-D bulk copy (cp.async.bulk) for the tiles and one 3-D TMA
//    load for the four X slices (one 2-D load per slice when K is not a
//    multiple of 64); 8 consumer warps each own 16 of the tile's 128
//    channels.
//  - Consumers widen int8 to fp16 in registers (prmt into the exponent
//    pattern of 1024, then one fp16x2 subtraction) and accumulate in fp32
//    with mma.sync m16n8k16 (channels as the MMA rows, tokens as its 8
//    columns, up to 8 token tiles), so conversion plus multiply-add stay a
//    small fraction of the issue budget; up to 64 tokens the weight stream
//    still sets the pace.  The stage's tiles are unrolled and
//    each 16-wide k slice has its own accumulator, so the mma results do not
//    form one long dependency chain.
//  - Only a CTA's first and last channel block can be split with other
//    CTAs.  A split part is published to the workspace (fp32 partial sums,
//    one fence, an atomic counter per block) as soon as it is done, and the
//    last contributor to arrive adds all parts in CTA order (so the result
//    does not depend on arrival order), applies scale and bias and resets
//    the counter.  The common two-way split (this CTA streams the first K
//    blocks of its last channel block last, the next CTA streams the rest
//    first) short-cuts this: when this CTA reaches that block the next CTA
//    has normally published already, so its part is loaded into registers
//    during the stream and the block is finished with no fence or atomic.
//  - Few channel blocks (a 4096 x 4096 layer has 32 for 148 SMs): the
//    cluster form.  A thread-block cluster of C CTAs owns one channel block
//    and splits its K range evenly; at the end CTAs 1..C-1 store their fp32
//    parts into CTA 0's shared memory with asynchronous distributed-shared-
//    memory stores whose bytes complete CTA 0's barrier, and CTA 0 adds the
//    parts in rank order, scales and stores.  No workspace, no counter, no
//    global round trip, no fence.
//  - The global round trips of a split never stall the stream: a helper
//    warp counts the part a CTA publishes mid-stream (its first block) and
//    watches for the next CTA's part of its last block; the consumers only
//    store their part and read the helper's verdicts, and a CTA that turns
//    out to be the last contributor of its first block finishes that block
//    after its stream.
#pragma once

#include "common.cuh"

namespace w8 {
namespace decode {

constexpr int kConsumerWarps = 8;
// warps 0-7 consumers, warp 8 producer, warp 9 helper
constexpr int kThreads = (kConsumerWarps + 2) * 32;
constexpr int kTilesPerStage = 4;
constexpr int kMaxStages = 4;
constexpr int kTileBytes = 8192;
constexpr int kStageW = kTilesPerStage * kTileBytes;
constexpr int kMaxTokens = 64;     // MT <= 8 token tiles of 8
constexpr int kMaxClusterDec = 8;  // CTAs per channel block in the cluster form
constexpr int kMaxTokensCluster = 16;   // the cluster form takes MT <= 2

// MT = token tiles of 8 (1, 2, 4 or 8: up to 8, 16, 32 or 64 tokens).
template <int MT>
struct Cfg {
    static constexpr int kXRows = 8 * MT;                // token rows per X box
    static constexpr int kXBoxBytes = kXRows * 128;      // box {64 fp16, kXRows}
    static constexpr int kStageX = kTilesPerStage * kXBoxBytes;
    static constexpr int kStageBytes = kStageW + kStageX;
    static constexpr int kStages = MT <= 4 ? 4 : 3;      // ring within shared memory
    static constexpr int kSmemBytes = kStages * kStageBytes + 1024;
    static constexpr int kPartialFloats = kConsumerWarps * 4 * MT * 32;   // per slot
    // independent accumulators per token tile: one per 16-wide k slice for
    // few tokens (otherwise one long mma chain), one when the token tiles
    // already give enough independent chains
    static constexpr int kNS = MT <= 2 ? 4 : 1;
    // cluster form: the parts of CTAs 1..C-1 in CTA 0, after the ring
    static constexpr int kSmemBytesCluster = kSmemBytes + (kMaxClusterDec - 1) * kPartialFloats * 4;
};

// Workspace: [partials: 2 slots per SM, sized for MT = 8][counters: one
// int32 per channel block].  The same size for every M and N, so the
// counters always sit at the same offset.
constexpr int kMaxPartialFloats = Cfg<8>::kPartialFloats;
// Partial slot size when at most 16 tokens are allowed.
constexpr int kPartialFloats16 = Cfg<2>::kPartialFloats;

// Test hook (0 in normal use): the helper waits this long before counting
// the CTA's first part, so that the next-CTA fallback and the finish of a
// first block after the stream run deterministically.
__device__ unsigned long long g_helper_delay_ns = 0;

struct Params {
    const uint8_t *packed;
    const uint16_t *scales;
    const int8_t *zeros;    // zero points (asymmetric codes), else unused
    const uint16_t *bias;   // may be null
    uint16_t *Y;
    int *counters;
    float *partials;
    // outlier split (all null otherwise): Y += X[:, rows] . vals per channel
    const uint16_t *X;           // [M, K] fp16, the activations
    const int32_t *o_count;      // [N]
    const int32_t *o_rows;       // [N][o_cap]
    const uint16_t *o_vals;      // [N][o_cap] fp16
    int o_cap;
    int64_t K;
    // 1: tmap_x is the 3-D view X[kb][m][c] = X[m][64 kb + c] (K % 64 == 0),
    // and a stage's X slices come in one load; 0: the 2-D map, one load per
    // 64-wide slice
    int x3;
    int M;
    int64_t N;
    int KB;        // ceil(K / 64)
    uint32_t T;    // tiles; the host guarantees T * (G + 1) < 2^32
    uint32_t G;    // CTAs
};

// Stream-K split in 32-bit arithmetic (64-bit division is a long software
// sequence and sat on the critical path of every stage).
__device__ __forceinline__ uint32_t range_start(uint32_t i, uint32_t T, uint32_t G) {
    return i * T / G;
}
// CTA whose range holds tile t.
__device__ __forceinline__ uint32_t owner_of(uint32_t t, uint32_t T, uint32_t G) {
    return ((t + 1) * G - 1) / T;
}

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint16_t out_f16(float acc, float s, float b) {
    return __half_as_ushort(__float2half_rn(fmaf(acc, s, b)));
}

// Thread (g = lane/4, t = lane%4) of consumer warp w holds, for token tile
// mt, acc[mt] = Y^T[n][m] at n = 16w+g (+8 for elements 2,3) and
// m = 8mt + 2t (+1 for elements 1,3).
template <int MT>
__device__ __forceinline__ void store_y(const Params &p, uint32_t b, int warp, int lane,
                                        const float (&acc)[MT][4]) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int64_t n = (int64_t)b * 128 + 16 * warp + g + 8 * half;
        if (n >= p.N) continue;
        const float s = __half2float(__ushort_as_half(p.scales[n]));
        const float bb = p.bias ? __half2float(__ushort_as_half(p.bias[n])) : 0.0f;
        // outlier split: the kept weights' products, added before rounding
        float extra[MT][2] = {};
        if (p.o_count) {
            const int cnt = p.o_count[n];
            for (int j = 0; j < cnt; ++j) {
                const int64_t k = p.o_rows[n * p.o_cap + j];
                const float v = __half2float(__ushort_as_half(p.o_vals[n * p.o_cap + j]));
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int m = 8 * mt + 2 * t + e;
                        if (m < p.M) extra[mt][e] = fmaf(__half2float(__ushort_as_half(p.X[m * p.K + k])), v,
                                                         extra[mt][e]);
                    }
            }
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int m = 8 * mt + 2 * t + e;
                if (m < p.M) p.Y[(int64_t)m * p.N + n] = out_f16(acc[mt][2 * half + e], s, bb + extra[mt][e]);
            }
        }
    }
}

// Sum of the parts of channel block b held by CTAs jf..jl, added in CTA
// order whoever finishes the block (so the result does not depend on who
// does).  The part of CTA `self` comes from `own` when use_own, otherwise
// it is read back like the others.  Up to kPar parts are loaded together
// (one L2 round trip).
template <int MT>
__device__ __forceinline__ void gather_parts(const Params &p, uint32_t b, uint32_t jf, uint32_t jl, uint32_t self,
                                             bool use_own, const float (&own)[MT][4], int warp, int lane,
                                             float (&sum)[MT][4]) {
    constexpr int kPar = MT <= 2 ? 8 : 2;
    const uint32_t KB = (uint32_t)p.KB;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sum[mt][e] = 0.0f;
    for (uint32_t j0 = jf; j0 <= jl; j0 += kPar) {
        float part[kPar][MT][4];
#pragma unroll
        for (int u = 0; u < kPar; ++u) {
            const uint32_t j = j0 + u;
            if (j <= jl && !(use_own && j == self)) {
                const uint32_t sj = (range_start(j, p.T, p.G) / KB == b) ? 2 * j : 2 * j + 1;
                const float *src = p.partials + (int64_t)sj * Cfg<MT>::kPartialFloats;
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        part[u][mt][e] = __ldcg(&src[(warp * 4 * MT + 4 * mt + e) * 32 + lane]);
            } else {
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) part[u][mt][e] = own[mt][e];
            }
        }
#pragma unroll
        for (int u = 0; u < kPar; ++u) {
            if (j0 + u <= jl) {
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) sum[mt][e] += part[u][mt][e];
            }
        }
    }
}

// Sum the per-k-slice accumulators of each token tile.
template <int MT, int NS>
__device__ __forceinline__ void fold(const float (&acc)[MT][NS][4], float (&out)[MT][4]) {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if constexpr (NS == 4)
                out[mt][e] = (acc[mt][0][e] + acc[mt][1][e]) + (acc[mt][2][e] + acc[mt][3][e]);
            else
                out[mt][e] = acc[mt][0][e];
        }
}

// kZp: asymmetric codes -- every weight is widened to q - z_n (exact in
// fp16) instead of q; nothing else changes.
// kCl: the cluster form -- grid = channel blocks x C CTAs, cluster dims
// (C, 1, 1), C <= kMaxClusterDec, MT <= 2; Cfg::kSmemBytesCluster of
// dynamic shared memory; the workspace is not used.
template <int MT, bool kZp, bool kCl = false>
__global__ void __launch_bounds__(kThreads, 1)
decode_kernel(const __grid_constant__ CUtensorMap tmap_x, const Params p) {
    using C = Cfg<MT>;
    static_assert(!kCl || MT <= 2, "cluster form: up to 16 tokens");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    __shared__ uint64_t full[kMaxStages], empty[kMaxStages];
    __shared__ uint64_t fix_bar;
    __shared__ int last_flag[2];   // [1]: last contributor (general path)
    // helper handshakes: pub_bar -- the consumers stored their first part;
    // start_bar -- the helper counted it (helper_flag[1]: this CTA was the
    // last contributor); tail_bar -- the consumers reached the last block;
    // pre_bar -- the helper's verdict on the next CTA's part (helper_flag[0])
    __shared__ uint64_t pub_bar, start_bar, tail_bar, pre_bar;
    __shared__ int helper_flag[2];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t cta = blockIdx.x;
    const uint32_t KB = (uint32_t)p.KB;
    // cluster form: rank crank of csz CTAs takes the crank-th of csz even
    // shares of channel block blockIdx.x / csz
    uint32_t crank = 0, csz = 1;
    if constexpr (kCl) {
        crank = cluster_rank();
        csz = cluster_size();
    }
    const uint32_t t_begin = kCl ? (cta / csz) * KB + crank * KB / csz : range_start(cta, p.T, p.G);
    const uint32_t t_end = kCl ? (cta / csz) * KB + (crank + 1) * KB / csz : range_start(cta + 1, p.T, p.G);
    const uint32_t first_b = t_begin / KB;
    const uint32_t last_b = (t_end - 1) / KB;
    // The first channel block starts past K block 0 and more work follows:
    // its part is published mid-stream (the helper counts it).
    const bool start_pub = !kCl && (t_begin % KB != 0) && ((first_b + 1) * KB < t_end);
    // The last channel block, when only its first K blocks are here and the
    // rest belongs to the next CTA alone (a two-way split with this CTA
    // holding the part that is streamed last): the next CTA publishes its
    // part early in its stream, so this CTA can usually pick it up while
    // streaming its own part and finish the block without any fence or
    // atomic at the end.
    const bool tail_pair = !kCl && (t_end - last_b * KB < KB) && (last_b * KB >= t_begin) &&
                           owner_of((last_b + 1) * KB - 1, p.T, p.G) == cta + 1;
    // cluster form: the parts of ranks 1..csz-1, in rank 0 (after the ring)
    float *red_parts = reinterpret_cast<float *>(base + C::kStages * C::kStageBytes);
    __shared__ uint64_t red_bar;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        mbar_init(&fix_bar, kConsumerWarps * 32);
        mbar_init(&pub_bar, kConsumerWarps * 32);
        mbar_init(&start_bar, 1);
        mbar_init(&tail_bar, 1);
        mbar_init(&pre_bar, 1);
        if constexpr (kCl) {
            // one arrival (below) plus the bytes of every peer's part
            mbar_init(&red_bar, 1);
            if (crank == 0 && csz > 1)
                mbar_arrive_expect_tx(&red_bar, (csz - 1) * C::kPartialFloats * (uint32_t)sizeof(float));
        }
        fence_barrier_init();
        prefetch_tensormap(&tmap_x);
    }
    __syncthreads();
    // cluster form: every thread arrives here; a peer waits for the phase
    // (rank 0's barrier initialised) before its first remote access
    if constexpr (kCl) cluster_arrive_relaxed();
    // The next call may start as soon as SMs free up; it only touches this
    // call's data after its own pdl_wait.
    pdl_launch_dependents();

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            // The weights are not written by the previous kernel in any
            // sane use, but only an L2 prefetch (never stale) runs before
            // the wait: the first ring's worth of this CTA's range.
            const uint32_t pre_tiles = min(t_end - t_begin, (uint32_t)(C::kStages * kTilesPerStage));
            prefetch_l2(p.packed + (size_t)t_begin * kTileBytes, pre_tiles * kTileBytes);
            pdl_wait();
            const uint64_t policy = policy_evict_first();
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            uint32_t kb = t_begin % KB;
            for (uint32_t t = t_begin; t < t_end;) {
                const int cnt = (int)min(min((uint32_t)kTilesPerStage, t_end - t), KB - kb);
                if (!mbar_wait(&empty[stage], phase ^ 1u, SITE_DEC_EMPTY)) break;
                uint8_t *ws = base + stage * C::kStageBytes;
                uint8_t *xs = ws + kStageW;
                if (p.x3) {
                    // one box of four 64-wide slices (beyond the last K
                    // block the fill is zero, and those bytes count too)
                    mbar_arrive_expect_tx(&full[stage], cnt * kTileBytes + kTilesPerStage * C::kXBoxBytes);
                    bulk_g2s_hint(ws, p.packed + (size_t)t * kTileBytes, cnt * kTileBytes, &full[stage], policy);
                    tma_load_3d(xs, &tmap_x, 0, 0, (int)kb, &full[stage]);
                } else {
                    mbar_arrive_expect_tx(&full[stage], cnt * (kTileBytes + C::kXBoxBytes));
                    bulk_g2s_hint(ws, p.packed + (size_t)t * kTileBytes, cnt * kTileBytes, &full[stage], policy);
                    for (int j = 0; j < cnt; ++j)
                        tma_load_2d(xs + j * C::kXBoxBytes, &tmap_x, (int)(kb + j) * 64, 0, &full[stage]);
                }
                t += cnt;
                kb += cnt;
                if (kb == KB) kb = 0;
                ++issued;
                if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
            }
            // every copy this CTA issued has landed before the CTA can exit
            // (normally long since consumed; matters only after a timeout)
            for (int i = 0; i < C::kStages && i < issued; ++i) {
                if (--stage < 0) { stage = C::kStages - 1; phase ^= 1u; }
                mbar_wait(&full[stage], phase, SITE_DEC_DRAIN, 10000000ull);
            }
        }
        return;
    }

    if (warp == kConsumerWarps + 1) {
        // -------------------------------------------------------- helper
        if (lane == 0 && (start_pub || tail_pair)) {
            pdl_wait();
            if (start_pub) {
                // count the first part once every consumer has stored its
                // share of it (their arrivals release the stores; the
                // atomic publishes them at GPU scope)
                int last = 0;
                if (mbar_wait_parked(&pub_bar, 0, SITE_DEC_PUB)) {
                    const unsigned long long delay = g_helper_delay_ns;
                    if (delay) {
                        const unsigned long long t1 = globaltimer_ns();
#pragma unroll 1
                        while (globaltimer_ns() - t1 < delay) __nanosleep(1000);
                    }
                    const uint32_t jf = owner_of(first_b * KB, p.T, p.G);
                    const uint32_t jl = owner_of((first_b + 1) * KB - 1, p.T, p.G);
                    const int old = atomic_add_acq_rel_gpu(&p.counters[first_b], 1);
                    last = ((uint32_t)old == jl - jf);
                }
                helper_flag[1] = last;
                mbar_arrive(&start_bar);
            }
            if (tail_pair) {
                // poll until the next CTA's part is counted, or until the
                // consumers reach the block (then one last look)
                int pub = 0;
                const unsigned long long t0 = globaltimer_ns();
#pragma unroll 1
                while (true) {
                    const bool reached = mbar_test_wait(&tail_bar, 0);
                    if (ld_acquire_gpu(&p.counters[last_b]) == 1) {
                        pub = 1;
                        break;
                    }
                    if (reached) break;
                    if (globaltimer_ns() - t0 > kWaitLimitNs) {
                        record_timeout(SITE_DEC_POLL);
                        break;
                    }
                    __nanosleep(256);
                }
                helper_flag[0] = pub;
                mbar_arrive(&pre_bar);
            }
        }
        return;
    }

    // ---------------------------------------------------------- consumers
    pdl_wait();   // before any global access of this grid's consumers
    const int g = lane >> 2, tq = lane & 3;
    const int h = (g >> 1) & 3;                     // chunk swizzle of rows 16w+g, 16w+g+8
    const int row_lo = 16 * warp + g;
    const int a_off_lo = row_lo * 64 + ((tq ^ h) << 4);
    const int a_off_hi = (row_lo + 8) * 64 + ((tq ^ h) << 4);
    int x_off[MT][2];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const int m = 8 * mt + g;
        x_off[mt][0] = m * 128 + (((2 * tq) ^ (m & 7)) << 4);
        x_off[mt][1] = m * 128 + (((2 * tq + 1) ^ (m & 7)) << 4);
    }

    // independent accumulators (see Cfg::kNS)
    constexpr int NS = C::kNS;
    float acc[MT][NS][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int jj = 0; jj < NS; ++jj)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[mt][jj][e] = 0.0f;

    uint32_t fix_phase = 0;
    // all 256 consumer threads meet (bounded); false if the wait ran out
    auto consumers_sync = [&]() -> bool {
        mbar_arrive(&fix_bar);
        const bool ok = mbar_wait(&fix_bar, fix_phase, SITE_DEC_FIX);
        fix_phase ^= 1u;
        return ok;
    };

    float pre[MT][4];
    bool have_pre = false;
    bool pre_pending = false;   // the helper's verdict on it not read yet
    // the next CTA's part of the last block, into registers
    auto load_pre = [&]() {
        const float *src = p.partials + (int64_t)(2 * (cta + 1)) * C::kPartialFloats;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) pre[mt][e] = __ldcg(&src[(warp * 4 * MT + 4 * mt + e) * 32 + lane]);
    };

    int stage = 0;
    uint32_t phase = 0;
    uint32_t b = first_b;                       // channel block of tile t
    uint32_t kb = t_begin - first_b * KB;       // its K block
    bool seg_whole = (kb == 0);                 // segment started at K block 0
    bool seg_new = true;
    // asymmetric codes: 1152 + z of this thread's two channels (rows g, g+8)
    uint32_t zc_lo = 0x64806480u, zc_hi = 0x64806480u;

    for (uint32_t t = t_begin; t < t_end;) {
        if (seg_new) {
            seg_new = false;
            if constexpr (kZp) {
                const int64_t n_lo = (int64_t)b * 128 + row_lo;
                zc_lo = zp_bias2(n_lo < p.N ? p.zeros[n_lo] : 0);
                zc_hi = zp_bias2(n_lo + 8 < p.N ? p.zeros[n_lo + 8] : 0);
            }
            if (tail_pair && b == last_b) {
                if (threadIdx.x == 0) mbar_arrive(&tail_bar);
                pre_pending = true;
            }
        }
        // the helper's verdict, picked up without waiting; the part itself
        // then arrives during the rest of the stream
        if (pre_pending && warp_all(mbar_test_wait(&pre_bar, 0))) {
            pre_pending = false;
            have_pre = helper_flag[0] != 0;
            if (have_pre) load_pre();
        }
        const int cnt = (int)min(min((uint32_t)kTilesPerStage, t_end - t), KB - kb);
        // parked, not spinning: eight warps polling one barrier take issue
        // slots from the warps that have data
        if (!mbar_wait_parked(&full[stage], phase, SITE_DEC_FULL)) return;
        const uint8_t *ws = base + stage * C::kStageBytes;
        const uint8_t *xs = ws + kStageW;
#pragma unroll
        for (int j = 0; j < kTilesPerStage; ++j) {
            if (j < cnt) {
                const uint8_t *tile = ws + j * kTileBytes;
                const uint4 alo = *reinterpret_cast<const uint4 *>(tile + a_off_lo);
                const uint4 ahi = *reinterpret_cast<const uint4 *>(tile + a_off_hi);
                uint4 xv[MT][2];
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    xv[mt][0] = *reinterpret_cast<const uint4 *>(xs + j * C::kXBoxBytes + x_off[mt][0]);
                    xv[mt][1] = *reinterpret_cast<const uint4 *>(xs + j * C::kXBoxBytes + x_off[mt][1]);
                }
                const uint32_t wl[4] = {alo.x, alo.y, alo.z, alo.w};
                const uint32_t wh[4] = {ahi.x, ahi.y, ahi.z, ahi.w};
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    uint32_t a0, a1, a2, a3;
                    if constexpr (kZp) {
                        a0 = unbias2_by(widen_lo2(wl[jj]), zc_lo);
                        a1 = unbias2_by(widen_lo2(wh[jj]), zc_hi);
                        a2 = unbias2_by(widen_hi2(wl[jj]), zc_lo);
                        a3 = unbias2_by(widen_hi2(wh[jj]), zc_hi);
                    } else {
                        a0 = unbias2(widen_lo2(wl[jj]));   // row g,   k +0,+1
                        a1 = unbias2(widen_lo2(wh[jj]));   // row g+8, k +0,+1
                        a2 = unbias2(widen_hi2(wl[jj]));   // row g,   k +2,+3
                        a3 = unbias2(widen_hi2(wh[jj]));   // row g+8, k +2,+3
                    }
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        const uint4 &xq = xv[mt][jj >> 1];
                        const uint32_t b0 = (jj & 1) ? xq.z : xq.x;
                        const uint32_t b1 = (jj & 1) ? xq.w : xq.y;
                        mma_16816(acc[mt][jj % NS], a0, a1, a2, a3, b0, b1);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);
        t += cnt;
        kb += cnt;
        if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        if (t != t_end && kb != KB) continue;

        // ------------------------------------------------ end of a segment
        // This CTA's part of channel block b is done.  It is the whole block
        // if it started at K block 0 and reached the end.
        float sum[MT][4];
        fold<MT, NS>(acc, sum);
        if constexpr (kCl) {
            // the cluster's parts of channel block b, added in rank order in
            // rank 0 (this is the CTA's only segment)
            if (csz == 1) {
                store_y<MT>(p, b, warp, lane, sum);
            } else if (crank != 0) {
                cluster_wait();
                const uint32_t dst =
                    mapa_shared(smem_u32(red_parts + (crank - 1) * C::kPartialFloats), 0);
                const uint32_t bar0 = mapa_shared(smem_u32(&red_bar), 0);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
                    st_async_dsmem_v4(dst + 16u * (uint32_t)((warp * MT + mt) * 32 + lane), sum[mt][0], sum[mt][1],
                                      sum[mt][2], sum[mt][3], bar0);
            } else {
                if (!warp_all(mbar_wait(&red_bar, 0, SITE_DEC_CLUSTER))) return;
                for (uint32_t r = 1; r < csz; ++r) {
                    const float *src = red_parts + (r - 1) * C::kPartialFloats;
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        const float4 v = *reinterpret_cast<const float4 *>(src + 4 * ((warp * MT + mt) * 32 + lane));
                        sum[mt][0] += v.x;
                        sum[mt][1] += v.y;
                        sum[mt][2] += v.z;
                        sum[mt][3] += v.w;
                    }
                }
                store_y<MT>(p, b, warp, lane, sum);
            }
            break;
        }
        if (!(seg_whole && kb == KB) && pre_pending) {
            // end of the last block before the verdict was seen (a short
            // block): wait for it here
            if (!warp_all(mbar_wait(&pre_bar, 0, SITE_DEC_PRE))) return;
            pre_pending = false;
            have_pre = helper_flag[0] != 0;
            if (have_pre) load_pre();
        }
        if (seg_whole && kb == KB) {
            store_y<MT>(p, b, warp, lane, sum);
        } else if (have_pre && b == last_b) {
            // partner's part already in registers: own part first, then the
            // partner's, the same order the general path uses
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e) sum[mt][e] += pre[mt][e];
            store_y<MT>(p, b, warp, lane, sum);
            if (threadIdx.x == 0) p.counters[b] = 0;
        } else if (start_pub && b == first_b) {
            // publish the first part and stream on: the helper counts it,
            // and says after the stream whether this CTA completed the count
            float *mine = p.partials + (int64_t)(2 * cta) * C::kPartialFloats;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    __stcg(&mine[(warp * 4 * MT + 4 * mt + e) * 32 + lane], sum[mt][e]);
            mbar_arrive(&pub_bar);
        } else {
            // publish this part; the last contributor to arrive adds all
            // parts in CTA order (independent of arrival order), scales and
            // stores, then resets the block's counter
            const int slot = (b == first_b) ? 2 * cta : 2 * cta + 1;
            float *mine = p.partials + (int64_t)slot * C::kPartialFloats;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    __stcg(&mine[(warp * 4 * MT + 4 * mt + e) * 32 + lane], sum[mt][e]);
            if (!consumers_sync()) return;
            const uint32_t j_first = owner_of(b * KB, p.T, p.G);
            const uint32_t j_last = owner_of((b + 1) * KB - 1, p.T, p.G);
            if (threadIdx.x == 0) {
                // release (with the barrier above: every thread's part) and
                // acquire (the parts are read after the count) in one atomic
                const int old = atomic_add_acq_rel_gpu(&p.counters[b], 1);
                last_flag[1] = ((uint32_t)old == j_last - j_first);
            }
            if (!consumers_sync()) return;
            if (last_flag[1]) {
                // this CTA's own part is still in registers
                float own[MT][4];
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) own[mt][e] = sum[mt][e];
                gather_parts<MT>(p, b, j_first, j_last, cta, true, own, warp, lane, sum);
                store_y<MT>(p, b, warp, lane, sum);
                if (threadIdx.x == 0) p.counters[b] = 0;
            }
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int jj = 0; jj < NS; ++jj)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[mt][jj][e] = 0.0f;
        if (kb == KB) { kb = 0; ++b; }
        seg_whole = true;
        seg_new = true;
    }

    if (start_pub) {
        // The helper's count of the first part (normally long done).  If it
        // completed the count, every other part was already published and
        // this CTA finishes the block.
        if (!warp_all(mbar_wait(&start_bar, 0, SITE_DEC_START))) return;
        if (helper_flag[1]) {
            const uint32_t jf = owner_of(first_b * KB, p.T, p.G);
            const uint32_t jl = owner_of((first_b + 1) * KB - 1, p.T, p.G);
            float none[MT][4] = {};
            float sum[MT][4];
            gather_parts<MT>(p, first_b, jf, jl, cta, false, none, warp, lane, sum);
            store_y<MT>(p, first_b, warp, lane, sum);
            if (threadIdx.x == 0) p.counters[first_b] = 0;
        }
    }
}

}  // namespace decode
}  // namespace w8
