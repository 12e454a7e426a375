// Prefill-regime W8A16 linear on CTA pairs (tcgen05 cta_group::2):
// Y = X . dequant(q) (+ bias).  The TPU-MLIR article (section 4) gives the
// W8A16 MatMul as load -> cast int8 to F16 -> scale -> matmul -> store,
// with the load overlapped with compute through ping-pong local memory; on
// sm_100a the same five steps become a warp-specialised, persistent
// pipeline in which each MMA spans the two SMs of a cluster of two CTAs.
//
// One thread issues a tcgen05.mma only about every 100 cycles, so the MMA
// shape must carry enough work: 128 x 256 x 16 per SM (136 cycles) keeps
// the tensor pipe busy where 128 x 128 x 16 (64 cycles) cannot.  A pair
// tile is 256 channels x 256 tokens: each CTA holds its
// own 128 channels (widened weights in its tensor memory, accumulator rows
// in its tensor memory) and HALF of the tokens' X tile (128 x 64, 16 KB) in
// its shared memory; one 256 x 256 x 16 MMA issued by the pair's first CTA
// reads the A halves from both tensor memories and the B halves from both
// shared memories.  Compared with one SM per 128 x 256 tile this halves the
// X tile each SM pulls from L2 per K step; no TMA multicast is used.
//
// Roles in each CTA (16 warps):
//   warp 0      weight producer: bulk copy of this CTA's four 8 KB packed
//               tiles per 256-wide K step into a local 2-stage ring.
//   warp 3      activation producer: four 2-D TMA loads of this CTA's 128
//               tokens x 64 X halves per K step into a local 2-stage ring of
//               64 KB slots; the completion is counted on the FIRST CTA's
//               barrier (both CTAs' halves must land before the pair MMAs).
//   warps 4-7   converters: widen the int8 codes into this CTA's tensor
//               memory A buffer, then arrive on the first CTA's barrier.
//   warp 1      (first CTA only) MMA issuer; its commits arrive on the
//               barriers of both CTAs.
//   warps 8-15  epilogue: drain this CTA's 128 accumulator lanes, release
//               the accumulator on the first CTA's barrier, scale, and store
//               Y through a shared-memory stage as whole 256-byte rows.
//   warp 2      tensor-memory allocation for the pair.
//
// Schedule.  The pairs are persistent.  Whole tiles go round robin over the
// pairs for all but the last wave ("data-parallel" part); the 256-wide K
// steps of the tiles that remain are then split evenly over all pairs
// (a stream-K split), so that the work per pair differs by at most one K
// step whatever the tile count.  A pair's share of a tile ends in one of
// two fp32 partial-sum slots of the workspace; the pair that brings a
// tile's arrival count to its number of contributors adds the partial sums
// in K order (a fixed order: results do not depend on timing), scales and
// stores the tile.  No pair ever waits for another.
#pragma once

#include "common.cuh"

namespace w8 {
namespace prefill2 {

constexpr int kBNc = 128;                // channels per CTA
constexpr int kBNp = 2 * kBNc;           // channels per pair tile (MMA M)
constexpr int kBT = 256;                 // tokens per pair tile (MMA N)
constexpr int kBTc = kBT / 2;            // tokens held by each CTA
// One pipeline stage covers a 256-wide K step: four packed tiles, four
// 64-wide X boxes and sixteen MMAs.  Every stage costs a handful of barrier
// handoffs (a few hundred cycles each, measured: arrive, wake-up, commit),
// so the step is made long enough (about 2200 cycles of tensor work) to
// hide them; 64- and 128-wide steps left the tensor pipe half and a fifth
// idle.
constexpr int kKStep = 4;                // 64-wide K blocks per stage
// Two weight stages measured as fast as three (and faster on short-K
// shapes); the 32 KB this frees holds the epilogue's Y stage.
constexpr int kWStages = 2;
constexpr int kXStages = 2;
constexpr int kWTile = 8192;             // packed int8 tile, 128 x 64
constexpr int kWBytes = kKStep * kWTile;
constexpr int kXBox = kBTc * 128;        // 128 tokens x 64 fp16
constexpr int kXBytes = kKStep * kXBox;
// Epilogue stage: per half of the tile's tokens, two buffers of 32 tokens x
// 128 channels fp16 (8 KB), double-buffered.
constexpr int kYChunk = 32;
constexpr int kYStageBytes = kYChunk * kBNc * 2;
constexpr int kYBytes = 2 * 2 * kYStageBytes;
constexpr int kSmemBytes = kXStages * kXBytes + kWStages * kWBytes + kYBytes + 1024;
constexpr int kABuf = 2;                 // A buffers of 32 kKStep columns
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAcol0 = kBT;         // first A buffer column
constexpr int kThreads = 512;
constexpr int kEpiWarps = 8;
constexpr uint32_t kIdesc = idesc_f16_f32(kBNp, kBT);
constexpr uint16_t kBoth = 0x3;          // CTA mask of the pair

static_assert(kXBox % 1024 == 0 && kWBytes % 1024 == 0, "stage alignment");
static_assert(kAcol0 + 32 * kKStep * kABuf <= kTmemCols, "tensor memory budget");
static_assert(kSmemBytes <= 227 * 1024 - 512, "shared memory budget");

// fp32 partial sums of one CTA's share of a pair tile: [256 tokens][128 channels]
constexpr int kPartFloats = kBT * kBNc;


struct Params {
    const uint8_t *packed;
    const uint16_t *scales;
    const int8_t *zeros;    // zero points (asymmetric codes), else unused
    const uint16_t *bias;   // may be null
    uint16_t *Y;
    float *partials;        // [pairs][2 slots][2 CTAs][kPartFloats]
    int *counters;          // [stream-K tiles][2 CTAs], zero between calls
    int M;
    int64_t N;
    int NB;        // ceil(N/128): packed channel blocks
    int KB;        // ceil(K/64)
    int KS;        // ceil(KB/4): 256-wide K steps
    int TT;        // token tiles = ceil(M/256)
    int tiles;     // ceil(NB/2) * TT pair tiles
    int dp_tiles;  // tiles [0, dp_tiles) run whole, round robin
    int sk_iters;  // K steps of tiles [dp_tiles, tiles), split evenly
    // outlier split (kMode == kOutliers): Y += X[:, rows] . vals per channel
    const uint16_t *XT;          // [K][Mp] fp16: X transposed, zero for m >= M
    int64_t Mp;                  // multiple of kBT
    const int32_t *o_count;      // [N]
    const int32_t *o_rows;       // [N][o_cap]
    const uint16_t *o_vals;      // [N][o_cap] fp16
    int o_cap;
    float *o_extra;              // per CTA kExtraFloats: the current tile's bias + outlier terms
};

// Outlier term of one CTA's share of a tile, written while its MMAs run and
// read back in the drain: [128 tokens][256 epilogue threads] fp32.
constexpr int kExtraFloats = 32 * kEpiWarps * 128;

// Code forms the converters and the epilogue handle.
constexpr int kSym = 0;        // symmetric codes
constexpr int kZeroPoint = 1;  // asymmetric codes: the converters widen to q - z
constexpr int kOutliers = 2;   // symmetric codes plus a sparse fp16 side list

// X^T for the outlier term: XT[k][m] = X[m][k] for m < M, 0 up to Mp.
// grid (ceil(K/32), Mp/32), 32 x 8 threads.
__global__ void transpose_x_kernel(const uint16_t *__restrict__ X, uint16_t *__restrict__ XT, int M, int64_t K,
                                   int64_t Mp) {
    __shared__ uint16_t tile[32][33];
    const int64_t k0 = (int64_t)blockIdx.x * 32, m0 = (int64_t)blockIdx.y * 32;
    for (int i = threadIdx.y; i < 32; i += 8) {
        const int64_t m = m0 + i, k = k0 + threadIdx.x;
        tile[i][threadIdx.x] = (m < M && k < K) ? X[m * K + k] : (uint16_t)0;
    }
    __syncthreads();
    for (int i = threadIdx.y; i < 32; i += 8) {
        const int64_t k = k0 + i, m = m0 + threadIdx.x;
        if (k < K) XT[k * Mp + m] = tile[threadIdx.x][i];
    }
}

// First stream-K step of pair q (steps numbered from tile dp_tiles' first).
// The host keeps tiles, sk_iters and sk_iters x pairs below 2^31.
__device__ __forceinline__ int sk_begin(int q, int pairs, int iters) {
    return (int)((int64_t)q * iters / pairs);
}
// The pair whose share holds stream-K step it: the largest q with
// sk_begin(q) <= it.  Every pair has at least one step (iters >= pairs).
__device__ __forceinline__ int sk_owner(int it, int pairs, int iters) {
    return (int)(((int64_t)(it + 1) * pairs - 1) / iters);
}
// Partial-sum slot that pair q uses for stream-K tile t: 0 for the tile its
// share starts in, 1 for the tile it ends in (every tile between is whole).
__device__ __forceinline__ int sk_slot(int q, int t, int pairs, int iters, int KS) {
    return sk_begin(q, pairs, iters) / KS == t ? 0 : 1;
}

// One segment of a pair's work: K steps [ks0, ks1) of one pair tile.
struct Seg {
    int tile;
    int ks0, ks1;
    int slot;     // -1: the whole tile; else the partial-sum slot
    bool final;   // the pair's last segment
};

struct Sched {
    int tile, pairs, dp_tiles, it, it_end, it_first, KS;
    __device__ Sched(int q, int npairs, int dp, int sk_iters, int ks)
        : tile(q), pairs(npairs), dp_tiles(dp), KS(ks) {
        it_first = it = sk_iters > 0 ? sk_begin(q, npairs, sk_iters) : 0;
        it_end = sk_iters > 0 ? sk_begin(q + 1, npairs, sk_iters) : 0;
    }
    __device__ bool more() const { return tile < dp_tiles || it < it_end; }
    __device__ bool next(Seg &s) {
        if (tile < dp_tiles) {
            s.tile = tile;
            s.ks0 = 0;
            s.ks1 = KS;
            s.slot = -1;
            tile += pairs;
        } else if (it < it_end) {
            const int t = it / KS;
            s.tile = dp_tiles + t;
            s.ks0 = it - t * KS;
            s.ks1 = min(KS, s.ks0 + (it_end - it));
            s.slot = (s.ks0 == 0 && s.ks1 == KS) ? -1 : (t == it_first / KS ? 0 : 1);
            it += s.ks1 - s.ks0;
        } else {
            return false;
        }
        s.final = !more();
        return true;
    }
};

struct Ring {
    int s = 0;
    uint32_t ph = 0;
    __device__ __forceinline__ void next(int n) {
        if (++s == n) { s = 0; ph ^= 1u; }
    }
    __device__ __forceinline__ void prev(int n) {
        if (--s < 0) { s = n - 1; ph ^= 1u; }
    }
};

// The epilogue's part in one share of a stream-K tile (all kEpiWarps
// warps call it together, once the share's accumulator is complete):
// publish the share's fp32 partial sums, count it, and when it is the
// tile's last share to be counted add all shares in K order, scale and
// store Y.  A pair on its last segment keeps its accumulator (nothing
// waits for it) and, if every other share is already counted, completes
// the tile from tensor memory without publishing its own.
__device__ __forceinline__ void stream_k_share(float *partials, int *counters, uint16_t *Y, const int M,
                                               const int64_t N, const int dp_tiles, const int sk_iters,
                                               const int KS, const Seg &sg, const int pair0, const int pstep,
                                               const uint32_t tmem, const uint32_t rank, const int warp,
                                               const int lane, int *fix_last, const uint32_t d_empty_leader,
                                               const float sc, const float bi, const bool n_ok, const int64_t n,
                                               const int tb) {
    const int q4 = warp & 3;
    const int half = (warp - 8) >> 2;
    const int r = 32 * q4 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * q4) << 16) + 128 * half;
    const int m0 = tb * kBT + 128 * half;
    const int t = sg.tile - dp_tiles;
    const int j_first = sk_owner(t * KS, pstep, sk_iters);
    const int j_last = sk_owner(t * KS + KS - 1, pstep, sk_iters);
    const int others = j_last - j_first;
    int *cnt = counters + t * 2 + rank;
    const int64_t elem = 128 * half * kBNc + r;   // this thread's first element of a share
    auto part_of = [&](int j) -> float * {
        const int slot = sk_slot(j, t, pstep, sk_iters, KS);
        return partials + (int64_t)((j * 2 + slot) * 2 + (int)rank) * kPartFloats + elem;
    };
    if (sg.final) {
        if (warp == 8 && lane == 0) *fix_last = ld_acquire_gpu(cnt) == others;
        named_bar_sync(1, 32 * kEpiWarps);
    }
    const bool publish = !(sg.final && *fix_last);
    if (publish) {
        float *mine = part_of(pair0);
#pragma unroll
        for (int cchunk = 0; cchunk < 4; ++cchunk) {
            uint32_t v[32];
            tmem_load_32(lane_addr + 32 * cchunk, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) __stcg(mine + (32 * cchunk + i) * kBNc, __uint_as_float(v[i]));
        }
    }
    if (!sg.final) {   // more work follows: free the accumulator now
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(d_empty_leader);
    }
    if (publish) {
        named_bar_sync(1, 32 * kEpiWarps);   // every part of this CTA is written
        if (warp == 8 && lane == 0) {
            // release (with the barrier above) and acquire in one atomic
            const int last = atomic_add_acq_rel_gpu(cnt, 1) == others;
            if (last) *cnt = 0;   // every share is counted: ready for the next call
            *fix_last = last;
        }
        named_bar_sync(1, 32 * kEpiWarps);
    } else if (warp == 8 && lane == 0) {
        *cnt = 0;
    }
    if (*fix_last) {
#pragma unroll 1
        for (int cchunk = 0; cchunk < 4; ++cchunk) {
            float acc[32];
#pragma unroll 1
            for (int j = j_first; j <= j_last; ++j) {
                uint32_t v[32];
                if (j == pair0 && sg.final) {
                    tmem_load_32(lane_addr + 32 * cchunk, v);
                } else {
                    const float *src = part_of(j) + 32 * cchunk * kBNc;
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__ldcg(src + i * kBNc));
                }
                if (j == j_first) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) acc[i] = __uint_as_float(v[i]);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) acc[i] += __uint_as_float(v[i]);
                }
            }
            if (n_ok) {
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int m = m0 + 32 * cchunk + i;
                    if (m < M) Y[(int64_t)m * N + n] = __half_as_ushort(__float2half_rn(fmaf(acc[i], sc, bi)));
                }
            }
        }
    }
    if (sg.final) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(d_empty_leader);
    }
}

// grid = 2 x pairs CTAs, cluster dims (2, 1, 1), kThreads threads,
// kSmemBytes dynamic shared memory.  tmap_x: X [M, K] fp16, box {64, 128},
// 128-byte swizzle.
// kMode == kZeroPoint: the converters widen every weight to q - z_n (exact
// in fp16) instead of q.  kMode == kOutliers: the epilogue adds each
// channel's kept weights times the matching X columns before rounding (no
// K split with it).
template <bool kSplit, int kMode>
__global__ void __launch_bounds__(kThreads, 1)
prefill2_kernel(const __grid_constant__ CUtensorMap tmap_x, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *x_ring = base;                                  // kXStages x 16 KB
    uint8_t *w_ring = base + kXStages * kXBytes;             // kWStages x 32 KB
    uint8_t *y_stage = w_ring + kWStages * kWBytes;          // epilogue: 2 halves x 2 x 8 KB
    __shared__ uint64_t w_full[kWStages], w_empty[kWStages];
    __shared__ uint64_t x_full[kXStages], x_empty[kXStages];
    __shared__ uint64_t a_full[kABuf], a_empty[kABuf];
    __shared__ uint64_t d_full, d_empty, drain;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int fix_last;       // this CTA completes the current tile

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();     // 0: issues the pair MMAs
    const int pair0 = blockIdx.x >> 1;
    const int pstep = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kWStages; ++i) {
            mbar_init(&w_full[i], 1);
            mbar_init(&w_empty[i], 4);         // this CTA's converter warps
        }
        for (int i = 0; i < kXStages; ++i) {
            mbar_init(&x_full[i], 1);          // first CTA: expect both halves
            mbar_init(&x_empty[i], 1);         // pair MMA commit
        }
        for (int i = 0; i < kABuf; ++i) {
            mbar_init(&a_full[i], 8);          // converter warps of both CTAs
            mbar_init(&a_empty[i], 1);
        }
        mbar_init(&d_full, 1);
        mbar_init(&d_empty, 2 * kEpiWarps);    // epilogue warps of both CTAs
        mbar_init(&drain, 1);
        fence_barrier_init();
        prefetch_tensormap(&tmap_x);
    }
    if (warp == 2) {
        tmem_alloc_pair(&tmem_base_sh, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();   // barriers initialised in both CTAs, TMEM allocated
    // The next call may start its prologue as SMs free up.  Every global
    // access of this call waits for the previous kernel in the stream to
    // complete: the producers, the epilogue and (for the zero points) the
    // converters call pdl_wait first (otherwise the converters and the MMA
    // issuer touch only shared and tensor memory).
    pdl_launch_dependents();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    // the first CTA's copy of a barrier, as a shared::cluster address
    auto leader = [](uint64_t *bar) -> uint32_t { return mapa_shared(smem_u32(bar), 0); };

    if (warp == 0) {
        // ---------------------------------------------------- weight producer
        if (lane == 0) {
            pdl_wait();
            Ring r;
            int issued = 0;
            bool ok = true;
            Sched sched(pair0, pstep, p.dp_tiles, p.sk_iters, p.KS);
            Seg sg;
            while (ok && sched.next(sg)) {
                const int64_t blk = (sg.tile / p.TT) * 2 + rank;
                const bool valid = blk < p.NB;
                const uint8_t *wsrc = p.packed + blk * p.KB * (int64_t)kWTile;
                for (int ks = sg.ks0; ks < sg.ks1; ++ks) {
                    const int cnt = min(kKStep, p.KB - kKStep * ks);   // tiles in this step
                    if (!mbar_wait(&w_empty[r.s], r.ph ^ 1u, SITE_P2_WEMPTY)) { ok = false; break; }
                    if (valid) {
                        mbar_arrive_expect_tx(&w_full[r.s], cnt * kWTile);
                        bulk_g2s(w_ring + r.s * kWBytes, wsrc + (int64_t)kKStep * ks * kWTile, cnt * kWTile,
                                 &w_full[r.s]);
                        ++issued;
                    } else {
                        mbar_arrive(&w_full[r.s]);   // no block: converters write zeros
                    }
                    r.next(kWStages);
                }
            }
            for (int i = 0; i < kWStages && i < issued; ++i) {
                r.prev(kWStages);
                mbar_wait(&w_full[r.s], r.ph, SITE_P2_DRAIN, 10000000ull);
            }
        }
    } else if (warp == 3) {
        // ---------------------------------------------------- activation producer
        if (lane == 0) {
            pdl_wait();
            Ring r;
            int issued = 0;
            bool ok = true;
            Sched sched(pair0, pstep, p.dp_tiles, p.sk_iters, p.KS);
            Seg sg;
            while (ok && sched.next(sg)) {
                const int tb = (int)(sg.tile % p.TT);
                for (int ks = sg.ks0; ks < sg.ks1; ++ks) {
                    const int cnt = min(kKStep, p.KB - kKStep * ks);
                    if (!mbar_wait(&x_empty[r.s], r.ph ^ 1u, SITE_P2_XEMPTY)) { ok = false; break; }
                    if (rank == 0) mbar_arrive_expect_tx(&x_full[r.s], 2 * cnt * kXBox);
                    for (int t = 0; t < cnt; ++t)
                        tma_load_2d_pair(x_ring + r.s * kXBytes + t * kXBox, &tmap_x, (kKStep * ks + t) * 64,
                                         tb * kBT + (int)rank * kBTc, leader(&x_full[r.s]));
                    ++issued;
                    r.next(kXStages);
                }
            }
            // every X half has landed before the pair can leave: the first
            // CTA sees both halves complete on its barrier; the MMA issuer
            // consumed them, or after a timeout the final cluster barrier
            // below orders the exit after this wait in the first CTA
            if (rank == 0) {
                for (int i = 0; i < kXStages && i < issued; ++i) {
                    r.prev(kXStages);
                    mbar_wait(&x_full[r.s], r.ph, SITE_P2_DRAIN, 10000000ull);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------- MMA issuer (first CTA)
        if (lane == 0 && rank == 0) {
            Ring xr, ar;
            int it = 0;
            bool ok = true;
            Sched sched(pair0, pstep, p.dp_tiles, p.sk_iters, p.KS);
            Seg sg;
            for (; ok && sched.next(sg); ++it) {
                if (!mbar_wait(&d_empty, (it & 1) ^ 1u, SITE_P2_DEMPTY)) { ok = false; break; }
                tc_fence_after();
                for (int ks = sg.ks0; ks < sg.ks1; ++ks) {
                    const int cnt = min(kKStep, p.KB - kKStep * ks);
                    if (!mbar_wait(&x_full[xr.s], xr.ph, SITE_P2_XFULL)) { ok = false; break; }
                    if (!mbar_wait(&a_full[ar.s], ar.ph, SITE_P2_AFULL)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_tmem = tmem + kAcol0 + 32 * kKStep * ar.s;
                    const uint32_t x_addr = smem_u32(x_ring + xr.s * kXBytes);
                    for (int t = 0; t < cnt; ++t) {
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            tc_mma_ts_f16_pair(tmem, a_tmem + 32 * t + 8 * j,
                                               smem_desc_kmajor_sw128(x_addr + t * kXBox + 32 * j), kIdesc,
                                               ((ks - sg.ks0) | t | j) != 0);
                    }
                    tc_commit_pair_mc(&x_empty[xr.s], kBoth);
                    tc_commit_pair_mc(&a_empty[ar.s], kBoth);
                    xr.next(kXStages);
                    ar.next(kABuf);
                }
                if (!ok) break;
                tc_commit_pair_mc(&d_full, kBoth);
            }
            // every pair MMA is complete before either CTA frees its TMEM
            tc_commit_pair(&drain);
            mbar_wait(&drain, 0, SITE_P2_DRAIN);
        }
    } else if (warp >= 4 && warp < 8) {
        // ---------------------------------------------------- converters
        const int q4 = warp & 3;
        const int r = 32 * q4 + lane;         // channel within this CTA's block
        const int h = (r >> 1) & 3;
        const uint32_t lane_addr = tmem + ((uint32_t)(32 * q4) << 16);
        Ring wr, ar;
        bool ok = true;
        // the zero points may have been written by the previous kernel
        if constexpr (kMode == kZeroPoint) pdl_wait();
        Sched sched(pair0, pstep, p.dp_tiles, p.sk_iters, p.KS);
        Seg sg;
        while (ok && sched.next(sg)) {
            const bool valid = (sg.tile / p.TT) * 2 + rank < p.NB;
            uint32_t zc = 0x64806480u;   // 1152 + z of this thread's channel
            if constexpr (kMode == kZeroPoint) {
                const int64_t n = ((int64_t)(sg.tile / p.TT) * 2 + rank) * kBNc + r;
                if (valid && n < p.N) zc = zp_bias2(p.zeros[n]);
            }
            for (int ks = sg.ks0; ks < sg.ks1; ++ks) {
                const int cnt = min(kKStep, p.KB - kKStep * ks);
                if (!warp_all(mbar_wait(&w_full[wr.s], wr.ph, SITE_P2_WFULL))) { ok = false; break; }
                uint4 c[kKStep][4];
#pragma unroll
                for (int t = 0; t < kKStep; ++t) {
                    if (valid && t < cnt) {
                        const uint8_t *row = w_ring + wr.s * kWBytes + t * kWTile + r * 64;
#pragma unroll
                        for (int i = 0; i < 4; ++i) c[t][i] = *reinterpret_cast<const uint4 *>(row + ((i ^ h) << 4));
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            c[t][i] = make_uint4(0x80808080u, 0x80808080u, 0x80808080u, 0x80808080u);
                    }
                }
                if (!warp_all(mbar_wait(&a_empty[ar.s], ar.ph ^ 1u, SITE_P2_AEMPTY))) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int t = 0; t < kKStep; ++t) {
                    uint32_t v[32];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint32_t w[4] = {c[t][i].x, c[t][i].y, c[t][i].z, c[t][i].w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            if constexpr (kMode == kZeroPoint) {
                                v[8 * i + 2 * j] = unbias2_by(widen_lo2(w[j]), zc);
                                v[8 * i + 2 * j + 1] = unbias2_by(widen_hi2(w[j]), zc);
                            } else {
                                v[8 * i + 2 * j] = unbias2(widen_lo2(w[j]));
                                v[8 * i + 2 * j + 1] = unbias2(widen_hi2(w[j]));
                            }
                        }
                    }
                    tmem_store_32(lane_addr + kAcol0 + 32 * kKStep * ar.s + 32 * t, v);
                }
                tc_fence_before();
                __syncwarp();
                // the slot is released only now that every lane's codes are
                // used: released right after the shared loads were issued, a
                // load still in flight could see the next bulk copy's bytes
                if (lane == 0) mbar_arrive(&w_empty[wr.s]);
                if (lane == 0) mbar_arrive_remote(leader(&a_full[ar.s]));
                wr.next(kWStages);
                ar.next(kABuf);
            }
        }
    } else if (warp >= 8) {
        // ---------------------------------------------------- epilogue
        pdl_wait();
        const int q4 = warp & 3;
        const int half = (warp - 8) >> 2;     // token columns [128 half, 128 half + 128)
        const int r = 32 * q4 + lane;
        const uint32_t lane_addr = tmem + ((uint32_t)(32 * q4) << 16) + 128 * half;
        int it = 0;
        Sched sched(pair0, pstep, p.dp_tiles, p.sk_iters, p.KS);
        Seg sg;
        for (; sched.next(sg); ++it) {
            if constexpr (kMode == kOutliers) {
                // this tile's bias + outlier terms, formed while its MMAs run
                // (the gathers from X^T are off the accumulator's path)
                const int64_t nb = ((int64_t)(sg.tile / p.TT) * 2 + rank) * kBNc + r;
                const int mb = (int)(sg.tile % p.TT) * kBT + 128 * half;
                const bool nb_ok = nb < p.N;
                const float bb = (nb_ok && p.bias) ? __half2float(__ushort_as_half(p.bias[nb])) : 0.0f;
                const int cnt = nb_ok ? p.o_count[nb] : 0;
                // the parked terms are token-major, [token][epilogue thread],
                // so a warp's access at one token is one 128-byte line
                float *park = p.o_extra + (int64_t)blockIdx.x * kExtraFloats + (threadIdx.x - 256);
                // up to four outliers (the common case): their rows and
                // values are read once for the whole tile
                int64_t krow[4];
                float kval[4];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int j = jj < cnt ? jj : 0;
                    krow[jj] = (cnt > 0 && cnt <= 4) ? p.o_rows[nb * p.o_cap + j] : 0;
                    kval[jj] = (jj < cnt && cnt <= 4) ? __half2float(__ushort_as_half(p.o_vals[nb * p.o_cap + j])) : 0.0f;
                }
                for (int cchunk = 0; cchunk < 4; ++cchunk) {
                    float ex[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) ex[i] = bb;
                    // four outliers per round: their X^T rows are loaded
                    // together (a padding slot reuses a listed row, weight 0)
                    for (int j0 = 0; j0 < cnt; j0 += 4) {
                        uint4 xv[4][4];
                        float ov[4];
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj) {
                            const int j = j0 + jj < cnt ? j0 + jj : j0;
                            const int64_t k = cnt <= 4 ? krow[jj] : p.o_rows[nb * p.o_cap + j];
                            ov[jj] = cnt <= 4 ? kval[jj]
                                              : (j0 + jj < cnt ? __half2float(__ushort_as_half(p.o_vals[nb * p.o_cap + j]))
                                                               : 0.0f);
                            const uint4 *src = reinterpret_cast<const uint4 *>(p.XT + k * p.Mp + mb + 32 * cchunk);
#pragma unroll
                            for (int u = 0; u < 4; ++u) xv[jj][u] = src[u];
                        }
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj)
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const uint32_t xw[4] = {xv[jj][u].x, xv[jj][u].y, xv[jj][u].z, xv[jj][u].w};
#pragma unroll
                                for (int h = 0; h < 4; ++h) {
                                    const __half2 x2 = *reinterpret_cast<const __half2 *>(&xw[h]);
                                    ex[8 * u + 2 * h] = fmaf(__low2float(x2), ov[jj], ex[8 * u + 2 * h]);
                                    ex[8 * u + 2 * h + 1] = fmaf(__high2float(x2), ov[jj], ex[8 * u + 2 * h + 1]);
                                }
                            }
                    }
#pragma unroll
                    for (int i = 0; i < 32; ++i) park[(32 * cchunk + i) * (32 * kEpiWarps)] = ex[i];
                }
            }
            const bool got = warp_all(mbar_wait(&d_full, it & 1, SITE_P2_DFULL));
            if constexpr (kSplit) {
                // all epilogue warps give up together: the stream-K share
                // below has barriers over all of them
                if (!named_bar_all(1, 32 * kEpiWarps, got)) break;
            } else {
                if (!got) break;
            }
            tc_fence_after();
            const int64_t blk = (sg.tile / p.TT) * 2 + rank;
            const int tb = (int)(sg.tile % p.TT);
            const int64_t n = blk * kBNc + r;
            const bool n_ok = n < p.N;
            const float sc = n_ok ? __half2float(__ushort_as_half(p.scales[n])) : 0.0f;
            const float bi = (n_ok && p.bias) ? __half2float(__ushort_as_half(p.bias[n])) : 0.0f;
            const int m0 = tb * kBT + 128 * half;
            if (kMode == kOutliers && sg.slot < 0) {
                // the parked terms of chunk c + 1 load while chunk c converts;
                // each chunk is stored right away (no results held)
                const float *park = p.o_extra + (int64_t)blockIdx.x * kExtraFloats + (threadIdx.x - 256);
                float exn[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) exn[i] = park[i * (32 * kEpiWarps)];
                // Y through the shared-memory stage, as in the plain path
                const int64_t nb0 = blk * kBNc;
                const int cl = 8 * (lane & 15);
#pragma unroll
                for (int cchunk = 0; cchunk < 4; ++cchunk) {
                    float ex[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) ex[i] = exn[i];
                    if (cchunk < 3) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) exn[i] = park[(32 * (cchunk + 1) + i) * (32 * kEpiWarps)];
                    }
                    uint32_t v[32];
                    tmem_load_32(lane_addr + 32 * cchunk, v);
                    if (cchunk == 3) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_remote(leader(&d_empty));
                    }
                    uint16_t *stg = reinterpret_cast<uint16_t *>(y_stage + (2 * half + (cchunk & 1)) * kYStageBytes);
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        stg[i * kBNc + r] = __half_as_ushort(__float2half_rn(fmaf(__uint_as_float(v[i]), sc, ex[i])));
                    named_bar_sync(2 + half, 128);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int row = 8 * q4 + 2 * j + (lane >> 4);
                        const int m = m0 + kYChunk * cchunk + row;
                        const uint4 val = *reinterpret_cast<const uint4 *>(stg + row * kBNc + cl);
                        if (m < p.M && nb0 + cl < p.N)
                            *reinterpret_cast<uint4 *>(p.Y + (int64_t)m * p.N + nb0 + cl) = val;
                    }
                }
            } else if (sg.slot < 0) {
                uint32_t y2[64];
#pragma unroll
                for (int cchunk = 0; cchunk < 4; ++cchunk) {
                    uint32_t v[32];
                    tmem_load_32(lane_addr + 32 * cchunk, v);
                    {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const __half2 hv = __floats2half2_rn(fmaf(__uint_as_float(v[2 * i]), sc, bi),
                                                                 fmaf(__uint_as_float(v[2 * i + 1]), sc, bi));
                            y2[16 * cchunk + i] = *reinterpret_cast<const uint32_t *>(&hv);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(leader(&d_empty));
                // Y through shared memory: each thread holds one channel of
                // 128 tokens, so direct stores would be 64 bytes per warp
                // store, one row apart.  The four warps of a half write a
                // 32-token chunk as [token][channel] into a stage buffer;
                // then each warp stores 8 whole token rows (128 channels,
                // 256 bytes) with 16-byte stores.  Two buffers per half: a
                // warp refills one only after the barrier of the next
                // chunk, which every warp passes after its stores from it.
                const int64_t nb0 = blk * kBNc;               // first channel of the block
                const int cl = 8 * (lane & 15);               // this lane's 8 channels in a row
#pragma unroll
                for (int cchunk = 0; cchunk < 4; ++cchunk) {
                    uint16_t *stg = reinterpret_cast<uint16_t *>(y_stage + (2 * half + (cchunk & 1)) * kYStageBytes);
#pragma unroll
                    for (int i = 0; i < kYChunk / 2; ++i) {
                        const uint32_t w2 = y2[16 * cchunk + i];
                        stg[(2 * i) * kBNc + r] = (uint16_t)(w2 & 0xFFFFu);
                        stg[(2 * i + 1) * kBNc + r] = (uint16_t)(w2 >> 16);
                    }
                    named_bar_sync(2 + half, 128);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int row = 8 * q4 + 2 * j + (lane >> 4);
                        const int m = m0 + kYChunk * cchunk + row;
                        const uint4 val = *reinterpret_cast<const uint4 *>(stg + row * kBNc + cl);
                        if (m < p.M && nb0 + cl < p.N)
                            *reinterpret_cast<uint4 *>(p.Y + (int64_t)m * p.N + nb0 + cl) = val;
                    }
                }
            } else if constexpr (kSplit && kMode != kOutliers) {
                stream_k_share(p.partials, p.counters, p.Y, p.M, p.N, p.dp_tiles, p.sk_iters, p.KS, sg, pair0,
                               pstep, tmem, rank, warp, lane, &fix_last, leader(&d_empty), sc, bi, n_ok, n, tb);
            }
        }
    }

    // neither CTA frees the pair's tensor memory, nor leaves while the
    // other may still signal its barriers, before both are done
    tc_fence_before();
    cluster_sync_all();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

}  // namespace prefill2
}  // namespace w8
