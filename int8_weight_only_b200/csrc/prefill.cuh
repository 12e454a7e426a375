// Prefill-regime W8A16 linear (M > 16 tokens) on the 5th-generation tensor
// cores: Y = X . dequant(q) (+ bias).
//
// The TPU-MLIR article (section 4) gives the W8A16 MatMul as load -> cast
// int8 to F16 -> scale -> matmul -> store, with the load overlapped with
// compute through ping-pong local memory.  On sm_100a the same five steps
// become a warp-specialised pipeline per CTA (one CTA per SM, persistent):
//
//   warp 0      weight producer: one 1-D bulk copy per 64-wide K block of
//               the 8 KB packed int8 tile (128 channels x 64) into an
//               8-stage ring.
//   warp 3      activation producer: one 2-D TMA load per K block of the X
//               tile (256 tokens x 64, 128-byte swizzle) into a 5-stage
//               ring of 32 KB slots.
//   warps 4-7   converters ("cast"): thread r owns channel r of the tile,
//               reads its 64 int8 codes, widens them to fp16 in registers
//               and writes them with tcgen05.st into tensor memory, where
//               they are the A operand of the MMA.  The widened weights
//               never pass through shared memory.
//   warp 1      MMA issuer ("matmul"): tcgen05.mma kind::f16 with A (128
//               channels x 16) in tensor memory and B (256 tokens x 16) the
//               swizzled X tile, fp32 accumulator D (128 x 256) in tensor
//               memory; four MMAs per K block.  N = 256 matters: one thread
//               issues an MMA only about every 100 cycles, so a 128 x 128
//               MMA (64 cycles of tensor work) would leave the tensor pipe
//               a third idle, while a 128 x 256 MMA keeps it busy.
//   warps 8-15  epilogue ("scale" + "store"): warp w drains TMEM lanes
//               32 (w % 4) .. +31 and half of the 256 columns into
//               registers, releases the accumulator to the next tile, then
//               writes y = acc * s_n + bias_n (fp32, one rounding to fp16).
//
// Tensor memory (512 columns): the accumulator at [0, 256) and eight A
// buffers of 32 columns (64 fp16 per channel) at [256, 512), so the
// converters run up to eight K blocks ahead of the MMAs.
// Tiles: 128 channels x 256 tokens; tile id = channel block * token tiles +
// token tile, so CTAs running together share a channel block (its weight
// tiles are read from HBM once and then hit in L2; X stays in L2).
#pragma once

#include "common.cuh"

namespace w8 {
namespace prefill {

constexpr int kBN = 128;                 // channels per tile (MMA M)
constexpr int kBT = 256;                 // tokens per tile (MMA N)
constexpr int kWStages = 8;
constexpr int kXStages = 5;
constexpr int kWBytes = 8192;            // packed int8 tile, 128 x 64
constexpr int kXBytes = kBT * 128;       // 256 tokens x 64 fp16
constexpr int kSmemBytes = kXStages * kXBytes + kWStages * kWBytes + 1024;
constexpr int kABuf = 8;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAcol0 = kBT;         // first A buffer column
constexpr int kThreads = 512;
constexpr int kEpiWarps = 8;
constexpr uint32_t kIdesc = idesc_f16_f32(kBN, kBT);

static_assert(kXBytes % 1024 == 0 && kWBytes % 1024 == 0, "stage alignment");
static_assert(kAcol0 + 32 * kABuf <= kTmemCols, "tensor memory budget");
static_assert(kSmemBytes <= 227 * 1024 - 512, "shared memory budget");

struct Params {
    const uint8_t *packed;
    const uint16_t *scales;
    const uint16_t *bias;   // may be null
    uint16_t *Y;
    int M;
    int64_t N;
    int KB;        // ceil(K/64)
    int TT;        // token tiles = ceil(M/256)
    int64_t tiles; // ceil(N/128) * TT
};

// Ring position: slot index and the parity of its current phase.
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

__global__ void __launch_bounds__(kThreads, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tmap_x, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *x_ring = base;                                  // kXStages x 32 KB
    uint8_t *w_ring = base + kXStages * kXBytes;             // kWStages x 8 KB
    __shared__ uint64_t w_full[kWStages], w_empty[kWStages];
    __shared__ uint64_t x_full[kXStages], x_empty[kXStages];
    __shared__ uint64_t a_full[kABuf], a_empty[kABuf];
    __shared__ uint64_t d_full, d_empty, drain;
    __shared__ uint32_t tmem_base_sh;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kWStages; ++i) {
            mbar_init(&w_full[i], 1);
            mbar_init(&w_empty[i], 4);        // the 4 converter warps
        }
        for (int i = 0; i < kXStages; ++i) {
            mbar_init(&x_full[i], 1);
            mbar_init(&x_empty[i], 1);        // MMA commit
        }
        for (int i = 0; i < kABuf; ++i) {
            mbar_init(&a_full[i], 4);
            mbar_init(&a_empty[i], 1);
        }
        mbar_init(&d_full, 1);
        mbar_init(&d_empty, kEpiWarps);
        mbar_init(&drain, 1);
        fence_barrier_init();
        prefetch_tensormap(&tmap_x);
    }
    if (warp == 2) {
        tmem_alloc(&tmem_base_sh, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    const int64_t tile0 = blockIdx.x;
    const int64_t tstep = gridDim.x;

    if (warp == 0 || warp == 3) {
        // ---------------------------------------------------- producers
        if (lane == 0) {
            const bool is_w = warp == 0;
            const int n = is_w ? kWStages : kXStages;
            uint64_t *fullb = is_w ? w_full : x_full;
            uint64_t *emptyb = is_w ? w_empty : x_empty;
            Ring r;
            int issued = 0;
            bool ok = true;
            for (int64_t tile = tile0; tile < p.tiles && ok; tile += tstep) {
                const int64_t nb = tile / p.TT;
                const int tb = (int)(tile % p.TT);
                const uint8_t *wsrc = p.packed + nb * p.KB * (int64_t)kWBytes;
                for (int kb = 0; kb < p.KB; ++kb) {
                    if (!mbar_wait(&emptyb[r.s], r.ph ^ 1u, is_w ? SITE_PF_EMPTY : SITE_PF_XEMPTY)) {
                        ok = false;
                        break;
                    }
                    if (is_w) {
                        mbar_arrive_expect_tx(&w_full[r.s], kWBytes);
                        bulk_g2s(w_ring + r.s * kWBytes, wsrc + (int64_t)kb * kWBytes, kWBytes, &w_full[r.s]);
                    } else {
                        mbar_arrive_expect_tx(&x_full[r.s], kXBytes);
                        tma_load_2d(x_ring + r.s * kXBytes, &tmap_x, kb * 64, tb * kBT, &x_full[r.s]);
                    }
                    ++issued;
                    r.next(n);
                }
            }
            // the copies this thread issued have landed before the CTA exits
            // (normally long since consumed; matters only after a timeout)
            for (int i = 0; i < n && i < issued; ++i) {
                r.prev(n);
                mbar_wait(&fullb[r.s], r.ph, SITE_PF_DRAIN, 10000000ull);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------- MMA issuer
        if (lane == 0) {
            Ring xr, ar;
            int it = 0;
            bool ok = true;
            for (int64_t tile = tile0; tile < p.tiles && ok; tile += tstep, ++it) {
                if (!mbar_wait(&d_empty, (it & 1) ^ 1u, SITE_PF_DEMPTY)) { ok = false; break; }
                tc_fence_after();
                for (int kb = 0; kb < p.KB; ++kb) {
                    if (!mbar_wait(&x_full[xr.s], xr.ph, SITE_PF_FULL_MMA)) { ok = false; break; }
                    if (!mbar_wait(&a_full[ar.s], ar.ph, SITE_PF_AFULL)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_tmem = tmem + kAcol0 + 32 * ar.s;
                    const uint32_t x_addr = smem_u32(x_ring + xr.s * kXBytes);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        tc_mma_ts_f16(tmem, a_tmem + 8 * j, smem_desc_kmajor_sw128(x_addr + 32 * j), kIdesc,
                                      (kb | j) != 0);
                    tc_commit(&x_empty[xr.s]);
                    tc_commit(&a_empty[ar.s]);
                    xr.next(kXStages);
                    ar.next(kABuf);
                }
                if (!ok) break;
                tc_commit(&d_full);
            }
            // all MMAs issued by this thread are complete before TMEM is freed
            tc_commit(&drain);
            mbar_wait(&drain, 0, SITE_PF_DRAIN);
        }
    } else if (warp >= 4 && warp < 8) {
        // ---------------------------------------------------- converters
        const int q4 = warp & 3;              // TMEM lane quarter of this warp
        const int r = 32 * q4 + lane;         // channel within the tile
        const int h = (r >> 1) & 3;
        const uint32_t lane_addr = tmem + ((uint32_t)(32 * q4) << 16);
        Ring wr, ar;
        bool ok = true;
        for (int64_t tile = tile0; tile < p.tiles && ok; tile += tstep) {
            for (int kb = 0; kb < p.KB; ++kb) {
                if (!mbar_wait(&w_full[wr.s], wr.ph, SITE_PF_FULL_CVT)) { ok = false; break; }
                const uint8_t *row = w_ring + wr.s * kWBytes + r * 64;
                uint4 c[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) c[i] = *reinterpret_cast<const uint4 *>(row + ((i ^ h) << 4));
                __syncwarp();
                if (lane == 0) mbar_arrive(&w_empty[wr.s]);
                uint32_t v[32];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t w[4] = {c[i].x, c[i].y, c[i].z, c[i].w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        v[8 * i + 2 * j] = unbias2(widen_lo2(w[j]));
                        v[8 * i + 2 * j + 1] = unbias2(widen_hi2(w[j]));
                    }
                }
                if (!mbar_wait(&a_empty[ar.s], ar.ph ^ 1u, SITE_PF_AEMPTY)) { ok = false; break; }
                tc_fence_after();
                tmem_st_32x32b_x32(lane_addr + kAcol0 + 32 * ar.s, v);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&a_full[ar.s]);
                wr.next(kWStages);
                ar.next(kABuf);
            }
        }
    } else if (warp >= 8) {
        // ---------------------------------------------------- epilogue
        const int q4 = warp & 3;
        const int half = (warp - 8) >> 2;     // columns [128 half, 128 half + 128)
        const int r = 32 * q4 + lane;
        const uint32_t lane_addr = tmem + ((uint32_t)(32 * q4) << 16) + 128 * half;
        int it = 0;
        for (int64_t tile = tile0; tile < p.tiles; tile += tstep, ++it) {
            if (!mbar_wait(&d_full, it & 1, SITE_PF_DFULL)) break;
            tc_fence_after();
            const int64_t nb = tile / p.TT;
            const int tb = (int)(tile % p.TT);
            const int64_t n = nb * kBN + r;
            const bool n_ok = n < p.N;
            const float sc = n_ok ? __half2float(__ushort_as_half(p.scales[n])) : 0.0f;
            const float bi = (n_ok && p.bias) ? __half2float(__ushort_as_half(p.bias[n])) : 0.0f;
            // drain this warp's 32 lanes x 128 columns into fp16 pairs
            uint32_t y2[64];
#pragma unroll
            for (int cchunk = 0; cchunk < 4; ++cchunk) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(lane_addr + 32 * cchunk, v);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const __half2 hv = __floats2half2_rn(fmaf(__uint_as_float(v[2 * i]), sc, bi),
                                                         fmaf(__uint_as_float(v[2 * i + 1]), sc, bi));
                    y2[16 * cchunk + i] = *reinterpret_cast<const uint32_t *>(&hv);
                }
            }
            // the accumulator may now take the next tile
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&d_empty);
            if (n_ok) {
                const int m0 = tb * kBT + 128 * half;
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    const int m = m0 + 2 * i;
                    if (m < p.M) p.Y[(int64_t)m * p.N + n] = (uint16_t)(y2[i] & 0xFFFFu);
                    if (m + 1 < p.M) p.Y[(int64_t)(m + 1) * p.N + n] = (uint16_t)(y2[i] >> 16);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace prefill
}  // namespace w8
