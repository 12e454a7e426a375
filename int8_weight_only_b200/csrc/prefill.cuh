// Prefill-regime W8A16 linear (M > 16 tokens) on the 5th-generation tensor
// cores: Y = X . dequant(q) (+ bias).
//
// The TPU-MLIR article (section 4) gives the W8A16 MatMul as load -> cast
// int8 to F16 -> scale -> matmul -> store, with the load overlapped with
// compute through ping-pong local memory.  On sm_100a the same five steps
// become a warp-specialised pipeline per CTA (one CTA per SM, persistent):
//
//   warp 0      TMA producer: per 64-wide K block, one 1-D bulk copy of the
//               8 KB packed int8 tile (128 channels x 64) and one 2-D TMA
//               load of the X tile (128 tokens x 64, 128-byte swizzle) into
//               a 6-stage shared-memory ring.
//   warps 4-7   converters ("cast"): thread r owns channel r of the tile,
//               reads its 64 int8 codes, widens them to fp16 in registers
//               and writes them with tcgen05.st into tensor memory, where
//               they are the A operand of the MMA.  The widened weights
//               therefore never pass through shared memory.
//   warp 1      MMA issuer ("matmul"): tcgen05.mma kind::f16, A (128
//               channels x 16) from tensor memory, B (128 tokens x 16) from
//               the swizzled X tile, fp32 accumulator D (128 x 128) in
//               tensor memory; four MMAs per K block.
//   warps 8-11  epilogue ("scale" + "store"): tcgen05.ld of the accumulator,
//               y = acc * s_n + bias_n in fp32, one rounding to fp16, store.
//
// Tensor memory: two accumulators (columns [0,128) and [128,256)) so the
// epilogue of tile i overlaps the main loop of tile i+1, and two A buffers
// of 32 columns (64 fp16 per channel) at [256, 320).
// Tiles: 128 channels x 128 tokens; tile id = channel block * token tiles +
// token tile, so CTAs running together share a channel block (its weight
// tile is read from HBM once and then hit in L2).
#pragma once

#include "common.cuh"

namespace w8 {
namespace prefill {

constexpr int kBN = 128;                 // channels per tile (MMA M)
constexpr int kBT = 128;                 // tokens per tile (MMA N)
constexpr int kStages = 6;
constexpr int kWBytes = 8192;            // packed int8 tile
constexpr int kXBytes = kBT * 128;       // 128 tokens x 64 fp16
constexpr int kStageBytes = kWBytes + kXBytes;
constexpr int kSmemBytes = kStages * kStageBytes + 1024;
constexpr int kABuf = 2;
constexpr int kDBuf = 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAcol0 = kDBuf * kBT; // first A buffer column
constexpr int kThreads = 384;
constexpr uint32_t kIdesc = idesc_f16_f32(kBN, kBT);

static_assert(kStageBytes % 1024 == 0, "stage alignment");
static_assert(kAcol0 + 32 * kABuf <= kTmemCols, "tensor memory budget");

struct Params {
    const uint8_t *packed;
    const uint16_t *scales;
    const uint16_t *bias;   // may be null
    uint16_t *Y;
    int M;
    int64_t N;
    int KB;        // ceil(K/64)
    int TT;        // token tiles = ceil(M/128)
    int64_t tiles; // ceil(N/128) * TT
};

__global__ void __launch_bounds__(kThreads, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tmap_x, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    __shared__ uint64_t full[kStages], empty[kStages];
    __shared__ uint64_t a_full[kABuf], a_empty[kABuf];
    __shared__ uint64_t d_full[kDBuf], d_empty[kDBuf];
    __shared__ uint64_t drain;
    __shared__ uint32_t tmem_base_sh;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 4 + 1);     // 4 converter warps + 1 MMA commit
        }
        for (int i = 0; i < kABuf; ++i) {
            mbar_init(&a_full[i], 4);
            mbar_init(&a_empty[i], 1);
        }
        for (int i = 0; i < kDBuf; ++i) {
            mbar_init(&d_full[i], 1);
            mbar_init(&d_empty[i], 4);
        }
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

    if (warp == 0) {
        // ---------------------------------------------------- TMA producer
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int64_t tile = tile0; tile < p.tiles && ok; tile += tstep) {
                const int64_t nb = tile / p.TT;
                const int tb = (int)(tile % p.TT);
                const uint8_t *wsrc = p.packed + nb * p.KB * (int64_t)kWBytes;
                for (int kb = 0; kb < p.KB; ++kb) {
                    if (!mbar_wait(&empty[s], ph ^ 1u, SITE_PF_EMPTY)) { ok = false; break; }
                    uint8_t *xs = base + s * kStageBytes;
                    uint8_t *ws = xs + kXBytes;
                    mbar_arrive_expect_tx(&full[s], kWBytes + kXBytes);
                    bulk_g2s(ws, wsrc + (int64_t)kb * kWBytes, kWBytes, &full[s]);
                    tma_load_2d(xs, &tmap_x, kb * 64, tb * kBT, &full[s]);
                    if (++s == kStages) { s = 0; ph ^= 1u; }
                }
            }
            if (!ok) {
                // let the copies already issued land before the CTA can exit
                for (int i = 0; i < kStages; ++i) {
                    if (--s < 0) { s = kStages - 1; ph ^= 1u; }
                    mbar_wait(&full[s], ph, SITE_PF_DRAIN, 10000000ull);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------- MMA issuer
        if (lane == 0) {
            int s = 0, ab = 0;
            uint32_t ph = 0, aph = 0;
            int it = 0;
            bool ok = true;
            for (int64_t tile = tile0; tile < p.tiles && ok; tile += tstep, ++it) {
                const int d = it & 1;
                const uint32_t dph = (it >> 1) & 1;
                if (!mbar_wait(&d_empty[d], dph ^ 1u, SITE_PF_DEMPTY)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem + d * kBT;
                for (int kb = 0; kb < p.KB; ++kb) {
                    if (!mbar_wait(&full[s], ph, SITE_PF_FULL_MMA)) { ok = false; break; }
                    if (!mbar_wait(&a_full[ab], aph, SITE_PF_AFULL)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_tmem = tmem + kAcol0 + 32 * ab;
                    const uint32_t x_addr = smem_u32(base + s * kStageBytes);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        tc_mma_ts_f16(d_tmem, a_tmem + 8 * j, smem_desc_kmajor_sw128(x_addr + 32 * j),
                                      kIdesc, (kb | j) != 0);
                    tc_commit(&empty[s]);
                    tc_commit(&a_empty[ab]);
                    if (++s == kStages) { s = 0; ph ^= 1u; }
                    if (++ab == kABuf) { ab = 0; aph ^= 1u; }
                }
                if (!ok) break;
                tc_commit(&d_full[d]);
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
        int s = 0, ab = 0;
        uint32_t ph = 0, aph = 0;
        bool ok = true;
        for (int64_t tile = tile0; tile < p.tiles && ok; tile += tstep) {
            for (int kb = 0; kb < p.KB; ++kb) {
                if (!mbar_wait(&full[s], ph, SITE_PF_FULL_CVT)) { ok = false; break; }
                const uint8_t *row = base + s * kStageBytes + kXBytes + r * 64;
                uint4 c[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) c[i] = *reinterpret_cast<const uint4 *>(row + ((i ^ h) << 4));
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
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
                if (!mbar_wait(&a_empty[ab], aph ^ 1u, SITE_PF_AEMPTY)) { ok = false; break; }
                tc_fence_after();
                tmem_st_32x32b_x32(lane_addr + kAcol0 + 32 * ab, v);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&a_full[ab]);
                if (++s == kStages) { s = 0; ph ^= 1u; }
                if (++ab == kABuf) { ab = 0; aph ^= 1u; }
            }
        }
    } else if (warp >= 8) {
        // ---------------------------------------------------- epilogue
        const int q4 = warp & 3;
        const int r = 32 * q4 + lane;
        const uint32_t lane_addr = tmem + ((uint32_t)(32 * q4) << 16);
        int it = 0;
        for (int64_t tile = tile0; tile < p.tiles; tile += tstep, ++it) {
            const int d = it & 1;
            const uint32_t dph = (it >> 1) & 1;
            if (!mbar_wait(&d_full[d], dph, SITE_PF_DFULL)) break;
            tc_fence_after();
            const int64_t nb = tile / p.TT;
            const int tb = (int)(tile % p.TT);
            const int64_t n = nb * kBN + r;
            const bool n_ok = n < p.N;
            const float sc = n_ok ? __half2float(__ushort_as_half(p.scales[n])) : 0.0f;
            const float bi = (n_ok && p.bias) ? __half2float(__ushort_as_half(p.bias[n])) : 0.0f;
#pragma unroll 1
            for (int cchunk = 0; cchunk < kBT / 32; ++cchunk) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(lane_addr + d * kBT + 32 * cchunk, v);
                tmem_wait_ld();
                const int m0 = tb * kBT + 32 * cchunk;
                if (n_ok) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int m = m0 + i;
                        if (m < p.M)
                            p.Y[(int64_t)m * p.N + n] =
                                __half_as_ushort(__float2half_rn(fmaf(__uint_as_float(v[i]), sc, bi)));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&d_empty[d]);
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
