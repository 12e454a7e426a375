// Per-output-channel symmetric int8 quantization (TPU-MLIR ChatGLM2 W8A16
// article, sections 2-3; LightSeq 2020 slides "clipping + symmetric").
//
//   s_n = fp16_rne( fp32(max_k |W[k,n]|) / 127 )
//   q[k,n] = clamp( rne( W[k,n] / float(s_n) ), -127, 127 ),  q = 0 if s_n == 0
//
// HBM-bound: the algorithmic traffic is one read of W (4 or 2 bytes per
// weight) plus one write of q (1 byte per weight).  To read W only once,
// a thread-block cluster of CQ CTAs owns a strip of BN columns: CTA r of the
// cluster stages rows [r*kc, (r+1)*kc) of the strip in shared memory with
// 2-D TMA loads, reduces its per-column |max|, the cluster combines the CQ
// partial maxima through distributed shared memory, and every CTA then
// quantizes its rows straight from shared memory.  When K is too large for
// the strip to stay resident (K * BN * elem > cluster shared memory), the
// same kernel streams the rows twice (max pass, then quantize pass).
#pragma once

#include "common.cuh"

namespace w8 {
namespace quant {

constexpr int kThreads = 256;
constexpr int kBoxRows = 64;          // rows per TMA box
constexpr int kMaxBoxes = 32;         // mbarriers per CTA

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }

// 4 consecutive elements of one row, widened to fp32.
template <typename T>
__device__ __forceinline__ void load4(const T *p, float (&v)[4]);
template <>
__device__ __forceinline__ void load4<float>(const float *p, float (&v)[4]) {
    float4 t = *reinterpret_cast<const float4 *>(p);
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
}
template <>
__device__ __forceinline__ void load4<__half>(const __half *p, float (&v)[4]) {
    uint2 t = *reinterpret_cast<const uint2 *>(p);
    __half2 a = *reinterpret_cast<__half2 *>(&t.x);
    __half2 b = *reinterpret_cast<__half2 *>(&t.y);
    v[0] = __low2float(a); v[1] = __high2float(a);
    v[2] = __low2float(b); v[3] = __high2float(b);
}

__device__ __forceinline__ int quantize_one(float w, float s) {
    if (s == 0.0f) return 0;
    int v = __float2int_rn(__fdiv_rn(w, s));   // IEEE division, ties to even
    return max(-127, min(127, v));
}

// Launch: grid.x = CQ * ceil(N / BN) with cluster dims (CQ, 1, 1); the
// cluster rank is the K slice.  Dynamic shared memory: nbuf boxes of
// kBoxRows x BN elements plus 1 KB of alignment slack.
//   kc      rows per CTA (multiple of kBoxRows)
//   nbuf    boxes held in shared memory (== kc / kBoxRows when resident)
template <typename T, int BN>
__global__ void __launch_bounds__(kThreads)
quantize_kernel(const __grid_constant__ CUtensorMap tmap_w, int64_t K, int64_t N, int kc,
                int nbuf, int8_t *__restrict__ q, uint16_t *__restrict__ scales) {
    static_assert(BN % 4 == 0 && (kThreads / (BN / 4)) * (BN / 4) == kThreads, "layout");
    constexpr int kColGroups = BN / 4;                  // threads per row
    constexpr int kRowsPerPass = kThreads / kColGroups; // rows per sweep
    constexpr int kBoxElems = kBoxRows * BN;
    constexpr uint32_t kBoxBytes = kBoxElems * sizeof(T);

    extern __shared__ uint8_t smem_raw[];
    T *buf = reinterpret_cast<T *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    __shared__ uint64_t bars[kMaxBoxes];
    __shared__ float red[kRowsPerPass][BN + 1];
    __shared__ float cta_amax[BN];
    __shared__ float col_scale[BN];
    __shared__ int abort_flag;

    uint32_t rank;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
    uint32_t csize;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(csize));
    const int64_t strip = blockIdx.x / csize;
    const int64_t n0 = strip * BN;
    const int64_t k_begin = (int64_t)rank * kc;
    const int64_t k_end = min64(K, k_begin + (int64_t)kc);
    const int rows = (int)max64(0, k_end - k_begin);
    const int nbox = (rows + kBoxRows - 1) / kBoxRows;
    const bool resident = nbox <= nbuf;
    const int tid = threadIdx.x;
    const int cg = tid % kColGroups;     // column group: columns 4cg .. 4cg+3
    const int rg = tid / kColGroups;     // row within a sweep

    if (tid == 0) {
        abort_flag = 0;
        for (int i = 0; i < nbuf; ++i) mbar_init(&bars[i], 1);
        fence_barrier_init();
        prefetch_tensormap(&tmap_w);
    }
    __syncthreads();

    uint32_t phase_bits = 0;   // bit i: parity of the next completion of bars[i]

    // Issue box `i` into buffer slot i % nbuf (thread 0 only).
    auto issue = [&](int i) {
        const int slot = i % nbuf;
        mbar_arrive_expect_tx(&bars[slot], kBoxBytes);
        tma_load_2d(buf + (size_t)slot * kBoxElems, &tmap_w, (int32_t)n0,
                    (int32_t)(k_begin + (int64_t)i * kBoxRows), &bars[slot]);
    };
    auto wait_box = [&](int i) -> bool {
        const int slot = i % nbuf;
        const bool ok = mbar_wait(&bars[slot], (phase_bits >> slot) & 1u, SITE_Q_LOAD);
        phase_bits ^= 1u << slot;
        return ok;
    };

    // ---------------- pass 1: per-column |max| over this CTA's rows
    float amax[4] = {0.f, 0.f, 0.f, 0.f};
    for (int g0 = 0; g0 < nbox; g0 += nbuf) {
        const int g1 = min(nbox, g0 + nbuf);
        if (tid == 0)
            for (int i = g0; i < g1; ++i) issue(i);
        for (int i = g0; i < g1; ++i) {
            if (!wait_box(i)) abort_flag = 1;
            const T *box = buf + (size_t)(i % nbuf) * kBoxElems;
            const int box_rows = min(kBoxRows, rows - i * kBoxRows);
            for (int r = rg; r < box_rows; r += kRowsPerPass) {
                float v[4];
                load4<T>(box + r * BN + 4 * cg, v);
#pragma unroll
                for (int j = 0; j < 4; ++j) amax[j] = fmaxf(amax[j], fabsf(v[j]));
            }
        }
        if (!resident) __syncthreads();   // slots are reused by the next group
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) red[rg][4 * cg + j] = amax[j];
    __syncthreads();
    if (tid < BN) {
        float m = 0.f;
        for (int r = 0; r < kRowsPerPass; ++r) m = fmaxf(m, red[r][tid]);
        cta_amax[tid] = m;
    }
    // ---------------- cluster-wide maximum through distributed shared memory
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    if (tid < BN) {
        float m = 0.f;
        const uint32_t local = smem_u32(&cta_amax[tid]);
        for (uint32_t r = 0; r < csize; ++r) {
            uint32_t remote;
            asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(r));
            float v;
            asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
            m = fmaxf(m, v);
        }
        const __half s16 = __float2half_rn(__fdiv_rn(m, 127.0f));
        col_scale[tid] = __half2float(s16);
        if (rank == 0 && n0 + tid < N) scales[n0 + tid] = __half_as_ushort(s16);
    }
    // no CTA may leave while a peer still reads its cta_amax
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");

    // ---------------- pass 2: quantize (from shared memory when resident)
    float s[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) s[j] = col_scale[4 * cg + j];
    const bool col_ok = (n0 + 4 * cg) < N;   // N % 8 == 0: groups of 4 are all in or all out
    for (int g0 = 0; g0 < nbox; g0 += nbuf) {
        const int g1 = min(nbox, g0 + nbuf);
        if (!resident) {
            if (tid == 0)
                for (int i = g0; i < g1; ++i) issue(i);
        }
        for (int i = g0; i < g1; ++i) {
            if (!resident && !wait_box(i)) abort_flag = 1;
            const T *box = buf + (size_t)(i % nbuf) * kBoxElems;
            const int box_rows = min(kBoxRows, rows - i * kBoxRows);
            for (int r = rg; r < box_rows; r += kRowsPerPass) {
                float v[4];
                load4<T>(box + r * BN + 4 * cg, v);
                uint32_t packed = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    packed |= (uint32_t)(quantize_one(v[j], s[j]) & 0xFF) << (8 * j);
                const int64_t k = k_begin + (int64_t)i * kBoxRows + r;
                if (col_ok)
                    *reinterpret_cast<uint32_t *>(q + k * N + n0 + 4 * cg) = packed;
            }
        }
        if (!resident) __syncthreads();
    }
}

}  // namespace quant
}  // namespace w8
