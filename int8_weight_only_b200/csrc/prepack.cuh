// Reorder the int8 codes q[K, N] into the tiled layout the linear kernels
// stream (layout specified in w8a16.h, w8_prepack).  One CTA per 8 KB tile;
// done once per weight, so the kernel favours simplicity over bandwidth.
#pragma once

#include "common.cuh"

namespace w8 {
namespace pack {

constexpr int kThreads = 128;
constexpr int kTileN = 128;
constexpr int kTileK = 64;
constexpr int kTileBytes = kTileN * kTileK;
constexpr int kPitch = kTileN + 4;   // shared row pitch (bytes), keeps 4-byte alignment

__device__ __forceinline__ int chunk_slot(int r, int c) { return c ^ ((r >> 1) & 3); }

// grid = (ceil(K/64), ceil(N/128))
__global__ void __launch_bounds__(kThreads)
prepack_kernel(const int8_t *__restrict__ q, int64_t K, int64_t N, int KB,
               uint8_t *__restrict__ packed) {
    __shared__ __align__(16) uint8_t tile[kTileK][kPitch];   // [k][n]
    const int kb = blockIdx.x;
    const int64_t b = blockIdx.y;
    const int64_t k0 = (int64_t)kb * kTileK;
    const int64_t n0 = b * kTileN;
    const int tid = threadIdx.x;

    for (int idx = tid; idx < kTileK * (kTileN / 4); idx += kThreads) {
        const int r = idx / (kTileN / 4);
        const int w = idx % (kTileN / 4);
        const int64_t k = k0 + r;
        const int64_t n = n0 + 4 * w;
        uint32_t v = 0;
        if (k < K && n < N)   // N % 8 == 0: the 4 bytes are all in range
            v = *reinterpret_cast<const uint32_t *>(q + k * N + n);
        *reinterpret_cast<uint32_t *>(&tile[r][4 * w]) = v;
    }
    __syncthreads();

    uint8_t *dst = packed + (b * KB + kb) * (int64_t)kTileBytes;
    const int r = tid;   // one output row (channel) per thread
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t v = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                v |= (uint32_t)(uint8_t)(tile[16 * c + 4 * i + j][r] ^ 0x80u) << (8 * j);
            w[i] = v;
        }
        *reinterpret_cast<uint4 *>(dst + r * 64 + chunk_slot(r, c) * 16) =
            make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// Inverse of prepack_kernel.  grid = (ceil(K/64), ceil(N/128))
__global__ void __launch_bounds__(kThreads)
unpack_kernel(const uint8_t *__restrict__ packed, int64_t K, int64_t N, int KB,
              int8_t *__restrict__ q) {
    __shared__ __align__(16) uint8_t tile[kTileK][kPitch];
    const int kb = blockIdx.x;
    const int64_t b = blockIdx.y;
    const int64_t k0 = (int64_t)kb * kTileK;
    const int64_t n0 = b * kTileN;
    const int tid = threadIdx.x;
    const uint8_t *src = packed + (b * KB + kb) * (int64_t)kTileBytes;
    const int r = tid;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint4 v = *reinterpret_cast<const uint4 *>(src + r * 64 + chunk_slot(r, c) * 16);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j)
                tile[16 * c + 4 * i + j][r] = (uint8_t)((w[i] >> (8 * j)) & 0xFFu) ^ 0x80u;
    }
    __syncthreads();
    for (int idx = tid; idx < kTileK * (kTileN / 4); idx += kThreads) {
        const int rr = idx / (kTileN / 4);
        const int w = idx % (kTileN / 4);
        const int64_t k = k0 + rr;
        const int64_t n = n0 + 4 * w;
        if (k < K && n < N)
            *reinterpret_cast<uint32_t *>(q + k * N + n) =
                *reinterpret_cast<const uint32_t *>(&tile[rr][4 * w]);
    }
}

}  // namespace pack
}  // namespace w8
