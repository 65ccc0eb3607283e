// 16-byte vectorised row-slice loads and stores (bf16 or fp32 in memory,
// fp32 in registers).  Slices must start on a 16-byte boundary.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

namespace hga {

template <typename T, int N>
__device__ __forceinline__ void load_slice(const T *__restrict__ p, float (&x)[N]) {
    if constexpr (sizeof(T) == 2) {
        static_assert(N % 8 == 0, "bf16 slices are multiples of 8");
#pragma unroll
        for (int v = 0; v < N / 8; ++v) {
            uint4 w = __ldg(reinterpret_cast<const uint4 *>(p) + v);
            const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&w);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float2 f = __bfloat1622float2(h[e]);
                x[v * 8 + 2 * e] = f.x;
                x[v * 8 + 2 * e + 1] = f.y;
            }
        }
    } else {
        static_assert(N % 4 == 0, "f32 slices are multiples of 4");
#pragma unroll
        for (int v = 0; v < N / 4; ++v) {
            float4 w = __ldg(reinterpret_cast<const float4 *>(p) + v);
            x[v * 4 + 0] = w.x;
            x[v * 4 + 1] = w.y;
            x[v * 4 + 2] = w.z;
            x[v * 4 + 3] = w.w;
        }
    }
}

template <typename T, int N>
__device__ __forceinline__ void store_slice(T *__restrict__ p, const float (&x)[N]) {
    if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int v = 0; v < N / 8; ++v) {
            uint4 w;
            __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&w);
#pragma unroll
            for (int e = 0; e < 4; ++e)
                h[e] = __floats2bfloat162_rn(x[v * 8 + 2 * e], x[v * 8 + 2 * e + 1]);
            reinterpret_cast<uint4 *>(p)[v] = w;
        }
    } else {
#pragma unroll
        for (int v = 0; v < N / 4; ++v)
            reinterpret_cast<float4 *>(p)[v] =
                make_float4(x[v * 4 + 0], x[v * 4 + 1], x[v * 4 + 2], x[v * 4 + 3]);
    }
}

// Unpack N elements held as 16-byte words (8 bf16 or 4 fp32 per word).
template <typename T, int N>
__device__ __forceinline__ void unpack_words(const uint4 (&w)[N * sizeof(T) / 16], float (&x)[N]) {
    if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int v = 0; v < N / 8; ++v) {
            const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&w[v]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h[e]);
                x[v * 8 + 2 * e] = f.x;
                x[v * 8 + 2 * e + 1] = f.y;
            }
        }
    } else {
#pragma unroll
        for (int v = 0; v < N / 4; ++v) {
            x[v * 4 + 0] = __uint_as_float(w[v].x);
            x[v * 4 + 1] = __uint_as_float(w[v].y);
            x[v * 4 + 2] = __uint_as_float(w[v].z);
            x[v * 4 + 3] = __uint_as_float(w[v].w);
        }
    }
}

}  // namespace hga
