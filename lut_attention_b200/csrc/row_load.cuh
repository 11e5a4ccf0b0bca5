// Loads of key rows for the CUDA-core kernels: 8 consecutive elements of a
// row-major fp32 / fp16 / bf16 matrix as fp32, in 16-byte loads.  elem is the
// index of the first of the 8 elements and must be a multiple of 8 in a 16-byte
// aligned buffer.  kStream marks data read once (evict-first); otherwise the
// loads keep the lines in cache for other CTAs that read the same keys.
#pragma once

#include <cstring>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace axr {

template <bool kStream, typename V>
__device__ __forceinline__ V ld16(const V *p)
{
    if constexpr (kStream) return __ldcs(p);
    else return __ldg(p);
}

template <typename T, bool kStream = true>
struct Load8;

template <bool kStream>
struct Load8<float, kStream> {
    __device__ static void run(const void *base, int64_t elem, float *v)
    {
        const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(base) + elem);
        const float4 a = ld16<kStream>(p);
        const float4 b = ld16<kStream>(p + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
};

template <bool kStream>
struct Load8<__nv_bfloat16, kStream> {
    __device__ static void run(const void *base, int64_t elem, float *v)
    {
        const uint4 *p = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(base) + elem);
        const uint4 w = ld16<kStream>(p);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(ws[i] << 16);
            v[2 * i + 1] = __uint_as_float(ws[i] & 0xffff0000u);
        }
    }
};

template <bool kStream>
struct Load8<__half, kStream> {
    __device__ static void run(const void *base, int64_t elem, float *v)
    {
        const uint4 *p = reinterpret_cast<const uint4 *>(static_cast<const __half *>(base) + elem);
        const uint4 w = ld16<kStream>(p);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __half2 h2;
            memcpy(&h2, &ws[i], 4);
            const float2 f = __half22float2(h2);
            v[2 * i] = f.x;
            v[2 * i + 1] = f.y;
        }
    }
};

}  // namespace axr
