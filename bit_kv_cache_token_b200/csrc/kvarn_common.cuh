// kvarn_common.cuh -- record layout and small device helpers shared by the
// KVarN kernels (quantise, append, dequantise, decode attention).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvarn.h"

namespace kvarn {

// Tokens per quantised block and channels per quantisation group.  The
// pages leave both open; the library fixes them at 128 and 32.
constexpr int kBlockTokens = 128;
constexpr int kGroup = 32;

// Byte layout of one block record (see kvarn.h): codes, (s, m) pairs,
// token scales r, channel scales c, padded to 128 bytes.
template <int D>
struct Record {
    static constexpr int kCodes = kBlockTokens * D / 4;
    static constexpr int kGroups = D / kGroup;
    static constexpr int kGpOff = kCodes;
    static constexpr int kROff = kGpOff + kBlockTokens * kGroups * 4;
    static constexpr int kCOff = kROff + 2 * kBlockTokens;
    static constexpr int kRaw = kCOff + 2 * D;
    static constexpr int kBytes = (kRaw + 127) / 128 * 128;
};

__host__ __device__ inline size_t record_bytes_rt(int D)
{
    const size_t raw = (size_t)kBlockTokens * D / 4 + (size_t)kBlockTokens * (D / kGroup) * 4 +
                       2 * (size_t)kBlockTokens + 2 * (size_t)D;
    return (raw + 127) / 128 * 128;
}

// ---- input element access (fp32 or bf16) --------------------------------
template <typename T>
struct In;

template <>
struct In<float> {
    // load 8 consecutive elements (32 bytes, 16-byte aligned) as fp32
    static __device__ __forceinline__ void load8(const float *p, float (&o)[8])
    {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(p));
        const float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
        o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
        o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
    }
    static __device__ __forceinline__ float load1(const float *p) { return *p; }
    static __device__ __forceinline__ void store1(float *p, float v) { *p = v; }
};

template <>
struct In<__nv_bfloat16> {
    static __device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&o)[8])
    {
        const uint4 a = __ldg(reinterpret_cast<const uint4 *>(p));
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            o[2 * i] = __uint_as_float(w[i] << 16);
            o[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
    static __device__ __forceinline__ float load1(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void store1(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }
};

// Same-type element copy (bit-exact, no rounding): used for the tail.
template <typename T>
__device__ __forceinline__ void copy_elems(T *dst, const T *src, int n, int tid, int nthreads)
{
    for (int i = tid; i < n; i += nthreads) dst[i] = src[i];
}

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

__device__ __forceinline__ void status_or(int32_t *status, int bits)
{
    if (status) atomicOr(reinterpret_cast<int *>(status), bits);
}

}  // namespace kvarn
