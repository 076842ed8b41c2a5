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

// Byte layout of one block record (see kvarn.h): 2-bit codes in the K or V
// fragment order, binary16 steps s[t][g], minima m[t][g], token scales r,
// channel scales c, padded to 128 bytes.
template <int D>
struct Record {
    static constexpr int kCodes = kBlockTokens * D / 4;
    static constexpr int kGroups = D / kGroup;
    static constexpr int kSOff = kCodes;
    static constexpr int kMOff = kSOff + kBlockTokens * kGroups * 2;
    static constexpr int kROff = kMOff + kBlockTokens * kGroups * 2;
    static constexpr int kCOff = kROff + 2 * kBlockTokens;
    static constexpr int kRaw = kCOff + 2 * D;
    static constexpr int kBytes = (kRaw + 127) / 128 * 128;
};

// Bit index, inside the code area, of the code of (token t, channel k) of a
// K record (fragment order of kvarn.h).
template <int D>
__host__ __device__ constexpr int k_code_bit(int t, int k)
{
    constexpr int F = D / 64;
    const int u = t / 16, n = (t % 16) / 8, lane = 4 * (t % 8) + (k % 8) / 2, half = k % 2, q = k / 8;
    int word, pos;
    if (q < 8 * F) { word = n * F + q / 8; pos = q % 8; }
    else { word = 2 * F; pos = q - 8 * F + 4 * n; }
    return ((u * 32 + lane) * (D / 32) + word) * 32 + 16 * half + 2 * pos;
}

// Same for a V record (token t, channel d).
__host__ __device__ constexpr int v_code_bit(int t, int d)
{
    const int j = d / 8, lane = 4 * (d % 8) + (t % 8) / 2, half = t % 2, a = (t % 32) / 8;
    const int word = a / 2, pos = 4 * (a % 2) + t / 32;
    return ((j * 32 + lane) * 2 + word) * 32 + 16 * half + 2 * pos;
}

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
    // load 8 consecutive elements (32 bytes, 16-byte aligned) as fp32; COHERENT
    // reads through L2 (data this kernel may have written), else the read-only path
    template <bool COHERENT = false>
    static __device__ __forceinline__ void load8(const float *p, float (&o)[8])
    {
        const float4 *q = reinterpret_cast<const float4 *>(p);
        const float4 a = COHERENT ? __ldcg(q) : __ldg(q);
        const float4 b = COHERENT ? __ldcg(q + 1) : __ldg(q + 1);
        o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
        o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
    }
    // load 4 consecutive elements (16 bytes, 16-byte aligned)
    static __device__ __forceinline__ float4 load4(const float *p) { return __ldg(reinterpret_cast<const float4 *>(p)); }
    // the same as raw bits, widened later (fewer registers while loads are in flight)
    using Raw4 = float4;
    static __device__ __forceinline__ Raw4 load4_raw(const float *p) { return load4(p); }
    static __device__ __forceinline__ float4 widen4(Raw4 r) { return r; }
    static __device__ __forceinline__ float load1(const float *p) { return *p; }
    static __device__ __forceinline__ void store1(float *p, float v) { *p = v; }
};

template <>
struct In<__nv_bfloat16> {
    template <bool COHERENT = false>
    static __device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&o)[8])
    {
        const uint4 *q = reinterpret_cast<const uint4 *>(p);
        const uint4 a = COHERENT ? __ldcg(q) : __ldg(q);
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            o[2 * i] = __uint_as_float(w[i] << 16);
            o[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
    // load 4 consecutive elements (8 bytes, 8-byte aligned) as fp32
    static __device__ __forceinline__ float4 load4(const __nv_bfloat16 *p)
    {
        const uint2 a = __ldg(reinterpret_cast<const uint2 *>(p));
        return make_float4(__uint_as_float(a.x << 16), __uint_as_float(a.x & 0xFFFF0000u),
                           __uint_as_float(a.y << 16), __uint_as_float(a.y & 0xFFFF0000u));
    }
    using Raw4 = uint2;
    static __device__ __forceinline__ Raw4 load4_raw(const __nv_bfloat16 *p)
    {
        return __ldg(reinterpret_cast<const uint2 *>(p));
    }
    static __device__ __forceinline__ float4 widen4(Raw4 a)
    {
        return make_float4(__uint_as_float(a.x << 16), __uint_as_float(a.x & 0xFFFF0000u),
                           __uint_as_float(a.y << 16), __uint_as_float(a.y & 0xFFFF0000u));
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

// Programmatic dependent launch.  A kernel launched by launch_overlapped has
// its launch prepared while the kernel before it in the stream is still
// running; grid_dep_wait blocks until that kernel has completed and its
// writes are visible, so it comes before the kernel's first access to global
// memory (in a kernel launched the ordinary way it returns at once).  No
// kernel here releases its dependents early (griddepcontrol.launch_dependents):
// with an early release the next kernel's blocks took the first SMs that the
// running kernel's blocks left, several to an SM, and the Qwen3-4B-shaped
// batch-8 step ran 0.7-4% slower; without it the step runs 0.6% faster than
// with ordinary launches.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
static cudaError_t launch_overlapped(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                     Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace kvarn
