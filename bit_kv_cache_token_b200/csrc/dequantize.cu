// dequantize.cu -- packed records -> fp32 K / V (rotated or original basis).
//
// Dequantisation with both scales (rndamp.com article, "Numbers": the
// second scale is fused into dequantisation):
//   x_rot[t][d] = r_t * c_d * (s_{t,g} * code + m_{t,g}),
// then, for the original basis, the normalised Hadamard rotation again (it is
// its own inverse).  Not on the decode hot path: decode attention unpacks
// codes itself.  One thread per token.
#include "kvarn_common.cuh"
#include "kvarn_internal.h"

namespace kvarn {

template <int D, int HB>
__global__ void __launch_bounds__(128)
dequantize_kernel(DequantArgs a)
{
    using R = Record<D>;
    const int b = blockIdx.x % a.num_blocks;
    const int sh = blockIdx.x / a.num_blocks;
    const int tensor = blockIdx.y;
    float *out = tensor ? a.v_out : a.k_out;
    if (!out) return;
    const unsigned char *rec = static_cast<const unsigned char *>(tensor ? a.v_records : a.k_records) +
                               ((size_t)sh * a.max_blocks + a.first_block + b) * R::kBytes;
    const int t = threadIdx.x;
    const float r = __half2float(*reinterpret_cast<const __half *>(rec + R::kROff + 2 * t));
    const uint32_t *codes = reinterpret_cast<const uint32_t *>(rec);
    float x[D];
#pragma unroll
    for (int g = 0; g < D / kGroup; ++g) {
        const float s = __half2float(reinterpret_cast<const __half *>(rec + R::kSOff)[t * (D / kGroup) + g]);
        const float m = __half2float(reinterpret_cast<const __half *>(rec + R::kMOff)[t * (D / kGroup) + g]);
#pragma unroll
        for (int i = 0; i < kGroup; ++i) {
            const int d = g * kGroup + i;
            const int bit = tensor ? v_code_bit(t, d) : k_code_bit<D>(t, d);
            const float code = (float)((codes[bit >> 5] >> (bit & 31)) & 3u);
            const float c = __half2float(*reinterpret_cast<const __half *>(rec + R::kCOff + 2 * d));
            x[d] = r * c * fmaf(s, code, m);
        }
    }
    if (HB > 0 && !a.rotated) {
#pragma unroll
        for (int base = 0; base < D; base += (HB > 0 ? HB : D)) {
#pragma unroll
            for (int h = 1; h < HB; h <<= 1) {
#pragma unroll
                for (int i = 0; i < HB; ++i) {
                    if (i & h) continue;
                    const float p = x[base + i], q = x[base + i + h];
                    x[base + i] = p + q;
                    x[base + i + h] = p - q;
                }
            }
        }
        const float nrm = HB == 32 ? 0.17677669529663688f : HB == 64 ? 0.125f : 0.08838834764831845f;
#pragma unroll
        for (int d = 0; d < D; ++d) x[d] *= nrm;
    }
    float *o = out + (((size_t)sh * a.num_blocks + b) * kBlockTokens + t) * D;
#pragma unroll
    for (int d = 0; d < D; d += 4) *reinterpret_cast<float4 *>(o + d) = make_float4(x[d], x[d + 1], x[d + 2], x[d + 3]);
}

template <int D, int HB>
static cudaError_t launch_dq(const DequantArgs &a, int S, int Hkv, cudaStream_t st)
{
    dim3 grid((unsigned)(S * Hkv * a.num_blocks), 2);
    dequantize_kernel<D, HB><<<grid, kBlockTokens, 0, st>>>(a);
    return cudaGetLastError();
}

template <int D>
static cudaError_t dispatch_dq(int hb, const DequantArgs &a, int S, int Hkv, cudaStream_t st)
{
    switch (hb) {
    case 0: return launch_dq<D, 0>(a, S, Hkv, st);
    case 32: return launch_dq<D, 32>(a, S, Hkv, st);
    case 64: if constexpr (D % 64 == 0) return launch_dq<D, 64>(a, S, Hkv, st); break;
    case 128: if constexpr (D % 128 == 0) return launch_dq<D, 128>(a, S, Hkv, st); break;
    }
    return cudaErrorInvalidValue;
}

cudaError_t run_dequantize(const kvarn_config &c, const DequantArgs &a, cudaStream_t st)
{
    if (a.num_blocks == 0) return cudaSuccess;
    switch (c.head_dim) {
    case 64: return dispatch_dq<64>(c.hadamard, a, c.num_seqs, c.num_kv_heads, st);
    case 96: return dispatch_dq<96>(c.hadamard, a, c.num_seqs, c.num_kv_heads, st);
    case 128: return dispatch_dq<128>(c.hadamard, a, c.num_seqs, c.num_kv_heads, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace kvarn
