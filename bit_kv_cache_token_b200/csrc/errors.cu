// errors.cu -- per-token quantisation error of stored blocks, split into
// magnitude and direction.
//
// The article on KVarN ("The Problem"; "How It Works") attributes the drift of
// long generations to errors in the magnitude of the cached vectors rather
// than in their direction; the abstract frames the method as removing that
// accumulation.  For each token of a block this kernel compares the original
// row x (as given to the quantiser) with its dequantised record x^:
//   magnitude error |‖x^‖ / ‖x‖ − 1|,  direction error 1 − x^·x / (‖x^‖ ‖x‖).
// Both are unchanged by the orthogonal Hadamard rotation, so they are taken
// in the rotated basis: x is rotated exactly as the quantiser rotates it and
// x^ = r c (s code + m) from the record's binary16 scales, with no inverse
// rotation.  A zero row gives (0, 0).
#include "kvarn_internal.h"
#include "quantize_block.cuh"

namespace kvarn {

// One CTA of D threads per (sequence, kv head, block) and tensor (blockIdx.y).
template <int D, int HB, typename Tin>
__global__ void __launch_bounds__(D, 2)
token_errors_kernel(ErrorArgs a)
{
    using R = Record<D>;
    constexpr int W = D / 32;
    constexpr int NG = D / kGroup;
    QuantSmem<D> &sm = quant_smem<D>();
    __shared__ float red[3][W][kBlockTokens];
    const int j = threadIdx.x >> 5, l = threadIdx.x & 31;
    const int nb = a.num_blocks;
    const int b = blockIdx.x % nb;
    const int sh = blockIdx.x / nb;
    const int tensor = blockIdx.y;
    const Tin *src = static_cast<const Tin *>(tensor ? a.v : a.k) + ((size_t)sh * nb + b) * kBlockTokens * D;
    const unsigned char *rec = static_cast<const unsigned char *>(tensor ? a.v_records : a.k_records) +
                               ((size_t)sh * a.max_blocks + a.first_block + b) * R::kBytes;

    float2 X[4][16];
    load_block<D>(src, X);
    rotate_block<D, HB>(X, sm);

    const __half *sh16 = reinterpret_cast<const __half *>(rec + R::kSOff);
    const __half *mh16 = reinterpret_cast<const __half *>(rec + R::kMOff);
    const __half *rh16 = reinterpret_cast<const __half *>(rec + R::kROff);
    const __half *ch16 = reinterpret_cast<const __half *>(rec + R::kCOff);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int t = qtok(l) + 32 * r;
        const float rt = __half2float(rh16[t]);
        const float s = __half2float(sh16[t * NG + j]), m = __half2float(mh16[t * NG + j]);
        float xx = 0.f, yy = 0.f, xy = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int d = 32 * j + 2 * k + e;
                const int bit = tensor ? v_code_bit(t, d) : k_code_bit<D>(t, d);
                const float code = (float)((rec[bit >> 3] >> (bit & 7)) & 3);
                const float y = rt * __half2float(ch16[d]) * fmaf(s, code, m);
                const float x = e ? X[r][k].y : X[r][k].x;
                xx = fmaf(x, x, xx);
                yy = fmaf(y, y, yy);
                xy = fmaf(x, y, xy);
            }
        }
        red[0][j][t] = xx;
        red[1][j][t] = yy;
        red[2][j][t] = xy;
    }
    __syncthreads();
    for (int t = threadIdx.x; t < kBlockTokens; t += D) {  // D may be below 128
        float xx = 0.f, yy = 0.f, xy = 0.f;
#pragma unroll
        for (int jj = 0; jj < W; ++jj) {
            xx += red[0][jj][t];
            yy += red[1][jj][t];
            xy += red[2][jj][t];
        }
        float mag = 0.f, dir = 0.f;
        if (xx > 0.f) {
            const float nx = sqrtf(xx), ny = sqrtf(yy);
            mag = fabsf(ny / nx - 1.f);
            dir = ny > 0.f ? 1.f - xy / (nx * ny) : 1.f;
        }
        float *out = (tensor ? a.err_v : a.err_k) + (((size_t)sh * nb + b) * kBlockTokens + t) * 2;
        out[0] = mag;
        out[1] = dir;
    }
}

template <int D, int HB, typename Tin>
static cudaError_t launch_err(const ErrorArgs &a, int units, cudaStream_t st)
{
    dim3 grid((unsigned)(units * a.num_blocks), 2);
    constexpr int kSmem = (int)sizeof(QuantSmem<D>);
    const cudaError_t e =
        cudaFuncSetAttribute(token_errors_kernel<D, HB, Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    token_errors_kernel<D, HB, Tin><<<grid, D, kSmem, st>>>(a);
    return cudaGetLastError();
}

template <int D, int HB>
static cudaError_t err_dtype(int dtype, const ErrorArgs &a, int units, cudaStream_t st)
{
    return dtype == KVARN_BF16 ? launch_err<D, HB, __nv_bfloat16>(a, units, st) : launch_err<D, HB, float>(a, units, st);
}

template <int D>
static cudaError_t err_hb(int hb, int dtype, const ErrorArgs &a, int units, cudaStream_t st)
{
    switch (hb) {
    case 0: return err_dtype<D, 0>(dtype, a, units, st);
    case 32: return err_dtype<D, 32>(dtype, a, units, st);
    case 64: if constexpr (D % 64 == 0) return err_dtype<D, 64>(dtype, a, units, st); break;
    case 128: if constexpr (D % 128 == 0) return err_dtype<D, 128>(dtype, a, units, st); break;
    }
    return cudaErrorInvalidValue;
}

cudaError_t run_token_errors(const kvarn_config &c, const ErrorArgs &a, cudaStream_t st)
{
    if (a.num_blocks == 0) return cudaSuccess;
    const int units = c.num_seqs * c.num_kv_heads;
    switch (c.head_dim) {
    case 64: return err_hb<64>(c.hadamard, c.dtype, a, units, st);
    case 96: return err_hb<96>(c.hadamard, c.dtype, a, units, st);
    case 128: return err_hb<128>(c.hadamard, c.dtype, a, units, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace kvarn
