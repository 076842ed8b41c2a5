// decode.cu -- split-K single-token decode attention over the packed cache.
//
// KVarN decode (abstract: attention over the 2-bit cache during long-horizon
// decoding; rndamp.com article, "Numbers": the second scale is fused into the
// dequantisation kernel).  The keys are stored rotated, so the query is
// rotated once (normalised Hadamard, per Hadamard block) and the scores are
// taken in the rotated basis, where q . k is unchanged.  With
// k_rot[t][d] = r_t c_d (s_{t,g} code + m_{t,g}):
//   score_t = r_t * sum_g ( s_{t,g} * sum_{d in g} q'_d code_{t,d} + m_{t,g} Q_g ),
//   q'_d = q_rot,d * c_d * scale,   Q_g = sum_{d in g} q'_d,
// so c^K folds into the query once per block and r^K, s^K, m^K into one FMA
// per (token, group).  For V, with p_t the softmax weight:
//   o_rot,d += c^V_d * sum_t ( p_t r^V_t s^V_{t,g} code_{t,d} + p_t r^V_t m^V_{t,g} ).
// The residual tail (unrotated, input dtype) is attended with the unrotated
// query in its own split; the combine merges all splits with log-sum-exp
// weights, rotates the block part back and adds the tail part.
//
// Grid: (S * Hkv, nsplit + 1); split nsplit is the tail.  The query heads of
// one kv head (GQA group) share every code load.  The last CTA of a
// (sequence, kv head) to finish, found with an atomic ticket, combines.  No
// CTA ever waits for another.
#include <math.h>

#include "kvarn_common.cuh"
#include "kvarn_internal.h"

namespace kvarn {

constexpr int kDecThreads = 128;

template <int D, int GRP>
struct DecSmem {
    unsigned char krec[Record<D>::kBytes];
    unsigned char vrec[Record<D>::kBytes];
    float qrot[GRP][D];          // rotated (blocks) or plain (tail) query, pre-scaled
    float qp[GRP][D];            // q' for the current block
    float Qg[GRP][D / kGroup];
    float pw[kBlockTokens][D / kGroup][GRP];  // p_t r_t s_{t,g} per head
    float pr[kBlockTokens][GRP];              // p_t r_t per head
    float bias[GRP][D / kGroup];
    float red[kDecThreads / 32][GRP];
    float mnew[GRP], alpha[GRP], lsum[GRP];
    int last;
};

__device__ __forceinline__ float code_f(uint32_t word, int i)
{
    // (word >> 2i) & 3 as an exact float: OR the code into the mantissa of 2^23
    return __uint_as_float(0x4B000000u | ((word >> (2 * i)) & 3u)) - 8388608.f;
}

// In-place normalised Walsh-Hadamard transform of nvec vectors of length D
// in shared memory, Hadamard block hb (0 = none).  All threads call it.
__device__ void smem_fwht(float *x, int nvec, int D, int hb)
{
    if (hb == 0) return;
    for (int h = 1; h < hb; h <<= 1) {
        for (int idx = threadIdx.x; idx < nvec * D / 2; idx += blockDim.x) {
            const int v = idx / (D / 2), p = idx % (D / 2);
            // p-th pair of this stage: index with bit h cleared
            const int lo = (p / h) * 2 * h + (p % h);
            float *row = x + v * D;
            const float a = row[lo], b = row[lo + h];
            row[lo] = a + b;
            row[lo + h] = a - b;
        }
        __syncthreads();
    }
    const float nrm = rsqrtf((float)hb);
    for (int idx = threadIdx.x; idx < nvec * D; idx += blockDim.x) x[idx] *= nrm;
    __syncthreads();
}

template <int GRP>
__device__ __forceinline__ void block_reduce(float (&v)[GRP], float (*red)[GRP], bool is_max)
{
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
#pragma unroll
    for (int h = 0; h < GRP; ++h) {
        float x = v[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float y = __shfl_xor_sync(0xffffffffu, x, o);
            x = is_max ? fmaxf(x, y) : x + y;
        }
        if (l == 0) red[w][h] = x;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < GRP; ++h) {
        float x = red[0][h];
#pragma unroll
        for (int ww = 1; ww < kDecThreads / 32; ++ww) x = is_max ? fmaxf(x, red[ww][h]) : x + red[ww][h];
        v[h] = x;
    }
    __syncthreads();
}

template <int D, int GRP, typename Tin>
__global__ void __launch_bounds__(kDecThreads)
decode_kernel(DecodeArgs a, int hb)
{
    using R = Record<D>;
    constexpr int NG = D / kGroup;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    DecSmem<D, GRP> &sm = *reinterpret_cast<DecSmem<D, GRP> *>(smem_raw);
    const int tid = threadIdx.x;
    const int sh = blockIdx.x, split = blockIdx.y;
    const int s = sh / a.num_kv_heads;
    const bool is_tail = split == a.nsplit;

    int n = a.n_tokens[s];
    if (n > a.max_tokens) {
        if (tid == 0 && split == 0) status_or(a.status, KVARN_STATUS_LENGTH);
        n = a.max_tokens;
    }
    const int nblk = n / kBlockTokens;
    const int ntail = n - nblk * kBlockTokens;

    // query of the GQA group, times softmax scale * log2(e)
    const Tin *q = static_cast<const Tin *>(a.q) + ((size_t)sh * GRP) * D;
    for (int idx = tid; idx < GRP * D; idx += kDecThreads)
        (&sm.qrot[0][0])[idx] = In<Tin>::load1(q + idx) * a.scale_log2;
    __syncthreads();
    if (!is_tail) smem_fwht(&sm.qrot[0][0], GRP, D, hb);

    float m_run[GRP], l_run[GRP], acc[GRP];
#pragma unroll
    for (int h = 0; h < GRP; ++h) { m_run[h] = -INFINITY; l_run[h] = 0.f; acc[h] = 0.f; }

    if (!is_tail) {
        const int b0 = split * a.blocks_per_split;
        const int b1 = min(b0 + a.blocks_per_split, nblk);
        const unsigned char *kbase = static_cast<const unsigned char *>(a.k_records) + (size_t)sh * a.max_blocks * R::kBytes;
        const unsigned char *vbase = static_cast<const unsigned char *>(a.v_records) + (size_t)sh * a.max_blocks * R::kBytes;
        for (int b = b0; b < b1; ++b) {
            // -- stage both records in shared memory (coalesced 16-byte loads)
            const uint4 *ks = reinterpret_cast<const uint4 *>(kbase + (size_t)b * R::kBytes);
            const uint4 *vs = reinterpret_cast<const uint4 *>(vbase + (size_t)b * R::kBytes);
            for (int i = tid; i < R::kBytes / 16; i += kDecThreads) {
                reinterpret_cast<uint4 *>(sm.krec)[i] = __ldcs(ks + i);
                reinterpret_cast<uint4 *>(sm.vrec)[i] = __ldcs(vs + i);
            }
            __syncthreads();
            // -- q' = q_rot * c^K and its group sums
            const __half *cK = reinterpret_cast<const __half *>(sm.krec + R::kCOff);
            for (int idx = tid; idx < GRP * D; idx += kDecThreads) {
                const int d = idx % D;
                (&sm.qp[0][0])[idx] = (&sm.qrot[0][0])[idx] * __half2float(cK[d]);
            }
            __syncthreads();
            if (tid < GRP * NG) {
                const int h = tid / NG, g = tid % NG;
                float t = 0.f;
#pragma unroll 8
                for (int i = 0; i < kGroup; ++i) t += sm.qp[h][g * kGroup + i];
                sm.Qg[h][g] = t;
            }
            __syncthreads();
            // -- scores, one token per thread
            const int t = tid;
            float sc[GRP];
            {
                const float rK = __half2float(reinterpret_cast<const __half *>(sm.krec + R::kROff)[t]);
#pragma unroll
                for (int h = 0; h < GRP; ++h) sc[h] = 0.f;
#pragma unroll
                for (int g = 0; g < NG; ++g) {
                    const __half2 gp = reinterpret_cast<const __half2 *>(sm.krec + R::kGpOff)[t * NG + g];
                    const float sK = __low2float(gp), mK = __high2float(gp);
                    const uint2 cw = *reinterpret_cast<const uint2 *>(sm.krec + t * (D / 4) + 8 * g);
                    float dot[GRP];
#pragma unroll
                    for (int h = 0; h < GRP; ++h) dot[h] = 0.f;
#pragma unroll
                    for (int i = 0; i < kGroup; ++i) {
                        const float c = code_f(i < 16 ? cw.x : cw.y, i & 15);
#pragma unroll
                        for (int h = 0; h < GRP; ++h) dot[h] = fmaf(sm.qp[h][g * kGroup + i], c, dot[h]);
                    }
#pragma unroll
                    for (int h = 0; h < GRP; ++h) sc[h] += fmaf(sK, dot[h], mK * sm.Qg[h][g]);
                }
#pragma unroll
                for (int h = 0; h < GRP; ++h) sc[h] *= rK;
            }
            // -- online softmax over this block
            float bm[GRP];
#pragma unroll
            for (int h = 0; h < GRP; ++h) bm[h] = sc[h];
            block_reduce<GRP>(bm, sm.red, true);
            float p[GRP], ps[GRP];
#pragma unroll
            for (int h = 0; h < GRP; ++h) {
                const float mn = fmaxf(m_run[h], bm[h]);
                p[h] = exp2f(sc[h] - mn);
                ps[h] = p[h];
            }
            block_reduce<GRP>(ps, sm.red, false);
            {
                const float rV = __half2float(reinterpret_cast<const __half *>(sm.vrec + R::kROff)[t]);
#pragma unroll
                for (int h = 0; h < GRP; ++h) sm.pr[t][h] = p[h] * rV;
#pragma unroll
                for (int g = 0; g < NG; ++g) {
                    const __half2 gp = reinterpret_cast<const __half2 *>(sm.vrec + R::kGpOff)[t * NG + g];
                    const float sV = __low2float(gp);
#pragma unroll
                    for (int h = 0; h < GRP; ++h) sm.pw[t][g][h] = p[h] * rV * sV;
                }
            }
#pragma unroll
            for (int h = 0; h < GRP; ++h) {
                const float mn = fmaxf(m_run[h], bm[h]);
                const float al = exp2f(m_run[h] - mn);
                l_run[h] = l_run[h] * al + ps[h];
                m_run[h] = mn;
                if (tid == 0) sm.alpha[h] = al;
            }
            __syncthreads();
            if (tid < GRP * NG) {  // bias_{h,g} = sum_t p_t r_t m^V_{t,g}
                const int h = tid / NG, g = tid % NG;
                float bsum = 0.f;
                for (int tt = 0; tt < kBlockTokens; ++tt) {
                    const __half2 gp = reinterpret_cast<const __half2 *>(sm.vrec + R::kGpOff)[tt * NG + g];
                    bsum = fmaf(sm.pr[tt][h], __high2float(gp), bsum);
                }
                sm.bias[h][g] = bsum;
            }
            __syncthreads();
            // -- P V, one channel per thread
            if (tid < D) {
                const int d = tid, g = d / kGroup;
                const float cV = __half2float(reinterpret_cast<const __half *>(sm.vrec + R::kCOff)[d]);
                float pv[GRP];
#pragma unroll
                for (int h = 0; h < GRP; ++h) pv[h] = sm.bias[h][g];
#pragma unroll 4
                for (int tt = 0; tt < kBlockTokens; ++tt) {
                    const uint32_t byte = sm.vrec[tt * (D / 4) + d / 4];
                    const float c = code_f(byte, d & 3);
#pragma unroll
                    for (int h = 0; h < GRP; ++h) pv[h] = fmaf(sm.pw[tt][g][h], c, pv[h]);
                }
#pragma unroll
                for (int h = 0; h < GRP; ++h) acc[h] = fmaf(acc[h], sm.alpha[h], cV * pv[h]);
            }
            __syncthreads();
        }
    } else if (ntail > 0) {
        // -- residual tail: unrotated query against the stored tokens
        const Tin *kt = static_cast<const Tin *>(a.k_tail) + (size_t)sh * kBlockTokens * D;
        const Tin *vt = static_cast<const Tin *>(a.v_tail) + (size_t)sh * kBlockTokens * D;
        const int t = tid;
        float sc[GRP];
#pragma unroll
        for (int h = 0; h < GRP; ++h) sc[h] = -INFINITY;
        if (t < ntail) {
#pragma unroll
            for (int h = 0; h < GRP; ++h) sc[h] = 0.f;
            for (int d = 0; d < D; ++d) {
                const float kv = In<Tin>::load1(kt + (size_t)t * D + d);
#pragma unroll
                for (int h = 0; h < GRP; ++h) sc[h] = fmaf(sm.qrot[h][d], kv, sc[h]);
            }
        }
        float bm[GRP];
#pragma unroll
        for (int h = 0; h < GRP; ++h) bm[h] = sc[h];
        block_reduce<GRP>(bm, sm.red, true);
        float ps[GRP];
#pragma unroll
        for (int h = 0; h < GRP; ++h) {
            const float p = t < ntail ? exp2f(sc[h] - bm[h]) : 0.f;
            sm.pr[t][h] = p;
            ps[h] = p;
        }
        block_reduce<GRP>(ps, sm.red, false);
#pragma unroll
        for (int h = 0; h < GRP; ++h) { m_run[h] = bm[h]; l_run[h] = ps[h]; }
        if (tid < D) {
            for (int tt = 0; tt < ntail; ++tt) {
                const float vv = In<Tin>::load1(vt + (size_t)tt * D + tid);
#pragma unroll
                for (int h = 0; h < GRP; ++h) acc[h] = fmaf(sm.pr[tt][h], vv, acc[h]);
            }
        }
    }

    // ---- write this split's partial (m, l, o) per head -------------------
    float *part = a.partials + ((size_t)sh * (a.nsplit + 1) + split) * GRP * (D + 2);
#pragma unroll
    for (int h = 0; h < GRP; ++h) {
        if (tid < D) part[h * (D + 2) + 2 + tid] = acc[h];
        if (tid == 0) { part[h * (D + 2)] = m_run[h]; part[h * (D + 2) + 1] = l_run[h]; }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const unsigned prev = atomicAdd(a.tickets + sh, 1u);
        sm.last = prev == (unsigned)a.nsplit;
        if (sm.last) a.tickets[sh] = 0u;  // every CTA of this (s, kv head) has arrived
    }
    __syncthreads();
    if (!sm.last) return;
    __threadfence();

    // ---- combine: log-sum-exp over splits, un-rotate, add the tail --------
    const float *pbase = a.partials + (size_t)sh * (a.nsplit + 1) * GRP * (D + 2);
    float *obuf = &sm.qp[0][0];   // [GRP][D] rotated part
    float *otail = &sm.pw[0][0][0];  // [GRP][D] tail part (fits: T*NG*GRP >= GRP*D)
    for (int idx = tid; idx < GRP * D; idx += kDecThreads) {
        const int h = idx / D, d = idx % D;
        float M = -INFINITY;
        for (int i = 0; i <= a.nsplit; ++i) M = fmaxf(M, __ldcg(pbase + ((size_t)i * GRP + h) * (D + 2)));
        float L = 0.f, orot = 0.f, otl = 0.f;
        if (M > -INFINITY) {
            for (int i = 0; i <= a.nsplit; ++i) {
                const float *pp = pbase + ((size_t)i * GRP + h) * (D + 2);
                const float wgt = exp2f(__ldcg(pp) - M);
                L = fmaf(__ldcg(pp + 1), wgt, L);
                const float o = __ldcg(pp + 2 + d) * wgt;
                if (i < a.nsplit) orot += o; else otl += o;
            }
        }
        const float inv = L > 0.f ? 1.f / L : 0.f;
        obuf[idx] = orot * inv;
        otail[idx] = otl * inv;
    }
    __syncthreads();
    smem_fwht(obuf, GRP, D, hb);
    float *out = a.out + (size_t)sh * GRP * D;
    for (int idx = tid; idx < GRP * D; idx += kDecThreads) out[idx] = obuf[idx] + otail[idx];
}

template <int D, int GRP, typename Tin>
static cudaError_t launch_dec(const DecodeArgs &a, int hb, int S, int Hkv, cudaStream_t st)
{
    const size_t smem = sizeof(DecSmem<D, GRP>);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, GRP, Tin>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    dim3 grid((unsigned)(S * Hkv), (unsigned)(a.nsplit + 1));
    decode_kernel<D, GRP, Tin><<<grid, kDecThreads, smem, st>>>(a, hb);
    return cudaGetLastError();
}

template <int D, int GRP>
static cudaError_t dispatch_dtype(int dtype, const DecodeArgs &a, int hb, int S, int Hkv, cudaStream_t st)
{
    return dtype == KVARN_BF16 ? launch_dec<D, GRP, __nv_bfloat16>(a, hb, S, Hkv, st)
                               : launch_dec<D, GRP, float>(a, hb, S, Hkv, st);
}

template <int D>
static cudaError_t dispatch_grp(int dtype, const DecodeArgs &a, int hb, int S, int Hkv, cudaStream_t st)
{
    switch (a.grp) {
    case 1: return dispatch_dtype<D, 1>(dtype, a, hb, S, Hkv, st);
    case 2: return dispatch_dtype<D, 2>(dtype, a, hb, S, Hkv, st);
    case 4: return dispatch_dtype<D, 4>(dtype, a, hb, S, Hkv, st);
    case 8: return dispatch_dtype<D, 8>(dtype, a, hb, S, Hkv, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t run_decode(const kvarn_config &c, const DecodeArgs &a, cudaStream_t st)
{
    switch (c.head_dim) {
    case 64: return dispatch_grp<64>(c.dtype, a, c.hadamard, c.num_seqs, c.num_kv_heads, st);
    case 96: return dispatch_grp<96>(c.dtype, a, c.hadamard, c.num_seqs, c.num_kv_heads, st);
    case 128: return dispatch_grp<128>(c.dtype, a, c.hadamard, c.num_seqs, c.num_kv_heads, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace kvarn
