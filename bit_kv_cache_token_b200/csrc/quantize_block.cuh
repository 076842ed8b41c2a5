// quantize_block.cuh -- one 128-token block of K or V -> packed 2-bit record.
//
// KVarN quantiser (paper "KVarN: Variance-Normalized KV-Cache Quantization
// Mitigates Error Accumulation in Reasoning Tasks"; rndamp.com article,
// "How It Works" items 1-2; abstract):
//   1. rotate every token along the channels with a Hadamard transform,
//      computed as a fast Walsh-Hadamard transform (O(N log N));
//   2. dual-axis variance normalisation: starting from c = 1, each sweep sets
//      r_t = std_d(X/c) for every token, then c_d = std_t(X/r) for every channel
//      (population std; a zero variance gives scale 1);
//   3. Y = X / (r c); per token and group of 32 channels: m = min Y,
//      s = (max Y - m)/3, code = rint((Y - m)/s) in 0..3 (s = 0 -> code 0);
//   4. store codes, binary16 (s, m), r and c in one block record.
//
// Thread layout (D threads = D/32 warps; warp j owns channel group j):
// lane l holds tokens l, l+32, l+64, l+96 and channels 32j .. 32j+31 of each,
// as 16 float2 per token.  So a quantisation group sits entirely in one
// thread, the 32-point Hadamard butterflies are in registers, a larger
// Hadamard block adds one exchange across warps through shared memory, the
// per-token (row) sums cross warps through shared memory and the
// per-channel (column) sums cross the 32 lanes through a swizzled
// shared-memory transpose.  Arithmetic is fp32; packed f32x2 operations
// (sm_100) halve the issue count of the elementwise work.
#pragma once

#include "kvarn_common.cuh"

namespace kvarn {

template <int D>
struct QuantSmem {
    static constexpr int W = D / 32;
    union {
        float4 xch[W][2][8][32];               // Hadamard exchange [warp][token pair][chunk][lane]
        float4 col[W][32][16];                 // column-sum transpose [warp][lane][chunk]
        unsigned char rec[Record<D>::kBytes];  // record staging
    } u;
    float2 part[2][W][kBlockTokens];           // per-token partial (sum, sum of squares)
    float ubuf[D];                             // 1 / c broadcast
};

__device__ __forceinline__ float2 sub2(float2 a, float2 b) { return __ffma2_rn(b, f2(-1.f, -1.f), a); }

__device__ __forceinline__ float min3(float a, float b, float c)
{
    float r;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ float max3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// In-register 32-point Walsh-Hadamard butterflies (unnormalised) on one token.
__device__ __forceinline__ void fwht32_regs(float2 (&x)[16])
{
#pragma unroll
    for (int k = 0; k < 16; ++k) {  // channel bit 0: inside each pair
        const float a = x[k].x, b = x[k].y;
        x[k] = f2(a + b, a - b);
    }
#pragma unroll
    for (int h = 1; h < 16; h <<= 1) {  // channel bits 1..4: across pairs
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            if (k & h) continue;
            const float2 a = x[k], b = x[k + h];
            x[k] = __fadd2_rn(a, b);
            x[k + h] = sub2(a, b);
        }
    }
}

// Load a block of 128 rows x D channels (row stride D elements) into the
// thread layout described above.  `rows` may be a device or tail buffer.
// COHERENT: the rows may have been written by this kernel (the append path's
// tail), so they are read through L2 rather than the read-only path.
template <int D, typename Tin, bool COHERENT = false>
__device__ __forceinline__ void load_block(const Tin *rows, float2 (&X)[4][16])
{
    const int j = threadIdx.x >> 5, l = threadIdx.x & 31;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const Tin *p = rows + (size_t)(l + 32 * r) * D + 32 * j;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float v[8];
            In<Tin>::template load8<COHERENT>(p + 8 * q, v);
#pragma unroll
            for (int e = 0; e < 4; ++e) X[r][4 * q + e] = f2(v[2 * e], v[2 * e + 1]);
        }
    }
}

// Step 1 of the quantiser on the block held in X: the Hadamard rotation
// along the channels (blockdiag(H_HB) / sqrt(HB); HB = 0 leaves X as it is).
// All D threads of the CTA must call this.
template <int D, int HB>
__device__ __forceinline__ void rotate_block(float2 (&X)[4][16], QuantSmem<D> &sm)
{
    const int j = threadIdx.x >> 5, l = threadIdx.x & 31;
    (void)j; (void)l;
    if constexpr (HB >= 32) {
#pragma unroll
        for (int r = 0; r < 4; ++r) fwht32_regs(X[r]);
        if constexpr (HB > 32) {
            // the remaining butterflies pair warps j and j ^ m (channel bit 5 + log2 m),
            // one stage per bit, two tokens at a time through shared memory
#pragma unroll
            for (int m = 1; m < HB / 32; m <<= 1) {
                const float sg = (j & m) ? -1.f : 1.f;  // upper half of the pair: partner - own
#pragma unroll
                for (int rp = 0; rp < 4; rp += 2) {
#pragma unroll
                    for (int r = 0; r < 2; ++r)
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            sm.u.xch[j][r][q][l] = make_float4(X[rp + r][2 * q].x, X[rp + r][2 * q].y,
                                                               X[rp + r][2 * q + 1].x, X[rp + r][2 * q + 1].y);
                    __syncthreads();
#pragma unroll
                    for (int r = 0; r < 2; ++r)
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float4 p = sm.u.xch[j ^ m][r][q][l];
                            X[rp + r][2 * q] = __ffma2_rn(f2(sg, sg), X[rp + r][2 * q], f2(p.x, p.y));
                            X[rp + r][2 * q + 1] = __ffma2_rn(f2(sg, sg), X[rp + r][2 * q + 1], f2(p.z, p.w));
                        }
                    __syncthreads();
                }
            }
        }
        const float nrm = HB == 32 ? 0.17677669529663688f : HB == 64 ? 0.125f : 0.08838834764831845f;  // 1/sqrt(HB)
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int k = 0; k < 16; ++k) X[r][k] = __fmul2_rn(X[r][k], f2(nrm, nrm));
    }

}

// Quantise the block held in X (destroyed) into rec_out (global, 16-byte
// aligned, Record<D>::kBytes); TENSOR 0 = K code order, 1 = V code order.  dbg: NULL or fp32 [T + D + 2*T*D/32] unrounded
// r, c, s, m.  All D threads of the CTA must call this.
template <int D, int HB, int TENSOR>
__device__ void quantize_block(float2 (&X)[4][16], QuantSmem<D> &sm, int sweeps,
                               unsigned char *__restrict__ rec_out, float *__restrict__ dbg,
                               int32_t *status)
{
    constexpr int W = D / 32;
    using R = Record<D>;
    const int j = threadIdx.x >> 5, l = threadIdx.x & 31;

    // ---- 1. Hadamard rotation along the channels --------------------------
    rotate_block<D, HB>(X, sm);

    // ---- 2. dual-axis variance normalisation ------------------------------
    float2 u[16];  // 1 / c for this thread's 32 channels
#pragma unroll
    for (int k = 0; k < 16; ++k) u[k] = f2(1.f, 1.f);
    float w[4] = {1.f, 1.f, 1.f, 1.f};    // 1 / r for this thread's 4 tokens
    float rt[4] = {1.f, 1.f, 1.f, 1.f};   // r for this thread's 4 tokens
    float cd = 1.f;                       // c of channel 32j + l (lane-owned)

    for (int sw = 0; sw < sweeps; ++sw) {
        // row step: r_t = std over the D channels of X / c
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            float2 s1 = f2(0.f, 0.f), s2 = f2(0.f, 0.f);
            if (sw == 0) {  // c = 1: X / c is X
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    s1 = __fadd2_rn(s1, X[r][k]);
                    s2 = __ffma2_rn(X[r][k], X[r][k], s2);
                }
            } else {
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const float2 z = __fmul2_rn(X[r][k], u[k]);
                    s1 = __fadd2_rn(s1, z);
                    s2 = __ffma2_rn(z, z, s2);
                }
            }
            sm.part[sw & 1][j][l + 32 * r] = f2(s1.x + s1.y, s2.x + s2.y);
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            float S1 = 0.f, S2 = 0.f;
#pragma unroll
            for (int jj = 0; jj < W; ++jj) {
                const float2 p = sm.part[sw & 1][jj][l + 32 * r];
                S1 += p.x;
                S2 += p.y;
            }
            const float mean = S1 * (1.f / D);
            const float var = fmaf(-mean, mean, S2 * (1.f / D));
            w[r] = var > 0.f ? rsqrtf(var) : 1.f;  // 1 / r_t
            rt[r] = var > 0.f ? var * w[r] : 1.f;  // r_t = sqrt(var)
        }
        // column step: c_d = std over the 128 tokens of X / r
#pragma unroll
        for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int k = 8 * half + kk;
                float2 c1 = f2(0.f, 0.f), c2 = f2(0.f, 0.f);
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const float2 z = __fmul2_rn(X[r][k], f2(w[r], w[r]));
                    c1 = __fadd2_rn(c1, z);
                    c2 = __ffma2_rn(z, z, c2);
                }
                // chunk k of row l holds channels 2k, 2k+1 as (sum, sumsq) pairs
                sm.u.col[j][l][k ^ (l & 15)] = make_float4(c1.x, c2.x, c1.y, c2.y);
            }
        }
        __syncwarp();
        {
            // lane l sums column l (channel 32j + l) over the 32 rows
            float2 acc = f2(0.f, 0.f);
            const int k = l >> 1, hi = l & 1;
#pragma unroll
            for (int row = 0; row < 32; ++row) {
                const float2 *chunk = reinterpret_cast<const float2 *>(&sm.u.col[j][row][k ^ (row & 15)]);
                acc = __fadd2_rn(acc, chunk[hi]);
            }
            const float mean = acc.x * (1.f / kBlockTokens);
            const float var = fmaf(-mean, mean, acc.y * (1.f / kBlockTokens));
            const float ud = var > 0.f ? rsqrtf(var) : 1.f;  // 1 / c_d
            cd = var > 0.f ? var * ud : 1.f;
            __syncwarp();
            sm.ubuf[32 * j + l] = ud;
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 v = reinterpret_cast<const float4 *>(&sm.ubuf[32 * j])[q];
                u[2 * q] = f2(v.x, v.y);
                u[2 * q + 1] = f2(v.z, v.w);
            }
        }
    }
    __syncthreads();  // every warp is done with the shared transposes

    // ---- 3. 2-bit asymmetric round-to-nearest per (token, group) ----------
    // Codes go to the record in the fragment order the decode kernel reads
    // (see kvarn.h).  K: the 4 codes of channels 8x + 2*tig + half (x = 0..3)
    // of one token fill one byte.  V: the codes of one channel for this
    // thread's 4 tokens (l + 32r) fill one byte.
    unsigned char *rec = sm.u.rec;
    // Codes are read from the low mantissa bits of lev = 1.5*2^23 + code, whose
    // bit pattern is 0x4B400000 + code: multiply-adding the raw patterns with the
    // code weights and subtracting the pattern's share once packs them.
    uint32_t vacc[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};  // V: channel i in byte i%4 of vacc[i/4]
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int t = l + 32 * r;
        float2 z[16];
        float mn = INFINITY, mx = -INFINITY;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            z[k] = __fmul2_rn(X[r][k], u[k]);
            mn = min3(mn, z[k].x, z[k].y);
            mx = max3(mx, z[k].x, z[k].y);
        }
        const float range = mx - mn;
        // level = (Z - min) * 3 / range: Z = Y * r_t, so this equals (Y - m) / s
        const float kq = range > 0.f ? 3.f / range : 0.f;
        const float2 kq2 = f2(kq, kq);
        const float2 nmk = f2(-mn * kq, -mn * kq);
        // 12582912 = 1.5 * 2^23: adding it rounds the level to an integer
        // (ties to even) and leaves that integer in the low mantissa bits.
        const float2 magic = f2(12582912.f, 12582912.f);
        uint32_t kacc[4] = {0u, 0u, 0u, 0u};  // K: byte (tig, half) at bits 8*half of kacc[tig]
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float2 lev = __fadd2_rn(__ffma2_rn(z[k], kq2, nmk), magic);
            const uint32_t b0 = __float_as_uint(lev.x), b1 = __float_as_uint(lev.y);
            // local channels 2k (b0) and 2k+1 (b1): x = k/4, tig = k%4
            if constexpr (TENSOR == 0) {
                kacc[k & 3] += b0 * (1u << (2 * (k >> 2))) + b1 * (1u << (8 + 2 * (k >> 2)));
            } else {
                vacc[k >> 1] += b0 * (1u << (16 * (k & 1) + 2 * r)) + b1 * (1u << (16 * (k & 1) + 8 + 2 * r));
            }
        }
        if constexpr (TENSOR == 0) {
            // remove 0x4B400000 * (1 + 4 + 16 + 64) * (1 + 256) from each word
            constexpr uint32_t kBias = 0x4B400000u * 85u * 257u;
#pragma unroll
            for (int tig = 0; tig < 4; ++tig) {
                const uint32_t v = kacc[tig] - kBias;
                const int kch = 32 * j + 2 * tig;  // channel with x = 0, half = 0
                rec[k_code_bit<D>(t, kch) / 8] = (unsigned char)(v & 0xFFu);
                rec[k_code_bit<D>(t, kch + 1) / 8] = (unsigned char)((v >> 8) & 0xFFu);
            }
        }
        const float s = range * w[r] * (1.f / 3.f);
        const float m = mn * w[r];
        const __half hs = __float2half_rn(s), hm = __float2half_rn(m);
        if (__hisinf(hs) || __hisnan(hs) || __hisinf(hm) || __hisnan(hm))
            status_or(status, KVARN_STATUS_NONFINITE);
        reinterpret_cast<__half *>(rec + R::kSOff)[t * (D / 32) + j] = hs;
        reinterpret_cast<__half *>(rec + R::kMOff)[t * (D / 32) + j] = hm;
        if (j == 0) {
            const __half hr = __float2half_rn(rt[r]);
            if (__hisinf(hr) || __hisnan(hr)) status_or(status, KVARN_STATUS_NONFINITE);
            *reinterpret_cast<__half *>(rec + R::kROff + 2 * t) = hr;
        }
        if (dbg) {
            if (j == 0) dbg[t] = rt[r];
            dbg[kBlockTokens + D + t * (D / 32) + j] = s;
            dbg[kBlockTokens + D + kBlockTokens * (D / 32) + t * (D / 32) + j] = m;
        }
    }
    if constexpr (TENSOR == 1) {
        // each vacc word took 0x4B400000 * (1 + 4 + 16 + 64) * (1 + 256 + 65536 + 2^24)
        constexpr uint32_t kBias = 0x4B400000u * 85u * 16843009u;
#pragma unroll
        for (int q = 0; q < 8; ++q) vacc[q] -= kBias;
#pragma unroll
        for (int i = 0; i < 32; ++i)
            rec[v_code_bit(l, 32 * j + i) / 8] = (unsigned char)(vacc[i >> 2] >> (8 * (i & 3)));
    }
    {
        const __half hc = __float2half_rn(cd);
        if (__hisinf(hc) || __hisnan(hc)) status_or(status, KVARN_STATUS_NONFINITE);
        *reinterpret_cast<__half *>(rec + R::kCOff + 2 * (32 * j + l)) = hc;
        if (dbg) dbg[kBlockTokens + 32 * j + l] = cd;
    }
    if constexpr (R::kBytes > R::kRaw) {  // zero the padding
        if (threadIdx.x < (R::kBytes - R::kRaw) / 4) reinterpret_cast<uint32_t *>(rec + R::kRaw)[threadIdx.x] = 0u;
    }
    __syncthreads();
    // ---- 4. coalesced 16-byte copy of the record to global ---------------
    for (int i = threadIdx.x; i < R::kBytes / 16; i += D)
        reinterpret_cast<uint4 *>(rec_out)[i] = reinterpret_cast<const uint4 *>(rec)[i];
    __syncthreads();  // staging may be reused by the caller
}

}  // namespace kvarn
