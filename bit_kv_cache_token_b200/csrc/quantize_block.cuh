// quantize_block.cuh -- one 128-token block of K or V -> packed 2-bit record.
//
// KVarN quantiser (paper "KVarN: Variance-Normalized KV-Cache Quantization
// Mitigates Error Accumulation in Reasoning Tasks"; rndamp.com article,
// "How It Works" items 1-2; abstract):
//   1. rotate every token along the channels with a Hadamard transform,
//      computed as a fast Walsh-Hadamard transform (O(N log N));
//   2. dual-axis variance normalisation: starting from c = 1, each sweep sets
//      r_t = std_d(X/c) for every token, then c_d = std_t(X/r) for every channel
//      (population std), then divides c by g, the geometric mean of the channel
//      scales, and multiplies r by g (only r_t c_d enters Y, and the split
//      between the two is otherwise free to drift out of binary16); a row or
//      column with zero variance takes scale 1 and stays out of the gauge;
//   3. Y = X / (r c); per token and group of 32 channels: m = min Y,
//      s = (max Y - m)/3, code = rint((Y - m)/s) in 0..3 (s = 0 -> code 0);
//      a token whose largest |Y| reaches 2^14 moves a power of two from its
//      (s, m) into r_t (token gauge, exact);
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
    float part[2][W][kBlockTokens];            // per-token partial row sums: [0] of z, [1] of (z - mean)^2
    float ubuf[D];                             // 1 / c broadcast
    float kbuf[D];                             // column shifts z[0][d]
    float2 gpart[W];                           // per-warp (sum of log2 c, count) of nonzero-variance channels
    float ymax[W][kBlockTokens];               // per-(group, token) largest |Y| (token gauge)
};

// A variance at most this fraction of the mean square counts as zero.  In
// fp32, values that are all equal leave a residual of order 2^-48 of their
// mean square through the fused shifts and sums; spreads of real data (bf16
// or fp32 inputs, rotated) sit far above 2^-40.
constexpr float kZeroVarRel = 9.094947e-13f;  // 2^-40

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
// aligned, Record<D>::kBytes); TENSOR 0 = K code order, 1 = V code order.
// dbg: NULL or fp32 [T + D + 2*T*D/32] unrounded r, c, s, m (as stored, token
// gauge included).  All D threads of the CTA must call this.
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
    // Rows: two passes (mean, then mean square deviation) over the D channels,
    // whose partial sums cross the warps through shared memory.  Columns: one
    // pass over the 128 tokens on values shifted by token 0's (lane 0's) z,
    // whose partials cross the lanes through a shared-memory transpose.  Then
    // the gauge: g = geometric mean of the nonzero-variance channel scales,
    // c <- c / g (1 for a zero-variance column), r <- r g at the end.
    float2 u[16];  // 1 / c for this thread's 32 channels
#pragma unroll
    for (int k = 0; k < 16; ++k) u[k] = f2(1.f, 1.f);
    float w[4] = {1.f, 1.f, 1.f, 1.f};    // 1 / r for this thread's 4 tokens
    float rt[4] = {1.f, 1.f, 1.f, 1.f};   // r for this thread's 4 tokens (0 marks zero variance)
    float cd = 1.f;                       // c of channel 32j + l (lane-owned, gauged)
    float g = 1.f;                        // gauge factor of the last column step

    for (int sw = 0; sw < sweeps; ++sw) {
        // row step, pass 1: mean over the D channels of z = X u
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            float2 s1 = f2(0.f, 0.f), s1b = f2(0.f, 0.f);
#pragma unroll
            for (int k = 0; k < 16; k += 2) {
                s1 = __ffma2_rn(X[r][k], u[k], s1);
                s1b = __ffma2_rn(X[r][k + 1], u[k + 1], s1b);
            }
            s1 = __fadd2_rn(s1, s1b);
            sm.part[0][j][l + 32 * r] = s1.x + s1.y;
        }
        __syncthreads();
        float mean[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            float S1 = 0.f;
#pragma unroll
            for (int jj = 0; jj < W; ++jj) S1 += sm.part[0][jj][l + 32 * r];
            mean[r] = S1 * (1.f / D);
        }
        // row step, pass 2: mean square deviation from that mean
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const float2 nm = f2(-mean[r], -mean[r]);
            float2 s2 = f2(0.f, 0.f), s2b = f2(0.f, 0.f);
#pragma unroll
            for (int k = 0; k < 16; k += 2) {
                const float2 e = __ffma2_rn(X[r][k], u[k], nm);
                const float2 eb = __ffma2_rn(X[r][k + 1], u[k + 1], nm);
                s2 = __ffma2_rn(e, e, s2);
                s2b = __ffma2_rn(eb, eb, s2b);
            }
            s2 = __fadd2_rn(s2, s2b);
            sm.part[1][j][l + 32 * r] = s2.x + s2.y;
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            float S2 = 0.f;
#pragma unroll
            for (int jj = 0; jj < W; ++jj) S2 += sm.part[1][jj][l + 32 * r];
            const float var = S2 * (1.f / D);
            const bool nz = var > kZeroVarRel * fmaf(mean[r], mean[r], var);
            const float is = rsqrtf(var);
            w[r] = nz ? is : 1.f;         // 1 / r_t
            rt[r] = nz ? var * is : 0.f;  // r_t = sqrt(var); 0 marks a zero-variance row (scale 1)
        }
        // column step: c_d = std over the 128 tokens of z = X / r, on values
        // shifted by token 0's z (lane 0, r = 0) for precision
        if (l == 0) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float2 a = __fmul2_rn(X[0][2 * q], f2(w[0], w[0]));
                const float2 b = __fmul2_rn(X[0][2 * q + 1], f2(w[0], w[0]));
                reinterpret_cast<float4 *>(&sm.kbuf[32 * j])[q] = make_float4(a.x, a.y, b.x, b.y);
            }
        }
        __syncwarp();
#pragma unroll
        for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int k = 8 * half + kk;
                const float2 kv = reinterpret_cast<const float2 *>(&sm.kbuf[32 * j])[k];
                const float2 nk = f2(-kv.x, -kv.y);
                float2 c1 = f2(0.f, 0.f), c2 = f2(0.f, 0.f);
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const float2 e = __ffma2_rn(X[r][k], f2(w[r], w[r]), nk);
                    c1 = __fadd2_rn(c1, e);
                    c2 = __ffma2_rn(e, e, c2);
                }
                // chunk k of row l holds channels 2k, 2k+1 as (sum, sumsq) pairs
                sm.u.col[j][l][k ^ (l & 15)] = make_float4(c1.x, c2.x, c1.y, c2.y);
            }
        }
        __syncwarp();
        bool znz;  // this lane's channel has nonzero variance
        {
            // lane l sums column l (channel 32j + l) over the 32 rows
            float2 acc[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};
            const int k = l >> 1, hi = l & 1;
#pragma unroll
            for (int row = 0; row < 32; ++row) {
                const float2 *chunk = reinterpret_cast<const float2 *>(&sm.u.col[j][row][k ^ (row & 15)]);
                acc[row & 3] = __fadd2_rn(acc[row & 3], chunk[hi]);
            }
            const float2 tot = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
            const float me = tot.x * (1.f / kBlockTokens);  // mean of the shifted values
            const float var = fmaf(-me, me, tot.y * (1.f / kBlockTokens));
            const float mz = sm.kbuf[32 * j + l] + me;      // mean of z
            znz = var > kZeroVarRel * fmaf(mz, mz, fmaxf(var, 0.f));
            cd = znz ? sqrtf(var) : 1.f;
            float lg = znz ? log2f(cd) : 0.f;
            float cnt = znz ? 1.f : 0.f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                lg += __shfl_xor_sync(0xffffffffu, lg, o);
                cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
            }
            if (l == 0) sm.gpart[j] = f2(lg, cnt);
        }
        __syncthreads();  // every warp's gauge partial is in
        {
            float2 tot = f2(0.f, 0.f);
#pragma unroll
            for (int jj = 0; jj < W; ++jj) tot = __fadd2_rn(tot, sm.gpart[jj]);
            g = tot.y > 0.f ? exp2f(tot.x / tot.y) : 1.f;
            cd = znz ? cd / g : 1.f;
            sm.ubuf[32 * j + l] = 1.f / cd;
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 v = reinterpret_cast<const float4 *>(&sm.ubuf[32 * j])[q];
                u[2 * q] = f2(v.x, v.y);
                u[2 * q + 1] = f2(v.z, v.w);
            }
        }
    }
    // last gauge on the token scales: r <- r g (a zero-variance row keeps 1)
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        rt[r] = rt[r] > 0.f ? rt[r] * g : 1.f;
        w[r] = 1.f / rt[r];
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
    float gs[4], gm[4];  // this group's s and m in Y units, before the token gauge
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
        // level = (Z - min) * 3 / range: Z = Y * r_t, so this equals (Y - m) / s.
        // Z - min is formed first: it lies in [0, range] whatever the offset of
        // the group, so the level stays in [0, 3] and cannot spill into the
        // neighbouring 2-bit fields of the packed words.
        const float kq = range > 0.f ? 3.f / range : 0.f;
        const float2 kq2 = f2(kq, kq);
        const float2 mn2 = f2(mn, mn);
        // 12582912 = 1.5 * 2^23: adding it rounds the level to an integer
        // (ties to even) and leaves that integer in the low mantissa bits.
        const float2 magic = f2(12582912.f, 12582912.f);
        uint32_t kacc[4] = {0u, 0u, 0u, 0u};  // K: byte (tig, half) at bits 8*half of kacc[tig]
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float2 lev = __ffma2_rn(sub2(z[k], mn2), kq2, magic);
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
        gs[r] = range * w[r] * (1.f / 3.f);
        gm[r] = mn * w[r];
        sm.ymax[j][t] = fmaxf(fabsf(mn), fabsf(mx)) * w[r];  // this group's largest |Y|
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
    __syncthreads();  // every group's largest |Y| is in
    // Token gauge: r_t times the token's (s, m) is what dequantises; when the
    // token's largest |Y| reaches 2^14, the power of two 2^k with k =
    // floor(log2 max|Y|) - 13 moves from (s, m) into r_t (exact: codes and
    // products unchanged), which keeps s and m inside binary16.
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int t = l + 32 * r;
        float ym = 0.f;
#pragma unroll
        for (int jj = 0; jj < W; ++jj) ym = fmaxf(ym, sm.ymax[jj][t]);
        float tg = 1.f, itg = 1.f;
        if (ym >= 16384.f) {
            const int e = (int)((__float_as_uint(ym) >> 23) & 0xFFu) - 127;  // floor(log2 ym)
            tg = __uint_as_float((uint32_t)(e - 13 + 127) << 23);
            itg = __uint_as_float((uint32_t)(127 - (e - 13)) << 23);
        }
        const float s = gs[r] * itg, m = gm[r] * itg;
        const __half hs = __float2half_rn(s), hm = __float2half_rn(m);
        if (__hisinf(hs) || __hisnan(hs) || __hisinf(hm) || __hisnan(hm))
            status_or(status, KVARN_STATUS_NONFINITE);
        reinterpret_cast<__half *>(rec + R::kSOff)[t * (D / 32) + j] = hs;
        reinterpret_cast<__half *>(rec + R::kMOff)[t * (D / 32) + j] = hm;
        const float rr = rt[r] * tg;
        if (j == 0) {
            const __half hr = __float2half_rn(rr);
            if (__hisinf(hr) || __hisnan(hr)) status_or(status, KVARN_STATUS_NONFINITE);
            *reinterpret_cast<__half *>(rec + R::kROff + 2 * t) = hr;
        }
        if (dbg) {
            if (j == 0) dbg[t] = rr;
            dbg[kBlockTokens + D + t * (D / 32) + j] = s;
            dbg[kBlockTokens + D + kBlockTokens * (D / 32) + t * (D / 32) + j] = m;
        }
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
