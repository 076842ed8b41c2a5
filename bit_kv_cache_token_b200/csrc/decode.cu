// decode.cu -- decode attention (one or a few query tokens per sequence) over
// the packed 2-bit cache.
//
// KVarN decode (abstract: attention over the 2-bit cache in long-horizon
// decoding; rndamp.com article, "Numbers": the second scale is fused into the
// dequantisation kernel).  Keys are stored rotated, so the query is rotated
// once and scores are taken in the rotated basis, where q . k is unchanged.
// With k_rot[t][d] = r_t c_d (s_{t,g} code + m_{t,g}):
//   score_t = r_t * sum_g ( s_{t,g} * sum_{d in g} q'_d code_{t,d} + m_{t,g} Q_g ),
//   q'_d = q_rot,d * c^K_d * scale,  Q_g = sum_{d in g} q'_d;
// and with p_t the softmax weight,
//   o_rot,d = c^V_d * sum_t ( p_t r^V_t s^V_{t,g} code_{t,d} + p_t r^V_t m^V_{t,g} ).
// The residual tail (unrotated, input dtype) is attended with the unrotated
// query; the combine merges all partials with log-sum-exp weights, rotates
// the block part back and adds the tail part.
//
// B200 mapping.  The work of a launch is a list of items, unit by unit (a
// unit is one (sequence, kv head)): the unit's max_tokens / 128 blocks, then
// kTailSlots items for its residual tail, 32 tokens each.  Every warp of a persistent grid (one CTA
// per SM) takes an equal contiguous range of that list, so the load is even
// whatever the number of units and their lengths relative to the SM count.
// Where a range crosses into a new unit the warp starts a new online softmax.
// The records reach shared memory by cp.async.bulk (TMA), one buffer each
// for K and V guarded by mbarriers: the next K record is requested as soon
// as the scores are done, the next V record as soon as P V is done, so each
// copy overlaps half a block of this warp's work and the whole work of the
// SM's other warps.  Both contractions run on tensor cores (mma.sync
// m16n8k16, fp16 in, fp32 accumulate):
//   scores: A = K codes (16 tokens x 16 channels), B = q' (16 channels x 8
//           columns: a column per head and hi/lo fp16 part), one accumulator
//           per 32-channel group, scaled by s r in the epilogue;
//   P V:    A = p r s (rows: heads and hi/lo parts), B = V codes (k = 16
//           tokens, n = 8 channels); the probabilities move from the score
//           layout to these rows by shuffles.
// A 2-bit code becomes an exact fp16 operand with a shift and an AND: the
// record stores every code in a 32-bit word at bit 16*half + 2*pos (see
// kvarn.h), and masking a shifted copy of the word puts both codes of a pair
// on bits 8-9 or 6-7 of their halves, i.e. fp16 subnormals c * 2^-16 or
// c * 2^-18.  The factor 4 between the two is folded into the other operand
// (it depends only on the contracted index), the remaining 2^-16 into the
// scales.  When the GQA group has fewer than 8 heads, the spare P V rows
// carry copies of the heads working on other channel groups.  A tail slot is
// attended on CUDA cores and its output rotated, so that it merges like a
// block partial.  Several query tokens
// per sequence (MQ instantiations) are more rows on the same kv head, with a
// causal limit applied in the last block and the tail.
//
// Merging.  Every (warp, unit) segment writes one partial (m, l, o_rot per
// head); every tail slot writes one more.  A per-unit ticket
// counts the items whose partials are written; the warp that completes it
// merges the unit itself when few warps covered it, and otherwise marks the
// unit for its CTA, whose warps merge it together after they have all
// finished their ranges.  No warp ever waits for another CTA.
#include <math.h>

#include "kvarn_common.cuh"
#include "kvarn_internal.h"

namespace kvarn {

constexpr float kTwo16 = 65536.f;           // 2^16
constexpr float kTwoM16 = 1.f / 65536.f;    // 2^-16
// Longest wait for a staged record, in ns of the global timer (a record
// normally lands within microseconds).
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

template <int D, int GRP>
struct alignas(128) DecWarpSmem {
    unsigned char rec[2][Record<D>::kBytes];  // [K, V] of the current block
    float scr[4 * kBlockTokens + kBlockTokens + D];  // K: srK[128][4], rK, cK; V: rsV[NG][128], rV, cV
    float qbuf[GRP][D];
    unsigned long long mbar[2];               // K record, V record
};

// Channel groups a lane's P V rows cover (its copy's groups): the lane keeps
// the running output of those groups' n-tiles only.
template <int D, int GRP>
__host__ __device__ constexpr int dec_sets()
{
    return (D / kGroup + 8 / GRP - 1) / (8 / GRP);
}

// Warps per CTA: up to 12 (16 for one row per kv head, 8 for eight rows), as
// many as fit in 227 KB of shared memory.
template <int D, int GRP>
__host__ __device__ constexpr int dec_warps()
{
    // Registers are reserved for warps in groups of four: 9 to 12 warps per
    // SM all leave 168 registers a thread.  The 8-row instantiation needs
    // more than that (it spills over 200 bytes at 168), so it runs 8 warps
    // with up to 255 registers and no spills: 156 against 170 us for two
    // query tokens at 32705 cached tokens (Qwen3-4B shapes, batch 8).  One
    // row per kv head (MHA) needs fewer: where 16 warps fit in shared memory
    // (head_dim 64 and 96) it runs 16 with 128 registers, a few words spilled
    // at head_dim 96: 257 against 279 us per Phi-3-mini-shaped layer (batch
    // 16, 32 heads, 16384 tokens).
    constexpr int fit = (227 * 1024) / (int)sizeof(DecWarpSmem<D, GRP>);
    constexpr int cap = GRP == 8 ? 8 : (GRP == 1 && fit >= 16) ? 16 : 12;
    return fit < cap ? fit : cap;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// A pure register operation: not volatile, so that independent MMA chains
// may be interleaved by the compiler.
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// fp32 pair -> fp16 pairs (hi, lo) with x = hi + lo to about 2^-22 relative.
// (lo may be subnormal: the lo rows of an MMA only need about 11 bits.)
__device__ __forceinline__ void split_hilo(float x, float y, uint32_t &hi, uint32_t &lo)
{
    const __half2 h = __floats2half2_rn(x, y);
    const float2 hf = __half22float2(h);
    const float2 d = __ffma2_rn(hf, make_float2(-1.f, -1.f), make_float2(x, y));  // x - hi, exact, both at once
    const __half2 l = __floats2half2_rn(d.x, d.y);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    lo = *reinterpret_cast<const uint32_t *>(&l);
}

// hi rows (c0, c1) plus lo rows (c2, c3) of an accumulator
__device__ __forceinline__ float2 hilo_sum(const float (&c)[4]) { return __fadd2_rn(f2(c[0], c[1]), f2(c[2], c[3])); }

// Four binary16 values (8 bytes) -> fp32 times `mul`.
__device__ __forceinline__ float4 h4_to_f4(uint2 w, float mul)
{
    const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&w.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&w.y));
    return make_float4(a.x * mul, a.y * mul, b.x * mul, b.y * mul);
}

// Per-token scales of one record to fp32, one lane per 4 consecutive tokens:
// out_s[g][t] = s[t][g] * rmul(t) * smul and out_r[t] = r[t]; out_c[d] = c[d] * cmul.
// rmul(t) is r[t] * tmul when with_r, else 1; tmul is the same for the
// lane's 4 tokens.
template <int D, bool WITH_R>
__device__ __forceinline__ void convert_scales(const unsigned char *rec, float *out_s, float *out_r, float *out_c,
                                               float smul, float tmul, float cmul)
{
    using R = Record<D>;
    constexpr int NG = D / kGroup;
    const int lane = threadIdx.x & 31, t0 = 4 * lane;
    const float4 r4 = h4_to_f4(reinterpret_cast<const uint2 *>(rec + R::kROff)[lane], 1.f);
    *reinterpret_cast<float4 *>(out_r + t0) = r4;
    const float rr[4] = {r4.x * tmul, r4.y * tmul, r4.z * tmul, r4.w * tmul};
    // s of tokens t0..t0+3: 4*NG halves at half index t0*NG (8-byte aligned)
    const uint2 *sp = reinterpret_cast<const uint2 *>(rec + R::kSOff) + lane * NG;
    float sv[4 * NG];
#pragma unroll
    for (int i = 0; i < NG; ++i) {
        const float4 f = h4_to_f4(sp[i], smul);
        sv[4 * i] = f.x; sv[4 * i + 1] = f.y; sv[4 * i + 2] = f.z; sv[4 * i + 3] = f.w;
    }
#pragma unroll
    for (int g = 0; g < NG; ++g) {
        float4 o;
        o.x = sv[0 * NG + g] * (WITH_R ? rr[0] : 1.f);
        o.y = sv[1 * NG + g] * (WITH_R ? rr[1] : 1.f);
        o.z = sv[2 * NG + g] * (WITH_R ? rr[2] : 1.f);
        o.w = sv[3 * NG + g] * (WITH_R ? rr[3] : 1.f);
        *reinterpret_cast<float4 *>(out_s + g * kBlockTokens + t0) = o;
    }
    if (4 * lane < D) {  // c of channels 4 lane .. 4 lane + 3 (D <= 128)
        const uint2 cw = reinterpret_cast<const uint2 *>(rec + R::kCOff)[lane];
        *reinterpret_cast<float4 *>(out_c + 4 * lane) = h4_to_f4(cw, cmul);
    }
}

// The five shifted copies of a code word from which every position is one AND.
struct CodeWord {
    uint32_t l8, l4, w, r4, r8;
    __device__ __forceinline__ explicit CodeWord(uint32_t x) : l8(x << 8), l4(x << 4), w(x), r4(x >> 4), r8(x >> 8) {}
    __device__ __forceinline__ CodeWord() : l8(0), l4(0), w(0), r4(0), r8(0) {}
};

// Two codes at position pos (0..7) of a word as an fp16 pair.  The code bits
// land on bits 8-9 (even pos: value c * 2^-16) or 6-7 (odd pos: c * 2^-18) of
// each half: the largest fp16 subnormals.  Smaller subnormal encodings lose
// accumulation precision in the tensor core, whose alignment goes by the
// encoded exponent.
__device__ __forceinline__ uint32_t code_pair(const CodeWord &c, int pos)
{
    constexpr uint32_t kEven = 0x03000300u, kOdd = 0x00C000C0u;
    switch (pos) {
    case 0: return c.l8 & kEven;
    case 1: return c.l4 & kOdd;
    case 2: return c.l4 & kEven;
    case 3: return c.w & kOdd;
    case 4: return c.w & kEven;
    case 5: return c.r4 & kOdd;
    case 6: return c.r4 & kEven;
    default: return c.r8 & kOdd;
    }
}

__device__ __forceinline__ void mbar_init(unsigned long long *bar)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_u32(bar)));
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}

// Lane 0 only: stage one record (bytes, multiple of 16) into shared memory.
__device__ __forceinline__ void issue_record(unsigned long long *bar, unsigned char *dst, const unsigned char *src,
                                             uint32_t bytes)
{
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ bool mbar_try(unsigned long long *bar, uint32_t parity)
{
    uint32_t done;
    asm volatile("{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\nselp.u32 %0, 1, 0, p;\n}\n"
                 : "=r"(done)
                 : "r"(smem_u32(bar)), "r"(parity)
                 : "memory");
    return done != 0u;
}

// A hint that the 128-byte line holding p be brought into L2.
__device__ __forceinline__ void prefetch_l2(const void *p)
{
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait for phase `parity` of an mbarrier: false once limit_ns of the
// global timer have passed without it.  The timer is read only when the
// first try does not succeed.
__device__ __forceinline__ bool mbar_wait(unsigned long long *bar, uint32_t parity, unsigned long long limit_ns)
{
    if (mbar_try(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (unsigned it = 1;; ++it) {
        if (mbar_try(bar, parity)) return true;
        if ((it & 63u) == 0u && global_ns() - t0 > limit_ns) return false;
    }
}

// Normalised Walsh-Hadamard transform (block hb, 0 = none) of nvec rows of
// length D in shared memory, by one warp.  Lane l holds channels l + 32i of a
// row: channel bits 0-4 pair lanes (shuffles), bits 5 and 6 pair the lane's
// own values.
template <int D>
__device__ __forceinline__ void fwht_rows(float *x, int nvec, int hb)
{
    constexpr int NV = D / 32;
    const int lane = threadIdx.x & 31;
    if (hb == 0) return;
    const float nrm = rsqrtf((float)hb);
    for (int v = 0; v < nvec; ++v) {
        float *row = x + v * D;
        float r[NV];
#pragma unroll
        for (int i = 0; i < NV; ++i) r[i] = row[lane + 32 * i];
#pragma unroll
        for (int bit = 1; bit < 32; bit <<= 1) {
            const bool upper = lane & bit;  // the upper element of the pair takes (partner - own)
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                const float o = __shfl_xor_sync(0xffffffffu, r[i], bit);
                r[i] = upper ? o - r[i] : r[i] + o;
            }
        }
        if (hb >= 64) {
#pragma unroll
            for (int i = 0; i + 1 < NV; i += 2) {
                const float a0 = r[i], a1 = r[i + 1];
                r[i] = a0 + a1;
                r[i + 1] = a0 - a1;
            }
        }
        if (hb >= 128 && NV == 4) {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const float a0 = r[i], a2 = r[i + 2];
                r[i] = a0 + a2;
                r[i + 2] = a0 - a2;
            }
        }
#pragma unroll
        for (int i = 0; i < NV; ++i) row[lane + 32 * i] = r[i] * nrm;
    }
    __syncwarp();
}

// One out-of-line copy of the transform, shared by the query preparation
// (every segment) and the merges and tails at the end of a launch, which then
// find it in the instruction cache: about 1 us per launch at GQA 4 (Qwen3-4B
// shapes, 32K context).  MHA (Phi-3 shapes) ran 1% slower with it and the
// 8-row instantiation spills around the call, so the others keep inline copies.
template <int D>
__device__ __noinline__ void fwht_rows_shared(float *x, int nvec, int hb)
{
    fwht_rows<D>(x, nvec, hb);
}

template <int D, int GRP>
__device__ __forceinline__ void warp_fwht(float *x, int nvec, int hb)
{
    if constexpr (GRP == 4) fwht_rows_shared<D>(x, nvec, hb);
    else fwht_rows<D>(x, nvec, hb);
}


// ---- the partition of the item list over the warps of the grid -----------
// warp w takes items [w * total / nw, (w + 1) * total / nw)
__device__ __forceinline__ long long part_begin(long long w, long long total, long long nw)
{
    return w * total / nw;
}

// the warp whose range holds item i
__device__ __forceinline__ long long part_owner(long long i, long long total, long long nw)
{
    return ((i + 1) * nw + total - 1) / total - 1;
}

// The block partials of one unit.  When every warp holds at least one item
// (total >= nw) they are the slots of the contiguous warps wf .. wf + n - 1.
// With fewer items than warps every warp holds at most one, so the unit's
// per_unit items have per_unit distinct owners, spread over the grid; only
// their slots were written, and only those are enumerated.
struct UnitSlots {
    long long ibase, wf, total, nw;
    int n;  // partials
    __device__ UnitSlots(long long unit, long long per_unit, long long total_, long long nw_)
        : ibase(unit * per_unit), total(total_), nw(nw_)
    {
        wf = part_owner(ibase, total, nw);
        n = total >= nw ? (int)(part_owner(ibase + per_unit - 1, total, nw) - wf + 1) : (int)per_unit;
    }
    // warp whose slot holds partial k
    __device__ long long warp(int k) const { return total >= nw ? wf + k : part_owner(ibase + k, total, nw); }
};

// Element offset of row v (query v / heads_per_kv, head v % heads_per_kv) of
// unit (sequence s, kv head hk) in q and out, laid out [S][num_queries][Hq][D].
template <int D, int GRP, bool MQ>
__device__ __forceinline__ size_t qo_row(const DecodeArgs &a, int unit, int v)
{
    if constexpr (!MQ) return ((size_t)unit * GRP + v) * D;  // one query: [S][Hq][D]
    const int s = unit / a.num_kv_heads, hk = unit % a.num_kv_heads;
    const int qi = v / a.heads_per_kv, h = v % a.heads_per_kv;
    const int hq = a.num_kv_heads * a.heads_per_kv;
    return (((size_t)s * a.num_queries + qi) * hq + (size_t)hk * a.heads_per_kv + h) * D;
}

// Slot layout of a partial: per head [m, l, pad, pad, o[D]] (16-byte aligned rows).
template <int D>
__host__ __device__ constexpr int slot_row() { return D + 4; }

// Partials (block and tail) that the completing warp merges alone.
constexpr int kWarpMergeMax = 12;
// Item slots of a unit's residual tail in the work list: slot j stands for
// tail tokens [32j, 32j + 32).  A warp attends the tokens of all the slots in
// its range at once and writes their partial into the first (the others get
// empty partials), so a long batch keeps one pass per tail while a short
// one, whose items sit on separate warps, has the tail spread over up to four.
constexpr int kTailSlots = kDecodeTailSlots;
static_assert(kTailSlots * 32 >= kBlockTokens - 1, "the tail slots cover a tail of 127 tokens");
// Most merges a CTA takes over from its warps (its contiguous range touches
// at most three units that need a CTA merge: one it ends, one it covers
// whole, one it starts); a warp that finds the list full merges alone.
constexpr int kCtaMergeCap = 8;

// 2^x for x <= 0 (softmax weights): the hardware approximation, subnormal
// results flushed to zero (relative error about 2^-22).
__device__ __forceinline__ float exp2_ftz(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// fp32 pair -> the fp16 pair of its high part (hl = 0) or of its remainder (hl = 1).
__device__ __forceinline__ uint32_t hilo_part(float x, float y, bool hl)
{
    const __half2 hi = __floats2half2_rn(x, y);
    const float2 hf = __half22float2(hi);
    const __half2 lo = __floats2half2_rn(x - hf.x, y - hf.y);
    return hl ? *reinterpret_cast<const uint32_t *>(&lo) : *reinterpret_cast<const uint32_t *>(&hi);
}

// K scales of one record to fp32, one lane per 4 consecutive tokens:
// srK[t][g] = s[t][g] r[t] 2^16 (rows of 4, zero-padded), rK[t] = r[t], cK[d] = c[d].
template <int D>
__device__ __forceinline__ void convert_k_scales(const unsigned char *rec, float *srK, float *rK, float *cK)
{
    using R = Record<D>;
    constexpr int NG = D / kGroup;
    static_assert(NG <= 4, "score epilogue reads four groups per token");
    const int lane = threadIdx.x & 31, t0 = 4 * lane;
    const float4 r4 = h4_to_f4(reinterpret_cast<const uint2 *>(rec + R::kROff)[lane], 1.f);
    *reinterpret_cast<float4 *>(rK + t0) = r4;
    const uint2 *sp = reinterpret_cast<const uint2 *>(rec + R::kSOff) + lane * NG;
    const float rr[4] = {r4.x, r4.y, r4.z, r4.w};
    if constexpr (NG == 4) {
        // token t0 + j's four groups are sp[j]: s times (r 2^16) in packed pairs
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float rs = rr[j] * kTwo16;
            const float2 a = __fmul2_rn(__half22float2(*reinterpret_cast<const __half2 *>(&sp[j].x)), f2(rs, rs));
            const float2 b = __fmul2_rn(__half22float2(*reinterpret_cast<const __half2 *>(&sp[j].y)), f2(rs, rs));
            *reinterpret_cast<float4 *>(srK + 4 * (t0 + j)) = make_float4(a.x, a.y, b.x, b.y);
        }
    } else {
        float sv[4 * NG];
#pragma unroll
        for (int i = 0; i < NG; ++i) {
            const float4 f = h4_to_f4(sp[i], kTwo16);
            sv[4 * i] = f.x; sv[4 * i + 1] = f.y; sv[4 * i + 2] = f.z; sv[4 * i + 3] = f.w;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float4 o;
            o.x = sv[j * NG] * rr[j];
            o.y = NG > 1 ? sv[j * NG + 1] * rr[j] : 0.f;
            o.z = NG > 2 ? sv[j * NG + 2] * rr[j] : 0.f;
            o.w = NG > 3 ? sv[j * NG + 3] * rr[j] : 0.f;
            *reinterpret_cast<float4 *>(srK + 4 * (t0 + j)) = o;
        }
    }
    // c of channels 4 lane .. 4 lane + 3 (D <= 128): one 8-byte load, one 16-byte store
    if (4 * lane < D) {
        const uint2 cw = reinterpret_cast<const uint2 *>(rec + R::kCOff)[lane];
        *reinterpret_cast<float4 *>(cK + 4 * lane) = h4_to_f4(cw, 1.f);
    }
}

// Blocks [b0, b1) of one unit into the running state.  Returns false if a
// staged copy did not arrive in time (after letting the copies still in
// flight land, bounded); the warp then stops using TMA.
//
// Scores (tensor cores): A = K codes of 16 tokens x 16 channels, B = q' of
// 16 channels x 8 columns, a column per (head, hi/lo part) of four heads
// (two n-tiles for eight); the accumulators of each 32-channel group take
// their scale s r 2^16 in the epilogue, the m term is one more MMA with
// A = m (tokens x groups) and B = Q (groups x columns).  A lane then holds
// the scores of tokens 16u + gl and 16u + gl + 8 for head 4j + tig, so
// m_run[j], l_run[j] (identical in the lanes of one tig) are those of that
// head.  P V keeps the head-rows layout (A = p r s rows, B = V codes), whose
// lanes get their probabilities from the score lanes by shuffles; orun is
// in that layout (head gl % GRP).
template <int D, int GRP, typename Tin, bool MQ>
__device__ bool run_blocks(DecWarpSmem<D, GRP> &sm, const unsigned char *kbase, const unsigned char *vbase, int b0,
                           int b1, uint32_t &kph, uint32_t &vph, float (&m_run)[(GRP + 3) / 4],
                           float (&l_run)[(GRP + 3) / 4], float2 (&orun)[dec_sets<D, GRP>()][kGroup / 8],
                           int blim0, int hpk, unsigned long long wait_ns, bool withhold_k)
{
    using R = Record<D>;
    constexpr int NG = D / kGroup;          // channel groups
    constexpr int NKT = D / 16;             // k-tiles of the score MMA
    constexpr int C = 8 / GRP;              // head copies in the 8 rows of the P V MMA
    constexpr int SETS = (NG + C - 1) / C;  // groups handled per copy
    constexpr int KW = D / 32;              // K code words per (16-token unit, lane)
    constexpr int F = D / 64;
    constexpr int NTN = (GRP + 3) / 4;      // score n-tiles (four heads each)
    const int lane = threadIdx.x & 31;
    const int gl = lane >> 2, tig = lane & 3;  // mma groupID, thread in group
    const int copy = gl / GRP, h = gl % GRP;   // P V layout
    const int hq = gl >> 1;                    // score B column: head 4j + hq, part hl
    const bool hl = gl & 1;

    if (b0 >= b1) return true;
    if (lane == 0) {
        if (!withhold_k)  // self-test of the bounded wait: the first K record is never requested
            issue_record(&sm.mbar[0], sm.rec[0], kbase + (size_t)b0 * R::kBytes, R::kBytes);
        issue_record(&sm.mbar[1], sm.rec[1], vbase + (size_t)b0 * R::kBytes, R::kBytes);
    }
    for (int b = b0; b < b1; ++b) {
        if (!mbar_wait(&sm.mbar[0], kph, wait_ns)) {
            // in flight: K (unless withheld) and V of block b
            if (lane == 0) {
                if (!withhold_k) mbar_wait(&sm.mbar[0], kph, wait_ns);
                mbar_wait(&sm.mbar[1], vph, wait_ns);
            }
            __syncwarp();
            return false;
        }
        kph ^= 1u;
        const unsigned char *krec = sm.rec[0];
        const unsigned char *vrec = sm.rec[1];
        float *scr = sm.scr;
        // several queries: row v sees positions <= blim0 + v / hpk; only a block
        // reaching past blim0 needs the mask
        const bool masked = b * kBlockTokens + kBlockTokens - 1 > blim0;

        // ---- K scales: srK[t][4] = s r 2^16, rK[t], cK[d]
        float *srK = scr, *rK = scr + 4 * kBlockTokens, *cK = scr + 5 * kBlockTokens;
        convert_k_scales<D>(krec, srK, rK, cK);
        __syncwarp();

        // ---- q' B fragments (column part hl of head 4j + hq) and the group sums Q_g.
        // Lanes g = 2hq and 2hq + 1 (lane ^ 4) need the same products, one the
        // fp16 high part, the other the low part: each computes half the k-tiles
        // (hl = 0 the first half) with both parts, keeps its own and passes its
        // partner the other through one shuffle per register.
        uint32_t Bq[NTN][NKT][2];
        uint32_t BQ[NTN];
        constexpr int HK = (NKT + 1) / 2;  // k-tiles per lane of the pair
#pragma unroll
        for (int j = 0; j < NTN; ++j) {
            const int hh = 4 * j + hq;
            const bool hv = hh < GRP;
            const float *qh = sm.qbuf[hv ? hh : 0];
            float Qg[NG];
#pragma unroll
            for (int g = 0; g < NG; ++g) Qg[g] = 0.f;
            uint32_t own[HK][2], give[HK][2];
#pragma unroll
            for (int kk = 0; kk < HK; ++kk) {
                const int kt = kk + (hl ? HK : 0);
                const bool kv = kt < NKT;
                const int k = 16 * (kv ? kt : 0) + 2 * tig;
                const float2 q01 = *reinterpret_cast<const float2 *>(qh + k);
                const float2 q89 = *reinterpret_cast<const float2 *>(qh + k + 8);
                const float2 c01 = *reinterpret_cast<const float2 *>(cK + k);
                const float2 c89 = *reinterpret_cast<const float2 *>(cK + k + 8);
                const float2 v01 = __fmul2_rn(q01, c01);
                // channels 8..15 of a k-tile sit at odd code positions (scale 2^-18): times 4
                const float2 v89 = __fmul2_rn(__fmul2_rn(q89, c89), f2(4.f, 4.f));
#pragma unroll
                for (int g = 0; g < NG; ++g)
                    if (kv && g == kt / 2) Qg[g] += (v01.x + v01.y) + 0.25f * (v89.x + v89.y);
                uint32_t h0, l0, h1, l1;
                split_hilo(v01.x, v01.y, h0, l0);
                split_hilo(v89.x, v89.y, h1, l1);
                own[kk][0] = hl ? l0 : h0;
                own[kk][1] = hl ? l1 : h1;
                give[kk][0] = hl ? h0 : l0;  // the partner's part of these products
                give[kk][1] = hl ? h1 : l1;
            }
#pragma unroll
            for (int kk = 0; kk < HK; ++kk) {
                const uint32_t r0 = __shfl_xor_sync(0xffffffffu, give[kk][0], 4);
                const uint32_t r1 = __shfl_xor_sync(0xffffffffu, give[kk][1], 4);
                // k-tile kk is this lane's own when hl = 0, the partner's when hl = 1; k-tile HK + kk the reverse
                Bq[j][kk][0] = hv ? (hl ? r0 : own[kk][0]) : 0u;
                Bq[j][kk][1] = hv ? (hl ? r1 : own[kk][1]) : 0u;
                if (HK + kk < NKT) {
                    Bq[j][HK + kk][0] = hv ? (hl ? own[kk][0] : r0) : 0u;
                    Bq[j][HK + kk][1] = hv ? (hl ? own[kk][1] : r1) : 0u;
                }
            }
#pragma unroll
            for (int g = 0; g < NG; ++g) {
                Qg[g] += __shfl_xor_sync(0xffffffffu, Qg[g], 1);
                Qg[g] += __shfl_xor_sync(0xffffffffu, Qg[g], 2);
                Qg[g] += __shfl_xor_sync(0xffffffffu, Qg[g], 4);  // the pair's other half of the k-tiles
            }
            float q0 = 0.f, q1 = 0.f;
#pragma unroll
            for (int g = 0; g < NG; ++g) {
                if (g == 2 * tig) q0 = Qg[g];
                if (g == 2 * tig + 1) q1 = Qg[g];
            }
            BQ[j] = hv ? hilo_part(q0, q1, hl) : 0u;
        }

        // ---- scores of tokens 16u + gl, 16u + gl + 8 for heads 4j + tig
        float sc[NTN][8][2];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            CodeWord kw[KW];
            const uint32_t *wp = reinterpret_cast<const uint32_t *>(krec) + (u * 32 + lane) * KW;
#pragma unroll
            for (int w = 0; w < KW; ++w) kw[w] = CodeWord(wp[w]);
            float acc[NTN][NG][4];
#pragma unroll
            for (int j = 0; j < NTN; ++j)
#pragma unroll
                for (int g = 0; g < NG; ++g) acc[j][g][0] = acc[j][g][1] = acc[j][g][2] = acc[j][g][3] = 0.f;
#pragma unroll
            for (int kt = 0; kt < NKT; ++kt) {
                uint32_t aa[4];
#pragma unroll
                for (int cs = 0; cs < 2; ++cs)
#pragma unroll
                    for (int ntl = 0; ntl < 2; ++ntl) {
                        const int q = 2 * kt + cs;
                        int word, pos;
                        if (q < 8 * F) { word = ntl * F + q / 8; pos = q % 8; }
                        else { word = 2 * F; pos = q - 8 * F + 4 * ntl; }
                        aa[2 * cs + ntl] = code_pair(kw[word], pos);
                    }
#pragma unroll
                for (int j = 0; j < NTN; ++j) mma16816(acc[j][kt / 2], aa, Bq[j][kt][0], Bq[j][kt][1]);
            }
            // m term: A = m of tokens gl, gl + 8 and groups 2tig, 2tig + 1
            uint32_t am[4] = {0u, 0u, 0u, 0u};
            {
                const __half *mh = reinterpret_cast<const __half *>(krec + R::kMOff);
                const int ta = 16 * u + gl, tb = ta + 8;
                if constexpr (NG % 2 == 0) {
                    if (2 * tig < NG) {
                        am[0] = *reinterpret_cast<const uint32_t *>(mh + ta * NG + 2 * tig);
                        am[1] = *reinterpret_cast<const uint32_t *>(mh + tb * NG + 2 * tig);
                    }
                } else {
                    const __half z = __float2half(0.f);
                    __half2 pa = __halves2half2(2 * tig < NG ? mh[ta * NG + 2 * tig] : z,
                                                2 * tig + 1 < NG ? mh[ta * NG + 2 * tig + 1] : z);
                    __half2 pb = __halves2half2(2 * tig < NG ? mh[tb * NG + 2 * tig] : z,
                                                2 * tig + 1 < NG ? mh[tb * NG + 2 * tig + 1] : z);
                    am[0] = *reinterpret_cast<uint32_t *>(&pa);
                    am[1] = *reinterpret_cast<uint32_t *>(&pb);
                }
            }
            const float4 sra = *reinterpret_cast<const float4 *>(srK + 4 * (16 * u + gl));
            const float4 srb = *reinterpret_cast<const float4 *>(srK + 4 * (16 * u + gl + 8));
            const float ra = rK[16 * u + gl], rb = rK[16 * u + gl + 8];
            const float swa[4] = {sra.x, sra.y, sra.z, sra.w}, swb[4] = {srb.x, srb.y, srb.z, srb.w};
#pragma unroll
            for (int j = 0; j < NTN; ++j) {
                float accM[4] = {0.f, 0.f, 0.f, 0.f};
                mma16816(accM, am, BQ[j], 0u);
                float s0 = (accM[0] + accM[1]) * ra, s1 = (accM[2] + accM[3]) * rb;
#pragma unroll
                for (int g = 0; g < NG; ++g) {
                    s0 = fmaf(acc[j][g][0] + acc[j][g][1], swa[g], s0);
                    s1 = fmaf(acc[j][g][2] + acc[j][g][3], swb[g], s1);
                }
                sc[j][u][0] = s0;
                sc[j][u][1] = s1;
            }
        }

        if (MQ && masked) {  // only the last block, when several queries end inside it
#pragma unroll
            for (int j = 0; j < NTN; ++j) {
                const int lim = blim0 + (4 * j + tig) / hpk;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int pa = b * kBlockTokens + 16 * u + gl;
                    if (pa > lim) sc[j][u][0] = -INFINITY;
                    if (pa + 8 > lim) sc[j][u][1] = -INFINITY;
                }
            }
        }

        // ---- online softmax (base 2; the scale carries log2(e)), per head 4j + tig
        float alpha[NTN];
#pragma unroll
        for (int j = 0; j < NTN; ++j) {
            float mb = -INFINITY;
#pragma unroll
            for (int u = 0; u < 8; ++u) mb = fmaxf(mb, fmaxf(sc[j][u][0], sc[j][u][1]));
            mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 4));
            mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 8));
            mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 16));
            const float mnew = fmaxf(m_run[j], mb);
            // several queries: a row may see nothing yet, and its weights must stay 0
            const float msub = (MQ && mnew == -INFINITY) ? 0.f : mnew;
            alpha[j] = exp2_ftz(m_run[j] - msub);
            float ls = 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                sc[j][u][0] = exp2_ftz(sc[j][u][0] - msub);
                sc[j][u][1] = exp2_ftz(sc[j][u][1] - msub);
                ls += sc[j][u][0] + sc[j][u][1];
            }
            ls += __shfl_xor_sync(0xffffffffu, ls, 4);
            ls += __shfl_xor_sync(0xffffffffu, ls, 8);
            ls += __shfl_xor_sync(0xffffffffu, ls, 16);
            l_run[j] = fmaf(l_run[j], alpha[j], ls);
            m_run[j] = mnew;
        }
        // ---- probabilities into the P V layout: head h, tokens 16ks + 2tig + {0, 1, 8, 9}
        float pv[8][4];
        const int src0 = 8 * tig + (h & 3), src1 = src0 + 4;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
            for (int j = 0; j < NTN; ++j) {
                const float x0 = __shfl_sync(0xffffffffu, sc[j][ks][0], src0);
                const float x1 = __shfl_sync(0xffffffffu, sc[j][ks][0], src1);
                const float x8 = __shfl_sync(0xffffffffu, sc[j][ks][1], src0);
                const float x9 = __shfl_sync(0xffffffffu, sc[j][ks][1], src1);
                if (j == 0 || (h >> 2) == j) {
                    pv[ks][0] = x0; pv[ks][1] = x1; pv[ks][2] = x8; pv[ks][3] = x9;
                }
            }
        }
        float alphaV = __shfl_sync(0xffffffffu, alpha[0], h & 3);
        if constexpr (NTN > 1) {
            const float a1 = __shfl_sync(0xffffffffu, alpha[NTN - 1], h & 3);
            if (h >= 4) alphaV = a1;
        }
        __syncwarp();  // every lane is done with the K record and the K scales
        if (lane == 0 && b + 1 < b1)
            issue_record(&sm.mbar[0], sm.rec[0], kbase + (size_t)(b + 1) * R::kBytes, R::kBytes);
        if (!mbar_wait(&sm.mbar[1], vph, wait_ns)) {
            // in flight: V of block b and K of block b + 1
            if (lane == 0) {
                mbar_wait(&sm.mbar[1], vph, wait_ns);
                if (b + 1 < b1) mbar_wait(&sm.mbar[0], kph, wait_ns);
            }
            __syncwarp();
            return false;
        }
        vph ^= 1u;

        // ---- V scales: rsV[g][t] = r^V_t s^V_{t,g} e(t), rV[t], cV[d] * 2^16, where
        //      tokens with odd t/32 sit at odd code positions (scale 2^-18): e = 4
        convert_scales<D, true>(vrec, scr, scr + NG * kBlockTokens, scr + (NG + 1) * kBlockTokens, 1.f,
                                ((lane >> 3) & 1) ? 4.f : 1.f, kTwo16);
        __syncwarp();
        const float *rsV = scr, *rV = scr + NG * kBlockTokens, *cV = scr + (NG + 1) * kBlockTokens;

        // ---- bias_{h,g} = sum_t p_t r_t m^V_{t,g} on the tensor cores (two chains)
        float accB[4] = {0.f, 0.f, 0.f, 0.f}, accB2[4] = {0.f, 0.f, 0.f, 0.f};
        {
            const __half *mh = reinterpret_cast<const __half *>(vrec + R::kMOff);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const int T0 = 16 * ks + 2 * tig, T1 = T0 + 8;
                uint32_t Ab[4] = {0u, 0u, 0u, 0u};
                if (copy == 0) {
                    const float2 a0 = __fmul2_rn(f2(pv[ks][0], pv[ks][1]), *reinterpret_cast<const float2 *>(rV + T0));
                    const float2 a1 = __fmul2_rn(f2(pv[ks][2], pv[ks][3]), *reinterpret_cast<const float2 *>(rV + T1));
                    split_hilo(a0.x, a0.y, Ab[0], Ab[1]);
                    split_hilo(a1.x, a1.y, Ab[2], Ab[3]);
                }
                uint32_t bb0 = 0u, bb1 = 0u;
                if (gl < NG) {
                    __half2 p0 = __halves2half2(mh[T0 * NG + gl], mh[(T0 + 1) * NG + gl]);
                    __half2 p1 = __halves2half2(mh[T1 * NG + gl], mh[(T1 + 1) * NG + gl]);
                    bb0 = *reinterpret_cast<uint32_t *>(&p0);
                    bb1 = *reinterpret_cast<uint32_t *>(&p1);
                }
                if (ks & 1) mma16816(accB2, Ab, bb0, bb1);
                else mma16816(accB, Ab, bb0, bb1);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) accB[i] += accB2[i];
        const float2 bpair = hilo_sum(accB);  // (h, groups 2tig, 2tig+1)

        // ---- P V, one group set at a time
#pragma unroll
        for (int st = 0; st < SETS; ++st)
#pragma unroll
            for (int jn = 0; jn < kGroup / 8; ++jn) orun[st][jn] = __fmul2_rn(orun[st][jn], f2(alphaV, alphaV));
#pragma unroll
        for (int st = 0; st < SETS; ++st) {
            const int g = st * C + copy;
            const bool gv = g < NG;
            uint32_t Av[8][4];
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const int T0 = 16 * ks + 2 * tig, T1 = T0 + 8;
                if (gv) {
                    const float2 r0 = *reinterpret_cast<const float2 *>(rsV + g * kBlockTokens + T0);
                    const float2 r1 = *reinterpret_cast<const float2 *>(rsV + g * kBlockTokens + T1);
                    const float2 p0 = __fmul2_rn(f2(pv[ks][0], pv[ks][1]), r0);
                    const float2 p1 = __fmul2_rn(f2(pv[ks][2], pv[ks][3]), r1);
                    split_hilo(p0.x, p0.y, Av[ks][0], Av[ks][1]);
                    split_hilo(p1.x, p1.y, Av[ks][2], Av[ks][3]);
                } else {
                    Av[ks][0] = Av[ks][1] = Av[ks][2] = Av[ks][3] = 0u;
                }
            }
            // bias of (h, g) lives in lane 4*h + g/2 (copy 0)
            const int gsrc = gv ? g : 0;
            const float bx = __shfl_sync(0xffffffffu, bpair.x, 4 * h + gsrc / 2);
            const float by = __shfl_sync(0xffffffffu, bpair.y, 4 * h + gsrc / 2);
            const float bias = ((gsrc & 1) ? by : bx) * kTwoM16;
            // two 8-channel n-tiles of every copy's group at a time: C x 2 independent
            // MMA chains, interleaved token slice by token slice
#pragma unroll
            for (int j4 = 0; j4 < kGroup / 8; j4 += 2) {
                float mine[2][4];
                CodeWord vw[C][2][2];
                float acc4[C][2][4];
#pragma unroll
                for (int cc = 0; cc < C; ++cc) {
                    const int gg = st * C + cc;
                    const int nt0 = (gg < NG ? gg : 0) * (kGroup / 8) + j4;
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        const uint2 vw2 = reinterpret_cast<const uint2 *>(vrec)[(nt0 + jj) * 32 + lane];
                        vw[cc][jj][0] = CodeWord(vw2.x);
                        vw[cc][jj][1] = CodeWord(vw2.y);
                        acc4[cc][jj][0] = acc4[cc][jj][1] = acc4[cc][jj][2] = acc4[cc][jj][3] = 0.f;
                    }
                }
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
                    for (int cc = 0; cc < C; ++cc) {
                        if (st * C + cc >= NG) continue;
#pragma unroll
                        for (int jj = 0; jj < 2; ++jj) {
                            uint32_t bb[2];
#pragma unroll
                            for (int cs = 0; cs < 2; ++cs) {
                                const int m = 2 * ks + cs, am = m % 4;
                                bb[cs] = code_pair(vw[cc][jj][am / 2], 4 * (am % 2) + m / 4);
                            }
                            mma16816(acc4[cc][jj], Av[ks], bb[0], bb[1]);
                        }
                    }
                }
                // the rows of this lane's copy carry the heads of group gg only when cc == copy
#pragma unroll
                for (int jj = 0; jj < 2; ++jj)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        float v = acc4[0][jj][i];
#pragma unroll
                        for (int cc = 1; cc < C; ++cc) v = cc == copy ? acc4[cc][jj][i] : v;
                        mine[jj][i] = v;
                    }
                if (gv) {
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        const int nt = g * (kGroup / 8) + j4 + jj;
                        const float2 cv = *reinterpret_cast<const float2 *>(cV + 8 * nt + 2 * tig);
                        const float2 hs = hilo_sum(mine[jj]);
                        const float2 o = f2(hs.x + bias, hs.y + bias);
                        orun[st][j4 + jj] = __ffma2_rn(o, cv, orun[st][j4 + jj]);
                    }
                }
            }
        }

        // ---- the V buffer is free: request the next V record
        __syncwarp();
        if (lane == 0 && b + 1 < b1)
            issue_record(&sm.mbar[1], sm.rec[1], vbase + (size_t)(b + 1) * R::kBytes, R::kBytes);
    }
    return true;
}

// Tail tokens [t0, t1) of one unit (at most 127), attended by one warp with
// the unrotated query on CUDA cores: lanes over tokens for the scores (a
// whole row's loads issued together), over channel quads for P V (VB rows'
// loads in flight).  The output is rotated before it is stored, so that the
// partial (m, l, o per head) is in the basis of the block partials and
// merges with them alike.  Runs after the segment's blocks: the record
// buffers and the query buffer are scratch.
template <int D, int GRP, typename Tin, bool MQ>
__device__ void tail_partial(const DecodeArgs &a, DecWarpSmem<D, GRP> &sm, int unit, int t0, int t1, int tlim0,
                             int hb, float *dst)
{
    constexpr int SR = slot_row<D>();
    constexpr int VB = 16;  // V rows per batch of loads
    const int lane = threadIdx.x & 31;
    float *ps = reinterpret_cast<float *>(sm.rec[0]);  // [128][GRP] scores, then weights (index t - t0), both buffers
    float *qt = &sm.qbuf[0][0];                        // [GRP][D] query, scaled (uniform reads: broadcasts)
    float *ob = qt;                                    // [GRP][D] output, rotated in place (once the scores are done)
    static_assert(sizeof(float) * kBlockTokens * GRP <= sizeof(sm.rec), "tail scratch");
    const int nt = t1 - t0;
    if (nt > 0) {
        // the range's K and V rows are prefetched into L2 while the query is staged
        const Tin *kt = static_cast<const Tin *>(a.k_tail) + (size_t)unit * kBlockTokens * D;
        const Tin *vt0 = static_cast<const Tin *>(a.v_tail) + (size_t)unit * kBlockTokens * D;
        constexpr int kLines = (D * (int)sizeof(Tin) + 127) / 128;  // 128-byte lines per row
        for (int i = lane; i < nt * kLines; i += 32) {
            const size_t off = (size_t)(t0 + i / kLines) * D * sizeof(Tin) + 128 * (i % kLines);
            prefetch_l2(reinterpret_cast<const unsigned char *>(kt) + off);
            prefetch_l2(reinterpret_cast<const unsigned char *>(vt0) + off);
        }
        if constexpr (MQ) {
#pragma unroll
            for (int v = 0; v < GRP; ++v) {
                const Tin *qv = static_cast<const Tin *>(a.q) + qo_row<D, GRP, MQ>(a, unit, v);
                for (int d = lane; d < D; d += 32) qt[v * D + d] = In<Tin>::load1(qv + d) * a.scale_log2;
            }
        } else {
            const Tin *qg = static_cast<const Tin *>(a.q) + (size_t)unit * GRP * D;
            for (int i = lane; i < GRP * D; i += 32) qt[i] = In<Tin>::load1(qg + i) * a.scale_log2;
        }
        __syncwarp();
        // scores: lanes over tokens, a row's loads issued together
        for (int u0 = 0; u0 < nt; u0 += 32) {
            const int u = u0 + lane, t = t0 + u;
            if (u < nt) {
                float acc[GRP];
#pragma unroll
                for (int hh = 0; hh < GRP; ++hh) acc[hh] = 0.f;
                float kv[D];
#pragma unroll
                for (int c8 = 0; c8 < D; c8 += 8) {
                    float k8[8];
                    In<Tin>::load8(kt + (size_t)t * D + c8, k8);
#pragma unroll
                    for (int e = 0; e < 8; ++e) kv[c8 + e] = k8[e];
                }
#pragma unroll
                for (int c4 = 0; c4 < D; c4 += 4) {
#pragma unroll
                    for (int hh = 0; hh < GRP; ++hh) {
                        const float4 qv = *reinterpret_cast<const float4 *>(qt + hh * D + c4);
                        acc[hh] = fmaf(qv.x, kv[c4], acc[hh]);
                        acc[hh] = fmaf(qv.y, kv[c4 + 1], acc[hh]);
                        acc[hh] = fmaf(qv.z, kv[c4 + 2], acc[hh]);
                        acc[hh] = fmaf(qv.w, kv[c4 + 3], acc[hh]);
                    }
                }
                // several queries: row hh sees tail tokens t <= tlim0 + hh / heads_per_kv
#pragma unroll
                for (int hh = 0; hh < GRP; ++hh)
                    ps[u * GRP + hh] = (!MQ || t <= tlim0 + hh / a.heads_per_kv) ? acc[hh] : -INFINITY;
            }
        }
        __syncwarp();
    }
    // softmax over the range, lanes over tokens
    float mt[GRP], lt[GRP];
#pragma unroll
    for (int hh = 0; hh < GRP; ++hh) {
        float sv[4], mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int u = lane + 32 * j;
            sv[j] = u < nt ? ps[u * GRP + hh] : -INFINITY;
            mx = fmaxf(mx, sv[j]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float sum = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int u = lane + 32 * j;
            const float p = sv[j] > -INFINITY ? exp2f(sv[j] - mx) : 0.f;
            if (u < nt) ps[u * GRP + hh] = p;
            sum += p;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        mt[hh] = mx;
        lt[hh] = sum;
    }
    __syncwarp();
    // P V: lanes over channel quads, VB rows' loads in flight
    const Tin *vt = static_cast<const Tin *>(a.v_tail) + (size_t)unit * kBlockTokens * D;
    const int c0 = 4 * lane;
    const bool act = c0 < D;
    float4 o[GRP];
#pragma unroll
    for (int hh = 0; hh < GRP; ++hh) o[hh] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int u0 = 0; u0 < nt; u0 += VB) {
        typename In<Tin>::Raw4 vr[VB];
#pragma unroll
        for (int u = 0; u < VB; ++u)
            vr[u] = In<Tin>::load4_raw(vt + (size_t)(t0 + min(u0 + u, nt - 1)) * D + (act ? c0 : 0));
#pragma unroll
        for (int u = 0; u < VB; ++u) {
            if (act && u0 + u < nt) {
                const float4 vv = In<Tin>::widen4(vr[u]);
#pragma unroll
                for (int hh = 0; hh < GRP; ++hh) {
                    const float p = ps[(u0 + u) * GRP + hh];
                    o[hh].x = fmaf(p, vv.x, o[hh].x);
                    o[hh].y = fmaf(p, vv.y, o[hh].y);
                    o[hh].z = fmaf(p, vv.z, o[hh].z);
                    o[hh].w = fmaf(p, vv.w, o[hh].w);
                }
            }
        }
    }
    // into the rotated basis of the block partials
#pragma unroll
    for (int hh = 0; hh < GRP; ++hh)
        if (act) *reinterpret_cast<float4 *>(ob + hh * D + c0) = o[hh];
    __syncwarp();
    warp_fwht<D, GRP>(ob, GRP, hb);
#pragma unroll
    for (int hh = 0; hh < GRP; ++hh) {
        float *row = dst + hh * SR;
        if (lane == 0) { row[0] = mt[hh]; row[1] = lt[hh]; }
        if (act) *reinterpret_cast<float4 *>(row + 4 + c0) = *reinterpret_cast<const float4 *>(ob + hh * D + c0);
    }
    __syncwarp();
}

// An empty partial (m = -inf, l = 0, o = 0) for GRP heads.
template <int D, int GRP>
__device__ __forceinline__ void empty_partial(float *dst)
{
    constexpr int SR = slot_row<D>();
    const int lane = threadIdx.x & 31;
    for (int i = lane; i < GRP * SR; i += 32) dst[i] = (i % SR == 0) ? -INFINITY : 0.f;
}

// Partial p of a unit: its block partials (p < us.n, in the slots of the
// warps that hold its items), then its kTailSlots tail partials.  All are in
// the rotated basis, and all were written (an empty one has m = -inf, l = 0).
template <int D, int GRP>
__device__ __forceinline__ const float *unit_partial(const DecodeArgs &a, int unit, const UnitSlots &us, int p)
{
    constexpr int SLOT = GRP * slot_row<D>();
    return p < us.n ? a.partials + (size_t)(us.warp(p) + unit) * SLOT
                    : a.tail_partials + ((size_t)unit * kTailSlots + (p - us.n)) * SLOT;
}

// Merge of one unit by a single warp (few partials): the log-sum-exp merge of
// its partials, the un-rotation, the output.  Uses the warp's record buffers
// as scratch.
template <int D, int GRP, bool MQ>
__device__ void warp_merge(const DecodeArgs &a, int hb, DecWarpSmem<D, GRP> &sm, int unit, const UnitSlots &us)
{
    constexpr int SR = slot_row<D>();
    const int lane = threadIdx.x & 31;
    float *obuf = reinterpret_cast<float *>(sm.rec[0]);  // [GRP][D]
    const int P = us.n + kTailSlots;
    // lanes over partials: the largest m of every head
    float M[GRP];
#pragma unroll
    for (int hh = 0; hh < GRP; ++hh) M[hh] = -INFINITY;
    for (int p = lane; p < P; p += 32) {
        const float *row = unit_partial<D, GRP>(a, unit, us, p);
#pragma unroll
        for (int hh = 0; hh < GRP; ++hh) M[hh] = fmaxf(M[hh], __ldcg(row + hh * SR));
    }
#pragma unroll
    for (int hh = 0; hh < GRP; ++hh)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M[hh] = fmaxf(M[hh], __shfl_xor_sync(0xffffffffu, M[hh], o));
    // 32 partials at a time: lane j fetches partial p0 + j's row address, weights and l, which the
    // warp then takes in order by shuffles; the rows' loads do not wait on one another
    float L[GRP], acc[GRP][D / 32];
#pragma unroll
    for (int hh = 0; hh < GRP; ++hh) {
        L[hh] = 0.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) acc[hh][c] = 0.f;
    }
    for (int p0 = 0; p0 < P; p0 += 32) {
        const int p = p0 + lane;
        const float *row = unit_partial<D, GRP>(a, unit, us, p < P ? p : p0);
        float w[GRP], lv[GRP];
#pragma unroll
        for (int hh = 0; hh < GRP; ++hh) {
            const float m = p < P ? __ldcg(row + hh * SR) : -INFINITY;
            w[hh] = (M[hh] > -INFINITY && m > -INFINITY) ? exp2f(m - M[hh]) : 0.f;
            lv[hh] = p < P ? __ldcg(row + hh * SR + 1) : 0.f;
        }
        const unsigned long long ra = reinterpret_cast<unsigned long long>(row);
        const int nj = min(32, P - p0);
#pragma unroll 4
        for (int j = 0; j < nj; ++j) {
            const float *rj = reinterpret_cast<const float *>(__shfl_sync(0xffffffffu, ra, j));
#pragma unroll
            for (int hh = 0; hh < GRP; ++hh) {
                const float wj = __shfl_sync(0xffffffffu, w[hh], j);
                const float lj = __shfl_sync(0xffffffffu, lv[hh], j);
                // a partial of weight 0 (empty, or far below the maximum) is left out
                L[hh] = wj == 0.f ? L[hh] : fmaf(lj, wj, L[hh]);
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    const float x = __ldcg(rj + hh * SR + 4 + 32 * c + lane);
                    acc[hh][c] = wj == 0.f ? acc[hh][c] : fmaf(x, wj, acc[hh][c]);
                }
            }
        }
    }
#pragma unroll
    for (int hh = 0; hh < GRP; ++hh) {
        const float linv = L[hh] > 0.f ? 1.f / L[hh] : 0.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) obuf[hh * D + 32 * c + lane] = acc[hh][c] * linv;
    }
    __syncwarp();
    warp_fwht<D, GRP>(obuf, GRP, hb);
    if constexpr (MQ) {
#pragma unroll
        for (int v = 0; v < GRP; ++v) {
            float *ov = a.out + qo_row<D, GRP, MQ>(a, unit, v);
            for (int d = lane; d < D; d += 32) ov[d] = obuf[v * D + d];
        }
    } else {
        float *out = a.out + (size_t)unit * GRP * D;
        for (int i = lane; i < GRP * D; i += 32) out[i] = obuf[i];
    }
    __syncwarp();
}

// Merge of one unit by all warps of the CTA (many partials).  Every thread
// of the CTA calls it with the same arguments; the whole dynamic shared
// memory is scratch.  The unit's partials (block partials, then tail
// partials) are copied into shared memory in one round of asynchronous
// 16-byte copies; everything after that is shared-memory arithmetic.
template <int D, int GRP>
struct CtaMergeLayout {
    static constexpr int SR = slot_row<D>();
    static constexpr int kSlot = GRP * SR;  // floats per partial
    // parts [P][GRP][SR], obuf [GRP][D], then 1/L and M per head (padded), then the weights [P][GRP]
    static __host__ __device__ constexpr size_t fixed_floats() { return GRP * D + 2 * ((GRP + 3) / 4 * 4); }
};

template <int D, int GRP, bool MQ>
__device__ void cta_merge(const DecodeArgs &a, int hb, unsigned char *smem, int unit, const UnitSlots &us)
{
    constexpr int W = dec_warps<D, GRP>();
    constexpr int NT = W * 32;
    constexpr int SR = slot_row<D>();
    constexpr int SLOT = GRP * SR;
    constexpr int GP = (GRP + 3) / 4 * 4;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int P = us.n + kTailSlots;
    float *parts = reinterpret_cast<float *>(smem);  // [P][GRP][SR]
    float *obuf = parts + (size_t)P * SLOT;          // [GRP][D] block part (rotated, then un-rotated)
    float *Li = obuf + GRP * D;                      // [GRP] 1 / L
    float *Mh = Li + GP;                             // [GRP]
    float *wts = Mh + GP;                            // [P][GRP] weights exp2(m - M)

    // ---- one round of copies: the block partials, then the tail partials (a warp per
    // partial, whose slot address is worked out once; lanes over its 16-byte pieces)
    static_assert(SLOT % 4 == 0, "a partial is a whole number of 16-byte pieces");
    for (int p = warp; p < P; p += W) {
        const float *g = unit_partial<D, GRP>(a, unit, us, p);
        const uint32_t d = smem_u32(parts + (size_t)p * SLOT);
        for (int c = lane; c < SLOT / 4; c += 32)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d + 16 * c), "l"(g + 4 * c) : "memory");
    }
    asm volatile("cp.async.commit_group;\n" ::: "memory");
    asm volatile("cp.async.wait_group 0;\n" ::: "memory");
    __syncthreads();
    // ---- per head: the largest m, the weights and the normaliser (warp h for head h)
    for (int h = warp; h < GRP; h += W) {
        float mx = -INFINITY;
        for (int p = lane; p < P; p += 32) mx = fmaxf(mx, parts[(size_t)p * SLOT + h * SR]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float M = mx;
        float ls = 0.f;
        for (int p = lane; p < P; p += 32) {
            const float m = parts[(size_t)p * SLOT + h * SR];
            const float wgt = (M > -INFINITY && m > -INFINITY) ? exp2f(m - M) : 0.f;
            ls = fmaf(parts[(size_t)p * SLOT + h * SR + 1], wgt, ls);
            wts[p * GRP + h] = wgt;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
        if (lane == 0) {
            Mh[h] = M;
            Li[h] = ls > 0.f ? 1.f / ls : 0.f;
        }
    }
    __syncthreads();
    // ---- weighted sum of the partials (an empty partial has weight 0 and zero rows), four
    // channels a thread, two chains over the partials
    for (int i = tid; i < GRP * (D / 4); i += NT) {
        const int h = i / (D / 4), c = 4 * (i % (D / 4));
        const float *src = parts + h * SR + 4 + c;
        float2 a01 = f2(0.f, 0.f), a23 = f2(0.f, 0.f), b01 = f2(0.f, 0.f), b23 = f2(0.f, 0.f);
        int p = 0;
        for (; p + 1 < P; p += 2) {
            const float w0 = wts[p * GRP + h], w1 = wts[(p + 1) * GRP + h];
            const float4 x0 = *reinterpret_cast<const float4 *>(src + (size_t)p * SLOT);
            const float4 x1 = *reinterpret_cast<const float4 *>(src + (size_t)(p + 1) * SLOT);
            a01 = __ffma2_rn(f2(x0.x, x0.y), f2(w0, w0), a01);
            a23 = __ffma2_rn(f2(x0.z, x0.w), f2(w0, w0), a23);
            b01 = __ffma2_rn(f2(x1.x, x1.y), f2(w1, w1), b01);
            b23 = __ffma2_rn(f2(x1.z, x1.w), f2(w1, w1), b23);
        }
        if (p < P) {
            const float w0 = wts[p * GRP + h];
            const float4 x0 = *reinterpret_cast<const float4 *>(src + (size_t)p * SLOT);
            a01 = __ffma2_rn(f2(x0.x, x0.y), f2(w0, w0), a01);
            a23 = __ffma2_rn(f2(x0.z, x0.w), f2(w0, w0), a23);
        }
        const float li = Li[h];
        const float2 o01 = __fmul2_rn(__fadd2_rn(a01, b01), f2(li, li));
        const float2 o23 = __fmul2_rn(__fadd2_rn(a23, b23), f2(li, li));
        *reinterpret_cast<float4 *>(obuf + h * D + c) = make_float4(o01.x, o01.y, o23.x, o23.y);
    }
    __syncthreads();
    if (warp < GRP) warp_fwht<D, GRP>(obuf + warp * D, 1, hb);
    __syncthreads();
    if constexpr (MQ) {
        if (tid < GRP * (D / 4)) {  // a float4 of one row per thread
            const int v = tid / (D / 4), d4 = tid % (D / 4);
            *reinterpret_cast<float4 *>(a.out + qo_row<D, GRP, MQ>(a, unit, v) + 4 * d4) =
                *reinterpret_cast<const float4 *>(obuf + v * D + 4 * d4);
        }
    } else {
        float *out = a.out + (size_t)unit * GRP * D;
        for (int i = tid; i < GRP * D; i += NT) out[i] = obuf[i];
    }
    __syncthreads();  // the scratch is free again
}

// Most partials the CTA merge holds in shared memory: beyond that (only when
// a unit is spread over nearly the whole grid at the largest GQA groups) the
// completing warp merges alone.
template <int D, int GRP>
__host__ __device__ constexpr int cta_merge_max()
{
    constexpr int W = dec_warps<D, GRP>();
    constexpr int SLOT = GRP * slot_row<D>();
    constexpr size_t avail = sizeof(DecWarpSmem<D, GRP>) * W / sizeof(float);
    return (int)((avail - CtaMergeLayout<D, GRP>::fixed_floats()) / (SLOT + GRP));
}

template <int D, int GRP, typename Tin, bool MQ>
__global__ void __launch_bounds__(dec_warps<D, GRP>() * 32, 1)
decode_kernel(DecodeArgs a, int hb)
{
    using R = Record<D>;
    constexpr int W = dec_warps<D, GRP>();
    constexpr int C = 8 / GRP;
    constexpr int NG = D / kGroup;
    constexpr int SETS = dec_sets<D, GRP>();
    constexpr int NTN = (GRP + 3) / 4;
    constexpr int SR = slot_row<D>();
    extern __shared__ __align__(128) unsigned char smem_raw[];
    grid_dep_wait();  // the previous kernel in the stream (an append, say) has completed
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    DecWarpSmem<D, GRP> &sm = reinterpret_cast<DecWarpSmem<D, GRP> *>(smem_raw)[warp];
    const int gl = lane >> 2, tig = lane & 3;
    const int copy = gl / GRP, h = gl % GRP;

    const long long nw = (long long)gridDim.x * W;
    const int nb_max = a.max_tokens / kBlockTokens;
    const long long per_unit = nb_max + kTailSlots;  // blocks, then the tail's slots
    const long long total = (long long)a.num_units * per_unit;
    const long long wg = (long long)blockIdx.x * W + warp;
    const long long i_begin = part_begin(wg, total, nw), i_end = part_begin(wg + 1, total, nw);

    // Units whose merge this CTA's warps hand to the CTA (filled by the warp
    // that completes the unit; read after the CTA's closing barrier).
    __shared__ int merge_list[kCtaMergeCap];
    __shared__ int merge_count;
    if (lane == 0) {
        mbar_init(&sm.mbar[0]);
        mbar_init(&sm.mbar[1]);
    }
    if (threadIdx.x == 0) merge_count = 0;
    __syncthreads();
    uint32_t kph = 0u, vph = 0u;
    bool dead = false;  // a staged copy timed out: no more TMA from this warp

    for (long long i = i_begin; i < i_end;) {
        const int unit = (int)(i / per_unit);
        const long long ibase = (long long)unit * per_unit;
        const long long seg_end = min(i_end, ibase + per_unit);
        const int s = unit / a.num_kv_heads;
        int n = a.n_tokens[s];
        if (n > a.max_tokens) {
            if (lane == 0 && i == ibase) status_or(a.status, KVARN_STATUS_LENGTH);
            n = a.max_tokens;
        }
        if (n < 0) n = 0;
        const int nblk = n / kBlockTokens;
        const int ntail = n - nblk * kBlockTokens;
        const int b0 = (int)(i - ibase);
        const int b1 = (int)min(seg_end - ibase, (long long)nb_max);
        const int b1r = min(b1, nblk);  // blocks beyond the sequence's length are skipped

        float m_run[NTN], l_run[NTN];
#pragma unroll
        for (int j = 0; j < NTN; ++j) { m_run[j] = -INFINITY; l_run[j] = 0.f; }
        float2 orun[SETS][kGroup / 8];  // this lane's groups st * C + copy, their four n-tiles
#pragma unroll
        for (int st = 0; st < SETS; ++st)
#pragma unroll
            for (int jn = 0; jn < kGroup / 8; ++jn) orun[st][jn] = f2(0.f, 0.f);
        if (b0 < b1r && !dead) {
            // rotated query of this GQA group, scaled by softmax scale * log2(e)
            if constexpr (MQ) {
#pragma unroll
                for (int v = 0; v < GRP; ++v) {
                    const Tin *qv = static_cast<const Tin *>(a.q) + qo_row<D, GRP, MQ>(a, unit, v);
                    for (int d = lane; d < D; d += 32) sm.qbuf[v][d] = In<Tin>::load1(qv + d) * a.scale_log2;
                }
            } else {
                const Tin *qg = static_cast<const Tin *>(a.q) + (size_t)unit * GRP * D;
                for (int j = lane; j < GRP * D; j += 32) (&sm.qbuf[0][0])[j] = In<Tin>::load1(qg + j) * a.scale_log2;
            }
            __syncwarp();
            warp_fwht<D, GRP>(&sm.qbuf[0][0], GRP, hb);
            const unsigned char *kbase =
                static_cast<const unsigned char *>(a.k_records) + (size_t)unit * a.max_blocks * R::kBytes;
            const unsigned char *vbase =
                static_cast<const unsigned char *>(a.v_records) + (size_t)unit * a.max_blocks * R::kBytes;
            if (!run_blocks<D, GRP, Tin, MQ>(sm, kbase, vbase, b0, b1r, kph, vph, m_run, l_run, orun, n - a.num_queries,
                                             a.heads_per_kv, a.wait_ns ? a.wait_ns : kWaitLimitNs,
                                             a.withhold_first_k != 0)) {
                dead = true;
                if (lane == 0) status_or(a.status, KVARN_STATUS_TIMEOUT);
#pragma unroll
                for (int j = 0; j < NTN; ++j) { m_run[j] = -INFINITY; l_run[j] = 0.f; }
#pragma unroll
                for (int st = 0; st < SETS; ++st)
#pragma unroll
                    for (int jn = 0; jn < kGroup / 8; ++jn) orun[st][jn] = f2(0.f, 0.f);
            }
        }
        // ---- this segment's block partial: (m, l, o_rot) per head
        {
            float *slot = a.partials + (size_t)(wg + unit) * GRP * SR;
            // (m, l) of head 4j + tig sit in every lane of that tig
#pragma unroll
            for (int j = 0; j < NTN; ++j)
                if (gl == 0 && 4 * j + tig < GRP) {
                    slot[(4 * j + tig) * SR] = m_run[j];
                    slot[(4 * j + tig) * SR + 1] = l_run[j];
                }
            float *pp = slot + h * SR;
#pragma unroll
            for (int st = 0; st < SETS; ++st) {
                const int g = st * C + copy;
                if (g < NG)
#pragma unroll
                    for (int jn = 0; jn < kGroup / 8; ++jn)
                        *reinterpret_cast<float2 *>(pp + 4 + 8 * (g * (kGroup / 8) + jn) + 2 * tig) = orun[st][jn];
            }
        }
        // its tail slots [j0, j1): one pass over their tokens into slot j0's partial, the others empty
        // (a warp with several slots attends their tokens at once; single slots spread a short batch's tail)
        const long long j0 = max(i - ibase - nb_max, 0ll), j1 = seg_end - ibase - nb_max;
        if (j0 < j1) {
            float *tp = a.tail_partials + (size_t)unit * kTailSlots * GRP * SR;
            tail_partial<D, GRP, Tin, MQ>(a, sm, unit, min(32 * (int)j0, ntail), min(32 * (int)j1, ntail),
                                          n - a.num_queries - nblk * kBlockTokens, hb, tp + j0 * GRP * SR);
            for (long long j = j0 + 1; j < j1; ++j) empty_partial<D, GRP>(tp + j * GRP * SR);
        }

        // ---- arrival: this segment's items are done
        __syncwarp();
        __threadfence();
        uint32_t prev = 0u;
        const uint32_t cnt = (uint32_t)(seg_end - i);
        if (lane == 0) prev = atomicAdd(a.tickets + unit, cnt);
        prev = __shfl_sync(0xffffffffu, prev, 0);
        if (prev + cnt == (uint32_t)per_unit) {
            __threadfence();
            const UnitSlots us(unit, per_unit, total, nw);
            const int np = us.n + kTailSlots;  // partials to merge
            bool alone = np <= kWarpMergeMax || np > cta_merge_max<D, GRP>();
            if (!alone) {  // hand it to the CTA, whose warps merge it together once they are all done
                int k = 0;
                if (lane == 0) {
                    k = atomicAdd(&merge_count, 1);
                    if (k < kCtaMergeCap) merge_list[k] = unit;
                }
                alone = __shfl_sync(0xffffffffu, k, 0) >= kCtaMergeCap;  // list full: merge alone
            }
            if (alone) {
                warp_merge<D, GRP, MQ>(a, hb, sm, unit, us);
                if (lane == 0) a.tickets[unit] = 0u;
            }
        }
        i = seg_end;
    }

    // ---- the merges this CTA's warps handed over
    __syncthreads();
    const int nmerge = min(merge_count, kCtaMergeCap);
    for (int j = 0; j < nmerge; ++j) {
        const int unit = merge_list[j];
        cta_merge<D, GRP, MQ>(a, hb, smem_raw, unit, UnitSlots(unit, per_unit, total, nw));
        if (threadIdx.x == 0) a.tickets[unit] = 0u;
    }
}

template <int D, int GRP, typename Tin, bool MQ>
static cudaError_t launch_dec_mq(const DecodeArgs &a, int hb, int ctas, cudaStream_t st)
{
    constexpr int W = dec_warps<D, GRP>();
    const size_t smem = sizeof(DecWarpSmem<D, GRP>) * W;
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, GRP, Tin, MQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_overlapped(decode_kernel<D, GRP, Tin, MQ>, dim3(ctas), dim3(W * 32), smem, st, a, hb);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// One query per sequence (the common case) runs the kernel without the
// causal masking and row mapping of several queries.
template <int D, int GRP, typename Tin>
static cudaError_t launch_dec(const DecodeArgs &a, int hb, int ctas, cudaStream_t st)
{
    return a.num_queries > 1 ? launch_dec_mq<D, GRP, Tin, true>(a, hb, ctas, st)
                             : launch_dec_mq<D, GRP, Tin, false>(a, hb, ctas, st);
}

template <int D, int GRP>
static cudaError_t dispatch_dtype(int dtype, const DecodeArgs &a, int hb, int ctas, cudaStream_t st)
{
    return dtype == KVARN_BF16 ? launch_dec<D, GRP, __nv_bfloat16>(a, hb, ctas, st)
                               : launch_dec<D, GRP, float>(a, hb, ctas, st);
}

template <int D>
static cudaError_t dispatch_grp(int dtype, const DecodeArgs &a, int hb, int ctas, cudaStream_t st)
{
    switch (a.grp) {
    case 1: return dispatch_dtype<D, 1>(dtype, a, hb, ctas, st);
    case 2: return dispatch_dtype<D, 2>(dtype, a, hb, ctas, st);
    case 4: return dispatch_dtype<D, 4>(dtype, a, hb, ctas, st);
    case 8: return dispatch_dtype<D, 8>(dtype, a, hb, ctas, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t run_decode(const kvarn_config &c, const DecodeArgs &a, int ctas, cudaStream_t st)
{
    switch (c.head_dim) {
    case 64: return dispatch_grp<64>(c.dtype, a, c.hadamard, ctas, st);
    case 96: return dispatch_grp<96>(c.dtype, a, c.hadamard, ctas, st);
    case 128: return dispatch_grp<128>(c.dtype, a, c.hadamard, ctas, st);
    }
    return cudaErrorInvalidValue;
}

template <int D>
static int warps_for(int grp)
{
    switch (grp) {
    case 1: return dec_warps<D, 1>();
    case 2: return dec_warps<D, 2>();
    case 4: return dec_warps<D, 4>();
    default: return dec_warps<D, 8>();
    }
}

int decode_warps_per_cta(int head_dim, int grp)
{
    return head_dim == 64 ? warps_for<64>(grp) : head_dim == 96 ? warps_for<96>(grp) : warps_for<128>(grp);
}

size_t decode_slot_bytes(int head_dim, int grp)
{
    return (size_t)grp * (head_dim + 4) * sizeof(float);
}

}  // namespace kvarn
