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
// lane l holds tokens qtok(l) + 32r (r = 0..3) and channels 32j .. 32j+31 of
// each, as 16 float2 per token.  So a quantisation group sits entirely in one
// thread, the per-token (row) sums cross warps through shared memory and the
// per-channel (column) sums cross the 32 lanes through a swizzled
// shared-memory transpose.
// Rotation.  bf16 blocks are rotated on the tensor cores: the Hadamard matrix
// is +-1, exact in bf16, and the products accumulate in fp32, so X H is a
// plain dense contraction (mma.sync m16n8k16).  Warp j computes its group's
// 32 outputs from the HB inputs of its Hadamard block, all 128 tokens, with
// A fragments read by ldmatrix from the block staged in shared memory.  fp32
// blocks take the CUDA-core path: 32-point butterflies in registers and one
// exchange across warps per further channel bit.  Arithmetic is fp32; packed
// f32x2 operations (sm_100) halve the issue count of the elementwise work.
#pragma once

#include "kvarn_common.cuh"

namespace kvarn {

// Lane l's first token: lanes 4g + tig hold tokens 8 tig + g (+ 32 r), the
// order in which the tensor-core rotation leaves them.
__host__ __device__ constexpr int qtok(int l) { return 8 * (l & 3) + (l >> 2); }

// Shared-memory stage of the tensor-core rotation: the bf16 block, rows padded
// by 16 bytes so that the eight row addresses of an ldmatrix hit distinct
// banks, and one 32-token x 32-channel fp32 transpose buffer per warp.
template <int D>
struct TcStage {
    static constexpr int kRowBytes = 2 * D + 16;
    unsigned char rows[kBlockTokens * kRowBytes];
    float4 xbuf[D / 32][32][8];
};

template <int D>
struct QuantSmem {
    static constexpr int W = D / 32;
    union {
        float4 xch[W][2][8][32];               // Hadamard exchange [warp][token pair][chunk][lane]
        float4 col[W][32][16];                 // column-sum transpose [warp][lane][chunk]
        unsigned char rec[Record<D>::kBytes];  // record staging
        TcStage<D> tc;                         // tensor-core rotation (bf16 blocks)
    } u;
    float part[2][W][kBlockTokens];            // per-token partial row sums: [0] of z, [1] of (z - mean)^2
    float ubuf[D];                             // 1 / c broadcast
    float kbuf[D];                             // column shifts z[0][d]
    float2 gpart[W];                           // per-warp (sum of log2 c, count) of nonzero-variance channels
    float ymax[W][kBlockTokens];               // per-(group, token) largest |Y| (token gauge)
};

// The block quantiser's shared memory lives in the dynamic segment (it exceeds
// the 48 KB static limit at D = 128); launches pass sizeof(QuantSmem<D>).
template <int D>
__device__ __forceinline__ QuantSmem<D> &quant_smem()
{
    extern __shared__ __align__(16) unsigned char quant_smem_raw[];
    return *reinterpret_cast<QuantSmem<D> *>(quant_smem_raw);
}

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
        const Tin *p = rows + (size_t)(qtok(l) + 32 * r) * D + 32 * j;
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

// ---- tensor-core rotation of a bf16 block --------------------------------
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The same with a zero accumulator in (the first k-tile of a chain).
__device__ __forceinline__ void mma_bf16_16816_z(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};\n"
        : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.f));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&a)[4], const void *p)
{
    const uint32_t addr = static_cast<uint32_t>(__cvta_generic_to_shared(p));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
                 : "r"(addr));
}

// Copy the 128 x D bf16 rows into the padded stage with asynchronous 16-byte
// copies (cp.async.cg: no register round trip, every copy of the thread in
// flight at once, read through L2 -- which also sees the append path's tail
// that this kernel wrote before a CTA barrier).  The caller waits and syncs.
template <int D>
__device__ __forceinline__ void stage_rows(const __nv_bfloat16 *rows, TcStage<D> &st)
{
    constexpr int CH = D / 8;  // 16-byte chunks per row
    constexpr int N = kBlockTokens * CH / D;  // copies per thread (D threads): 16 at every D
    static_assert(kBlockTokens * CH % D == 0, "stage split");
#pragma unroll
    for (int it = 0; it < N; ++it) {
        const int i = threadIdx.x + it * D;
        const int row = i / CH, ch = i % CH;
        const void *src = rows + (size_t)row * D + 8 * ch;
        const uint32_t dst = static_cast<uint32_t>(
            __cvta_generic_to_shared(st.rows + row * TcStage<D>::kRowBytes + 16 * ch));
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
    }
    asm volatile("cp.async.commit_group;\n" ::: "memory");
    asm volatile("cp.async.wait_group 0;\n" ::: "memory");
}

// Physical float4 slot of logical slot q in row `row` (t = row >> 3, g =
// row & 7) of a transpose buffer: q xor (t1 ^ g1, t0 ^ g0, g0).  A 16-byte
// read phase (eight lanes: rows 8 t + g for t = 0..3 and two g differing in
// bit 0) and an 8-byte write phase (sixteen lanes: rows 8 t + g for one t and
// four g, two slots each) then both meet every bank once.
__device__ __forceinline__ int xswz(int row, int q)
{
    return q ^ (((((row >> 4) ^ (row >> 1)) & 1) << 2) | ((((row >> 3) ^ row) & 1) << 1) | (row & 1));
}

// One warp's share of X H for a bf16 block: the 32 rotated channels of group j
// (unnormalised: the stored r takes the 1/sqrt(HB)), all 128 tokens, into X
// in the thread layout.  HB in {0, 32, 64, 128}.
//
// Output channel 32j + 8 nu + n of n-tile nu is column n of the MMA; input
// channel 16 kappa + k of the warp's Hadamard block is row k of k-tile kappa.
// With i = 16 kappa + k and o = 32 JP + 8 nu + n (both within the block,
// JP = j mod (HB / 32)),
//   (-1)^popcount(i & o) = (-1)^popcount(k & (8 (nu & 1) + n))
//                        * (-1)^popcount(kappa & (nu >> 1))
//                        * (-1)^popcount(kappa & 2 JP),
// a per-lane base fragment (two of them, by nu & 1), a sign fixed at compile
// time, and a sign set by the warp.  The last is either 1 for every kappa
// (JP = 0) or, once the k-tiles are visited in a warp-chosen order, kappa's
// bit 1 (JP = 2: bits 1 and 2 of kappa swapped; JP = 3: bit 1 replaced by
// bit 1 xor bit 2), so one code path serves every warp: the k-tiles with bit 1
// set use base registers whose signs the warp swapped once.
// m-tile mu of round rho holds tokens 32 rho + 16 mu + (0..15); the C
// fragments leave lane (g, tig) tokens g + {0, 8, 16, 24} x channels
// 8 nu + 2 tig + {0, 1}, and a transpose through the warp's buffer gives lane
// 4g + tig the token 8 tig + g = qtok(lane) with all 32 channels.
template <int D, int HB>
__device__ __forceinline__ void rotate_warp_tc(float2 (&X)[4][16], TcStage<D> &st)
{
    const int j = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tig = lane & 3;
    constexpr uint32_t kOne = 0x3F80u, kMinus = 0xBF80u;  // bf16 +1, -1
    // base B fragments: b0 holds rows k = 2 tig + {0, 1}, b1 rows k = 2 tig + 8 + {0, 1}, column n = g
    uint32_t bp[2][2], bn[2][2];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            uint32_t reg = 0u;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int k = 2 * tig + 8 * half + e;
                uint32_t v;
                if constexpr (HB == 0) v = (k == 8 * h + g) ? kOne : 0u;  // identity
                else v = (__popc(k & (8 * h + g)) & 1) ? kMinus : kOne;
                reg |= v << (16 * e);
            }
            bp[h][half] = reg;
            bn[h][half] = reg ^ 0x80008000u;
        }
    constexpr int NKT = HB == 0 ? 2 : HB / 16;  // k-tiles feeding this warp
    const int jp = HB >= 64 ? j % (HB / 32) : 0;
    // the warp's sign on k-tiles with bit 1 set: swap the bases' signs once
    const bool flip = jp != 0;
    uint32_t sp[2][2], sn[2][2];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            sp[h][half] = flip ? bn[h][half] : bp[h][half];
            sn[h][half] = flip ? bp[h][half] : bn[h][half];
        }
    // byte offset of each k-tile in a staged row, in the warp's visiting order
    const int kt0 = HB == 0 ? 2 * j : (32 * j / (HB == 0 ? 32 : HB)) * (HB / 16);
    int koff[NKT];
#pragma unroll
    for (int kap = 0; kap < NKT; ++kap) {
        int kk = kap;
        if (HB == 128 && jp == 2) kk = (kap & 1) | ((kap & 2) << 1) | ((kap & 4) >> 1);
        if (HB == 128 && jp == 3) kk = kap ^ ((kap & 4) >> 1);
        koff[kap] = 32 * (kt0 + kk);
    }
    float4(&xb)[32][8] = st.xbuf[j];
#pragma unroll
    for (int rho = 0; rho < 4; ++rho) {  // unrolled: X[rho] must stay in registers
#pragma unroll
        for (int mu = 0; mu < 2; ++mu) {
            float acc[4][4];
            const int arow = 32 * rho + 16 * mu + (lane & 7) + 8 * ((lane >> 3) & 1);
            const unsigned char *abase = st.rows + arow * TcStage<D>::kRowBytes + 16 * (lane >> 4);
#pragma unroll
            for (int kap = 0; kap < NKT; ++kap) {
                uint32_t a[4];
                ldmatrix_x4(a, abase + koff[kap]);
#pragma unroll
                for (int nu = 0; nu < 4; ++nu) {
                    if constexpr (HB == 0) {
                        // identity: k-tile 2j + (nu >> 1) alone feeds n-tile nu
                        if (kap != (nu >> 1)) continue;
                        mma_bf16_16816_z(acc[nu], a, bp[nu & 1][0], bp[nu & 1][1]);
                    } else {
                        const bool neg = __popc(kap & (nu >> 1)) & 1;  // compile-time
                        const uint32_t b0 = (kap & 2) == 0 ? (neg ? bn[nu & 1][0] : bp[nu & 1][0])
                                                           : (neg ? sn[nu & 1][0] : sp[nu & 1][0]);
                        const uint32_t b1 = (kap & 2) == 0 ? (neg ? bn[nu & 1][1] : bp[nu & 1][1])
                                                           : (neg ? sn[nu & 1][1] : sp[nu & 1][1]);
                        if (kap == 0) mma_bf16_16816_z(acc[nu], a, b0, b1);
                        else mma_bf16_16816(acc[nu], a, b0, b1);
                    }
                }
            }
            // C fragments -> transpose buffer: rows 16 mu + g (c0, c1) and 16 mu + g + 8 (c2, c3)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int row = 16 * mu + g + 8 * hh;
#pragma unroll
                for (int nu = 0; nu < 4; ++nu) {
                    const int q = 2 * nu + (tig >> 1);  // channel 8 nu + 2 tig sits in float4 q, half tig & 1
                    float2 *dst = reinterpret_cast<float2 *>(&xb[row][xswz(row, q)]) + (tig & 1);
                    *dst = f2(acc[nu][2 * hh], acc[nu][2 * hh + 1]);
                }
            }
        }
        __syncwarp();
        const int row = qtok(lane);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 v = xb[row][xswz(row, q)];
            X[rho][2 * q] = f2(v.x, v.y);
            X[rho][2 * q + 1] = f2(v.z, v.w);
        }
        __syncwarp();
    }
}

// Load and rotate a bf16 block on the tensor cores (all D threads call this).
template <int D, int HB>
__device__ __forceinline__ void load_rotate_tc(const __nv_bfloat16 *rows, float2 (&X)[4][16], QuantSmem<D> &sm)
{
    stage_rows<D>(rows, sm.u.tc);
    __syncthreads();
    rotate_warp_tc<D, HB>(X, sm.u.tc);
    __syncthreads();  // the stage is free for the union's next use
}

// Quantise the block held in X (destroyed) into rec_out (global, 16-byte
// aligned, Record<D>::kBytes); TENSOR 0 = K code order, 1 = V code order.
// dbg: NULL or fp32 [T + D + 2*T*D/32] unrounded r, c, s, m (as stored, token
// gauge included).  All D threads of the CTA must call this.
// PREROT: X already holds the rotation, unnormalised (tensor-core path); the
// 1/sqrt(HB) then goes into the stored r (Y, c, s and m do not depend on it).
template <int D, int HB, int TENSOR, bool PREROT = false>
__device__ void quantize_block(float2 (&X)[4][16], QuantSmem<D> &sm, int sweeps,
                               unsigned char *__restrict__ rec_out, float *__restrict__ dbg,
                               int32_t *status)
{
    constexpr int W = D / 32;
    using R = Record<D>;
    const int j = threadIdx.x >> 5, l = threadIdx.x & 31;
    const int t0 = qtok(l);  // this lane's tokens: t0 + 32 r
    // 1/sqrt(HB) of a rotation left unnormalised
    constexpr float kRNorm = !PREROT || HB == 0 ? 1.f : HB == 32 ? 0.17677669529663688f
                                                       : HB == 64 ? 0.125f : 0.08838834764831845f;
    // a token scale of 1 (no sweeps, zero-variance row) in the frame of X
    constexpr float kRUnit = 1.f / kRNorm;

    // ---- 1. Hadamard rotation along the channels --------------------------
    if constexpr (!PREROT) rotate_block<D, HB>(X, sm);

    // ---- 2. dual-axis variance normalisation ------------------------------
    // Rows: two passes (mean, then mean square deviation) over the D channels,
    // whose partial sums cross the warps through shared memory.  Columns: one
    // pass over the 128 tokens on values shifted by token 0's (lane 0's) z,
    // whose partials cross the lanes through a shared-memory transpose.  Then
    // the gauge: g = geometric mean of the nonzero-variance channel scales,
    // c <- c / g (1 for a zero-variance column), r <- r g at the end.
    // 1 / c of the warp's 32 channels lives in sm.ubuf (the same for every
    // lane of the warp: broadcast reads, channel-outer loops), not in registers
    sm.ubuf[32 * j + l] = 1.f;
    __syncwarp();
    const float2 *u2 = reinterpret_cast<const float2 *>(&sm.ubuf[32 * j]);
    float w[4] = {kRNorm, kRNorm, kRNorm, kRNorm};  // 1 / r for this thread's 4 tokens
    float rt[4] = {0.f, 0.f, 0.f, 0.f};   // r for this thread's 4 tokens (0: scale 1, kRUnit in X's frame)
    float cd = 1.f;                       // c of channel 32j + l (lane-owned, gauged)
    float g = 1.f;                        // gauge factor of the last column step

    for (int sw = 0; sw < sweeps; ++sw) {
        // row step, pass 1: mean over the D channels of z = X u
        {
            float2 s1[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
            for (int k = 0; k < 16; k += 2) {
                const float4 u4 = reinterpret_cast<const float4 *>(u2)[k >> 1];  // one broadcast read, two pairs
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    s1[r] = __ffma2_rn(X[r][k], f2(u4.x, u4.y), s1[r]);
                    s1[r] = __ffma2_rn(X[r][k + 1], f2(u4.z, u4.w), s1[r]);
                }
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) sm.part[0][j][t0 + 32 * r] = s1[r].x + s1[r].y;
        }
        __syncthreads();
        float mean[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            float S1 = 0.f;
#pragma unroll
            for (int jj = 0; jj < W; ++jj) S1 += sm.part[0][jj][t0 + 32 * r];
            mean[r] = S1 * (1.f / D);
        }
        // row step, pass 2: mean square deviation from that mean
        {
            float2 s2[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
            for (int k = 0; k < 16; k += 2) {
                const float4 u4 = reinterpret_cast<const float4 *>(u2)[k >> 1];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const float2 e = __ffma2_rn(X[r][k], f2(u4.x, u4.y), f2(-mean[r], -mean[r]));
                    const float2 e1 = __ffma2_rn(X[r][k + 1], f2(u4.z, u4.w), f2(-mean[r], -mean[r]));
                    s2[r] = __ffma2_rn(e, e, s2[r]);
                    s2[r] = __ffma2_rn(e1, e1, s2[r]);
                }
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) sm.part[1][j][t0 + 32 * r] = s2[r].x + s2[r].y;
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            float S2 = 0.f;
#pragma unroll
            for (int jj = 0; jj < W; ++jj) S2 += sm.part[1][jj][t0 + 32 * r];
            const float var = S2 * (1.f / D);
            const bool nz = var > kZeroVarRel * fmaf(mean[r], mean[r], var);
            const float is = rsqrtf(var);
            w[r] = nz ? is : kRNorm;      // 1 / r_t
            rt[r] = nz ? var * is : 0.f;  // r_t = sqrt(var); 0 marks a zero-variance row (scale 1)
        }
        // column step: c_d = std over the 128 tokens of z = X / r, on values
        // shifted by token 0's z (lane 0, r = 0: qtok(0) = 0) for precision
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
                const float4 kv4 = reinterpret_cast<const float4 *>(&sm.kbuf[32 * j])[k >> 1];
                const float2 nk = (k & 1) ? f2(-kv4.z, -kv4.w) : f2(-kv4.x, -kv4.y);
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
        }
    }
    // last gauge on the token scales: r <- r g (a zero-variance row keeps 1)
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        rt[r] = rt[r] > 0.f ? rt[r] * g : kRUnit;
        w[r] = 1.f / rt[r];
    }
    __syncthreads();  // every warp is done with the shared transposes

    // ---- 3. 2-bit asymmetric round-to-nearest per (token, group) ----------
    // Codes go to the record in the fragment order the decode kernel reads
    // (see kvarn.h).  K: the 4 codes of channels 8x + 2*tig + half (x = 0..3)
    // of one token fill one byte.  V: the codes of one channel for this
    // thread's 4 tokens (qtok(l) + 32r) fill one byte.
    unsigned char *rec = sm.u.rec;
    // Codes are read from the low mantissa bits of lev = 1.5*2^23 + code, whose
    // bit pattern is 0x4B400000 + code: multiply-adding the raw patterns with the
    // code weights and subtracting the pattern's share once packs them.
    uint32_t vacc[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};  // V: channel i in byte i%4 of vacc[i/4]
    // Z = X u = Y r_t, in place
#pragma unroll
    for (int k = 0; k < 16; k += 2) {
        const float4 u4 = reinterpret_cast<const float4 *>(u2)[k >> 1];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            X[r][k] = __fmul2_rn(X[r][k], f2(u4.x, u4.y));
            X[r][k + 1] = __fmul2_rn(X[r][k + 1], f2(u4.z, u4.w));
        }
    }
    float gs[4], gm[4];  // this group's s and m in Y units, before the token gauge
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int t = t0 + 32 * r;
        float2 (&z)[16] = X[r];
        float mn = INFINITY, mx = -INFINITY;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
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
            rec[v_code_bit(t0, 32 * j + i) / 8] = (unsigned char)(vacc[i >> 2] >> (8 * (i & 3)));
    }
    __syncthreads();  // every group's largest |Y| is in
    // Token gauge: r_t times the token's (s, m) is what dequantises; when the
    // token's largest |Y| reaches 2^14, the power of two 2^k with k =
    // floor(log2 max|Y|) - 13 moves from (s, m) into r_t (exact: codes and
    // products unchanged), which keeps s and m inside binary16.
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int t = t0 + 32 * r;
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
        const float rr = rt[r] * tg * kRNorm;
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
