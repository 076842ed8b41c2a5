// quantize.cu -- bulk quantisation (prefill) and append-with-quantise kernels.
#include "kvarn_internal.h"
#include "quantize_block.cuh"

namespace kvarn {

// Load a block and quantise it: bf16 blocks are rotated on the tensor cores,
// fp32 blocks on the CUDA cores.
template <int D, int HB, typename Tin, bool COHERENT>
__device__ __forceinline__ void load_quantize(const Tin *src, QuantSmem<D> &sm, int tensor, int sweeps,
                                              unsigned char *rec, float *dbg, int32_t *status)
{
    float2 X[4][16];
    if constexpr (sizeof(Tin) == 2) {
        load_rotate_tc<D, HB>(src, X, sm);  // reads through L2: coherent either way
        if (tensor) quantize_block<D, HB, 1, true>(X, sm, sweeps, rec, dbg, status);
        else quantize_block<D, HB, 0, true>(X, sm, sweeps, rec, dbg, status);
    } else {
        load_block<D, Tin, COHERENT>(src, X);
        if (tensor) quantize_block<D, HB, 1>(X, sm, sweeps, rec, dbg, status);
        else quantize_block<D, HB, 0>(X, sm, sweeps, rec, dbg, status);
    }
}

// One CTA per (sequence, kv head, block) and per tensor (blockIdx.y: 0 = K,
// 1 = V).  Block index nb (one past the full blocks) copies the ragged tail.
// 12 warps per SM: the register cap (168) spills a few words of the 128-float
// block a thread holds, yet the extra warps hide more of the dependent
// arithmetic's latency than the spills cost.
template <int D, int HB, typename Tin>
__global__ void __launch_bounds__(D, 384 / D)
quantize_blocks_kernel(QuantArgs a)
{
    QuantSmem<D> &sm = quant_smem<D>();
    const int nb = a.num_tokens / kBlockTokens;
    const int rem = a.num_tokens % kBlockTokens;
    const int nbx = nb + (rem > 0 ? 1 : 0);
    const int b = blockIdx.x % nbx;
    const int sh = blockIdx.x / nbx;  // s * Hkv + h
    const int tensor = blockIdx.y;
    const Tin *src = static_cast<const Tin *>(tensor ? a.v : a.k) +
                     (size_t)sh * a.num_tokens * D + (size_t)b * kBlockTokens * D;

    if (b == 0 && tensor == 0 && (sh % a.num_kv_heads) == 0 && threadIdx.x == 0)
        a.n_tokens[sh / a.num_kv_heads] = a.first_block * kBlockTokens + a.num_tokens;

    if (b == nb) {  // residual tail: copied as given, unrotated
        Tin *tail = static_cast<Tin *>(tensor ? a.v_tail : a.k_tail) + (size_t)sh * kBlockTokens * D;
        copy_elems(tail, src, rem * D, threadIdx.x, D);
        return;
    }
    const size_t slot = (size_t)sh * a.max_blocks + a.first_block + b;
    unsigned char *rec = static_cast<unsigned char *>(tensor ? a.v_records : a.k_records) +
                         slot * Record<D>::kBytes;
    float *dbg = tensor ? a.debug_v : a.debug_k;
    if (dbg) dbg += ((size_t)sh * nb + b) * (kBlockTokens + D + 2 * kBlockTokens * (D / kGroup));
    load_quantize<D, HB, Tin, false>(src, sm, tensor, a.sweeps, rec, dbg, a.status);
}

// One CTA per (sequence, kv head) and per tensor.  The token goes into tail
// slot n % T; if that completes the tail, the CTA quantises the tail into
// record n / T.  The last CTA of a sequence to finish advances n_tokens[s]
// (arrival counter, no waiting).
template <int D, int HB, typename Tin>
__global__ void __launch_bounds__(D, 2)
append_kernel(AppendArgs a)
{
    grid_dep_wait();  // the previous kernel in the stream (a decode, say) has completed
    QuantSmem<D> &sm = quant_smem<D>();
    __shared__ int s_n;
    const int sh = blockIdx.x;  // s * Hkv + h
    const int s = sh / a.num_kv_heads;
    const int tensor = blockIdx.y;
    if (threadIdx.x == 0) s_n = *reinterpret_cast<volatile int32_t *>(a.n_tokens + s);
    __syncthreads();
    const int n = s_n;
    const int pos = n % kBlockTokens, blk = n / kBlockTokens;
    const bool fills = pos == kBlockTokens - 1;
    const bool full = fills && blk >= a.max_blocks;

    if (!full) {
        Tin *tail = static_cast<Tin *>(tensor ? a.v_tail : a.k_tail) + (size_t)sh * kBlockTokens * D;
        const Tin *tok = static_cast<const Tin *>(tensor ? a.v : a.k) + (size_t)sh * D;
        copy_elems(tail + (size_t)pos * D, tok, D, threadIdx.x, D);
        if (fills) {
            __syncthreads();  // the new row is visible to the whole CTA
            unsigned char *rec = static_cast<unsigned char *>(tensor ? a.v_records : a.k_records) +
                                 ((size_t)sh * a.max_blocks + blk) * Record<D>::kBytes;
            // row pos was just written by this CTA: read the tail through L2
            load_quantize<D, HB, Tin, true>(tail, sm, tensor, a.sweeps, rec, nullptr, a.status);
        }
    } else if (threadIdx.x == 0 && tensor == 0 && (sh % a.num_kv_heads) == 0) {
        status_or(a.status, KVARN_STATUS_CAPACITY);
    }
    __syncthreads();
    // Arrival: the last of the sequence's 2 * Hkv CTAs advances its length.  It
    // only has to come after every CTA has read the old length (each read it
    // before arriving); what the CTAs wrote is read by later launches, which
    // the kernel boundary orders, so no fence is needed here.
    if (threadIdx.x == 0) {
        const unsigned prev = atomicAdd(a.arrive + s, 1u);
        if (prev == 2u * a.num_kv_heads - 1u) {
            a.arrive[s] = 0u;
            if (!full) a.n_tokens[s] = n + 1;
        }
    }
}

template <int D, int HB, typename Tin>
static cudaError_t launch_quant(const QuantArgs &a, int S, int Hkv, cudaStream_t st)
{
    const int nb = a.num_tokens / kBlockTokens;
    const int nbx = nb + (a.num_tokens % kBlockTokens ? 1 : 0);
    if (nbx == 0) return cudaSuccess;
    dim3 grid((unsigned)(S * Hkv * nbx), 2);
    constexpr int kSmem = (int)sizeof(QuantSmem<D>);
    const cudaError_t e =
        cudaFuncSetAttribute(quantize_blocks_kernel<D, HB, Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    // the largest shared-memory carveout, so that three CTAs fit on an SM
    cudaFuncSetAttribute(quantize_blocks_kernel<D, HB, Tin>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    quantize_blocks_kernel<D, HB, Tin><<<grid, D, kSmem, st>>>(a);
    return cudaGetLastError();
}

template <int D, int HB, typename Tin>
static cudaError_t launch_append(const AppendArgs &a, int S, int Hkv, cudaStream_t st)
{
    dim3 grid((unsigned)(S * Hkv), 2);
    constexpr int kSmem = (int)sizeof(QuantSmem<D>);
    const cudaError_t e =
        cudaFuncSetAttribute(append_kernel<D, HB, Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    // the largest shared-memory carveout, so that three CTAs fit on an SM
    cudaFuncSetAttribute(append_kernel<D, HB, Tin>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    const cudaError_t el = launch_overlapped(append_kernel<D, HB, Tin>, grid, dim3(D), (size_t)kSmem, st, a);
    return el != cudaSuccess ? el : cudaGetLastError();
}

// ---- dispatch over (D, Hadamard block, dtype) ---------------------------
#define KVARN_DISPATCH_HB(D, HB, FN, ...)                                            \
    (dtype == KVARN_BF16 ? FN<D, HB, __nv_bfloat16>(__VA_ARGS__) : FN<D, HB, float>(__VA_ARGS__))

template <int D>
static cudaError_t dispatch_quant(int hb, int dtype, const QuantArgs &a, int S, int Hkv, cudaStream_t st)
{
    switch (hb) {
    case 0: return KVARN_DISPATCH_HB(D, 0, launch_quant, a, S, Hkv, st);
    case 32: return KVARN_DISPATCH_HB(D, 32, launch_quant, a, S, Hkv, st);
    case 64: if constexpr (D % 64 == 0) return KVARN_DISPATCH_HB(D, 64, launch_quant, a, S, Hkv, st); break;
    case 128: if constexpr (D % 128 == 0) return KVARN_DISPATCH_HB(D, 128, launch_quant, a, S, Hkv, st); break;
    }
    return cudaErrorInvalidValue;
}

template <int D>
static cudaError_t dispatch_append(int hb, int dtype, const AppendArgs &a, int S, int Hkv, cudaStream_t st)
{
    switch (hb) {
    case 0: return KVARN_DISPATCH_HB(D, 0, launch_append, a, S, Hkv, st);
    case 32: return KVARN_DISPATCH_HB(D, 32, launch_append, a, S, Hkv, st);
    case 64: if constexpr (D % 64 == 0) return KVARN_DISPATCH_HB(D, 64, launch_append, a, S, Hkv, st); break;
    case 128: if constexpr (D % 128 == 0) return KVARN_DISPATCH_HB(D, 128, launch_append, a, S, Hkv, st); break;
    }
    return cudaErrorInvalidValue;
}

__global__ void set_length_kernel(int32_t *n_tokens, int num_seqs, int value)
{
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < num_seqs; i += gridDim.x * blockDim.x) n_tokens[i] = value;
}

cudaError_t run_set_length(int32_t *n_tokens, int num_seqs, int value, cudaStream_t st)
{
    set_length_kernel<<<(num_seqs + 255) / 256, 256, 0, st>>>(n_tokens, num_seqs, value);
    return cudaGetLastError();
}

cudaError_t run_quantize(const kvarn_config &c, const QuantArgs &a, cudaStream_t st)
{
    switch (c.head_dim) {
    case 64: return dispatch_quant<64>(c.hadamard, c.dtype, a, c.num_seqs, c.num_kv_heads, st);
    case 96: return dispatch_quant<96>(c.hadamard, c.dtype, a, c.num_seqs, c.num_kv_heads, st);
    case 128: return dispatch_quant<128>(c.hadamard, c.dtype, a, c.num_seqs, c.num_kv_heads, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t run_append(const kvarn_config &c, const AppendArgs &a, cudaStream_t st)
{
    switch (c.head_dim) {
    case 64: return dispatch_append<64>(c.hadamard, c.dtype, a, c.num_seqs, c.num_kv_heads, st);
    case 96: return dispatch_append<96>(c.hadamard, c.dtype, a, c.num_seqs, c.num_kv_heads, st);
    case 128: return dispatch_append<128>(c.hadamard, c.dtype, a, c.num_seqs, c.num_kv_heads, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace kvarn
