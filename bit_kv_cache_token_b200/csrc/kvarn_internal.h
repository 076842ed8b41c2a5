// kvarn_internal.h -- launch argument blocks passed from the C ABI layer to
// the kernels (by value, in kernel parameter space).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "kvarn.h"

namespace kvarn {

struct QuantArgs {
    const void *k, *v;          // [S][Hkv][num_tokens][D]
    void *k_records, *v_records;
    void *k_tail, *v_tail;
    int32_t *n_tokens;
    int32_t *status;
    float *debug_k, *debug_v;
    int num_tokens, first_block, max_blocks, num_kv_heads, sweeps;
};

struct AppendArgs {
    const void *k, *v;          // [S][Hkv][D]
    void *k_records, *v_records;
    void *k_tail, *v_tail;
    int32_t *n_tokens;
    uint32_t *arrive;
    int32_t *status;
    int max_blocks, num_kv_heads, sweeps;
};

struct DequantArgs {
    const void *k_records, *v_records;
    float *k_out, *v_out;
    int first_block, num_blocks, max_blocks, rotated;
};

struct DecodeArgs {
    const void *q;              // [S][Hq][D]
    const void *k_records, *v_records;
    const void *k_tail, *v_tail;
    const int32_t *n_tokens;
    int32_t *status;
    float *out;                 // [S][Hq][D]
    float *partials;            // [warps + units][grp][D+4]: one per (warp, unit) segment, at warp + unit
    float *tail_partials;       // [units][kDecodeTailSlots][grp][D+4]
    uint32_t *tickets;          // [units], zero between calls
    float scale_log2;           // softmax scale * log2(e)
    int num_kv_heads, grp, max_blocks, max_tokens;
    int num_units;              // S * Hkv
    // Several query tokens per sequence: grp = num_queries * heads_per_kv rows
    // share a kv head; row v is query v / heads_per_kv of head v % heads_per_kv.
    // q and out are [S][num_queries][Hq][D]; query i of a sequence with n
    // tokens sits at position n - num_queries + i and sees positions <= it.
    int num_queries, heads_per_kv;
    // Bounded waits: limit per staged-record wait in ns (0 = the default) and,
    // for the self-test only, a flag that withholds each segment's first K copy.
    unsigned long long wait_ns;
    int withhold_first_k;
};

struct ErrorArgs {
    const void *k, *v;          // [S][Hkv][num_blocks * T][D], the rows that were quantised
    const void *k_records, *v_records;
    float *err_k, *err_v;       // [S][Hkv][num_blocks * T][2]: magnitude, direction
    int num_blocks, first_block, max_blocks;
};

cudaError_t run_quantize(const kvarn_config &c, const QuantArgs &a, cudaStream_t st);
cudaError_t run_token_errors(const kvarn_config &c, const ErrorArgs &a, cudaStream_t st);
cudaError_t run_append(const kvarn_config &c, const AppendArgs &a, cudaStream_t st);
cudaError_t run_dequantize(const kvarn_config &c, const DequantArgs &a, cudaStream_t st);
cudaError_t run_decode(const kvarn_config &c, const DecodeArgs &a, int ctas, cudaStream_t st);
cudaError_t run_set_length(int32_t *n_tokens, int num_seqs, int value, cudaStream_t st);

// Item slots of a unit's residual tail in the decode work list, 32 tokens each.
constexpr int kDecodeTailSlots = 4;

// Warps per decode CTA (one CTA per SM by shared memory).
int decode_warps_per_cta(int head_dim, int grp);

// Bytes of one decode partial (grp heads x (m, l, pad, pad, o[D])).
size_t decode_slot_bytes(int head_dim, int grp);

}  // namespace kvarn
