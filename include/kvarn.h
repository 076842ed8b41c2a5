/*
 * kvarn.h -- C ABI of the KVarN hot path on B200 (sm_100a).
 *
 * KVarN ("KVarN: Variance-Normalized KV-Cache Quantization Mitigates Error
 * Accumulation in Reasoning Tasks") stores the KV cache in 2 bits.  Each
 * block of K and of V is (1) rotated along the channel axis with a Hadamard
 * transform (rndamp.com article, "How It Works", item 1; abstract), (2)
 * variance-normalised along both axes by an iterative row / column balancing
 * that yields a scale per token r_t and a scale per channel c_d ("How It
 * Works", item 2; abstract), and (3) quantised to 2-bit codes with a
 * per-group step and minimum (abstract: 2-bit precision).  Decode attention
 * reads the packed cache and dequantises it in registers with both scales
 * fused ("Numbers": the second scale fused into the dequantisation kernel),
 * scoring against the Hadamard-rotated query.
 *
 * Parameters the pages leave open and this library fixes: 128-token blocks,
 * 4 normalisation sweeps, groups of 32 contiguous channels of one token,
 * binary16 scales, a residual tail of not-yet-quantised tokens kept in the
 * input dtype (bf16 or fp32).
 *
 * Conventions for every call:
 *  - All buffers are caller-owned DEVICE memory unless stated otherwise; the
 *    library never allocates, frees or synchronises.  Pointers must be 16-byte
 *    aligned and tensors densely packed (row-major, last index fastest).
 *  - Every call is asynchronous on `stream` (a cudaStream_t passed as void*,
 *    NULL = legacy default stream).
 *  - Return value: KVARN_OK (0) or a negative KVARN_E* code.  Argument errors
 *    are detected on the host before anything is launched.  Conditions only
 *    the device can see (cache capacity exceeded, a scale that overflows
 *    binary16, a length above max_tokens) are OR-ed into *cache->status as
 *    KVARN_STATUS_* bits; the caller reads that word when it chooses.
 *  - Calls on different caches may run concurrently on different streams.
 *    Calls on the same cache must be ordered (same stream, or events).
 */
#ifndef KVARN_H
#define KVARN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KVARN_API __attribute__((visibility("default")))
#else
#define KVARN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- return codes ---------------------------------------------------- */
#define KVARN_OK            0
#define KVARN_EINVAL       (-1)  /* null pointer, misalignment, bad size    */
#define KVARN_EUNSUPPORTED (-2)  /* valid but not built: D, group, hadamard */
#define KVARN_EWORKSPACE   (-3)  /* decode workspace too small              */
#define KVARN_ECUDA        (-4)  /* a CUDA launch or runtime call failed    */

/* ---- device status bits (OR-ed into *kvarn_cache.status) ------------- */
#define KVARN_STATUS_CAPACITY  1  /* append needed block >= max_blocks     */
#define KVARN_STATUS_NONFINITE 2  /* a scale rounded to inf/nan in binary16 */
#define KVARN_STATUS_LENGTH    4  /* n_tokens[s] > max_tokens at decode     */
#define KVARN_STATUS_TIMEOUT   8  /* a staged copy did not arrive within  */
                                  /* 2 s; the affected partial is dropped   */

typedef enum { KVARN_F32 = 0, KVARN_BF16 = 1 } kvarn_dtype;

/*
 * Shape and method parameters of one cache (one model layer).
 *   head_dim      D: 64, 96 or 128.
 *   block_tokens  tokens per quantised block; 128.
 *   group         channels per quantisation group; 32 (must divide D).
 *   hadamard      Hadamard block along the channels: D (one rotation of the
 *                 whole head), 32 (block-diagonal, e.g. 3 x 32 at D = 96),
 *                 64, or 0 (no rotation).  Power of two, divides D.
 *   sweeps        row+column normalisation sweeps, 0..16; 4.  0 = no
 *                 normalisation (r = c = 1): plain group-wise RTN.
 *   max_blocks    capacity: quantised blocks per (sequence, kv head).
 *   dtype         kvarn_dtype of K, V, q and of the residual tail.
 */
typedef struct {
    int32_t num_seqs;
    int32_t num_kv_heads;
    int32_t head_dim;
    int32_t block_tokens;
    int32_t group;
    int32_t hadamard;
    int32_t sweeps;
    int32_t max_blocks;
    int32_t dtype;
} kvarn_config;

/*
 * The cache of one layer.  All members are device pointers.
 *
 * k_records, v_records: [num_seqs][num_kv_heads][max_blocks] block records of
 *   kvarn_record_bytes(cfg) bytes each.  A record holds, for one block of
 *   T = block_tokens tokens and D channels (G = D/group groups):
 *     codes    T*D/4 bytes of 2-bit codes (0..3), in the fragment order below
 *     s        T*G binary16 steps, token-major: s[t*G + g]
 *     m        T*G binary16 minima, token-major: m[t*G + g]
 *     r        T binary16 token scales
 *     c        D binary16 channel scales
 *     zero padding to a multiple of 128 bytes.
 *   The dequantised, still rotated value is r_t * c_d * (s * code + m).
 *   Code order.  Every code sits in a 32-bit little-endian word at bit
 *   16*half + 2*pos, 0 <= pos < 8, so that one AND of a word with
 *   0x00030003 << 2*(pos % 4) (after a shift by 8 when pos >= 4) yields two
 *   codes as the two halves of an exact binary16 pair.
 *   K record (token t, channel k):  u = t/16, l = 4*(t%8) + (k%8)/2,
 *     half = k%2, q = k/8, n = (t%16)/8, F = D/64;
 *     q < 8F:  word = n*F + q/8, pos = q%8;  else (D = 96): word = 2F,
 *     pos = q - 8F + 4n;  byte offset of the word = ((u*32 + l)*(D/32) + word)*4.
 *   V record (token t, channel d):  j = d/8, l = 4*(d%8) + (t%8)/2,
 *     half = t%2, a = (t%32)/8, word = a/2, pos = 4*(a%2) + t/32;
 *     byte offset of the word = ((j*32 + l)*2 + word)*4.
 * k_tail, v_tail: [num_seqs][num_kv_heads][block_tokens][D] in cfg->dtype;
 *   tokens n - n % T .. n - 1 of each sequence, unrotated, as given.
 * n_tokens: [num_seqs] int32, tokens held per sequence (blocks then tail).
 * arrive:   [num_seqs] uint32 scratch counters for kvarn_append_token;
 *   zero them once when the cache is created; every call leaves them zero.
 * status:   one int32; KVARN_STATUS_* bits, never cleared by the library.
 */
typedef struct {
    void *k_records;
    void *v_records;
    void *k_tail;
    void *v_tail;
    int32_t *n_tokens;
    uint32_t *arrive;
    int32_t *status;
} kvarn_cache;

/* Bytes of one block record (per tensor), as laid out above. */
KVARN_API size_t kvarn_record_bytes(const kvarn_config *cfg);

/*
 * Bytes of one cache component: part 0 = record area of one tensor
 * (num_seqs * num_kv_heads * max_blocks records), 1 = tail of one tensor,
 * 2 = n_tokens, 3 = arrive, 4 = status.  0 for an invalid cfg or part.
 */
KVARN_API size_t kvarn_cache_bytes(const kvarn_config *cfg, int part);

/*
 * Workspace bytes kvarn_decode_attention needs for num_q_heads query heads
 * on the current device: merge tickets (one uint32 per (sequence, kv head),
 * padded to 256 bytes), then partial results -- one per (warp, sequence x kv
 * head) segment of the persistent grid (at most SMs x warps per CTA + units)
 * and four per unit for the slots of its residual tail, each grp x (D + 4)
 * fp32.  The size
 * depends on the device's SM count: query it on the device that runs the
 * decode.  Zero the workspace once (e.g. cudaMemsetAsync) before its first
 * use; every decode call leaves the tickets zero again, so one workspace
 * serves any number of calls that are ordered on the GPU.
 */
KVARN_API size_t kvarn_decode_workspace_bytes(const kvarn_config *cfg, int num_q_heads);

/*
 * Bulk quantisation (prefill) of num_tokens tokens per sequence, written as
 * tokens first_block*T .. first_block*T + num_tokens - 1:
 *   k, v  [num_seqs][num_kv_heads][num_tokens][D] in cfg->dtype.
 * Source: the abstract (Hadamard rotation, dual-scaling variance
 * normalisation across the token and channel axes of K and V, 2-bit
 * codes) and the rndamp.com article, "How It Works", items 1 (Hadamard
 * transform in the channel dimension) and 2 (iterative balancing of rows
 * and columns until the variance is close to uniform).
 * Full blocks go through rotation -> normalisation -> 2-bit packing into
 * record slots first_block, first_block+1, ...; the last num_tokens % T
 * tokens are copied, unrotated, into the tail; n_tokens[s] is set to
 * first_block*T + num_tokens.  Needs first_block + floor(num_tokens/T) <=
 * max_blocks, and num_seqs*num_kv_heads*(floor(num_tokens/T) + 1) <= INT_MAX
 * (one CTA per block and tail; KVARN_EINVAL otherwise).
 * debug_k / debug_v: NULL, or fp32 buffers of
 *   num_seqs*num_kv_heads*(num_tokens/T) * (T + D + 2*T*(D/group)) floats
 *   receiving, per block, the unrounded r[T], c[D], s[T][D/group],
 *   m[T][D/group] (for parity tests).
 */
KVARN_API int kvarn_quantize_blocks(const kvarn_config *cfg, const void *k, const void *v,
                          int num_tokens, int first_block, const kvarn_cache *cache,
                          float *debug_k, float *debug_v, void *stream);

/*
 * Source: the abstract (the cache grows with every decoded token in
 * long-horizon decoding) and the rndamp.com article, "How It Works" (each
 * full block is rotated, normalised and coded as in kvarn_quantize_blocks).
 * Append one token per sequence (k, v: [num_seqs][num_kv_heads][D]) at
 * position n_tokens[s].  The token goes into tail slot n % T; when that fills
 * the tail, the tail is quantised into record n / T in the same launch.
 * n_tokens[s] is then advanced by one.  If that record slot is >= max_blocks
 * nothing is written for that sequence and KVARN_STATUS_CAPACITY is set.
 */
KVARN_API int kvarn_append_token(const kvarn_config *cfg, const void *k, const void *v,
                       const kvarn_cache *cache, void *stream);

/*
 * Source: the abstract (decode attention over the 2-bit cache, which is
 * what bounds long-horizon decoding) and the rndamp.com article, "Numbers"
 * (the second scale is fused into the dequantisation inside the attention
 * kernel); the query is rotated like the keys ("How It Works", item 1: the
 * rotation is orthogonal, so q . k is unchanged).
 * Single-token decode attention over the whole cache:
 *   q    [num_seqs][num_q_heads][D] in cfg->dtype, unrotated;
 *   out  [num_seqs][num_q_heads][D] fp32, unrotated;
 *   out_h = sum_t softmax_t(softmax_scale * q_h . k_t) v_t over the
 *   n_tokens[s] cached tokens (dequantised blocks, then the tail).
 * Query head h reads kv head h / (num_q_heads / num_kv_heads); num_q_heads
 * must be a multiple of num_kv_heads, at most 8 query heads per kv head.
 * softmax_scale <= 0 selects 1/sqrt(D).  max_tokens is an upper bound on
 * every n_tokens[s]: the work is split evenly over the warps of one CTA per
 * SM as if every sequence held max_tokens tokens, so the closer the bound,
 * the better the balance.  A sequence longer than that sets
 * KVARN_STATUS_LENGTH and is cut to it.
 * A sequence with n_tokens 0 gets zeros.
 */
KVARN_API int kvarn_decode_attention(const kvarn_config *cfg, const void *q, int num_q_heads,
                           float softmax_scale, const kvarn_cache *cache, int max_tokens,
                           float *out, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Decode attention for several query tokens per sequence at once (draft
 * tokens being verified, or a short chunk), the step next to single-token
 * decode.  The queries are the last num_queries tokens already appended to
 * the cache: for a sequence holding n tokens, query i (0-based) sits at
 * position n - num_queries + i and attends positions 0 .. n - num_queries + i.
 *   q    [num_seqs][num_queries][num_q_heads][D] in cfg->dtype, unrotated;
 *   out  [num_seqs][num_queries][num_q_heads][D] fp32, unrotated.
 * The num_queries x (num_q_heads / num_kv_heads) rows that share a kv head
 * read its blocks once and fill the tensor-core tiles together; that count
 * must be 1, 2, 4 or 8 (KVARN_EUNSUPPORTED otherwise).  Everything else --
 * softmax_scale, max_tokens, status, empty sequences -- is as in
 * kvarn_decode_attention; the workspace is
 * kvarn_decode_workspace_bytes(cfg, num_queries * num_q_heads) bytes.  A
 * query before position 0 (n < num_queries) gets zeros.
 */
KVARN_API int kvarn_decode_attention_multi(const kvarn_config *cfg, const void *q, int num_q_heads,
                                           int num_queries, float softmax_scale, const kvarn_cache *cache,
                                           int max_tokens, float *out, void *workspace, size_t workspace_bytes,
                                           void *stream);

/*
 * Self-test of the decode kernel's bounded waits (an engineering check; the
 * method has no counterpart).  Runs kvarn_decode_attention with every warp's
 * first K record copy withheld and each staged-record wait limited to 1 ms
 * of the global timer (the normal limit is 2 s).  The launch must end -- not
 * hang -- with KVARN_STATUS_TIMEOUT OR-ed into *cache->status; the outputs
 * are not meaningful.  Afterwards the context and the cache stay usable: a
 * normal decode on the same cache gives its usual result.  Arguments and
 * errors as kvarn_decode_attention (softmax scale 1/sqrt(D)).
 */
KVARN_API int kvarn_decode_selftest_timeout(const kvarn_config *cfg, const void *q, int num_q_heads,
                                            const kvarn_cache *cache, int max_tokens, float *out, void *workspace,
                                            size_t workspace_bytes, void *stream);

/*
 * Quantisation error of stored blocks, per token, split into magnitude and
 * direction (article on KVarN, "The Problem": the errors that compound in
 * K are those of the token magnitudes, not of the directions; "How It
 * Works": the dual scaling is there to cut the magnitude part).  Compares
 * the original rows
 *   k, v  [num_seqs][num_kv_heads][num_tokens][D] in cfg->dtype (the rows
 *         kvarn_quantize_blocks was given), num_tokens a multiple of T,
 * with records first_block .. first_block + num_tokens/T - 1, and writes
 *   err_k, err_v [num_seqs][num_kv_heads][num_tokens][2] fp32:
 *   (|norm(x^)/norm(x) - 1|, 1 - cos(x^, x)) per token; a zero row gives (0, 0).
 * Both quantities are invariant under the rotation, so x is rotated as the
 * quantiser rotates it and x^ = r c (s code + m) from the stored binary16
 * scales.  Useful with cfg->hadamard = 0 or cfg->sweeps = 0 to measure what
 * each stage removes.  Errors: KVARN_EINVAL for a ragged num_tokens, a block
 * range beyond max_blocks, num_seqs*num_kv_heads*num_tokens/T above INT_MAX,
 * or a NULL / unaligned pointer.
 */
KVARN_API int kvarn_token_errors(const kvarn_config *cfg, const void *k, const void *v, int num_tokens,
                                 int first_block, const kvarn_cache *cache, float *err_k, float *err_v,
                                 void *stream);

/*
 * Source: the rndamp.com article, "Numbers" (each value is rebuilt from its
 * code with both scales, r_t c_d (s code + m)) and "How It Works", item 1
 * (the rotation is its own inverse once normalised).
 * Dequantise records first_block .. first_block+num_blocks-1 of every
 * (sequence, kv head) into fp32 k_out / v_out
 * [num_seqs][num_kv_heads][num_blocks*T][D]; rotated != 0 keeps the rotated
 * basis, rotated == 0 rotates back.  Either output may be NULL.  Errors:
 * KVARN_EINVAL for a block range outside 0 .. max_blocks, or
 * num_seqs*num_kv_heads*num_blocks above INT_MAX.
 */
KVARN_API int kvarn_dequantize(const kvarn_config *cfg, const kvarn_cache *cache, int first_block,
                     int num_blocks, int rotated, float *k_out, float *v_out, void *stream);

/*
 * kvarn_decode_attention without a workspace argument, for callers that
 * cannot allocate device memory where they run decode (code running inside a
 * host callback or another runtime's allocator, or a process that must not
 * grow its device footprint after start-up).  There is no counterpart on the
 * pages: this is a deployment variant of the same kernel.
 * The workspace is a 16 MiB array that this library holds in device memory
 * on every GPU that loads it, until the process exits; a call whose
 * kvarn_decode_workspace_bytes(cfg, num_q_heads) exceeds 16 MiB returns
 * KVARN_EWORKSPACE.  Nothing is allocated or freed.
 * The first call in a CUDA context looks up the array's device address in
 * that context (with it current) and caches it for that context; make that
 * first call before any stream capture.  The cache is keyed by the driver's
 * context id, so other contexts on the same device, and a context created
 * again after cudaDeviceReset, get their own lookup.  Every
 * call clears the array's combine tickets on `stream` and then uses the
 * array, so calls whose work overlaps on the GPU (any two streams, any two
 * threads) race with each other: order them.  Arguments and results are as
 * for kvarn_decode_attention.
 */
KVARN_API int kvarn_decode_attention_noalloc(const kvarn_config *cfg, const void *q, int num_q_heads,
                                             float softmax_scale, const kvarn_cache *cache,
                                             int max_tokens, float *out, void *stream);

/* Static text for a KVARN_* return code. */
KVARN_API const char *kvarn_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* KVARN_H */
