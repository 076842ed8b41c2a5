// kvarn_api.cu -- the extern "C" boundary: validation, sizes, launches.
#include <limits.h>
#include <math.h>
#include <stdint.h>

#include "kvarn_common.cuh"
#include "kvarn_internal.h"

using namespace kvarn;

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape / method checks shared by every call.  EUNSUPPORTED for well-formed
// parameters the library has no kernel for, EINVAL for malformed ones.
int check_config(const kvarn_config *c)
{
    if (!c) return KVARN_EINVAL;
    if (c->num_seqs < 1 || c->num_kv_heads < 1 || c->max_blocks < 0) return KVARN_EINVAL;
    if ((long long)c->num_seqs * c->num_kv_heads > (1LL << 24)) return KVARN_EINVAL;
    if (c->dtype != KVARN_F32 && c->dtype != KVARN_BF16) return KVARN_EINVAL;
    if (c->sweeps < 0 || c->sweeps > 16) return KVARN_EINVAL;
    if (c->head_dim <= 0 || c->block_tokens <= 0 || c->group <= 0) return KVARN_EINVAL;
    if (c->head_dim % c->group) return KVARN_EINVAL;
    if (c->hadamard < 0 || (c->hadamard && (c->hadamard & (c->hadamard - 1)))) return KVARN_EINVAL;
    if (c->hadamard && c->head_dim % c->hadamard) return KVARN_EINVAL;
    if (c->head_dim != 64 && c->head_dim != 96 && c->head_dim != 128) return KVARN_EUNSUPPORTED;
    if (c->block_tokens != kBlockTokens || c->group != kGroup) return KVARN_EUNSUPPORTED;
    if (c->hadamard != 0 && c->hadamard < 32) return KVARN_EUNSUPPORTED;
    return KVARN_OK;
}

int check_cache(const kvarn_cache *k, bool need_arrive)
{
    if (!k) return KVARN_EINVAL;
    if (!k->k_records || !k->v_records || !k->k_tail || !k->v_tail || !k->n_tokens || !k->status)
        return KVARN_EINVAL;
    if (need_arrive && !k->arrive) return KVARN_EINVAL;
    if (!aligned16(k->k_records) || !aligned16(k->v_records) || !aligned16(k->k_tail) || !aligned16(k->v_tail))
        return KVARN_EINVAL;
    return KVARN_OK;
}

size_t elem_size(const kvarn_config *c) { return c->dtype == KVARN_BF16 ? 2 : 4; }

int num_sms()
{
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? KVARN_OK : KVARN_ECUDA; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// One CTA per (sequence, kv head, block): the grid's x extent must fit an int.
bool grid_fits(const kvarn_config *c, long long blocks_per_unit)
{
    return (long long)c->num_seqs * c->num_kv_heads * blocks_per_unit <= INT_MAX;
}

size_t ticket_bytes(const kvarn_config *c)
{
    return align_up((size_t)c->num_seqs * c->num_kv_heads * sizeof(uint32_t), 256);
}

}  // namespace

extern "C" {

size_t kvarn_record_bytes(const kvarn_config *cfg)
{
    if (check_config(cfg) == KVARN_EINVAL || !cfg) return 0;
    const size_t raw = (size_t)cfg->block_tokens * cfg->head_dim / 4 +
                       (size_t)cfg->block_tokens * (cfg->head_dim / cfg->group) * 4 +
                       2 * (size_t)cfg->block_tokens + 2 * (size_t)cfg->head_dim;
    return align_up(raw, 128);
}

size_t kvarn_cache_bytes(const kvarn_config *cfg, int part)
{
    if (check_config(cfg) == KVARN_EINVAL) return 0;
    const size_t sh = (size_t)cfg->num_seqs * cfg->num_kv_heads;
    switch (part) {
    case 0: return sh * cfg->max_blocks * kvarn_record_bytes(cfg);
    case 1: return sh * cfg->block_tokens * cfg->head_dim * elem_size(cfg);
    case 2: return (size_t)cfg->num_seqs * sizeof(int32_t);
    case 3: return (size_t)cfg->num_seqs * sizeof(uint32_t);
    case 4: return sizeof(int32_t);
    }
    return 0;
}

size_t kvarn_decode_workspace_bytes(const kvarn_config *cfg, int num_q_heads)
{
    if (check_config(cfg) != KVARN_OK || num_q_heads < cfg->num_kv_heads || num_q_heads % cfg->num_kv_heads)
        return 0;
    const int grp = num_q_heads / cfg->num_kv_heads;
    const size_t sh = (size_t)cfg->num_seqs * cfg->num_kv_heads;
    const size_t warps = (size_t)num_sms() * decode_warps_per_cta(cfg->head_dim, grp);
    // tickets, one block partial per (warp, unit) segment (at most warps + units), the tail slots' partials
    return ticket_bytes(cfg) + (warps + sh * (1 + kDecodeTailSlots)) * decode_slot_bytes(cfg->head_dim, grp);
}

int kvarn_quantize_blocks(const kvarn_config *cfg, const void *k, const void *v, int num_tokens,
                          int first_block, const kvarn_cache *cache, float *debug_k, float *debug_v,
                          void *stream)
{
    int rc = check_config(cfg);
    if (rc) return rc;
    if ((rc = check_cache(cache, false))) return rc;
    if (num_tokens < 0 || first_block < 0) return KVARN_EINVAL;
    if (num_tokens > 0 && (!k || !v || !aligned16(k) || !aligned16(v))) return KVARN_EINVAL;
    if ((long long)first_block + num_tokens / cfg->block_tokens > cfg->max_blocks) return KVARN_EINVAL;
    if (!grid_fits(cfg, num_tokens / cfg->block_tokens + 1)) return KVARN_EINVAL;
    if ((debug_k && !aligned16(debug_k)) || (debug_v && !aligned16(debug_v))) return KVARN_EINVAL;
    QuantArgs a;
    a.k = k; a.v = v;
    a.k_records = cache->k_records; a.v_records = cache->v_records;
    a.k_tail = cache->k_tail; a.v_tail = cache->v_tail;
    a.n_tokens = cache->n_tokens; a.status = cache->status;
    a.debug_k = debug_k; a.debug_v = debug_v;
    a.num_tokens = num_tokens; a.first_block = first_block; a.max_blocks = cfg->max_blocks;
    a.num_kv_heads = cfg->num_kv_heads; a.sweeps = cfg->sweeps;
    if (num_tokens == 0)  // nothing to quantise; only the lengths change
        return cuda_status(run_set_length(cache->n_tokens, cfg->num_seqs, first_block * cfg->block_tokens,
                                          static_cast<cudaStream_t>(stream)));
    return cuda_status(run_quantize(*cfg, a, static_cast<cudaStream_t>(stream)));
}

int kvarn_append_token(const kvarn_config *cfg, const void *k, const void *v, const kvarn_cache *cache,
                       void *stream)
{
    int rc = check_config(cfg);
    if (rc) return rc;
    if ((rc = check_cache(cache, true))) return rc;
    if (!k || !v || !aligned16(k) || !aligned16(v)) return KVARN_EINVAL;
    AppendArgs a;
    a.k = k; a.v = v;
    a.k_records = cache->k_records; a.v_records = cache->v_records;
    a.k_tail = cache->k_tail; a.v_tail = cache->v_tail;
    a.n_tokens = cache->n_tokens; a.arrive = cache->arrive; a.status = cache->status;
    a.max_blocks = cfg->max_blocks; a.num_kv_heads = cfg->num_kv_heads; a.sweeps = cfg->sweeps;
    return cuda_status(run_append(*cfg, a, static_cast<cudaStream_t>(stream)));
}

static int decode_impl(const kvarn_config *cfg, const void *q, int num_q_heads, int num_queries,
                       float softmax_scale, const kvarn_cache *cache, int max_tokens, float *out, void *workspace,
                       size_t workspace_bytes, void *stream, unsigned long long wait_ns = 0, int withhold = 0)
{
    int rc = check_config(cfg);
    if (rc) return rc;
    if ((rc = check_cache(cache, false))) return rc;
    if (!q || !out || !aligned16(q) || !aligned16(out)) return KVARN_EINVAL;
    if (num_q_heads < cfg->num_kv_heads || num_q_heads % cfg->num_kv_heads) return KVARN_EINVAL;
    if (num_queries < 1) return KVARN_EINVAL;
    const int hpk = num_q_heads / cfg->num_kv_heads;
    if ((long long)hpk * num_queries > 8) return KVARN_EUNSUPPORTED;
    const int rows = hpk * num_queries;  // rows sharing one kv head
    if (rows != 1 && rows != 2 && rows != 4 && rows != 8) return KVARN_EUNSUPPORTED;
    if (max_tokens < 0 || (long long)max_tokens > (long long)cfg->max_blocks * cfg->block_tokens + cfg->block_tokens - 1)
        return KVARN_EINVAL;
    if (!(softmax_scale == softmax_scale) || isinf(softmax_scale)) return KVARN_EINVAL;
    const size_t need = kvarn_decode_workspace_bytes(cfg, num_q_heads * num_queries);
    if (!workspace || !aligned16(workspace) || workspace_bytes < need) return KVARN_EWORKSPACE;

    // a persistent grid: one CTA of decode_warps_per_cta warps per SM, the
    // item list (blocks and tails of all units) split evenly over the warps
    const int units = cfg->num_seqs * cfg->num_kv_heads;
    const int ctas = num_sms();
    DecodeArgs a;
    a.q = q;
    a.k_records = cache->k_records; a.v_records = cache->v_records;
    a.k_tail = cache->k_tail; a.v_tail = cache->v_tail;
    a.n_tokens = cache->n_tokens; a.status = cache->status;
    a.out = out;
    a.tickets = static_cast<uint32_t *>(workspace);
    a.partials = reinterpret_cast<float *>(static_cast<unsigned char *>(workspace) + ticket_bytes(cfg));
    a.tail_partials = a.partials + ((size_t)ctas * decode_warps_per_cta(cfg->head_dim, rows) + units) *
                                       (decode_slot_bytes(cfg->head_dim, rows) / sizeof(float));
    const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf((float)cfg->head_dim);
    a.scale_log2 = scale * 1.4426950408889634f;
    a.num_kv_heads = cfg->num_kv_heads; a.grp = rows; a.max_blocks = cfg->max_blocks;
    a.max_tokens = max_tokens; a.num_units = units;
    a.num_queries = num_queries; a.heads_per_kv = hpk;
    a.wait_ns = wait_ns; a.withhold_first_k = withhold;
    return cuda_status(run_decode(*cfg, a, ctas, static_cast<cudaStream_t>(stream)));
}

int kvarn_decode_attention(const kvarn_config *cfg, const void *q, int num_q_heads, float softmax_scale,
                           const kvarn_cache *cache, int max_tokens, float *out, void *workspace,
                           size_t workspace_bytes, void *stream)
{
    return decode_impl(cfg, q, num_q_heads, 1, softmax_scale, cache, max_tokens, out, workspace, workspace_bytes,
                       stream);
}

int kvarn_decode_selftest_timeout(const kvarn_config *cfg, const void *q, int num_q_heads, const kvarn_cache *cache,
                                  int max_tokens, float *out, void *workspace, size_t workspace_bytes, void *stream)
{
    // every warp's first K record is withheld and its wait ends after 1 ms
    return decode_impl(cfg, q, num_q_heads, 1, 0.f, cache, max_tokens, out, workspace, workspace_bytes, stream,
                       1000000ull, 1);
}

int kvarn_decode_attention_multi(const kvarn_config *cfg, const void *q, int num_q_heads, int num_queries,
                                 float softmax_scale, const kvarn_cache *cache, int max_tokens, float *out,
                                 void *workspace, size_t workspace_bytes, void *stream)
{
    return decode_impl(cfg, q, num_q_heads, num_queries, softmax_scale, cache, max_tokens, out, workspace,
                       workspace_bytes, stream);
}

int kvarn_token_errors(const kvarn_config *cfg, const void *k, const void *v, int num_tokens, int first_block,
                       const kvarn_cache *cache, float *err_k, float *err_v, void *stream)
{
    int rc = check_config(cfg);
    if (rc) return rc;
    if ((rc = check_cache(cache, false))) return rc;
    if (num_tokens < 0 || num_tokens % cfg->block_tokens || first_block < 0) return KVARN_EINVAL;
    const int nb = num_tokens / cfg->block_tokens;
    if ((long long)first_block + nb > cfg->max_blocks || !grid_fits(cfg, nb)) return KVARN_EINVAL;
    if (nb == 0) return KVARN_OK;
    if (!k || !v || !err_k || !err_v || !aligned16(k) || !aligned16(v) || !aligned16(err_k) || !aligned16(err_v))
        return KVARN_EINVAL;
    ErrorArgs a;
    a.k = k; a.v = v;
    a.k_records = cache->k_records; a.v_records = cache->v_records;
    a.err_k = err_k; a.err_v = err_v;
    a.num_blocks = nb; a.first_block = first_block; a.max_blocks = cfg->max_blocks;
    return cuda_status(run_token_errors(*cfg, a, static_cast<cudaStream_t>(stream)));
}

int kvarn_dequantize(const kvarn_config *cfg, const kvarn_cache *cache, int first_block, int num_blocks,
                     int rotated, float *k_out, float *v_out, void *stream)
{
    int rc = check_config(cfg);
    if (rc) return rc;
    if (!cache || !cache->k_records || !cache->v_records) return KVARN_EINVAL;
    if (first_block < 0 || num_blocks < 0 || (long long)first_block + num_blocks > cfg->max_blocks)
        return KVARN_EINVAL;
    if (!grid_fits(cfg, num_blocks)) return KVARN_EINVAL;
    if ((k_out && !aligned16(k_out)) || (v_out && !aligned16(v_out))) return KVARN_EINVAL;
    DequantArgs a;
    a.k_records = cache->k_records; a.v_records = cache->v_records;
    a.k_out = k_out; a.v_out = v_out;
    a.first_block = first_block; a.num_blocks = num_blocks; a.max_blocks = cfg->max_blocks;
    a.rotated = rotated ? 1 : 0;
    return cuda_status(run_dequantize(*cfg, a, static_cast<cudaStream_t>(stream)));
}

const char *kvarn_strerror(int code)
{
    switch (code) {
    case KVARN_OK: return "ok";
    case KVARN_EINVAL: return "invalid argument (null or misaligned pointer, bad size or shape)";
    case KVARN_EUNSUPPORTED: return "unsupported parameter (head_dim, block_tokens, group, hadamard or GQA ratio)";
    case KVARN_EWORKSPACE: return "decode workspace missing, misaligned or too small";
    case KVARN_ECUDA: return "CUDA launch or runtime error";
    }
    return "unknown kvarn status code";
}

}  // extern "C"
