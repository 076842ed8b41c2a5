// noalloc.cu -- decode attention without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they run
// decode: code that runs inside a host callback or a signal-restricted
// context, embedders whose allocator is owned by another runtime, or code
// that must not grow the process's device footprint after start-up.  For
// them this entry point uses a workspace that lives in this library's own
// device image: a file-scope __device__ array, reserved on every GPU that
// loads the library and held until the process exits.
#include <cuda_runtime.h>

#include "kvarn.h"

namespace {

// Largest decode workspace the static array serves (16 MiB).
constexpr size_t kStaticScratchBytes = (size_t)16 << 20;

__device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

// Device address of g_decode_scratch, looked up once per device.  In host
// code the symbol name is only a host-side stand-in, never a device address.
void *g_scratch_ptr[64] = {nullptr};

int scratch_for_current_device(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return KVARN_ECUDA;
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return KVARN_ECUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return KVARN_OK;
}

}  // namespace

extern "C" {

int kvarn_decode_attention_noalloc(const kvarn_config *cfg, const void *q, int num_q_heads, float softmax_scale,
                                   const kvarn_cache *cache, int max_tokens, float *out, void *stream)
{
    const size_t need = kvarn_decode_workspace_bytes(cfg, num_q_heads);
    if (need == 0) return KVARN_EINVAL;
    if (need > kStaticScratchBytes) return KVARN_EWORKSPACE;
    void *ws = nullptr;
    const int rc = scratch_for_current_device(&ws);
    if (rc != KVARN_OK) return rc;
    // The array keeps the previous call's contents: the split tickets at its
    // start must be zero when a decode begins.
    const size_t tickets = ((size_t)cfg->num_seqs * cfg->num_kv_heads * sizeof(unsigned int) + 255) / 256 * 256;
    if (cudaMemsetAsync(ws, 0, tickets, static_cast<cudaStream_t>(stream)) != cudaSuccess) return KVARN_ECUDA;
    return kvarn_decode_attention(cfg, q, num_q_heads, softmax_scale, cache, max_tokens, out, ws,
                                  kStaticScratchBytes, stream);
}

}  // extern "C"
