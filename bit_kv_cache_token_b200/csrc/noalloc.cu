// noalloc.cu -- decode attention without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they run
// decode: code that runs inside a host callback or a signal-restricted
// context, embedders whose allocator is owned by another runtime, or code
// that must not grow the process's device footprint after start-up.  For
// them this entry point uses a workspace that lives in this library's own
// device image: a file-scope __device__ array, reserved on every GPU that
// loads the library and held until the process exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "kvarn.h"

namespace {

// Largest decode workspace the static array serves (16 MiB).
constexpr size_t kStaticScratchBytes = (size_t)16 << 20;

__device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

// In host code g_decode_scratch is only a host-side stand-in, never a device
// address.  Its device address belongs to one CUDA context (a second context
// on the same device, or the context created again after cudaDeviceReset,
// loads the module anew at another address), so the looked-up address is
// cached per context, keyed by the driver's unique context id.  The cache is
// shared by all host threads and guarded by a mutex.
struct ScratchEntry {
    unsigned long long ctx_id;
    void *ptr;
};
constexpr int kCacheSlots = 64;
std::mutex g_mu;
ScratchEntry g_cache[kCacheSlots];
int g_used = 0, g_next = 0;

using PfnCtxGetCurrent = CUresult (*)(CUcontext *);
using PfnCtxGetId = CUresult (*)(CUcontext, unsigned long long *);
PfnCtxGetCurrent g_get_current = nullptr;
PfnCtxGetId g_get_id = nullptr;
bool g_resolved = false;

// Driver entry points, resolved once through the runtime (no link-time
// dependency on the driver library).  Called with g_mu held.
void resolve_entry_points()
{
    if (g_resolved) return;
    g_resolved = true;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        g_get_current = reinterpret_cast<PfnCtxGetCurrent>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        g_get_id = reinterpret_cast<PfnCtxGetId>(fn);
}

// Unique id of the calling thread's current context; false when there is
// none yet or the driver cannot tell.
bool current_context_id(unsigned long long *id)
{
    if (!g_get_current || !g_get_id) return false;
    CUcontext ctx = nullptr;
    if (g_get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
    return g_get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_decode_scratch in the current context.  The first
// call in a context looks it up (cudaGetSymbolAddress, which also sets up the
// device's primary context if none is current) and caches it.
int scratch_for_current_context(void **out)
{
    std::lock_guard<std::mutex> lock(g_mu);
    resolve_entry_points();
    unsigned long long id = 0;
    bool have_id = current_context_id(&id);
    if (have_id) {
        for (int i = 0; i < g_used; ++i)
            if (g_cache[i].ctx_id == id) {
                *out = g_cache[i].ptr;
                return KVARN_OK;
            }
    }
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return KVARN_ECUDA;
    if (!have_id) have_id = current_context_id(&id);  // the lookup may have made the context current
    if (have_id) {
        g_cache[g_next] = ScratchEntry{id, p};
        g_next = (g_next + 1) % kCacheSlots;
        if (g_used < kCacheSlots) ++g_used;
    }
    *out = p;
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
    const int rc = scratch_for_current_context(&ws);
    if (rc != KVARN_OK) return rc;
    // The array keeps the previous call's contents: the split tickets at its
    // start must be zero when a decode begins.
    const size_t tickets = ((size_t)cfg->num_seqs * cfg->num_kv_heads * sizeof(unsigned int) + 255) / 256 * 256;
    if (cudaMemsetAsync(ws, 0, tickets, static_cast<cudaStream_t>(stream)) != cudaSuccess) return KVARN_ECUDA;
    return kvarn_decode_attention(cfg, q, num_q_heads, softmax_scale, cache, max_tokens, out, ws,
                                  kStaticScratchBytes, stream);
}

}  // extern "C"
