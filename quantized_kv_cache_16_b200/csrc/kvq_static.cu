// kvq_static.cu -- decode attention without any caller-provided or allocated
// workspace: the scratch lives in a fixed-size array in this library's own
// device memory.  For callers that cannot allocate device memory (see
// kvq_decode_attn_static in kvq.h).
#include <string.h>

#include "kvq_internal.cuh"

using kvq::decode_counter_bytes;

namespace {

// Decode workspace (split counters + split partials) for every call of
// kvq_decode_attn_static.  Each GPU that loads the library holds one copy of
// this array until the process exits.
constexpr size_t kStaticScratchBytes = 4u << 20;  // 4 MiB
__device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
void *g_scratch_ptr[kMaxDevices];  // device address of g_decode_scratch per device, set on first use

// In host code g_decode_scratch names a host-side stand-in, not device
// memory: its device address must come from cudaGetSymbolAddress, taken with
// the device current.
kvq_status scratch_for_current_device(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVQ_ERR_CUDA;
    if (!g_scratch_ptr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || !ptr) {
            cudaGetLastError();
            return KVQ_ERR_CUDA;
        }
        g_scratch_ptr[dev] = ptr;
    }
    *out = g_scratch_ptr[dev];
    return KVQ_OK;
}

}  // namespace

extern "C" kvq_status kvq_decode_attn_static(kvq_cache *c, const void *q, const int32_t *block_table,
                                             int32_t max_pages_per_seq, const int32_t *ctx_lens, int32_t batch,
                                             float softmax_scale, void *out, void *stream)
{
    if (!c || batch < 0 || max_pages_per_seq < 1) return KVQ_ERR_INVALID_ARG;
    if (batch == 0) return KVQ_OK;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return KVQ_ERR_CUDA;
    if (dev != c->device) return KVQ_ERR_INVALID_ARG;  // the cache's device must be current
    const size_t need = kvq_decode_workspace_bytes(c, batch, max_pages_per_seq);
    if (need == 0 || need > kStaticScratchBytes) return KVQ_ERR_CAPACITY;
    void *ws = nullptr;
    const kvq_status st = scratch_for_current_device(&ws);
    if (st != KVQ_OK) return st;
    // the counters must start at zero; the partials need no clearing
    const size_t counters = decode_counter_bytes(batch, c->L.hkv);
    if (cudaMemsetAsync(ws, 0, counters, static_cast<cudaStream_t>(stream)) != cudaSuccess) return KVQ_ERR_CUDA;
    return kvq_decode_attn(c, q, block_table, max_pages_per_seq, ctx_lens, batch, softmax_scale, nullptr, ws,
                           kStaticScratchBytes, out, nullptr, stream);
}
