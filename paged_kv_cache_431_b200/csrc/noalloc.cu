// noalloc.cu -- paged_decode_attn for callers that cannot allocate device memory.
//
// paged_decode_attn needs a caller-provided workspace for its split-K partials when a
// context spans more than one partition.  Some callers cannot provide one: code that
// runs inside a host runtime which owns every device allocation (a serving engine's
// memory planner that has already divided HBM among its pools, or a plugin that may
// only use the memory it is handed), and code on latency-critical paths where a
// cudaMalloc -- which may synchronize the whole device -- is not acceptable.
// paged_decode_attn_noalloc serves them: it runs the same kernels with the partials in
// a fixed buffer that lives in this library's device memory.
//
// The buffer is a file-scope __device__ array of PKV_NOALLOC_SCRATCH_BYTES.  Every GPU
// that loads the library holds it until the process exits.  In host code its name is
// only a host-side stand-in, so its device address is looked up with
// cudaGetSymbolAddress -- once per device, on that device's first call, with the
// device current -- and that address is passed to the kernels.
//
// All calls on a device share the one buffer and it keeps the last call's contents.
// Nothing in it has to start at zero: a call writes every partial it later reads.  Two
// calls whose kernels overlap on the GPU (different streams, or different host threads,
// without ordering between them) race on the buffer and give wrong results; callers must
// serialize them, e.g. by issuing them on one stream.
#include <mutex>

#include "internal.h"

namespace {

constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[PKV_NOALLOC_SCRATCH_BYTES];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the buffer on the current device (looked up on first use).
int scratch_on_current_device(void** out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return PKV_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return PKV_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return PKV_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return PKV_OK;
}

}  // namespace

extern "C" {

int paged_decode_attn_noalloc(pkv_pool_t pool, int layer, const void* q, int q_dtype, const int32_t* block_tables,
                              int block_table_width, const int32_t* context_lens, int num_seqs, int num_q_heads,
                              int max_context_len, float scale, float* out, const pkv_decode_opts* opts, void* stream)
{
    const size_t need = paged_decode_workspace_bytes(pool, num_seqs, num_q_heads, max_context_len, opts);
    if (need > (size_t)PKV_NOALLOC_SCRATCH_BYTES) return PKV_ERR_WORKSPACE;
    void* ws = nullptr;
    if (need > 0) {
        const int rc = scratch_on_current_device(&ws);
        if (rc != PKV_OK) return rc;
    }
    return paged_decode_attn(pool, layer, q, q_dtype, block_tables, block_table_width, context_lens, num_seqs,
                             num_q_heads, max_context_len, scale, out, ws, need > 0 ? (size_t)PKV_NOALLOC_SCRATCH_BYTES : 0,
                             opts, stream);
}

}  // extern "C"
