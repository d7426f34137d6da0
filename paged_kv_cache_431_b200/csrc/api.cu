// api.cu -- the C-ABI of libpkv: argument validation, pool handles, tensor maps,
// workspace layout and kernel launches.  Every entry point validates on the host
// before launching and returns a PKV_* status; nothing here synchronizes except
// pkv_read_device_status.
#include <cudaTypedefs.h>

#include <atomic>
#include <cstring>
#include <new>

#include "internal.h"
#include "../../include/pkv_block_manager.h"

namespace pkv {

namespace {
std::atomic<int> g_hold_tile{-1};
std::atomic<long long> g_wait_cycles{kDefaultWaitCycles};
}  // namespace

WaitHook wait_hook()
{
    return WaitHook{g_hold_tile.load(std::memory_order_relaxed), g_wait_cycles.load(std::memory_order_relaxed)};
}

int row_bytes_of(int dtype, int head_dim)
{
    switch (dtype) {
    case PKV_F16:
    case PKV_BF16: return 2 * head_dim;
    case PKV_INT8:
    case PKV_FP8E4M3: return head_dim;
    case PKV_INT4: return head_dim / 2;
    default: return -1;
    }
}

bool is_quantized(int dtype) { return dtype == PKV_INT8 || dtype == PKV_INT4 || dtype == PKV_FP8E4M3; }

int num_sms()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 148;
    return n;
}

PFN_encode tensor_map_encoder()
{
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// One layer's K or V pool as a 2-D tensor [N * H_kv * 16 rows][row elements], loaded in
// boxes of 16 rows x (at most) 128 bytes with the matching shared-memory swizzle.
static bool make_map(CUtensorMap* map, void* base, const pkv_pool_desc& d, int row_bytes)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const bool b16 = d.kv_dtype == PKV_F16 || d.kv_dtype == PKV_BF16;
    const int esize = b16 ? 2 : 1;
    const cuuint64_t dims[2] = {(cuuint64_t)(row_bytes / esize), (cuuint64_t)d.num_blocks * d.num_kv_heads * PKV_BLOCK_SIZE};
    const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    const int box_bytes = row_bytes < 128 ? row_bytes : 128;
    const cuuint32_t box[2] = {(cuuint32_t)(box_bytes / esize), (cuuint32_t)PKV_BLOCK_SIZE};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapSwizzle swz = box_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                 : box_bytes == 64  ? CU_TENSOR_MAP_SWIZZLE_64B
                                                    : CU_TENSOR_MAP_SWIZZLE_32B;
    CUresult r = enc(map, b16 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int layer_maps(pkv_pool* pool, int layer, const CUtensorMap** tmk, const CUtensorMap** tmv)
{
    std::lock_guard<std::mutex> lock(pool->mu);
    if (!pool->maps_ready) {
        const int L = pool->d.num_layers;
        pool->tmk.resize(L);
        pool->tmv.resize(L);
        for (int l = 0; l < L; ++l) {
            if (!make_map(&pool->tmk[l], pool->k_base[l], pool->d, pool->row_bytes) ||
                !make_map(&pool->tmv[l], pool->v_base[l], pool->d, pool->row_bytes))
                return PKV_ERR_CUDA;
        }
        pool->maps_ready = true;
    }
    *tmk = &pool->tmk[layer];
    *tmv = &pool->tmv[layer];
    return PKV_OK;
}

// Split-K partition size: about 256 KiB of K + V per partition for 16-bit pools (512 tokens
// at head_dim 128) and 192 KiB for quantized ones (768 tokens for int8 / fp8, 1536 for int4),
// so the partials stay near 1.6-2% of the bytes read; smaller (halved, down to 128 or 192
// tokens) when the batch is too small to fill the GPU with one-warp CTAs.  The quantized
// sizes were measured on the long-context layer: 768 against 1024 tokens took int8 from 495
// to 475 us per call and fp8 from 618 to 586, 1536 against 2048 took int4 from 560 to 524
// (partitions of 3 * 2^k tokens beat the powers of two on both sides of them).
static int choose_partition(int B, int ctas, int max_ctx, int row_bytes, bool quantized, const pkv_decode_opts* o)
{
    if (o && o->partition_tokens > 0) return o->partition_tokens;
    int P = (quantized ? 192 : 256) * 1024 / (2 * row_bytes);
    P = P < 128 ? 128 : (P > 4096 ? 4096 : P);
    const long target = 4L * num_sms() * 8;
    while (P >= 256) {   // halves down to 128 (powers of two) or 192 (3 * 2^k) tokens
        const long parts = (max_ctx + P - 1) / P;
        if ((long)B * ctas * (parts > 0 ? parts : 1) >= target) break;
        P /= 2;
    }
    return P;
}

static bool valid_partition(int P) { return P >= 64 && P <= 4096 && P % PKV_BLOCK_SIZE == 0; }

}  // namespace pkv

using namespace pkv;

extern "C" {

int pkv_version(void) { return 100; }

const char* pkv_strerror(int status)
{
    switch (status) {
    case PKV_OK: return "ok";
    case PKV_ERR_NULL: return "a required pointer is NULL";
    case PKV_ERR_ARG: return "an argument is out of range";
    case PKV_ERR_DTYPE: return "unsupported dtype or dtype combination";
    case PKV_ERR_SHAPE: return "inconsistent sizes";
    case PKV_ERR_WORKSPACE: return "workspace missing or too small";
    case PKV_ERR_CUDA: return "a CUDA call failed";
    case PKV_ERR_TIMEOUT: return "a kernel gave up waiting on a bulk copy";
    case PKV_ERR_INDEX: return "the device saw a block id, slot or context length out of range";
    case PKV_ERR_UNSUPPORTED: return "configuration not supported by the library";
    case PKV_ERR_NO_BLOCKS: return "not enough free blocks in the pool";
    case PKV_ERR_STATE: return "unknown, existing or swapped-out sequence, or a broken block-manager invariant";
    default: return "unknown status";
    }
}

static int validate_desc(const pkv_pool_desc* d)
{
    if (!d) return PKV_ERR_NULL;
    if (d->num_layers <= 0 || d->num_layers > PKV_MAX_LAYERS || d->num_blocks <= 0 || d->num_kv_heads <= 0)
        return PKV_ERR_ARG;
    if (d->block_size != PKV_BLOCK_SIZE) return PKV_ERR_ARG;
    if (d->head_dim != 64 && d->head_dim != 128) return PKV_ERR_UNSUPPORTED;
    if (row_bytes_of(d->kv_dtype, d->head_dim) <= 0) return PKV_ERR_DTYPE;
    if ((long long)d->num_blocks * d->num_kv_heads * PKV_BLOCK_SIZE > 0x7fffffffLL) return PKV_ERR_ARG;
    return PKV_OK;
}

size_t pkv_pool_bytes(const pkv_pool_desc* d, size_t* scale_bytes)
{
    if (scale_bytes) *scale_bytes = 0;
    if (validate_desc(d) != PKV_OK) return 0;
    const size_t per_layer = (size_t)d->num_blocks * d->num_kv_heads * PKV_BLOCK_SIZE * row_bytes_of(d->kv_dtype, d->head_dim);
    if (scale_bytes && is_quantized(d->kv_dtype))
        *scale_bytes = (size_t)d->num_layers * d->num_blocks * d->num_kv_heads * sizeof(float);
    return per_layer * d->num_layers;
}

// A handle over per-layer bases (validated by the caller), or null when out of memory.
static pkv_pool* new_pool(const pkv_pool_desc* d, void* const* k, void* const* v, float* const* ks, float* const* vs)
{
    pkv_pool* p = new (std::nothrow) pkv_pool();
    if (!p) return nullptr;
    p->d = *d;
    p->row_bytes = row_bytes_of(d->kv_dtype, d->head_dim);
    p->tile_bytes = (size_t)PKV_BLOCK_SIZE * p->row_bytes;
    p->layer_bytes = (size_t)d->num_blocks * d->num_kv_heads * p->tile_bytes;
    p->layer_scales = is_quantized(d->kv_dtype) ? (size_t)d->num_blocks * d->num_kv_heads : 0;
    const int L = d->num_layers;
    try {
        p->k_base.resize(L);
        p->v_base.resize(L);
        p->ks_base.assign(L, nullptr);
        p->vs_base.assign(L, nullptr);
    } catch (...) {
        delete p;
        return nullptr;
    }
    for (int l = 0; l < L; ++l) {
        p->k_base[l] = static_cast<uint8_t*>(k[l]);
        p->v_base[l] = static_cast<uint8_t*>(v[l]);
        if (p->layer_scales) {
            p->ks_base[l] = ks[l];
            p->vs_base[l] = vs[l];
        }
    }
    return p;
}

int kv_pool_create(const pkv_pool_desc* d, pkv_pool_t* out)
{
    if (!out) return PKV_ERR_NULL;
    *out = nullptr;
    int rc = validate_desc(d);
    if (rc != PKV_OK) return rc;
    if (!d->k_data || !d->v_data) return PKV_ERR_NULL;
    if (is_quantized(d->kv_dtype) && (!d->k_scale || !d->v_scale)) return PKV_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(d->k_data) | reinterpret_cast<uintptr_t>(d->v_data)) & 15) return PKV_ERR_ARG;
    // a dense pool: layer l starts l whole layers into each allocation
    const size_t lb = (size_t)d->num_blocks * d->num_kv_heads * PKV_BLOCK_SIZE * row_bytes_of(d->kv_dtype, d->head_dim);
    const size_t ls = (size_t)d->num_blocks * d->num_kv_heads;
    void* k[PKV_MAX_LAYERS];
    void* v[PKV_MAX_LAYERS];
    float* ks[PKV_MAX_LAYERS];
    float* vs[PKV_MAX_LAYERS];
    for (int l = 0; l < d->num_layers; ++l) {
        k[l] = static_cast<uint8_t*>(d->k_data) + (size_t)l * lb;
        v[l] = static_cast<uint8_t*>(d->v_data) + (size_t)l * lb;
        ks[l] = d->k_scale ? d->k_scale + (size_t)l * ls : nullptr;
        vs[l] = d->v_scale ? d->v_scale + (size_t)l * ls : nullptr;
    }
    pkv_pool* p = new_pool(d, k, v, ks, vs);
    if (!p) return PKV_ERR_ARG;
    *out = p;
    return PKV_OK;
}

int kv_pool_create_layers(const pkv_pool_desc* d, void* const* k_layers, void* const* v_layers,
                          float* const* k_scale_layers, float* const* v_scale_layers, pkv_pool_t* out)
{
    if (!out) return PKV_ERR_NULL;
    *out = nullptr;
    int rc = validate_desc(d);
    if (rc != PKV_OK) return rc;
    if (!k_layers || !v_layers) return PKV_ERR_NULL;
    const bool quant = is_quantized(d->kv_dtype);
    if (quant && (!k_scale_layers || !v_scale_layers)) return PKV_ERR_NULL;
    for (int l = 0; l < d->num_layers; ++l) {
        if (!k_layers[l] || !v_layers[l]) return PKV_ERR_NULL;
        if ((reinterpret_cast<uintptr_t>(k_layers[l]) | reinterpret_cast<uintptr_t>(v_layers[l])) & 15)
            return PKV_ERR_ARG;
        if (quant) {
            if (!k_scale_layers[l] || !v_scale_layers[l]) return PKV_ERR_NULL;
            if ((reinterpret_cast<uintptr_t>(k_scale_layers[l]) | reinterpret_cast<uintptr_t>(v_scale_layers[l])) & 3)
                return PKV_ERR_ARG;
        }
    }
    pkv_pool* p = new_pool(d, k_layers, v_layers, k_scale_layers, v_scale_layers);
    if (!p) return PKV_ERR_ARG;
    p->d.k_data = p->k_base[0];   // the first layer's, for callers that read the description back
    p->d.v_data = p->v_base[0];
    p->d.k_scale = p->ks_base[0];
    p->d.v_scale = p->vs_base[0];
    *out = p;
    return PKV_OK;
}

int kv_pool_destroy(pkv_pool_t pool)
{
    delete pool;
    return PKV_OK;
}

size_t kv_append_workspace_bytes(pkv_pool_t pool, int num_tokens)
{
    if (!pool || num_tokens < 0) return 0;
    return append_workspace_bytes(pool->d.num_blocks, pool->d.num_kv_heads, pool->d.kv_dtype);
}

int kv_append(pkv_pool_t pool, int layer, const void* k, const void* v, int src_dtype, const int32_t* slot_mapping,
              int num_tokens, void* workspace, size_t workspace_bytes, void* stream)
{
    if (!pool) return PKV_ERR_NULL;
    const pkv_pool_desc& d = pool->d;
    if (layer < 0 || layer >= d.num_layers || num_tokens < 0) return PKV_ERR_ARG;
    if (num_tokens == 0) return PKV_OK;
    if (!k || !v || !slot_mapping) return PKV_ERR_NULL;
    if (is_quantized(d.kv_dtype)) {
        if (src_dtype != PKV_BF16) return PKV_ERR_DTYPE;
        const size_t need = append_workspace_bytes(d.num_blocks, d.num_kv_heads, d.kv_dtype);
        if (!workspace || workspace_bytes < need) return PKV_ERR_WORKSPACE;
        if (reinterpret_cast<uintptr_t>(workspace) & 3) return PKV_ERR_ARG;
    } else if (src_dtype != d.kv_dtype) {
        return PKV_ERR_DTYPE;
    }
    const uintptr_t align = is_quantized(d.kv_dtype) ? 8 : 16;
    if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & (align - 1)) return PKV_ERR_ARG;
    if ((long long)num_tokens * d.num_kv_heads > 0x7fffffffLL / 32) return PKV_ERR_ARG;
    AppendArgs a;
    a.k = k;
    a.v = v;
    a.slots = slot_mapping;
    a.T = num_tokens;
    a.N = d.num_blocks;
    a.H_kv = d.num_kv_heads;
    a.d = d.head_dim;
    a.kv_dtype = d.kv_dtype;
    a.k_pool = pool->k_base[layer];
    a.v_pool = pool->v_base[layer];
    a.k_scale = pool->ks_base[layer];
    a.v_scale = pool->vs_base[layer];
    a.workspace = workspace;
    a.status = d.device_status;
    return launch_append(a, static_cast<cudaStream_t>(stream));
}

// CTAs the decode grid has per (sequence, partition): one per KV head and group of 16 query heads.
static int ctas_per_partition(pkv_pool_t pool, int num_q_heads)
{
    const int H_kv = pool->d.num_kv_heads;
    const int G = (num_q_heads > 0 && num_q_heads % H_kv == 0) ? num_q_heads / H_kv : 1;
    return H_kv * ((G + 15) / 16);
}

// Partition of the keys-on-M tcgen05 decodes (one or two CTAs per SM, a fixed cost per CTA): as
// few partitions per sequence as fill the SMs, each at most 4096 tokens, in whole 128-key tiles.
static int keys_tc_partition(int seq_heads, int span, int ctas_per_sm)
{
    int parts = (span + 4095) / 4096;
    const int fill = (ctas_per_sm * num_sms() + seq_heads - 1) / (seq_heads > 0 ? seq_heads : 1);
    parts = parts < fill ? fill : parts;
    parts = parts < 1 ? 1 : parts;
    const int P = ((span + parts - 1) / parts + 127) / 128 * 128;
    return P < 128 ? 128 : (P > 4096 ? 4096 : P);
}

static int decode_partitioning(pkv_pool_t pool, int num_seqs, int num_q_heads, int max_ctx,
                               const pkv_decode_opts* opts, int* P, int* max_parts)
{
    const int window = opts ? opts->sliding_window : 0;
    if (window < 0) return PKV_ERR_ARG;
    // with a window a sequence's partitions start at the block holding ctx - window
    const int span = (window > 0 && max_ctx > window + PKV_BLOCK_SIZE - 1) ? window + PKV_BLOCK_SIZE - 1 : max_ctx;
    const int H_kv = pool->d.num_kv_heads;
    const int keys_tc = ((!opts || opts->engine == 0) && window == 0 && num_q_heads % H_kv == 0)
                            ? decode_keys_tc_available(pool->d.head_dim, num_q_heads / H_kv, pool->d.kv_dtype)
                            : 0;
    if (keys_tc > 0 && !(opts && opts->partition_tokens > 0))
        *P = keys_tc_partition(num_seqs * H_kv, span, keys_tc);
    else
        *P = choose_partition(num_seqs, ctas_per_partition(pool, num_q_heads), span, pool->row_bytes,
                              is_quantized(pool->d.kv_dtype), opts);
    if (!valid_partition(*P)) return PKV_ERR_ARG;
    *max_parts = span > 0 ? (span + *P - 1) / *P : 1;
    return PKV_OK;
}

// Split-K workspace: partials o [B][H_q][parts][d] and (m, l) [B][H_q][parts][2] (fp32).
static size_t decode_ws_bytes(pkv_pool_t pool, int num_seqs, int num_q_heads, int parts)
{
    if (parts <= 1) return 0;
    return (size_t)num_seqs * num_q_heads * parts * (pool->d.head_dim + 2) * sizeof(float);
}

size_t paged_decode_workspace_bytes(pkv_pool_t pool, int num_seqs, int num_q_heads, int max_context_len,
                                    const pkv_decode_opts* opts)
{
    if (!pool || num_seqs < 0 || num_q_heads <= 0 || max_context_len < 0) return 0;
    int P, parts;
    if (decode_partitioning(pool, num_seqs, num_q_heads, max_context_len, opts, &P, &parts) != PKV_OK) return 0;
    return decode_ws_bytes(pool, num_seqs, num_q_heads, parts);
}

int paged_decode_attn(pkv_pool_t pool, int layer, const void* q, int q_dtype, const int32_t* block_tables,
                      int block_table_width, const int32_t* context_lens, int num_seqs, int num_q_heads,
                      int max_context_len, float scale, float* out, void* workspace, size_t workspace_bytes,
                      const pkv_decode_opts* opts, void* stream)
{
    if (!pool) return PKV_ERR_NULL;
    const pkv_pool_desc& d = pool->d;
    if (layer < 0 || layer >= d.num_layers || num_seqs < 0 || num_q_heads <= 0 || block_table_width <= 0 ||
        max_context_len < 0 || num_seqs > 65535)
        return PKV_ERR_ARG;
    if (num_q_heads % d.num_kv_heads) return PKV_ERR_SHAPE;
    const int G = num_q_heads / d.num_kv_heads;
    if ((long long)d.num_kv_heads * ((G + 15) / 16) > 65535) return PKV_ERR_UNSUPPORTED;
    if (num_seqs == 0) return PKV_OK;
    if (!q || !block_tables || !context_lens || !out) return PKV_ERR_NULL;
    if (q_dtype != PKV_F16 && q_dtype != PKV_BF16) return PKV_ERR_DTYPE;
    if (!is_quantized(d.kv_dtype) && q_dtype != d.kv_dtype) return PKV_ERR_DTYPE;
    if ((reinterpret_cast<uintptr_t>(q) & 3) || (reinterpret_cast<uintptr_t>(out) & 15)) return PKV_ERR_ARG;
    int engine = opts ? opts->engine : 0;
    if (engine < 0 || engine > 3) return PKV_ERR_ARG;
    int P, parts;
    int rc = decode_partitioning(pool, num_seqs, num_q_heads, max_context_len, opts, &P, &parts);
    if (rc != PKV_OK) return rc;
    const size_t need = decode_ws_bytes(pool, num_seqs, num_q_heads, parts);
    if (need && (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 15)))
        return PKV_ERR_WORKSPACE;
    const CUtensorMap *tmk = nullptr, *tmv = nullptr;
    rc = layer_maps(pool, layer, &tmk, &tmv);
    if (rc != PKV_OK) return rc;

    DecodeArgs a;
    a.q = q;
    a.q_dtype = q_dtype;
    a.tables = block_tables;
    a.W = block_table_width;
    a.ctx_lens = context_lens;
    a.B = num_seqs;
    a.H_q = num_q_heads;
    a.H_kv = d.num_kv_heads;
    a.G = G;
    a.N = d.num_blocks;
    a.d = d.head_dim;
    a.kv_dtype = d.kv_dtype;
    a.part_tokens = P;
    a.max_parts = parts;
    a.scale = scale;
    a.k_scale = pool->ks_base[layer];
    a.v_scale = pool->vs_base[layer];
    a.out = out;
    float* ws = static_cast<float*>(workspace);
    a.ws_o = need ? ws : nullptr;
    a.ws_ml = need ? ws + (size_t)num_seqs * num_q_heads * parts * d.head_dim : nullptr;
    a.status = d.device_status;
    a.engine = engine;
    a.window = opts ? opts->sliding_window : 0;
    return launch_decode(a, tmk, tmv, static_cast<cudaStream_t>(stream));
}

// ---- shared-prefix (cascade) decode ------------------------------------------------

static bool cascade_shape_ok(pkv_pool_t pool, int num_q_heads, int max_context_len, int prefix_len)
{
    const pkv_pool_desc& d = pool->d;
    if (num_q_heads <= 0 || num_q_heads % d.num_kv_heads) return false;
    const int G = num_q_heads / d.num_kv_heads;
    return prefill_tc_supported(d.head_dim, G, d.kv_dtype) && prefix_len > 0 && prefix_len % PKV_BLOCK_SIZE == 0 &&
           max_context_len >= prefix_len;
}

static int cascade_partitioning(pkv_pool_t pool, int num_seqs, int num_q_heads, int max_ctx, int prefix_len,
                                const pkv_decode_opts* opts, int* P, int* suffix_parts)
{
    const int rest = max_ctx - prefix_len;
    *P = choose_partition(num_seqs, ctas_per_partition(pool, num_q_heads), rest > 0 ? rest : 1, pool->row_bytes,
                          is_quantized(pool->d.kv_dtype), opts);
    if (!valid_partition(*P)) return PKV_ERR_ARG;
    *suffix_parts = rest > 0 ? (rest + *P - 1) / *P : 1;
    return PKV_OK;
}

size_t paged_decode_cascade_workspace_bytes(pkv_pool_t pool, int num_seqs, int num_q_heads, int max_context_len,
                                            int shared_prefix_len, const pkv_decode_opts* opts)
{
    if (!pool || num_seqs < 0 || max_context_len < 0 || shared_prefix_len < 0) return 0;
    if (shared_prefix_len == 0) return paged_decode_workspace_bytes(pool, num_seqs, num_q_heads, max_context_len, opts);
    if (!cascade_shape_ok(pool, num_q_heads, max_context_len, shared_prefix_len)) return 0;
    int P, parts;
    if (cascade_partitioning(pool, num_seqs, num_q_heads, max_context_len, shared_prefix_len, opts, &P, &parts) !=
        PKV_OK)
        return 0;
    const int splits = prefill_tc_key_splits(num_seqs, num_q_heads / pool->d.num_kv_heads, pool->d.num_kv_heads,
                                             shared_prefix_len);
    return (size_t)num_seqs * num_q_heads * (splits + parts) * (pool->d.head_dim + 2) * sizeof(float);
}

int paged_decode_attn_cascade(pkv_pool_t pool, int layer, const void* q, int q_dtype, const int32_t* block_tables,
                              int block_table_width, const int32_t* context_lens, int num_seqs, int num_q_heads,
                              int max_context_len, int shared_prefix_len, float scale, float* out, void* workspace,
                              size_t workspace_bytes, const pkv_decode_opts* opts, void* stream)
{
    if (!pool) return PKV_ERR_NULL;
    if (shared_prefix_len < 0) return PKV_ERR_ARG;
    if (shared_prefix_len == 0)
        return paged_decode_attn(pool, layer, q, q_dtype, block_tables, block_table_width, context_lens, num_seqs,
                                 num_q_heads, max_context_len, scale, out, workspace, workspace_bytes, opts, stream);
    const pkv_pool_desc& d = pool->d;
    if (layer < 0 || layer >= d.num_layers || num_seqs < 0 || num_q_heads <= 0 || block_table_width <= 0 ||
        max_context_len < 0 || num_seqs > 65535)
        return PKV_ERR_ARG;
    if (num_q_heads % d.num_kv_heads) return PKV_ERR_SHAPE;
    if (shared_prefix_len % PKV_BLOCK_SIZE || max_context_len < shared_prefix_len ||
        (long long)block_table_width * PKV_BLOCK_SIZE < shared_prefix_len)
        return PKV_ERR_SHAPE;
    if (!cascade_shape_ok(pool, num_q_heads, max_context_len, shared_prefix_len)) return PKV_ERR_UNSUPPORTED;
    if (opts && opts->sliding_window != 0) return PKV_ERR_UNSUPPORTED;
    if (num_seqs == 0) return PKV_OK;
    if (!q || !block_tables || !context_lens || !out) return PKV_ERR_NULL;
    if (q_dtype != d.kv_dtype) return PKV_ERR_DTYPE;
    if ((reinterpret_cast<uintptr_t>(q) & 15) || (reinterpret_cast<uintptr_t>(out) & 15)) return PKV_ERR_ARG;
    int engine = opts ? opts->engine : 0;
    if (engine < 0 || engine > 3) return PKV_ERR_ARG;
    int P, parts;
    int rc = cascade_partitioning(pool, num_seqs, num_q_heads, max_context_len, shared_prefix_len, opts, &P, &parts);
    if (rc != PKV_OK) return rc;
    const int G = num_q_heads / d.num_kv_heads;
    const int splits = prefill_tc_key_splits(num_seqs, G, d.num_kv_heads, shared_prefix_len);
    const int slots = splits + parts;   // prefix partials in slots 0 .. splits-1, then the suffix
    const size_t need = (size_t)num_seqs * num_q_heads * slots * (d.head_dim + 2) * sizeof(float);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 15)) return PKV_ERR_WORKSPACE;
    const CUtensorMap *tmk = nullptr, *tmv = nullptr;
    rc = layer_maps(pool, layer, &tmk, &tmv);
    if (rc != PKV_OK) return rc;
    float* ws_o = static_cast<float*>(workspace);
    float* ws_ml = ws_o + (size_t)num_seqs * num_q_heads * slots * d.head_dim;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    // 1. the shared prefix, once per KV group for the whole batch, on the tensor cores:
    //    rows = (sequence, head of the group), keys = the prefix blocks of table row 0
    PrefillArgs pa;
    pa.q = q;
    pa.q_dtype = q_dtype;
    pa.table = block_tables;
    pa.W = shared_prefix_len / PKV_BLOCK_SIZE;
    pa.P0 = 0;
    pa.C = num_seqs;
    pa.H_q = num_q_heads;
    pa.H_kv = d.num_kv_heads;
    pa.G = G;
    pa.N = d.num_blocks;
    pa.d = d.head_dim;
    pa.kv_dtype = d.kv_dtype;
    pa.scale = scale;
    pa.out = nullptr;
    pa.status = d.device_status;
    pa.cascade_nkeys = shared_prefix_len;
    pa.key_splits = splits;
    pa.ws_slots = slots;
    pa.ws_o = ws_o;
    pa.ws_ml = ws_ml;
    CUtensorMap tmq;
    auto enc = tensor_map_encoder();
    if (!enc || !make_q_map(&tmq, q, num_seqs, num_q_heads, G, enc)) return PKV_ERR_CUDA;
    rc = launch_prefill_tc(pa, &tmq, tmk, tmv, s);
    if (rc != PKV_OK) return rc;

    // 2. each sequence's own suffix as split-K partitions into slots 1.., then the merge
    DecodeArgs a;
    a.q = q;
    a.q_dtype = q_dtype;
    a.tables = block_tables;
    a.W = block_table_width;
    a.ctx_lens = context_lens;
    a.B = num_seqs;
    a.H_q = num_q_heads;
    a.H_kv = d.num_kv_heads;
    a.G = G;
    a.N = d.num_blocks;
    a.d = d.head_dim;
    a.kv_dtype = d.kv_dtype;
    a.part_tokens = P;
    a.max_parts = parts;
    a.scale = scale;
    a.k_scale = nullptr;
    a.v_scale = nullptr;
    a.out = out;
    a.ws_o = ws_o;
    a.ws_ml = ws_ml;
    a.status = d.device_status;
    a.engine = engine;
    a.tok_base = shared_prefix_len;
    a.part_base = splits;
    return launch_decode(a, tmk, tmv, s);
}

size_t paged_prefill_workspace_bytes(pkv_pool_t pool, int chunk_len, int num_q_heads, int ctx_before)
{
    (void)pool;
    (void)chunk_len;
    (void)num_q_heads;
    (void)ctx_before;
    return 0;
}

int paged_prefill_chunk_attn(pkv_pool_t pool, int layer, const void* q, int q_dtype, const int32_t* block_table,
                             int block_table_width, int ctx_before, int chunk_len, int num_q_heads, float scale,
                             float* out, void* workspace, size_t workspace_bytes, void* stream)
{
    (void)workspace;
    (void)workspace_bytes;
    return paged_prefill_chunk_attn_window(pool, layer, q, q_dtype, block_table, block_table_width, ctx_before,
                                           chunk_len, num_q_heads, scale, 0, out, stream);
}

int paged_prefill_chunk_attn_window(pkv_pool_t pool, int layer, const void* q, int q_dtype,
                                    const int32_t* block_table, int block_table_width, int ctx_before, int chunk_len,
                                    int num_q_heads, float scale, int sliding_window, float* out, void* stream)
{
    if (!pool) return PKV_ERR_NULL;
    if (sliding_window < 0) return PKV_ERR_ARG;
    const pkv_pool_desc& d = pool->d;
    if (layer < 0 || layer >= d.num_layers || ctx_before < 0 || chunk_len < 0 || num_q_heads <= 0 ||
        block_table_width <= 0)
        return PKV_ERR_ARG;
    if (num_q_heads % d.num_kv_heads) return PKV_ERR_SHAPE;
    if (is_quantized(d.kv_dtype)) return PKV_ERR_UNSUPPORTED;
    if (q_dtype != d.kv_dtype) return PKV_ERR_DTYPE;
    if ((long long)block_table_width * PKV_BLOCK_SIZE < (long long)ctx_before + chunk_len) return PKV_ERR_SHAPE;
    if (chunk_len == 0) return PKV_OK;
    if (!q || !block_table || !out) return PKV_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(q) & 15) || (reinterpret_cast<uintptr_t>(out) & 15)) return PKV_ERR_ARG;
    const CUtensorMap *tmk = nullptr, *tmv = nullptr;
    int rc = layer_maps(pool, layer, &tmk, &tmv);
    if (rc != PKV_OK) return rc;
    PrefillArgs a;
    a.q = q;
    a.q_dtype = q_dtype;
    a.table = block_table;
    a.W = block_table_width;
    a.P0 = ctx_before;
    a.C = chunk_len;
    a.H_q = num_q_heads;
    a.H_kv = d.num_kv_heads;
    a.G = num_q_heads / d.num_kv_heads;
    a.N = d.num_blocks;
    a.d = d.head_dim;
    a.kv_dtype = d.kv_dtype;
    a.scale = scale;
    a.out = out;
    a.status = d.device_status;
    a.window = sliding_window;
    if (sliding_window == 0 && prefill_tc_supported(a.d, a.G, a.kv_dtype)) {
        CUtensorMap tmq;
        auto enc = tensor_map_encoder();
        if (!enc || !make_q_map(&tmq, q, chunk_len, num_q_heads, a.G, enc)) return PKV_ERR_CUDA;
        return launch_prefill_tc(a, &tmq, tmk, tmv, static_cast<cudaStream_t>(stream));
    }
    return launch_prefill(a, tmk, tmv, static_cast<cudaStream_t>(stream));
}

int pkv_test_withhold_copy(int tile, long long wait_cycles)
{
    if (tile < 0) {
        g_hold_tile.store(-1);
        g_wait_cycles.store(kDefaultWaitCycles);
        return PKV_OK;
    }
    if (wait_cycles <= 0 || wait_cycles > kDefaultWaitCycles) return PKV_ERR_ARG;
    g_wait_cycles.store(wait_cycles);
    g_hold_tile.store(tile);
    return PKV_OK;
}

int pkv_get_device_status(pkv_pool_t pool, void* stream, int32_t* status_out)
{
    return pkv_read_device_status(pool, stream, status_out);
}

int pkv_read_device_status(pkv_pool_t pool, void* stream, int32_t* status_out)
{
    if (!pool || !status_out) return PKV_ERR_NULL;
    *status_out = 0;
    if (!pool->d.device_status) return PKV_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t host = 0;
    if (cudaMemcpyAsync(&host, pool->d.device_status, sizeof(host), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return PKV_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return PKV_ERR_CUDA;
    if (host != 0 && cudaMemsetAsync(pool->d.device_status, 0, sizeof(int32_t), s) != cudaSuccess) return PKV_ERR_CUDA;
    *status_out = host;
    if (host & PKV_DEV_TIMEOUT) return PKV_ERR_TIMEOUT;
    return host ? PKV_ERR_INDEX : PKV_OK;
}

}  // extern "C"
