// internal.h -- host-side types shared by the C-ABI implementation and the kernel launchers.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>
#include <vector>

#include "../../include/pkv.h"

struct pkv_pool {
    pkv_pool_desc d;
    int row_bytes;             // bytes of one token row of one KV head
    size_t tile_bytes;         // 16 rows: one (block, kv head) tile
    size_t layer_bytes;        // bytes of one layer's K (or V) pool
    size_t layer_scales;       // fp32 scales per layer (N * H_kv), 0 for 16-bit pools
    // Per layer: base of its K and V pools and of its K and V scales (null for 16-bit pools).
    // Dense pools: offsets into desc.k_data etc.; kv_pool_create_layers: the caller's pointers.
    std::vector<uint8_t*> k_base, v_base;
    std::vector<float*> ks_base, vs_base;
    std::mutex mu;             // guards the lazily built tensor maps
    bool maps_ready = false;
    std::vector<CUtensorMap> tmk, tmv;   // per layer: K and V pool as a 2-D tensor
};

namespace pkv {

// The test hook of pkv_test_withhold_copy, read by every attention launcher: the CTA-local
// index of the K/V tile whose copy is withheld (-1: none) and the wait bound in SM cycles.
struct WaitHook {
    int hold_tile;
    long long wait_cycles;
};
WaitHook wait_hook();
constexpr long long kDefaultWaitCycles = 2000000000LL;   // about 1 s at the B200's clock

int row_bytes_of(int dtype, int head_dim);
bool is_quantized(int dtype);

// Tensor maps for `layer` (built on first use). Returns PKV_OK or PKV_ERR_CUDA.
int layer_maps(pkv_pool* pool, int layer, const CUtensorMap** tmk, const CUtensorMap** tmv);

int num_sms();

struct DecodeArgs {
    const void* q;
    int q_dtype;
    const int32_t* tables;
    int W;
    const int32_t* ctx_lens;
    int B, H_q, H_kv, G, N, d;
    int kv_dtype;
    int part_tokens, max_parts;
    float scale;
    const float* k_scale;   // this layer's scales, or null
    const float* v_scale;
    float* out;
    float* ws_o;            // [B][H_q][max_parts][d]
    float* ws_ml;           // [B][H_q][max_parts][2]
    int32_t* status;
    int engine;             // 0 auto, 1 warp-level mma.sync, 2 / 3 CUDA-core FMA
    int tok_base = 0;       // first token the partitions cover (cascade: the prefix length)
    int part_base = 0;      // first workspace slot they write (cascade: 1)
    int window = 0;         // sliding window (tokens a query sees), 0 = whole context
};

int launch_decode(const DecodeArgs& a, const CUtensorMap* tmk, const CUtensorMap* tmv, cudaStream_t s);

struct AppendArgs {
    const void* k;
    const void* v;
    const int32_t* slots;
    int T, N, H_kv, d, kv_dtype;
    uint8_t* k_pool;        // this layer
    uint8_t* v_pool;
    float* k_scale;         // this layer, quantized only
    float* v_scale;
    void* workspace;        // quantized only: per-block scratch
    int32_t* status;
};

int launch_append(const AppendArgs& a, cudaStream_t s);
size_t append_workspace_bytes(int N, int H_kv, int kv_dtype);

struct PrefillArgs {
    const void* q;
    int q_dtype;
    const int32_t* table;
    int W, P0, C, H_q, H_kv, G, N, d;
    int kv_dtype;
    float scale;
    float* out;
    int32_t* status;
    // tcgen05 form only: shared-prefix (cascade) pass of the decode.  With cascade_nkeys > 0
    // the C positions are the decode batch, every row sees keys 0 .. cascade_nkeys-1, and the
    // partials (o, m, l) of the key_splits key ranges go to slots 0 .. key_splits-1 of decode
    // workspace rows of ws_slots slots.
    int window = 0;         // sliding window (warp-level form only)
    int cascade_nkeys = 0;
    int key_splits = 1;     // cascade: CTAs the prefix keys are split over (partials in slots 0..)
    int ws_slots = 0;
    float* ws_o = nullptr;
    float* ws_ml = nullptr;
};

int launch_prefill(const PrefillArgs& a, const CUtensorMap* tmk, const CUtensorMap* tmv, cudaStream_t s);

// CTAs per SM of the automatic decode engine for this shape when it is one of the keys-on-M
// tcgen05 kernels (decode_tc_keys.cu: 64 query heads per KV head, one CTA per SM;
// decode_tc_fp8.cu: fp8 pools with 8, two CTAs per SM), else 0.  Their split-K partitions
// follow their own rule.
int decode_keys_tc_available(int d, int G, int kv_dtype);

using PFN_encode = PFN_cuTensorMapEncodeTiled_v12000;
PFN_encode tensor_map_encoder();   // null when no driver is present

// tcgen05 / TMEM form of the chunked prefill (prefill_tc.cu)
bool prefill_tc_supported(int d, int G, int kv_dtype);
// Key splits of the cascade prefix pass that fill the GPU (>= 1, <= key tiles).
int prefill_tc_key_splits(int C, int G, int H_kv, int nkeys);
bool make_q_map(CUtensorMap* map, const void* q, int C, int H_q, int G, PFN_encode enc);
int launch_prefill_tc(const PrefillArgs& a, const CUtensorMap* tmq, const CUtensorMap* tmk, const CUtensorMap* tmv,
                      cudaStream_t s);

}  // namespace pkv
