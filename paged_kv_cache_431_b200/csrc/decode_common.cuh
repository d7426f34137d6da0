// decode_common.cuh -- pieces shared by the decode kernels (16-bit and quantized pools).
#pragma once

#include "common.cuh"
#include "internal.h"

namespace pkv {

constexpr int kMaxPartTiles = 256;   // partition_tokens <= 4096
constexpr float kLog2e = 1.4426950408889634f;

// L2 cache hints of the decode kernels: the K/V stream is read once (evict_first), the
// split-K partials are read back by the merge soon after (evict_last).
#ifndef PKV_L2_HINTS
#define PKV_L2_HINTS 3
#endif
constexpr bool kHintKV = (PKV_L2_HINTS & 1) != 0;
constexpr bool kHintPartials = (PKV_L2_HINTS & 2) != 0;

struct DecodeParams {
    const void* q;
    const int32_t* tables;
    const int32_t* ctx_lens;
    const float* k_scale;
    const float* v_scale;
    float* out;
    float* ws_o;
    float* ws_ml;
    int32_t* status;
    int W, H_q, H_kv, G, N, part_tokens, max_parts;
    int num_seqs;
    // Partitions cover tokens tok_base .. ctx-1 and write workspace slots part_base + part of
    // a row of `slots`.  Plain decode: 0, 0, max_parts.  Shared-prefix (cascade) decode:
    // tok_base = prefix length, part_base = key splits of the prefix (slots 0 .. part_base-1
    // hold the prefix's partials).
    int tok_base, part_base, slots;
    int prefix_blocks;      // cascade: table entries every sequence must share with row 0
    int window;             // sliding window: tokens a query sees (0: the whole context)
    int hgroups;            // CTAs per KV head, 16 query heads each (G > 16 takes several)
    int q_bf16;             // q dtype: 1 bf16, 0 f16
    float scale_log2;
    int hold_tile;          // test hook: this CTA-local tile's copy is never issued (-1: none)
    long long wait_cycles;  // bound of every wait on a copy (SM cycles)
};

// Context length of sequence b, clamped to what the table and the grid can cover (with a
// window the grid covers any context: a query reads at most window + 15 tokens' blocks).
__device__ __forceinline__ int checked_ctx(const DecodeParams& p, int b, bool report)
{
    int ctx = p.ctx_lens[b];
    const int cap = p.window ? p.W * kBlock : min(p.W * kBlock, p.tok_base + p.max_parts * p.part_tokens);
    if (ctx < p.tok_base || ctx > cap) {
        if (report) flag_status(p.status, PKV_DEV_BAD_LENGTH);
        ctx = ctx < p.tok_base ? p.tok_base : cap;
    }
    return ctx;
}

// First token the query sees: ctx - window with a sliding window, else 0.
__device__ __forceinline__ int visible_lo(const DecodeParams& p, int ctx)
{
    return (p.window > 0 && ctx > p.window) ? ctx - p.window : 0;
}

// First token of partition 0: the prefix end (cascade), or the block holding visible_lo.
__device__ __forceinline__ int seq_base(const DecodeParams& p, int ctx)
{
    return p.window > 0 ? (visible_lo(p, ctx) & ~(kBlock - 1)) : p.tok_base;
}

// Partitions of this launch that sequence b's context needs.
__device__ __forceinline__ int part_count(const DecodeParams& p, int ctx)
{
    return (ctx - seq_base(p, ctx) + p.part_tokens - 1) / p.part_tokens;
}

// Workspace slot (row = b * H_q + h) of partition `part` of this launch.
__device__ __forceinline__ size_t ws_slot(const DecodeParams& p, size_t row, int part)
{
    return row * p.slots + p.part_base + part;
}

// Byte address of 16-byte chunk `c` of row `t` in a tile stored as 128-byte-wide TMA
// boxes of 16 rows with the 128-byte swizzle (chunk index XOR row % 8).
__device__ __forceinline__ uint32_t swz128(uint32_t tile, int t, int c)
{
    return tile + (uint32_t)((c >> 3) * (16 * 128) + t * 128 + (((c & 7) ^ (t & 7)) << 4));
}


// CUDA-core (FP32 FMA) decode for 16-bit pools (decode_simt.cu); f2 = packed fp32x2 FMA.
bool decode_simt_supported(int d, int G, int kv_dtype);
int launch_decode_simt(const DecodeParams& p, int kv_dtype, int G, bool f2, dim3 grid, cudaStream_t s,
                       const CUtensorMap* tmk, const CUtensorMap* tmv);

// tcgen05 decode for groups of 64 or 128 query heads (decode_tc.cu).
bool decode_tc_supported(int d, int G, int kv_dtype);
int launch_decode_tc(const DecodeParams& p, int kv_dtype, const CUtensorMap* tmq, const CUtensorMap* tmk,
                     const CUtensorMap* tmv, cudaStream_t s);

// tcgen05 decode for groups of 64 query heads with the keys on the MMA's M side (decode_tc_keys.cu).
bool decode_tck_supported(int d, int G, int kv_dtype);
bool make_q_map_seq(CUtensorMap* map, const void* q, int B, int H_q, PFN_encode enc);
int launch_decode_tck(const DecodeParams& p, int kv_dtype, const CUtensorMap* tmq, const CUtensorMap* tmk,
                      const CUtensorMap* tmv, cudaStream_t s);

// tcgen05 decode for fp8 pools with 8 query heads per KV head, codes fed to kind::f8f6f4
// MMAs (decode_tc_fp8.cu).
bool decode_tc_fp8_supported(int d, int G, int kv_dtype);
int launch_decode_tc_fp8(const DecodeParams& p, const CUtensorMap* tmk, const CUtensorMap* tmv, cudaStream_t s);

// Launch the quantized-pool decode kernel (decode_quant.cu).
int launch_decode_quant(const DecodeParams& p, int kv_dtype, int d, int nht, dim3 grid, cudaStream_t s,
                        const CUtensorMap* tmk, const CUtensorMap* tmv);

}  // namespace pkv
