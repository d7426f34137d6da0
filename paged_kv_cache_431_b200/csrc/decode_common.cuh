// decode_common.cuh -- pieces shared by the decode kernels (16-bit and quantized pools).
#pragma once

#include "common.cuh"
#include "internal.h"

namespace pkv {

constexpr int kMaxPartTiles = 256;   // partition_tokens <= 4096
constexpr float kLog2e = 1.4426950408889634f;

struct DecodeParams {
    const void* q;
    const int32_t* tables;
    const int32_t* ctx_lens;
    const float* k_scale;
    const float* v_scale;
    float* out;
    float* ws_o;
    float* ws_ml;
    int* counters;          // fused merge: one per (sequence, CTA row of the grid), zero at entry; null:
                            // the separate decode_reduce_kernel merges (cascade, CUDA-core engines)
    int32_t* status;
    int W, H_q, H_kv, G, N, part_tokens, max_parts;
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

// Split-K merge of the partials of query heads row0 .. row0 + nh - 1 (rows b * H_q + h) over
// partitions 0 .. nparts-1 of this launch, by one warp:
//   out = sum_i 2^(m_i - M) o_i / sum_i 2^(m_i - M) l_i,  M = max_i m_i  (log2-domain m).
// The partials were written by other CTAs: loads bypass L1 (ld.global.cg).
template <int D>
__device__ __forceinline__ void merge_partials(const DecodeParams& p, size_t row0, int nh, int nparts, int lane)
{
    constexpr int V = D / 32;   // floats per lane
    for (int h = 0; h < nh; ++h) {
        const size_t base = (row0 + h) * p.slots + p.part_base;
        const float2* ml = reinterpret_cast<const float2*>(p.ws_ml) + base;
        float M = -INFINITY;
        for (int i = lane; i < nparts; i += 32) M = fmaxf(M, __ldcg(&ml[i]).x);
#pragma unroll
        for (int off = 16; off; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        float L = 0.f;
        for (int i = lane; i < nparts; i += 32) {
            const float2 v = __ldcg(&ml[i]);
            L += ex2(v.x - M) * v.y;
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
        float acc[V];
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] = 0.f;
        const float* po = p.ws_o + base * D + lane * V;
#pragma unroll 4
        for (int i = 0; i < nparts; ++i) {
            const float w = ex2(__ldcg(&ml[i]).x - M);
            if constexpr (V == 4) {
                const float4 v = __ldcg(reinterpret_cast<const float4*>(po + (size_t)i * D));
                acc[0] += w * v.x; acc[1] += w * v.y; acc[2] += w * v.z; acc[3] += w * v.w;
            } else {
                const float2 v = __ldcg(reinterpret_cast<const float2*>(po + (size_t)i * D));
                acc[0] += w * v.x; acc[1] += w * v.y;
            }
        }
        const float inv = 1.f / L;
        float* o = p.out + (row0 + h) * D + lane * V;
        if constexpr (V == 4) {
            *reinterpret_cast<float4*>(o) = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
        } else {
            *reinterpret_cast<float2*>(o) = make_float2(acc[0] * inv, acc[1] * inv);
        }
    }
}

// After this CTA's partials are written: count the partition done; true in the CTA that
// completes the (sequence, CTA row) -- it then merges, and leaves the counter at zero for the
// next call.  Every thread of the CTA calls it (one warp: `lane`-uniform; several warps: a CTA
// barrier inside); all return the same value.
__device__ __forceinline__ bool last_partition(const DecodeParams& p, int b, int nparts, int* s_flag)
{
    __threadfence();   // this thread's partial stores are visible device-wide before the count
    __syncthreads();
    if (threadIdx.x == 0) {
        int* c = p.counters + (size_t)b * gridDim.y + blockIdx.y;
        const int done = atomicAdd(c, 1) + 1;
        const bool last = done == nparts;
        if (last) atomicExch(c, 0);
        *s_flag = last;
    }
    __syncthreads();
    const bool last = *s_flag;
    if (last) __threadfence();   // the other CTAs' partials are read after their counts
    return last;
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

// Launch the quantized-pool decode kernel (decode_quant.cu).
int launch_decode_quant(const DecodeParams& p, int kv_dtype, int d, int nht, dim3 grid, cudaStream_t s,
                        const CUtensorMap* tmk, const CUtensorMap* tmv);

}  // namespace pkv
