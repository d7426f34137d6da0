// append.cu -- kv_append: write new tokens' K/V into their pool slots.
//
// "KV cache, continuous batching and paged attention", section "The KV cache": keys and
// values of earlier tokens never change, so each step only caches the new token's K/V.
// "KV cache, GQA, paging and continuous batching", section "PagedAttention": a block
// table maps logical positions to physical 16-token blocks; the caller passes the
// resulting slot (block * 16 + offset) of every new token.
//
// 16-bit pools: a scatter of 16-byte chunks, one thread per chunk, coalesced on the
// source side; each (token, head) row lands contiguously in its tile.
//
// Quantized pools (inference guide a2-inf-2, section "KV-cache quantization": integer
// codes sharing one scale), fused into the scatter, in three short kernels:
//   1. clear the per-block scratch of every block this call touches;
//   2. per (token, head) row: |x| max by warp shuffles, atomicMax into the block's
//      amax (non-negative floats order like their bit patterns), atomicOr of the
//      token's offset into the block's written-offsets mask;
//   3. per (token, head) row: s = max(S_old, amax / Q) with S_old = 0 for a block the
//      call starts (offset 0 written), codes = round-half-even(x / s) (int, clamped)
//      or e4m3 saturating (fp8).  The row with the lowest written offset of the block
//      re-quantizes the block's other (not written) rows once when s > S_old > 0 and
//      stores s.  Another row of the same block may read the scale before or after that
//      store: max(S_old, amax/Q) and max(s, amax/Q) are both s, so the result is the same.
// All arithmetic is IEEE fp32 with explicit round-to-nearest operations (no fast math).
#include <cuda_fp8.h>

#include "common.cuh"
#include "internal.h"

namespace pkv {

// ---------------------------------------------------------------- 16-bit ----

__global__ void append16_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                const int32_t* __restrict__ slots, int T, int H_kv, int chunks_per_row,
                                uint8_t* k_pool, uint8_t* v_pool, int N, int32_t* status)
{
    const int64_t per_tensor = (int64_t)T * H_kv * chunks_per_row;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= 2 * per_tensor) return;
    const bool is_v = i >= per_tensor;
    const int64_t e = is_v ? i - per_tensor : i;
    const int c = (int)(e % chunks_per_row);
    const int64_t row = e / chunks_per_row;          // token * H_kv + head
    const int h = (int)(row % H_kv);
    const int tok = (int)(row / H_kv);
    const int slot = slots[tok];
    if (slot < 0) return;
    if (slot >= N * kBlock) {
        if (c == 0 && h == 0 && !is_v) flag_status(status, PKV_DEV_BAD_SLOT);
        return;
    }
    const int blk = slot / kBlock, off = slot % kBlock;
    const size_t dst_row = ((size_t)blk * H_kv + h) * kBlock + off;
    uint4* dst = reinterpret_cast<uint4*>(is_v ? v_pool : k_pool) + dst_row * chunks_per_row + c;
    *dst = (is_v ? v : k)[e];
}

// ------------------------------------------------------------- quantized ----

struct QScratch {
    uint32_t* amax_k;   // [N][H_kv]
    uint32_t* amax_v;   // [N][H_kv]
    uint32_t* mask;     // [N]
};

__device__ __forceinline__ QScratch scratch_of(void* ws, int N, int H_kv)
{
    QScratch q;
    q.amax_k = static_cast<uint32_t*>(ws);
    q.amax_v = q.amax_k + (size_t)N * H_kv;
    q.mask = q.amax_v + (size_t)N * H_kv;
    return q;
}

__global__ void qappend_clear_kernel(const int32_t* __restrict__ slots, int T, int H_kv, int N, void* ws)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)T * H_kv) return;
    const int tok = (int)(i / H_kv), h = (int)(i % H_kv);
    const int slot = slots[tok];
    if (slot < 0 || slot >= N * kBlock) return;
    QScratch q = scratch_of(ws, N, H_kv);
    const int blk = slot / kBlock;
    q.amax_k[(size_t)blk * H_kv + h] = 0u;
    q.amax_v[(size_t)blk * H_kv + h] = 0u;
    if (h == 0) q.mask[blk] = 0u;
}

template <int D>
__device__ __forceinline__ void load_row_bf16(const __nv_bfloat16* src, int lane, float (&x)[D / 32])
{
    constexpr int E = D / 32;
    if constexpr (E == 4) {
        const uint2 u = *reinterpret_cast<const uint2*>(src + lane * E);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
        x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
    } else {
        const uint32_t u = *reinterpret_cast<const uint32_t*>(src + lane * E);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u));
        x[0] = a.x; x[1] = a.y;
    }
}

template <int D>
__global__ void qappend_reduce_kernel(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                                      const int32_t* __restrict__ slots, int T, int H_kv, int N, void* ws,
                                      int32_t* status)
{
    const int warp = (int)(((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
    const int lane = threadIdx.x & 31;
    if (warp >= T * H_kv) return;
    const int tok = warp / H_kv, h = warp % H_kv;
    const int slot = slots[tok];
    if (slot < 0) return;
    if (slot >= N * kBlock) {
        if (lane == 0 && h == 0) flag_status(status, PKV_DEV_BAD_SLOT);
        return;
    }
    float xk[D / 32], xv[D / 32];
    load_row_bf16<D>(k + (size_t)warp * D, lane, xk);
    load_row_bf16<D>(v + (size_t)warp * D, lane, xv);
    float ak = 0.f, av = 0.f;
#pragma unroll
    for (int e = 0; e < D / 32; ++e) {
        ak = fmaxf(ak, fabsf(xk[e]));
        av = fmaxf(av, fabsf(xv[e]));
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) {
        ak = fmaxf(ak, __shfl_xor_sync(0xffffffffu, ak, off));
        av = fmaxf(av, __shfl_xor_sync(0xffffffffu, av, off));
    }
    if (lane == 0) {
        QScratch q = scratch_of(ws, N, H_kv);
        const int blk = slot / kBlock;
        atomicMax(&q.amax_k[(size_t)blk * H_kv + h], __float_as_uint(ak));
        atomicMax(&q.amax_v[(size_t)blk * H_kv + h], __float_as_uint(av));
        if (h == 0) atomicOr(&q.mask[blk], 1u << (slot % kBlock));
    }
}

// Code of x / s for storage dtype DT, IEEE fp32 round-to-nearest throughout.
template <int DT>
__device__ __forceinline__ uint32_t quant_code(float x, float s)
{
    if (s == 0.f) return 0u;
    const float r = __fdiv_rn(x, s);
    if constexpr (DT == PKV_FP8E4M3) {
        return (uint32_t)__nv_cvt_float_to_fp8(r, __NV_SATFINITE, __NV_E4M3);
    } else {
        constexpr float Q = DT == PKV_INT8 ? 127.f : 7.f;
        const float c = fminf(fmaxf(rintf(r), -Q), Q);
        return (uint32_t)(int)c & (DT == PKV_INT8 ? 0xffu : 0xfu);
    }
}

template <int DT>
__device__ __forceinline__ float code_value(uint32_t c)
{
    if constexpr (DT == PKV_FP8E4M3) {
        return __half2float(__half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c, __NV_E4M3)));
    } else if constexpr (DT == PKV_INT8) {
        return (float)(int)(int8_t)c;
    } else {
        return (float)(((int)c ^ 8) - 8);   // 4-bit two's complement
    }
}

template <int DT>
__device__ __forceinline__ uint32_t requant_code(uint32_t c, float s_old, float s)
{
    const float r = __fdiv_rn(__fmul_rn(code_value<DT>(c), s_old), s);
    if constexpr (DT == PKV_FP8E4M3) {
        return (uint32_t)__nv_cvt_float_to_fp8(r, __NV_SATFINITE, __NV_E4M3);
    } else {
        constexpr float Q = DT == PKV_INT8 ? 127.f : 7.f;
        const float q = fminf(fmaxf(rintf(r), -Q), Q);
        return (uint32_t)(int)q & (DT == PKV_INT8 ? 0xffu : 0xfu);
    }
}

// Lane's E = D/32 codes of one row, packed little-endian: bytes for 8-bit codes,
// nibbles (element 2j low) for int4.
template <int DT, int E>
__device__ __forceinline__ void store_codes(uint8_t* row, int lane, const uint32_t (&c)[E])
{
    if constexpr (DT == PKV_INT4) {
        uint32_t w = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) w |= c[e] << (4 * e);
        if constexpr (E == 4) *reinterpret_cast<uint16_t*>(row + lane * 2) = (uint16_t)w;
        else row[lane] = (uint8_t)w;
    } else {
        uint32_t w = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) w |= c[e] << (8 * e);
        if constexpr (E == 4) *reinterpret_cast<uint32_t*>(row + lane * 4) = w;
        else *reinterpret_cast<uint16_t*>(row + lane * 2) = (uint16_t)w;
    }
}

template <int DT, int E>
__device__ __forceinline__ void load_codes(const uint8_t* row, int lane, uint32_t (&c)[E])
{
    if constexpr (DT == PKV_INT4) {
        const uint32_t w = E == 4 ? *reinterpret_cast<const uint16_t*>(row + lane * 2) : row[lane];
#pragma unroll
        for (int e = 0; e < E; ++e) c[e] = (w >> (4 * e)) & 0xfu;
    } else {
        const uint32_t w = E == 4 ? *reinterpret_cast<const uint32_t*>(row + lane * 4)
                                  : *reinterpret_cast<const uint16_t*>(row + lane * 2);
#pragma unroll
        for (int e = 0; e < E; ++e) c[e] = (w >> (8 * e)) & 0xffu;
    }
}

template <int DT, int D>
__device__ __forceinline__ void write_one(const __nv_bfloat16* src, uint8_t* tile, float* scale, uint32_t amax_bits,
                                          uint32_t mask, int off, int lane)
{
    constexpr int E = D / 32;
    constexpr int RB = DT == PKV_INT4 ? D / 2 : D;
    constexpr float Q = DT == PKV_INT8 ? 127.f : DT == PKV_INT4 ? 7.f : 448.f;
    const bool fresh = (mask & 1u) != 0u;
    const float s_old = fresh ? 0.f : *scale;
    const float s = fmaxf(s_old, __fdiv_rn(__uint_as_float(amax_bits), Q));
    float x[E];
    load_row_bf16<D>(src, lane, x);
    uint32_t c[E];
#pragma unroll
    for (int e = 0; e < E; ++e) c[e] = quant_code<DT>(x[e], s);
    store_codes<DT, E>(tile + off * RB, lane, c);
    const int leader = __ffs(mask) - 1;
    if (off == leader) {
        if (s > s_old && s_old > 0.f) {
            for (int o2 = 0; o2 < kBlock; ++o2) {
                if (mask & (1u << o2)) continue;
                uint32_t oc[E];
                load_codes<DT, E>(tile + o2 * RB, lane, oc);
#pragma unroll
                for (int e = 0; e < E; ++e) oc[e] = requant_code<DT>(oc[e], s_old, s);
                store_codes<DT, E>(tile + o2 * RB, lane, oc);
            }
        }
        if (lane == 0) *scale = s;
    }
}

template <int DT, int D>
__global__ void qappend_write_kernel(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                                     const int32_t* __restrict__ slots, int T, int H_kv, int N, const void* ws,
                                     uint8_t* k_pool, uint8_t* v_pool, float* k_scale, float* v_scale)
{
    const int warp = (int)(((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
    const int lane = threadIdx.x & 31;
    if (warp >= T * H_kv) return;
    const int tok = warp / H_kv, h = warp % H_kv;
    const int slot = slots[tok];
    if (slot < 0 || slot >= N * kBlock) return;
    const int blk = slot / kBlock, off = slot % kBlock;
    QScratch q = scratch_of(const_cast<void*>(ws), N, H_kv);
    const uint32_t mask = q.mask[blk];
    const size_t th = (size_t)blk * H_kv + h;
    constexpr int RB = DT == PKV_INT4 ? D / 2 : D;
    write_one<DT, D>(k + (size_t)warp * D, k_pool + th * kBlock * RB, k_scale + th, q.amax_k[th], mask, off, lane);
    write_one<DT, D>(v + (size_t)warp * D, v_pool + th * kBlock * RB, v_scale + th, q.amax_v[th], mask, off, lane);
}

// ---------------------------------------------------------------- launch ----

size_t append_workspace_bytes(int N, int H_kv, int kv_dtype)
{
    if (!is_quantized(kv_dtype)) return 0;
    return ((size_t)2 * N * H_kv + N) * sizeof(uint32_t);
}

template <int DT, int D>
static void launch_qwrite(const AppendArgs& a, int blocks, cudaStream_t s)
{
    qappend_write_kernel<DT, D><<<blocks, 128, 0, s>>>(
        static_cast<const __nv_bfloat16*>(a.k), static_cast<const __nv_bfloat16*>(a.v), a.slots, a.T, a.H_kv, a.N,
        a.workspace, a.k_pool, a.v_pool, a.k_scale, a.v_scale);
}

int launch_append(const AppendArgs& a, cudaStream_t s)
{
    if (a.T == 0) return PKV_OK;
    if (!is_quantized(a.kv_dtype)) {
        const int cpr = a.d * 2 / 16;
        const int64_t n = 2LL * a.T * a.H_kv * cpr;
        const int threads = 256;
        append16_kernel<<<(unsigned)((n + threads - 1) / threads), threads, 0, s>>>(
            static_cast<const uint4*>(a.k), static_cast<const uint4*>(a.v), a.slots, a.T, a.H_kv, cpr, a.k_pool,
            a.v_pool, a.N, a.status);
        return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
    }
    const int64_t rows = (int64_t)a.T * a.H_kv;
    qappend_clear_kernel<<<(unsigned)((rows + 255) / 256), 256, 0, s>>>(a.slots, a.T, a.H_kv, a.N, a.workspace);
    const int blocks = (int)((rows + 3) / 4);   // one warp per (token, head) row
    const __nv_bfloat16* k = static_cast<const __nv_bfloat16*>(a.k);
    const __nv_bfloat16* v = static_cast<const __nv_bfloat16*>(a.v);
    if (a.d == 128) qappend_reduce_kernel<128><<<blocks, 128, 0, s>>>(k, v, a.slots, a.T, a.H_kv, a.N, a.workspace, a.status);
    else qappend_reduce_kernel<64><<<blocks, 128, 0, s>>>(k, v, a.slots, a.T, a.H_kv, a.N, a.workspace, a.status);
    switch (a.kv_dtype * 1000 + a.d) {
    case PKV_INT8 * 1000 + 128: launch_qwrite<PKV_INT8, 128>(a, blocks, s); break;
    case PKV_INT8 * 1000 + 64: launch_qwrite<PKV_INT8, 64>(a, blocks, s); break;
    case PKV_INT4 * 1000 + 128: launch_qwrite<PKV_INT4, 128>(a, blocks, s); break;
    case PKV_INT4 * 1000 + 64: launch_qwrite<PKV_INT4, 64>(a, blocks, s); break;
    case PKV_FP8E4M3 * 1000 + 128: launch_qwrite<PKV_FP8E4M3, 128>(a, blocks, s); break;
    case PKV_FP8E4M3 * 1000 + 64: launch_qwrite<PKV_FP8E4M3, 64>(a, blocks, s); break;
    default: return PKV_ERR_UNSUPPORTED;
    }
    return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

}  // namespace pkv
