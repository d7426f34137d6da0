// blocks.cu -- whole-block moves: copy-on-write copies and swap to / from host memory.
//
// "KV cache, continuous batching and paged attention", section "Paged attention": blocks
// can be shared copy-on-write (parallel samples, beam search, common prefixes); a
// sequence that diverges from a shared block gets a private copy of it.
// "KV cache, GQA, paging and continuous batching", section "The scheduler, and
// preemption": a preempted sequence's blocks are swapped to host memory and back.
//
// A block is, for every layer, its H_kv tiles of K and of V (H_kv * 16 * row_bytes bytes
// each, contiguous) and, for quantized pools, its 2 * H_kv scales.  Layers may live in
// separate allocations: the kernels get every layer's base pointers as a parameter.  All
// moves are 16-byte vector copies.  A copy runs one CTA per (pair, layer, K/V) span with
// several loads in flight per thread, bound by HBM; a swap runs one thread per 16 bytes
// over the host link (the kernel reads / writes pinned host memory directly through its
// device mapping).
#include "common.cuh"
#include "internal.h"

namespace pkv {

namespace {

struct BlockGeom {
    size_t tile_row;      // bytes of one block's K (or V) in one layer: H_kv * 16 * row_bytes
    size_t scales;        // scales per block per layer per K/V (H_kv), 0 for 16-bit pools
    int L, N;
};

// Every layer's K / V pool and K / V scales (scales null for 16-bit pools), passed by value.
struct LayerBases {
    uint8_t* k[PKV_MAX_LAYERS];
    uint8_t* v[PKV_MAX_LAYERS];
    float* ks[PKV_MAX_LAYERS];
    float* vs[PKV_MAX_LAYERS];
};

// Host layout of one swapped block: [L][K, V][tile_row bytes], then [L][K, V][scales] fp32.
__host__ __device__ inline size_t swap_block_bytes(const BlockGeom& g)
{
    return (size_t)g.L * 2 * g.tile_row + (size_t)g.L * 2 * g.scales * sizeof(float);
}

// One CTA per (pair, layer, K/V): the block's contiguous H_kv * 16 * row_bytes bytes of
// that layer's K or V, copied with 16-byte vectors, each thread keeping kUnroll loads in
// flight before its stores; the first threads also copy the scales.
constexpr int kCopyThreads = 256;
constexpr int kUnroll = 4;

__global__ void __launch_bounds__(kCopyThreads)
copy_blocks_kernel(const __grid_constant__ LayerBases lb, BlockGeom g, const int32_t* __restrict__ src,
                   const int32_t* __restrict__ dst, int32_t* status)
{
    const int item = blockIdx.x;                 // (pair * L + layer) * 2 + is_v
    const bool is_v = item & 1;
    const int layer = (item >> 1) % g.L;
    const int pr = (item >> 1) / g.L;
    const int sb = src[pr], db = dst[pr];
    if ((unsigned)sb >= (unsigned)g.N || (unsigned)db >= (unsigned)g.N) {
        if (threadIdx.x == 0 && layer == 0 && !is_v) flag_status(status, PKV_DEV_BAD_BLOCK);
        return;
    }
    uint8_t* base = is_v ? lb.v[layer] : lb.k[layer];
    const uint4* from = reinterpret_cast<const uint4*>(base + (size_t)sb * g.tile_row);
    uint4* to = reinterpret_cast<uint4*>(base + (size_t)db * g.tile_row);
    const int chunks = (int)(g.tile_row / 16);
    for (int c0 = threadIdx.x; c0 < chunks; c0 += kCopyThreads * kUnroll) {
        uint4 t[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int c = c0 + u * kCopyThreads;
            if (c < chunks) t[u] = from[c];
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int c = c0 + u * kCopyThreads;
            if (c < chunks) to[c] = t[u];
        }
    }
    if (g.scales) {
        float* sc = is_v ? lb.vs[layer] : lb.ks[layer];
        for (size_t h = threadIdx.x; h < g.scales; h += kCopyThreads) sc[(size_t)db * g.scales + h] = sc[(size_t)sb * g.scales + h];
    }
}

// Swap out (to_host) or in: block blocks[j] <-> host slot j.
__global__ void swap_blocks_kernel(const __grid_constant__ LayerBases lb, BlockGeom g,
                                   const int32_t* __restrict__ blocks, int n, uint8_t* host, bool to_host,
                                   int32_t* status)
{
    const size_t chunks = g.tile_row / 16;
    const size_t per_blk = (size_t)g.L * 2 * chunks;
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= per_blk * n) return;
    const int j = (int)(i / per_blk);
    size_t rem = i % per_blk;
    const int layer = (int)(rem / (2 * chunks));
    rem %= 2 * chunks;
    const bool is_v = rem >= chunks;
    const size_t c = rem % chunks;
    const int blk = blocks[j];
    if ((unsigned)blk >= (unsigned)g.N) {
        if (c == 0 && layer == 0 && !is_v) flag_status(status, PKV_DEV_BAD_BLOCK);
        return;
    }
    uint8_t* hb = host + (size_t)j * swap_block_bytes(g);
    uint4* dev = reinterpret_cast<uint4*>((is_v ? lb.v[layer] : lb.k[layer]) + (size_t)blk * g.tile_row) + c;
    uint4* hst = reinterpret_cast<uint4*>(hb + ((size_t)layer * 2 + (is_v ? 1 : 0)) * g.tile_row) + c;
    if (to_host) *hst = *dev;
    else *dev = *hst;
    if (g.scales && c < g.scales) {
        float* sc = (is_v ? lb.vs[layer] : lb.ks[layer]) + (size_t)blk * g.scales + c;
        float* hs = reinterpret_cast<float*>(hb + (size_t)g.L * 2 * g.tile_row) + ((size_t)layer * 2 + (is_v ? 1 : 0)) * g.scales + c;
        if (to_host) *hs = *sc;
        else *sc = *hs;
    }
}

BlockGeom geom_of(const pkv_pool* pool)
{
    BlockGeom g;
    g.tile_row = (size_t)pool->d.num_kv_heads * pool->tile_bytes;
    g.scales = pool->layer_scales ? (size_t)pool->d.num_kv_heads : 0;
    g.L = pool->d.num_layers;
    g.N = pool->d.num_blocks;
    return g;
}

static int launch_moves(bool copy, const pkv_pool* pool, const int32_t* a, const int32_t* b, int n, uint8_t* host,
                        bool to_host, cudaStream_t s)
{
    const BlockGeom g = geom_of(pool);
    const size_t total = (size_t)n * g.L * 2 * (g.tile_row / 16);
    const int threads = 256;
    const size_t grid = (total + threads - 1) / threads;
    if (grid > 0x7fffffffULL) return PKV_ERR_ARG;
    LayerBases lb = {};
    for (int l = 0; l < g.L; ++l) {
        lb.k[l] = pool->k_base[l];
        lb.v[l] = pool->v_base[l];
        lb.ks[l] = pool->ks_base[l];
        lb.vs[l] = pool->vs_base[l];
    }
    if (copy) {
        const size_t items = (size_t)n * g.L * 2;
        if (items > 0x7fffffffULL) return PKV_ERR_ARG;
        copy_blocks_kernel<<<(unsigned)items, kCopyThreads, 0, s>>>(lb, g, a, b, pool->d.device_status);
    } else
        swap_blocks_kernel<<<(unsigned)grid, threads, 0, s>>>(lb, g, a, n, host, to_host, pool->d.device_status);
    return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

// Device address of a page-locked, mapped host buffer, or null.
static uint8_t* mapped_host(const void* host)
{
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, host) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    if (at.type != cudaMemoryTypeHost || !at.devicePointer) return nullptr;
    return static_cast<uint8_t*>(at.devicePointer);
}

static int swap(pkv_pool_t pool, const int32_t* blocks, int n, const void* host, bool to_host, void* stream)
{
    if (!pool) return PKV_ERR_NULL;
    if (n < 0) return PKV_ERR_ARG;
    if (n == 0) return PKV_OK;
    if (!blocks || !host) return PKV_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(host) & 15) return PKV_ERR_ARG;
    uint8_t* dev_view = mapped_host(host);
    if (!dev_view || (reinterpret_cast<uintptr_t>(dev_view) & 15)) return PKV_ERR_ARG;
    return launch_moves(false, pool, blocks, nullptr, n, dev_view, to_host, static_cast<cudaStream_t>(stream));
}

}  // namespace
}  // namespace pkv

using namespace pkv;

extern "C" {

int kv_copy_blocks(pkv_pool_t pool, const int32_t* src, const int32_t* dst, int num_pairs, void* stream)
{
    if (!pool) return PKV_ERR_NULL;
    if (num_pairs < 0) return PKV_ERR_ARG;
    if (num_pairs == 0) return PKV_OK;
    if (!src || !dst) return PKV_ERR_NULL;
    return launch_moves(true, pool, src, dst, num_pairs, nullptr, false, static_cast<cudaStream_t>(stream));
}

size_t kv_swap_bytes_per_block(pkv_pool_t pool) { return pool ? swap_block_bytes(geom_of(pool)) : 0; }

int kv_swap_out(pkv_pool_t pool, const int32_t* blocks, int num_blocks_to_move, void* host, void* stream)
{
    return swap(pool, blocks, num_blocks_to_move, host, true, stream);
}

int kv_swap_in(pkv_pool_t pool, const int32_t* blocks, int num_blocks_to_move, const void* host, void* stream)
{
    return swap(pool, blocks, num_blocks_to_move, host, false, stream);
}

}  // extern "C"
