// prefill.cu -- paged_prefill_chunk_attn: one chunk of a long prompt against the paged cache.
//
// Inference guide a2-inf-2, section "Chunked prefill", and "KV cache, continuous
// batching and paged attention", section "Scheduling prefill and decode": a long
// prompt is prefilled in chunks mixed with decode steps.  Query position P0 + i of
// the chunk attends causally to positions 0 .. P0 + i: the earlier paged context
// (which may be a shared prefix, section "Prefix caching") and its own chunk, whose
// K/V the caller has already appended to the pool.
//
// Here Q.K^T is a real dense contraction (C * G query rows against thousands of keys),
// so both products run on the tensor cores.  This is the warp-level form: each warp
// owns 16 query rows (row = position * G + head of one KV group), a CTA of 4 warps
// shares K/V tiles of 64 keys (4 paged blocks, TMA-loaded with the 128-byte swizzle,
// double-buffered), S = Q.K^T and O += P.V use mma.sync m16n8k16 with fp32
// accumulation, and the online softmax keeps per-row running max / sum.  It serves the
// shapes the tcgen05 form (prefill_tc.cu) does not: head dim 64, group sizes that do not
// divide 128, and sliding-window chunks (a row at position p sees p - window + 1 .. p;
// key tiles and blocks before every window of the CTA are not read).
#include <climits>

#include "common.cuh"
#include "internal.h"

namespace pkv {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kKeys = 64;        // keys per tile (4 blocks)
constexpr int kWarps = 4;
constexpr int kRows = 16 * kWarps;

template <int D>
struct PrefillCfg {
    static constexpr int TILE = 16 * 2 * D;            // one block-head tile (bytes)
    static constexpr int NBOX = D / 64;
    static constexpr int KBYTES = 4 * TILE;            // K of 64 keys
    static constexpr int STAGE = 2 * KBYTES;           // K and V
    static constexpr int STAGES = 2;
    static constexpr int SMEM = STAGES * STAGE + 1024;
};

struct PrefillParams {
    const void* q;
    const int32_t* table;
    float* out;
    int32_t* status;
    int W, P0, C, H_q, H_kv, G, N;
    int window;             // sliding window (keys a row sees, itself included); 0 = all earlier
    float scale_log2;
    int hold_tile;          // test hook: this CTA-local tile's copy is never issued (-1: none)
    long long wait_cycles;  // bound of every wait on a copy (SM cycles)
};

__device__ __forceinline__ uint32_t swz(uint32_t tile, int t, int c)
{
    return tile + (uint32_t)((c >> 3) * (16 * 128) + t * 128 + (((c & 7) ^ (t & 7)) << 4));
}

template <int D, bool BF16>
__global__ void __launch_bounds__(128)
prefill_mma_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV)
{
    using Cfg = PrefillCfg<D>;
    extern __shared__ uint8_t smem_dyn[];
    __shared__ __align__(8) uint64_t bars[Cfg::STAGES];
    __shared__ int s_fail_t;   // the first key tile whose copy a thread gave up on (INT_MAX: none)

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = blockIdx.y;
    const int rg = lane >> 2, qd = lane & 3;
    const int row_cta = blockIdx.x * kRows;
    const int rows_total = p.C * p.G;

    // key bound of the CTA: the last position it holds attends P0 + i_last + 1 keys
    const int i_last = min(p.C - 1, (row_cta + kRows - 1) / p.G);
    const int kend_cta = p.P0 + i_last + 1;
    const int ntiles = (kend_cta + kKeys - 1) / kKeys;
    // with a sliding window, tiles wholly before the first row's window are skipped
    const int lo_cta = p.window > 0 ? max(0, p.P0 + min(p.C - 1, row_cta / p.G) + 1 - p.window) : 0;
    const int t_begin = lo_cta / kKeys;
    const int seq_len = p.P0 + p.C;
    const int nblk_seq = (seq_len + kBlock - 1) / kBlock;

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    if (tid == 0) {
        s_fail_t = INT_MAX;
        for (int s = 0; s < Cfg::STAGES; ++s) mbar_init(smem_u32(&bars[s]), 1);
        mbar_fence_init();
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    __syncthreads();

    auto issue = [&](int t) {   // t: key tile; its ring stage counts from t_begin
        const int s = (t - t_begin) % Cfg::STAGES;
        const uint32_t bar = smem_u32(&bars[s]);
        const uint32_t kdst = smem_u32(smem + s * Cfg::STAGE);
        mbar_arrive_expect_tx(bar, Cfg::STAGE);
        if (t - t_begin == p.hold_tile) return;   // test hook: the stage's bytes never arrive
        // all four table entries first, so their loads overlap
        int rows[4];
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
            const int lb = t * 4 + kb;        // logical block of the sequence
            // past the sequence's last block, or wholly before every row's window (an engine
            // may have released it): load block 0 (in bounds); those keys are masked and
            // their V zeroed below
            int blk = (lb < nblk_seq && (lb + 1) * kBlock > lo_cta) ? p.table[lb] : 0;
            if ((unsigned)blk >= (unsigned)p.N) {
                flag_status(p.status, PKV_DEV_BAD_BLOCK);
                blk = 0;
            }
            rows[kb] = (blk * p.H_kv + g) * kBlock;
        }
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
#pragma unroll
            for (int x = 0; x < Cfg::NBOX; ++x) {
                tma_load_2d(kdst + kb * Cfg::TILE + x * 2048, &tmK, x * 64, rows[kb], bar);
                tma_load_2d(kdst + Cfg::KBYTES + kb * Cfg::TILE + x * 2048, &tmV, x * 64, rows[kb], bar);
            }
        }
    };
    if (tid == 0) {
        for (int t = t_begin; t < min(t_begin + Cfg::STAGES, ntiles); ++t) issue(t);
    }

    // this warp's rows: r0 = row of lane group rg, r1 = r0 + 8
    const int r0 = row_cta + warp * 16 + rg, r1 = r0 + 8;
    const bool v0 = r0 < rows_total, v1 = r1 < rows_total;
    const int i0 = v0 ? r0 / p.G : 0, i1 = v1 ? r1 / p.G : 0;
    const int kmax0 = p.P0 + i0 + 1, kmax1 = p.P0 + i1 + 1;   // exclusive key bounds
    const int klo0 = p.window > 0 ? max(0, kmax0 - p.window) : 0;   // first visible keys
    const int klo1 = p.window > 0 ? max(0, kmax1 - p.window) : 0;
    uint32_t qa[D / 16][4];
    {
        const uint16_t* qb = static_cast<const uint16_t*>(p.q);
        const uint16_t* q0 = qb + ((size_t)i0 * p.H_q + g * p.G + (v0 ? r0 % p.G : 0)) * D;
        const uint16_t* q1 = qb + ((size_t)i1 * p.H_q + g * p.G + (v1 ? r1 % p.G : 0)) * D;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            qa[ks][0] = v0 ? *reinterpret_cast<const uint32_t*>(q0 + 16 * ks + 2 * qd) : 0u;
            qa[ks][2] = v0 ? *reinterpret_cast<const uint32_t*>(q0 + 16 * ks + 8 + 2 * qd) : 0u;
            qa[ks][1] = v1 ? *reinterpret_cast<const uint32_t*>(q1 + 16 * ks + 2 * qd) : 0u;
            qa[ks][3] = v1 ? *reinterpret_cast<const uint32_t*>(q1 + 16 * ks + 8 + 2 * qd) : 0u;
        }
    }

    float o[D / 8][4];
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
#pragma unroll
        for (int c = 0; c < 4; ++c) o[n][c] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    const float sl = p.scale_log2;
    // the warp's smallest key bound: tiles entirely below it need no causal mask
    const int kmin_warp = p.P0 + min(p.C - 1, (row_cta + warp * 16) / p.G) + 1;
    // the warp's window starts: tiles wholly at or above the largest need no window mask,
    // tiles wholly below the smallest are skipped
    const int kwin_lo = p.window > 0 ? max(0, kmin_warp - p.window) : 0;
    const int kwin_hi = p.window > 0 ? max(0, p.P0 + min(p.C - 1, (row_cta + warp * 16 + 15) / p.G) + 1 - p.window) : 0;

    int t_stop = ntiles;   // the tile the CTA stopped at (ntiles: it did not)
    for (int t = t_begin; t < ntiles; ++t) {
        const int s = (t - t_begin) % Cfg::STAGES;
        if (!mbar_wait_bounded(smem_u32(&bars[s]), ((t - t_begin) / Cfg::STAGES) & 1, p.wait_cycles))
            atomicMin(&s_fail_t, t);   // this tile's data is not there: computed on, but never written out
        const uint32_t kb = smem_u32(smem + s * Cfg::STAGE);
        const uint32_t vb = kb + Cfg::KBYTES;
        const int key0 = t * kKeys;

        if (key0 < p.P0 + min(p.C - 1, (row_cta + warp * 16 + 15) / p.G) + 1 &&
            key0 + kKeys > kwin_lo) {   // warp has work here
            float sc[8][4];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int c = 0; c < 4; ++c) sc[nt][c] = 0.f;
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk) {
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
                    const int key = nt * 8 + (lane & 7);
                    uint32_t bk[4];
                    ldsm_x4(bk, swz(kb + (key >> 4) * Cfg::TILE, key & 15, 4 * kk + (lane >> 3)));
                    mma16816<BF16>(sc[nt], qa[2 * kk], bk[0], bk[1]);
                    mma16816<BF16>(sc[nt], qa[2 * kk + 1], bk[2], bk[3]);
                }
            }
            const bool need_mask = key0 + kKeys > kmin_warp || key0 < kwin_hi;
            float alpha[2];
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int kmax = hr ? kmax1 : kmax0;
                const int klo = hr ? klo1 : klo0;
                float mx = -INFINITY;
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int key = key0 + nt * 8 + 2 * qd + e;
                        float x = sc[nt][2 * hr + e] * sl;
                        if (need_mask && (key >= kmax || key < klo)) x = -INFINITY;
                        sc[nt][2 * hr + e] = x;
                        mx = fmaxf(mx, x);
                    }
                mx = warp_max_quad(mx);
                const float mn = fmaxf(m_run[hr], mx);
                const float mref = mn == -INFINITY ? 0.f : mn;
                alpha[hr] = ex2(m_run[hr] - mref);
                float sum = 0.f;
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const float pv = ex2(sc[nt][2 * hr + e] - mref);
                        sc[nt][2 * hr + e] = pv;
                        sum += pv;
                    }
                l_run[hr] = l_run[hr] * alpha[hr] + sum;
                m_run[hr] = mn;
            }
#pragma unroll
            for (int n = 0; n < D / 8; ++n) {
                o[n][0] *= alpha[0];
                o[n][1] *= alpha[0];
                o[n][2] *= alpha[1];
                o[n][3] *= alpha[1];
            }
            // O += P . V, P split into high and low 16-bit parts
#pragma unroll
            for (int kk = 0; kk < kKeys / 16; ++kk) {
                uint32_t ah[4], al[4];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {       // n-tiles 2kk (keys +0..7), 2kk+1 (keys +8..15)
#pragma unroll
                    for (int hr = 0; hr < 2; ++hr) {   // rows r0, r1
                        const float x0 = sc[2 * kk + hh][2 * hr], x1 = sc[2 * kk + hh][2 * hr + 1];
                        const uint32_t hi = pack2<BF16>(x0, x1);
                        const float2 back = unpack2<BF16>(hi);
                        ah[2 * hh + hr] = hi;
                        al[2 * hh + hr] = pack2<BF16>(x0 - back.x, x1 - back.y);
                    }
                }
                // V rows past the end of the sequence (or before every window) may hold anything: zero them
                uint32_t keep_lo = 0xffffffffu, keep_hi = 0xffffffffu;
                const int kb0 = key0 + 16 * kk + 2 * qd;
                if (key0 + kKeys > seq_len || key0 < lo_cta) {   // and keys no row of the CTA sees
                    auto in = [&](int key) { return key < seq_len && key >= lo_cta; };
                    keep_lo = (in(kb0) ? 0x0000ffffu : 0u) | (in(kb0 + 1) ? 0xffff0000u : 0u);
                    keep_hi = (in(kb0 + 8) ? 0x0000ffffu : 0u) | (in(kb0 + 9) ? 0xffff0000u : 0u);
                }
#pragma unroll
                for (int np = 0; np < D / 16; ++np) {
                    const int key = 16 * kk + (((lane >> 3) & 1) << 3) + (lane & 7);
                    const int chunk = 2 * np + (lane >> 4);
                    uint32_t bv[4];
                    ldsm_x4_trans(bv, swz(vb + (key >> 4) * Cfg::TILE, key & 15, chunk));
                    bv[0] &= keep_lo;
                    bv[1] &= keep_hi;
                    bv[2] &= keep_lo;
                    bv[3] &= keep_hi;
                    mma16816<BF16>(o[2 * np], ah, bv[0], bv[1]);
                    mma16816<BF16>(o[2 * np], al, bv[0], bv[1]);
                    mma16816<BF16>(o[2 * np + 1], ah, bv[2], bv[3]);
                    mma16816<BF16>(o[2 * np + 1], al, bv[2], bv[3]);
                }
            }
        }
        __syncthreads();
        // A give-up in this tile was recorded before the barrier; one in a later tile records a
        // larger index, so every thread takes the same decision here.
        if (s_fail_t <= t) {
            t_stop = t;
            break;
        }
        if (tid == 0 && t + Cfg::STAGES < ntiles) {
            fence_proxy_async_smem();
            issue(t + Cfg::STAGES);
        }
    }
    if (t_stop < ntiles) {   // no copy may still be landing in this CTA's shared memory when it exits
        if (tid == 0) {
            flag_status(p.status, PKV_DEV_TIMEOUT);
            for (int t = t_stop; t < min(ntiles, t_stop + Cfg::STAGES); ++t)
                mbar_wait_bounded(smem_u32(&bars[(t - t_begin) % Cfg::STAGES]), ((t - t_begin) / Cfg::STAGES) & 1,
                                  p.wait_cycles);
        }
        return;
    }
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) l_run[hr] = warp_sum_quad(l_run[hr]);
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
        const int rr = hr ? r1 : r0;
        if (rr >= rows_total) continue;
        const int i = rr / p.G, e = rr % p.G;
        const float inv = 1.f / l_run[hr];
        float* orow = p.out + ((size_t)i * p.H_q + g * p.G + e) * D;
#pragma unroll
        for (int n = 0; n < D / 8; ++n)
            *reinterpret_cast<float2*>(orow + 8 * n + 2 * qd) = make_float2(o[n][2 * hr] * inv, o[n][2 * hr + 1] * inv);
    }
}

template <int D, bool BF16>
int launch_prefill_mma(const PrefillParams& p, cudaStream_t s, const CUtensorMap* tmk, const CUtensorMap* tmv)
{
    constexpr int smem = PrefillCfg<D>::SMEM;
    auto kern = prefill_mma_kernel<D, BF16>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return PKV_ERR_CUDA;
    const dim3 grid((p.C * p.G + kRows - 1) / kRows, p.H_kv);
    kern<<<grid, 128, smem, s>>>(p, *tmk, *tmv);
    return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

}  // namespace

int launch_prefill(const PrefillArgs& a, const CUtensorMap* tmk, const CUtensorMap* tmv, cudaStream_t s)
{
    PrefillParams p;
    p.q = a.q;
    p.table = a.table;
    p.out = a.out;
    p.status = a.status;
    p.W = a.W;
    p.P0 = a.P0;
    p.C = a.C;
    p.H_q = a.H_q;
    p.H_kv = a.H_kv;
    p.G = a.G;
    p.N = a.N;
    p.scale_log2 = a.scale * kLog2e;
    p.window = a.window;
    const WaitHook hook = wait_hook();
    p.hold_tile = hook.hold_tile;
    p.wait_cycles = hook.wait_cycles;
    const bool bf = a.kv_dtype == PKV_BF16;
    if (a.d == 128) return bf ? launch_prefill_mma<128, true>(p, s, tmk, tmv) : launch_prefill_mma<128, false>(p, s, tmk, tmv);
    if (a.d == 64) return bf ? launch_prefill_mma<64, true>(p, s, tmk, tmv) : launch_prefill_mma<64, false>(p, s, tmk, tmv);
    return PKV_ERR_UNSUPPORTED;
}

}  // namespace pkv
