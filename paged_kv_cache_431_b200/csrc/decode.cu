// decode.cu -- paged_decode_attn: one query token per sequence against its paged cache.
//
// What is computed ("KV cache, continuous batching and paged attention", section "Paged
// attention": the attention kernel follows the block table; "KV cache, GQA, paging and
// continuous batching", section "Mechanics": G query heads share one KV head):
//   out[b][h] = softmax_t(scale * q[b][h] . K_b[t]) V_b[t],  lo_b <= t < context_lens[b],
// K_b[t] = tile (block_tables[b][t / 16], h / G), row t % 16; lo_b = 0, or ctx - window with a
// sliding window ("KV cache, continuous batching and paged attention", section "The KV
// cache": sliding-window attention layers).
//
// Design (B200):
//   * One warp per (partition of <= part_tokens tokens, KV head, sequence) and group of up
//     to 16 query heads (wider groups: one CTA of ceil(G/16) warps sharing the K/V ring up
//     to G = 64).  The CTA streams its partition's (block, KV head) tiles -- 16 rows of K
//     and of V, each tile contiguous in HBM -- into a ring of shared-memory stages with
//     tiled TMA loads (128-byte swizzle, completion on an mbarrier; no multicast).  One
//     thread keeps STAGES tiles in flight; the block-table slice is read once into shared
//     memory.
//   * All G query heads of the KV group are processed together, so each K/V byte is
//     read from HBM exactly once.  Q.K^T and P.V are small dense contractions
//     (G x d times d x 16 tokens); they run on the tensor cores with warp-level
//     mma.sync m16n8k16 (fp32 accumulate), which keeps the FP32 pipe free: at G = 8 the
//     CUDA-core form needs 8 flop per K/V byte, as much as the FP32 pipe can issue at
//     HBM speed.  Scores: S[16 heads][16 tokens] = Q . K^T with K from ldmatrix;
//     output: O^T[d][heads] += V^T . P^T with V from ldmatrix.trans.  P is split into a
//     high and a low 16-bit part (two MMAs) so the P.V product keeps ~16 mantissa bits.
//   * Online softmax in fp32 in the log2 domain (ex2 on the SFU), row maxima by quad
//     shuffles.  Masked (past-the-end) tokens get -inf scores and zeroed V, so stale or
//     poisoned slots never reach the result.
//   * Split-K: a sequence longer than one partition writes per-partition (o, m, l)
//     partials; decode_reduce merges them with the log-sum-exp rule.  The shared-prefix
//     (cascade) form starts the partitions after the prefix and merges them with the
//     prefix's partials written by the tensor-core prefill kernel.
#include "decode_common.cuh"

namespace pkv {

// ---------------------------------------------------------------------------
// Tensor-core engine, 16-bit pools.
// ---------------------------------------------------------------------------
template <int D, int STAGES, int NW>
struct Mma16Cfg {
    static constexpr int TILE = 16 * 2 * D;        // bytes of one K (or V) tile
    static constexpr int NBOX = D / 64;            // 128-byte boxes per row
    static constexpr int STAGE = 2 * TILE;
    static constexpr int RING = STAGES * STAGE;
    static constexpr int STAGING = NW * 16 * (D + 4) * 4;   // the epilogue's 16 O rows per warp
    static constexpr int BODY = RING > STAGING ? RING : STAGING;
    static constexpr int SMEM = BODY + 1024;
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
};

// NW = 1: one warp per (partition, KV head or group of 16 of its query heads, sequence).
// NW > 1 (groups of 17..64 query heads): NW warps share one K/V ring, warp w taking query
// heads 16w .. 16w+15 of the group, so every K/V tile crosses into the SM once; a stage is
// refilled once all warps have released it.
template <int D, bool BF16, int NHT, int STAGES, int NW>
__global__ void __launch_bounds__(32 * NW)
decode_mma16_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV)
{
    using Cfg = Mma16Cfg<D, STAGES, NW>;
    extern __shared__ uint8_t smem_dyn[];
    __shared__ __align__(8) uint64_t bars[STAGES];
    __shared__ __align__(8) uint64_t empty[STAGES];
    __shared__ int tbl[kMaxPartTiles];

    pdl_launch_dependents();   // the split-K merge may be scheduled behind the last wave
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int part = blockIdx.x, b = blockIdx.z;
    const int g = NW > 1 ? blockIdx.y : blockIdx.y / p.hgroups;               // KV head
    const int hg = NW > 1 ? warp : blockIdx.y - g * p.hgroups;                // group of 16 query heads
    const int GC = min(16, p.G - 16 * hg);                                   // query heads of this warp
    const int r = lane >> 2, qd = lane & 3;
    const int hbase = g * p.G + 16 * hg;

    const int ctx = checked_ctx(p, b, threadIdx.x == 0 && part == 0 && g == 0);
    const int nparts = part_count(p, ctx);
    const int tok0 = seq_base(p, ctx) + part * p.part_tokens;
    const int lo = visible_lo(p, ctx);   // tokens before lo are outside the window
    if (tok0 >= ctx) {
        if (part == 0 && p.part_base == 0) {   // empty context: a zero row
            float* o = p.out + ((size_t)b * p.H_q + hbase) * D;
            for (int i = lane; i < GC * D; i += 32) o[i] = 0.f;
        }
        return;
    }
    const int ntok = min(p.part_tokens, ctx - tok0);
    const int ntiles = (ntok + kBlock - 1) / kBlock;

    const int32_t* trow = p.tables + (size_t)b * p.W + tok0 / kBlock;
    for (int j = threadIdx.x; j < ntiles; j += 32 * NW) {
        int blk = trow[j];
        if ((unsigned)blk >= (unsigned)p.N) {
            flag_status(p.status, PKV_DEV_BAD_BLOCK);
            blk = 0;
        }
        tbl[j] = blk;
    }
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&bars[s]), 1);
            mbar_init(smem_u32(&empty[s]), NW);
        }
        mbar_fence_init();
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    __syncthreads();

    auto issue = [&](int j) {
        const int s = j % STAGES;
        const uint32_t bar = smem_u32(&bars[s]);
        const uint32_t kdst = smem_u32(smem + s * Cfg::STAGE);
        const int row = (tbl[j] * p.H_kv + g) * kBlock;
        mbar_arrive_expect_tx(bar, Cfg::STAGE);
        if (j == p.hold_tile) return;   // test hook: the stage's bytes never arrive
        if constexpr (kHintKV) {   // the K/V stream is read once: first out of L2
            const uint64_t pol = l2_evict_first();
#pragma unroll
            for (int x = 0; x < Cfg::NBOX; ++x) tma_load_2d_hint(kdst + x * 2048, &tmK, x * 64, row, bar, pol);
#pragma unroll
            for (int x = 0; x < Cfg::NBOX; ++x) tma_load_2d_hint(kdst + Cfg::TILE + x * 2048, &tmV, x * 64, row, bar, pol);
        } else {
#pragma unroll
            for (int x = 0; x < Cfg::NBOX; ++x) tma_load_2d(kdst + x * 2048, &tmK, x * 64, row, bar);
#pragma unroll
            for (int x = 0; x < Cfg::NBOX; ++x) tma_load_2d(kdst + Cfg::TILE + x * 2048, &tmV, x * 64, row, bar);
        }
    };
    if (threadIdx.x == 0) {
        for (int j = 0; j < min(STAGES, ntiles); ++j) issue(j);
    }

    // Q as the A operand of S = Q.K^T: rows = heads (r and r + 8), 16 dims per k-step.
    uint32_t qa[D / 16][4];
    {
        const uint32_t* q32 = reinterpret_cast<const uint32_t*>(
            static_cast<const uint16_t*>(p.q) + ((size_t)b * p.H_q + hbase) * D);
        const bool r0 = r < GC, r1 = (NHT == 2) && (r + 8 < GC);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            qa[ks][0] = r0 ? __ldg(q32 + (r * D + 16 * ks + 2 * qd) / 2) : 0u;
            qa[ks][2] = r0 ? __ldg(q32 + (r * D + 16 * ks + 8 + 2 * qd) / 2) : 0u;
            qa[ks][1] = r1 ? __ldg(q32 + ((r + 8) * D + 16 * ks + 2 * qd) / 2) : 0u;
            qa[ks][3] = r1 ? __ldg(q32 + ((r + 8) * D + 16 * ks + 8 + 2 * qd) / 2) : 0u;
        }
    }

    float o[D / 16][NHT][4];
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
        for (int hn = 0; hn < NHT; ++hn)
#pragma unroll
            for (int c = 0; c < 4; ++c) o[mt][hn][c] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    const float sl = p.scale_log2;

    int j = 0;
    bool ok = true;
    for (; j < ntiles; ++j) {
        const int s = j % STAGES;
        // the whole warp gives up together (its mma.sync needs every lane)
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&bars[s]), (j / STAGES) & 1, p.wait_cycles))) {
            ok = false;
            break;
        }
        const uint32_t kb = smem_u32(smem + s * Cfg::STAGE);
        const uint32_t vb = kb + Cfg::TILE;
        const int nv = min(kBlock, ntok - j * kBlock);
        const int nlo = lo - (tok0 + j * kBlock);   // tokens of this tile before the window: < nlo

        // S = Q . K^T  (two n-tiles of 8 tokens)
        float sc[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int c = 0; c < 4; ++c) sc[nt][c] = 0.f;
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk) {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                uint32_t bk[4];
                ldsm_x4(bk, swz128(kb, nt * 8 + (lane & 7), 4 * kk + (lane >> 3)));
                mma16816<BF16>(sc[nt], qa[2 * kk], bk[0], bk[1]);
                mma16816<BF16>(sc[nt], qa[2 * kk + 1], bk[2], bk[3]);
            }
        }

        // online softmax, rows r (c = 0, 1) and r + 8 (c = 2, 3)
        float pr[2][4];
        float alpha[2];
#pragma unroll
        for (int hr = 0; hr < NHT; ++hr) {
            float x[2][2];
            float mx = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int tok = nt * 8 + 2 * qd + e;
                    x[nt][e] = (tok < nv && tok >= nlo) ? sc[nt][2 * hr + e] * sl : -INFINITY;
                    mx = fmaxf(mx, x[nt][e]);
                }
            mx = warp_max_quad(mx);
            const float mn = fmaxf(m_run[hr], mx);   // finite: every tile has a valid token
            alpha[hr] = ex2(m_run[hr] - mn);
            float sum = 0.f;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    pr[nt][2 * hr + e] = ex2(x[nt][e] - mn);
                    sum += pr[nt][2 * hr + e];
                }
            l_run[hr] = l_run[hr] * alpha[hr] + sum;
            m_run[hr] = mn;
        }

        // rescale O^T columns (heads 2qd, 2qd + 1 of each head n-tile) when a max moved
        const bool moved = (alpha[0] != 1.f) || (NHT == 2 && alpha[1] != 1.f);
        if (__any_sync(0xffffffffu, moved)) {
#pragma unroll
            for (int hn = 0; hn < NHT; ++hn) {
                const float a_lo = __shfl_sync(0xffffffffu, alpha[hn], 8 * qd);
                const float a_hi = __shfl_sync(0xffffffffu, alpha[hn], 8 * qd + 4);
#pragma unroll
                for (int mt = 0; mt < D / 16; ++mt) {
                    o[mt][hn][0] *= a_lo;
                    o[mt][hn][1] *= a_hi;
                    o[mt][hn][2] *= a_lo;
                    o[mt][hn][3] *= a_hi;
                }
            }
        }

        // P^T as the B operand of O^T += V^T . P^T (k = tokens, n = heads), hi + lo parts
        uint32_t bh[NHT][2], bl[NHT][2];
#pragma unroll
        for (int hn = 0; hn < NHT; ++hn)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const float p0 = pr[nt][2 * hn], p1 = pr[nt][2 * hn + 1];
                bh[hn][nt] = pack2<BF16>(p0, p1);
                const float2 back = unpack2<BF16>(bh[hn][nt]);
                bl[hn][nt] = pack2<BF16>(p0 - back.x, p1 - back.y);
            }

        uint32_t keep01 = 0xffffffffu, keep23 = 0xffffffffu;
        if (nv < kBlock || nlo > 0) {   // zero V outside [nlo, nv): P is 0 there, V may be stale
            auto in = [&](int t) { return t >= nlo && t < nv; };
            keep01 = (in(2 * qd) ? 0x0000ffffu : 0u) | (in(2 * qd + 1) ? 0xffff0000u : 0u);
            keep23 = (in(8 + 2 * qd) ? 0x0000ffffu : 0u) | (in(9 + 2 * qd) ? 0xffff0000u : 0u);
        }
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
            uint32_t va[4];
            ldsm_x4_trans(va, swz128(vb, ((lane >> 4) << 3) + (lane & 7), 2 * mt + ((lane >> 3) & 1)));
            va[0] &= keep01;
            va[1] &= keep01;
            va[2] &= keep23;
            va[3] &= keep23;
#pragma unroll
            for (int hn = 0; hn < NHT; ++hn) {
                mma16816<BF16>(o[mt][hn], va, bh[hn][0], bh[hn][1]);
                mma16816<BF16>(o[mt][hn], va, bl[hn][0], bl[hn][1]);
            }
        }

        __syncwarp();
        if constexpr (NW == 1) {
            if (lane == 0 && j + STAGES < ntiles) {
                fence_proxy_async_smem();
                issue(j + STAGES);
            }
        } else {   // release the stage; thread 0 refills it once every warp has
            if (lane == 0) {
                fence_proxy_async_smem();
                mbar_arrive(smem_u32(&empty[s]));
            }
            bool refilled = true;
            if (threadIdx.x == 0 && j + STAGES < ntiles) {
                refilled = mbar_wait_bounded(smem_u32(&empty[s]), (j / STAGES) & 1, p.wait_cycles);
                if (refilled) issue(j + STAGES);
            }
            if (!__shfl_sync(0xffffffffu, refilled ? 1 : 0, 0)) {   // warp 0 stops; the others time out
                ok = false;
                ++j;
                break;
            }
        }
    }

    if (!ok) {   // no copy may still be landing in this CTA's shared memory when it exits
        if (lane == 0) flag_status(p.status, PKV_DEV_TIMEOUT);
        for (int jj = j; jj < min(ntiles, j + STAGES); ++jj)
            mbar_wait_bounded(smem_u32(&bars[jj % STAGES]), (jj / STAGES) & 1, p.wait_cycles);
    }
    if constexpr (NW > 1) {
        // every warp is done with the ring before the staging reuses it; a warp that gave up
        // stops the whole CTA (the epilogue's barriers need every warp)
        if (__syncthreads_or(!ok)) return;
    } else {
        if (!ok) return;
    }

    // ---- epilogue: O rows [head][dim] through shared memory, then coalesced stores
#pragma unroll
    for (int hr = 0; hr < NHT; ++hr) l_run[hr] = warp_sum_quad(l_run[hr]);
    const bool final_out = (p.part_base == 0 && nparts == 1);
    float* so = reinterpret_cast<float*>(smem) + warp * 16 * (D + 4);
    constexpr int SR = D + 4;   // padded row stride (floats)
    __syncwarp();
#pragma unroll
    for (int hn = 0; hn < NHT; ++hn) {
        float inv_lo = 1.f, inv_hi = 1.f;
        const float la = __shfl_sync(0xffffffffu, l_run[hn], 8 * qd);
        const float lb = __shfl_sync(0xffffffffu, l_run[hn], 8 * qd + 4);
        if (final_out) {
            inv_lo = 1.f / la;
            inv_hi = 1.f / lb;
        }
        const int h0 = 8 * hn + 2 * qd;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
            so[h0 * SR + 16 * mt + r] = o[mt][hn][0] * inv_lo;
            so[(h0 + 1) * SR + 16 * mt + r] = o[mt][hn][1] * inv_hi;
            so[h0 * SR + 16 * mt + 8 + r] = o[mt][hn][2] * inv_lo;
            so[(h0 + 1) * SR + 16 * mt + 8 + r] = o[mt][hn][3] * inv_hi;
        }
    }
    __syncwarp();
    const size_t row0 = (size_t)b * p.H_q + hbase;
    if (final_out) {
        for (int i = lane; i < GC * (D / 4); i += 32) {
            const int h = i / (D / 4), c4 = i % (D / 4);
            const float4 v = *reinterpret_cast<const float4*>(&so[h * SR + 4 * c4]);
            *reinterpret_cast<float4*>(p.out + (row0 + h) * D + 4 * c4) = v;
        }
    } else {
        for (int i = lane; i < GC * (D / 4); i += 32) {
            const int h = i / (D / 4), c4 = i % (D / 4);
            const float4 v = *reinterpret_cast<const float4*>(&so[h * SR + 4 * c4]);
            float4* dst = reinterpret_cast<float4*>(p.ws_o + ws_slot(p, row0 + h, part) * D + 4 * c4);
            if constexpr (kHintPartials) st_hint(dst, v, l2_evict_last());   // the merge reads it back soon
            else *dst = v;
        }
        if (qd == 0) {
#pragma unroll
            for (int hr = 0; hr < NHT; ++hr) {
                const int h = r + 8 * hr;
                if (h < GC) {
                    float2 ml = make_float2(m_run[hr], l_run[hr]);
                    float2* dst = reinterpret_cast<float2*>(p.ws_ml + ws_slot(p, row0 + h, part) * 2);
                    if constexpr (kHintPartials) st_hint(dst, ml, l2_evict_last());
                    else *dst = ml;
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Split-K merge: out = sum_i 2^(m_i - M) o_i / sum_i 2^(m_i - M) l_i, M = max_i m_i.
// One warp per (query head, sequence), four heads per CTA; sequences that fit one partition
// were written directly by the main kernel and are skipped.  In the shared-prefix (cascade)
// form slots 0 .. part_base-1 hold the prefix's partials (one per key split) and the suffix
// follows.  The context length (not written by the decode kernel) is read before the wait
// for the decode grid; after it, the (m, l) pairs and up to 8 partial rows per lane go out
// as one batch of independent loads.
// ---------------------------------------------------------------------------
constexpr int kMergeHeads = 4;   // warps (query heads) per merge CTA

template <int D>
__global__ void __launch_bounds__(32 * kMergeHeads) decode_reduce_kernel(const DecodeParams p)
{
    const int lane = threadIdx.x & 31;
    const int h = blockIdx.x * kMergeHeads + (threadIdx.x >> 5), b = blockIdx.y;
    const int ctx = checked_ctx(p, b, false);
    pdl_wait_primary();   // the partials of the decode kernel before this one
    if (h >= p.H_q) return;
    if (p.prefix_blocks > 0 && h == 0) {   // cascade: every table must start with row 0's prefix
        bool same = true;
        for (int j = lane; j < p.prefix_blocks; j += 32) same &= p.tables[(size_t)b * p.W + j] == p.tables[j];
        if (!__all_sync(0xffffffffu, same) && lane == 0) flag_status(p.status, PKV_DEV_BAD_PREFIX);
    }
    const int nparts = p.part_base + part_count(p, ctx);
    if (p.part_base == 0 && nparts <= 1) return;
    const size_t base = ((size_t)b * p.H_q + h) * p.slots;
    const float2* ml = reinterpret_cast<const float2*>(p.ws_ml) + base;
    constexpr int V = D / 32;   // floats per lane
    constexpr int kBatch = 8;   // partial rows loaded together
    const float* po = p.ws_o + base * D + lane * V;

    float M = -INFINITY, L = 0.f;
    float acc[V];
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = 0.f;
    for (int i0 = 0; i0 < nparts; i0 += kBatch) {
        // this batch's (m, l) (lane k < kBatch holds partial i0 + k) and o rows, all in flight at once
        const int nb = min(kBatch, nparts - i0);
        const float2 mlk = lane < nb ? ml[i0 + lane] : make_float2(-INFINITY, 0.f);
        float v[kBatch][V];
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
            if (k < nb) {
                if constexpr (V == 4) {
                    const float4 t = *reinterpret_cast<const float4*>(po + (size_t)(i0 + k) * D);
                    v[k][0] = t.x; v[k][1] = t.y; v[k][2] = t.z; v[k][3] = t.w;
                } else {
                    const float2 t = *reinterpret_cast<const float2*>(po + (size_t)(i0 + k) * D);
                    v[k][0] = t.x; v[k][1] = t.y;
                }
            } else {
#pragma unroll
                for (int e = 0; e < V; ++e) v[k][e] = 0.f;
            }
        }
        float mb = mlk.x;
#pragma unroll
        for (int off = 4; off; off >>= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, off));
        mb = __shfl_sync(0xffffffffu, mb, 0);             // the batch's max (lanes 0..7 hold it)
        const float Mn = fmaxf(M, mb);                     // finite: every partial has a visible key
        const float a = ex2(M - Mn);                       // rescale what the earlier batches summed
        float lb = lane < nb ? ex2(mlk.x - Mn) * mlk.y : 0.f;
#pragma unroll
        for (int off = 4; off; off >>= 1) lb += __shfl_xor_sync(0xffffffffu, lb, off);
        L = L * a + __shfl_sync(0xffffffffu, lb, 0);
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] *= a;
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
            const float w = k < nb ? ex2(__shfl_sync(0xffffffffu, mlk.x, k) - Mn) : 0.f;
#pragma unroll
            for (int e = 0; e < V; ++e) acc[e] += w * v[k][e];
        }
        M = Mn;
    }
    const float inv = 1.f / L;
    float* out = p.out + ((size_t)b * p.H_q + h) * D + lane * V;
    if constexpr (V == 4) {
        *reinterpret_cast<float4*>(out) = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    } else {
        *reinterpret_cast<float2*>(out) = make_float2(acc[0] * inv, acc[1] * inv);
    }
}

// ---------------------------------------------------------------------------
// launcher
// ---------------------------------------------------------------------------
namespace {

constexpr int kStages = 2;

// Groups of 64 query heads go to the keys-on-M tcgen05 kernel (decode_tc_keys.cu); 0 sends
// them to the two-sequences-per-CTA one (decode_tc.cu).
#ifndef PKV_DECODE_KEYS_TC
#define PKV_DECODE_KEYS_TC 1
#endif
constexpr bool kDecodeKeysTc = PKV_DECODE_KEYS_TC != 0;

// fp8 pools with 8 query heads per KV head go to the tcgen05 kernel that multiplies the stored
// codes (decode_tc_fp8.cu); 0 sends them to the warp-level one (decode_quant.cu).
#ifndef PKV_DECODE_TC_FP8
#define PKV_DECODE_TC_FP8 1
#endif
constexpr bool kDecodeTcFp8 = PKV_DECODE_TC_FP8 != 0;

}  // namespace

int decode_keys_tc_available(int d, int G, int kv_dtype)
{
    if (kDecodeKeysTc && decode_tck_supported(d, G, kv_dtype)) return 1;
    if (kDecodeTcFp8 && decode_tc_fp8_supported(d, G, kv_dtype)) return 2;
    return 0;
}

namespace {

template <typename K>
int launch_k(K kernel, int smem, dim3 grid, int threads, cudaStream_t s, const DecodeParams& p,
             const CUtensorMap* tmk, const CUtensorMap* tmv)
{
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return PKV_ERR_CUDA;
    kernel<<<grid, threads, smem, s>>>(p, *tmk, *tmv);
    return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

template <int D, bool BF16, int NW>
int launch_mma16_nw(const DecodeParams& p, int nht, dim3 grid, cudaStream_t s, const CUtensorMap* tmk,
                    const CUtensorMap* tmv)
{
    constexpr int smem = Mma16Cfg<D, kStages, NW>::SMEM;
    if (nht == 1)
        return launch_k(decode_mma16_kernel<D, BF16, 1, kStages, NW>, smem, grid, 32 * NW, s, p, tmk, tmv);
    return launch_k(decode_mma16_kernel<D, BF16, 2, kStages, NW>, smem, grid, 32 * NW, s, p, tmk, tmv);
}

// Groups of 17..64 query heads run as one CTA of ceil(G / 16) warps sharing the K/V ring;
// wider groups as one single-warp CTA per 16 heads.
template <int D, bool BF16>
int launch_mma16(const DecodeParams& p, int nht, dim3 grid, cudaStream_t s, const CUtensorMap* tmk,
                 const CUtensorMap* tmv)
{
    const dim3 g1(grid.x, grid.y / p.hgroups, grid.z);   // one CTA per KV head
    switch (p.hgroups) {
    case 2: return launch_mma16_nw<D, BF16, 2>(p, nht, g1, s, tmk, tmv);
    case 3: return launch_mma16_nw<D, BF16, 3>(p, nht, g1, s, tmk, tmv);
    case 4: return launch_mma16_nw<D, BF16, 4>(p, nht, g1, s, tmk, tmv);
    default: return launch_mma16_nw<D, BF16, 1>(p, nht, grid, s, tmk, tmv);
    }
}

}  // namespace

int launch_decode(const DecodeArgs& a, const CUtensorMap* tmk, const CUtensorMap* tmv, cudaStream_t s)
{
    DecodeParams p;
    p.q = a.q;
    p.tables = a.tables;
    p.ctx_lens = a.ctx_lens;
    p.k_scale = a.k_scale;
    p.v_scale = a.v_scale;
    p.out = a.out;
    p.ws_o = a.ws_o;
    p.ws_ml = a.ws_ml;
    p.status = a.status;
    p.W = a.W;
    p.H_q = a.H_q;
    p.H_kv = a.H_kv;
    p.G = a.G;
    p.N = a.N;
    p.part_tokens = a.part_tokens;
    p.max_parts = a.max_parts;
    p.tok_base = a.tok_base;
    p.part_base = a.part_base;
    p.slots = a.part_base + a.max_parts;
    p.prefix_blocks = a.part_base ? a.tok_base / kBlock : 0;
    p.window = a.window;
    p.hgroups = (a.G + 15) / 16;
    p.num_seqs = a.B;
    p.q_bf16 = a.q_dtype == PKV_BF16;
    p.scale_log2 = a.scale * kLog2e;
    const WaitHook hook = wait_hook();
    p.hold_tile = hook.hold_tile;
    p.wait_cycles = hook.wait_cycles;

    const dim3 grid(a.max_parts, a.H_kv * p.hgroups, a.B);
    const int nht = a.G <= 8 ? 1 : 2;   // 8 or 16 query heads per CTA
    int rc = PKV_ERR_UNSUPPORTED;
    if ((a.kv_dtype == PKV_BF16 || a.kv_dtype == PKV_F16) && (a.engine == 2 || a.engine == 3)) {
        if (!decode_simt_supported(a.d, a.G, a.kv_dtype) || (reinterpret_cast<uintptr_t>(a.q) & 15))
            return PKV_ERR_UNSUPPORTED;
        rc = launch_decode_simt(p, a.kv_dtype, a.G, a.engine == 2, grid, s, tmk, tmv);
    } else if (kDecodeTcFp8 && a.engine == 0 && a.window == 0 && a.part_base == 0 &&
               decode_tc_fp8_supported(a.d, a.G, a.kv_dtype) && (reinterpret_cast<uintptr_t>(a.q) & 15) == 0) {
        // fp8 pools, 8 query heads per KV head: the codes go to tcgen05 kind::f8f6f4 MMAs
        rc = launch_decode_tc_fp8(p, tmk, tmv, s);
    } else if (kDecodeKeysTc && a.engine == 0 && a.window == 0 && a.part_base == 0 &&
               decode_tck_supported(a.d, a.G, a.kv_dtype) && (reinterpret_cast<uintptr_t>(a.q) & 15) == 0) {
        // 64 query heads per KV head: tcgen05 with the keys on the MMA's M side
        CUtensorMap tmq;
        auto enc = tensor_map_encoder();
        if (!enc || !make_q_map_seq(&tmq, a.q, a.B, a.H_q, enc)) return PKV_ERR_CUDA;
        rc = launch_decode_tck(p, a.kv_dtype, &tmq, tmk, tmv, s);
    } else if ((a.kv_dtype == PKV_BF16 || a.kv_dtype == PKV_F16) && a.engine == 0 && a.window == 0 &&
               a.part_base == 0 && decode_tc_supported(a.d, a.G, a.kv_dtype) &&
               (reinterpret_cast<uintptr_t>(a.q) & 15) == 0) {
        // wide groups (MQA-like): Q.K^T and P.V as tcgen05 MMAs
        CUtensorMap tmq;
        auto enc = tensor_map_encoder();
        if (!enc || !make_q_map(&tmq, a.q, a.B, a.H_q, a.G, enc)) return PKV_ERR_CUDA;
        rc = launch_decode_tc(p, a.kv_dtype, &tmq, tmk, tmv, s);
    } else if (a.kv_dtype == PKV_BF16 || a.kv_dtype == PKV_F16) {
        if (a.engine > 1) return PKV_ERR_UNSUPPORTED;
        const bool bf = a.kv_dtype == PKV_BF16;
        if (a.d == 128) rc = bf ? launch_mma16<128, true>(p, nht, grid, s, tmk, tmv)
                                : launch_mma16<128, false>(p, nht, grid, s, tmk, tmv);
        else if (a.d == 64) rc = bf ? launch_mma16<64, true>(p, nht, grid, s, tmk, tmv)
                                    : launch_mma16<64, false>(p, nht, grid, s, tmk, tmv);
    } else if (is_quantized(a.kv_dtype)) {
        if (a.engine > 1) return PKV_ERR_UNSUPPORTED;
        rc = launch_decode_quant(p, a.kv_dtype, a.d, nht, grid, s, tmk, tmv);
    }
    if (rc != PKV_OK) return rc;
    if (a.max_parts > 1 || a.part_base > 0) {
        // programmatic dependent launch: scheduled while the decode grid's last wave runs
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((a.H_q + kMergeHeads - 1) / kMergeHeads, a.B);
        cfg.blockDim = dim3(32 * kMergeHeads);
        cfg.dynamicSmemBytes = 0;
        cfg.stream = s;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr.val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        const cudaError_t e = a.d == 128 ? cudaLaunchKernelEx(&cfg, decode_reduce_kernel<128>, p)
                                         : cudaLaunchKernelEx(&cfg, decode_reduce_kernel<64>, p);
        if (e != cudaSuccess) return PKV_ERR_CUDA;
    }
    return PKV_OK;
}

}  // namespace pkv
