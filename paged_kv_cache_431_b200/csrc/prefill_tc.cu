// prefill_tc.cu -- paged_prefill_chunk_attn on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// Inference guide a2-inf-2, section "Chunked prefill", and "KV cache, continuous
// batching and paged attention", section "Scheduling prefill and decode": a prompt
// chunk of C positions P0 .. P0+C-1 attends causally to the paged context (possibly a
// shared prefix, section "Prefix caching") and to itself.
//
// One CTA owns two query tiles A and B of 128 rows each -- 256/G positions x the G heads of
// one KV group -- and walks the keys in tiles of 128 (8 paged blocks) shared by both:
//   warp 0      TMA producer: Q once (3-D boxes over [position][head][dim]), then K and V
//               tiles block by block through the pool's tensor maps into separate 2-stage
//               rings (128-byte swizzle, no multicast): a K stage is free once its Q.K^T is
//               done, a V stage once its P.V is done;
//   warp 1      allocates all 512 TMEM columns -- per query tile 128 for S (later P) and
//               128 for the O accumulator -- and issues every MMA from one thread;
//   warps 2..5  softmax of tile A, warps 6..9 of tile B, one thread per query row (= TMEM
//               lane): read the row's 128 scores, mask (causal bound, window, end of
//               sequence), keep the running max lazily (it moves only when the new max
//               exceeds the old by 2^8, then O is rescaled in TMEM), and write P back into
//               the score's own TMEM columns, where the P . V MMA reads it as its A operand:
//               for bf16 pools as a high and a low bf16 part (two MMAs keep P . V at ~16
//               mantissa bits), for fp16 pools as one fp16 part (11 bits, one MMA).
// The two tiles ping-pong: while the softmax warps of one tile work, the tensor cores run
// the other tile's P . V and next Q.K^T, so neither unit waits for the other:
//   MMA order per key tile t:  P.V(A, t), Q.K^T(A, t+1), P.V(B, t), Q.K^T(B, t+1).
// Tensor-core instructions issued by one thread execute in order, so Q.K^T(A, t+1) may
// overwrite the columns P.V(A, t) reads.  Every wait is bounded; a timeout sets
// PKV_DEV_TIMEOUT and the CTA winds down.
#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace pkv {

namespace {

constexpr int kD = 128;             // head dim handled here
constexpr int kBM = 128;            // query rows per tile
constexpr int kQT = 2;              // query tiles per CTA
constexpr int kBN = 128;            // keys per tile
constexpr int kNS = 2;              // stages of each of the K and V rings
constexpr int kQBytes = kBM * kD * 2;            // 32 KiB per query tile
constexpr int kKVBytes = kBN * kD * 2;           // 32 KiB per K (or V) stage
constexpr int kSmem = kQT * kQBytes + kNS * 2 * kKVBytes + 1024;
constexpr uint32_t kTmemCols = 512;              // tile x: S/P at 256x, O at 256x + 128
constexpr int kThreads = 320;                    // producer, MMA, 2 x 4 softmax warps
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleSlack = 8.f;             // log2 units

struct TcParams {
    const int32_t* table;
    float* out;
    int32_t* status;
    int P0, C, H_q, H_kv, G, N;
    float scale_log2;
    // Shared-prefix (cascade) form: the C "positions" are C sequences whose query rows all
    // see the same nkeys keys (no causal mask); the unnormalized output and (m, l) go to
    // the decode workspace rows [C][H_q][slots] instead of `out`.
    // The cascade form may split the keys over gridDim.z CTAs per query tile pair, split z
    // writing slot z (a small batch alone would leave most SMs idle).
    int cascade, nkeys, slots;
    float* ws_o;
    float* ws_ml;
    int hold_tile;          // test hook: the K copy of this CTA-local key tile is never issued (-1: none)
    long long wait_cycles;  // bound of every wait (SM cycles)
};

struct Bars {
    uint64_t q_full;
    uint64_t k_full[kNS];
    uint64_t k_empty[kNS];
    uint64_t v_full[kNS];
    uint64_t v_empty[kNS];
    uint64_t s_full[kQT];      // S(x, t) is in TMEM (every earlier MMA of the CTA is done too)
    uint64_t p_full[kQT];      // P(x, t) stored by the four softmax warps of tile x
    uint64_t o_done[kQT];      // the last P . V of tile x is done
    uint64_t mma_drain;        // every MMA the issuer launched is done (before TMEM is freed)
};

template <bool BF16>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const TcParams p, const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV)
{
    extern __shared__ uint8_t smem_dyn[];
    __shared__ Bars bars;
    __shared__ uint32_t s_tmem_base;
    __shared__ volatile int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = blockIdx.y;
    const int pos_per_tile = kBM / p.G;
    const int i0 = blockIdx.x * kQT * pos_per_tile;          // first chunk position of this CTA
    const int i_end = min(p.C, i0 + kQT * pos_per_tile);
    const int seq_len = p.cascade ? p.nkeys : p.P0 + p.C;
    const int kend = p.cascade ? p.nkeys : p.P0 + i_end;     // exclusive key bound of the CTA's last row
    const int ntiles_all = (kend + kBN - 1) / kBN;
    const int t_lo = (int)((long)blockIdx.z * ntiles_all / gridDim.z);        // this CTA's key tiles
    const int t_hi = (int)((long)(blockIdx.z + 1) * ntiles_all / gridDim.z);
    const int ntiles = t_hi - t_lo;                          // tile t_lo + u is the u-th of this CTA
    const int nblk_seq = (seq_len + kBlock - 1) / kBlock;

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    const uint32_t sQ = smem_u32(smem);                      // kQT query tiles
    const uint32_t sK = sQ + kQT * kQBytes;                  // kNS stages of K
    const uint32_t sV = sK + kNS * kKVBytes;                 // kNS stages of V

    if (threadIdx.x == 0) {
        s_abort = 0;
        mbar_init(smem_u32(&bars.q_full), 1);
        for (int s = 0; s < kNS; ++s) {
            mbar_init(smem_u32(&bars.k_full[s]), 1);
            mbar_init(smem_u32(&bars.k_empty[s]), 1);
            mbar_init(smem_u32(&bars.v_full[s]), 1);
            mbar_init(smem_u32(&bars.v_empty[s]), 1);
        }
        for (int x = 0; x < kQT; ++x) {
            mbar_init(smem_u32(&bars.s_full[x]), 1);
            mbar_init(smem_u32(&bars.p_full[x]), 4);
            mbar_init(smem_u32(&bars.o_done[x]), 1);
        }
        mbar_init(smem_u32(&bars.mma_drain), 1);
        mbar_fence_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem_base)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        // The whole warp walks the tiles: its 32 lanes hold the block ids of the next 4
        // tiles (one coalesced load per 4 tiles, fetched a chunk ahead), lane 0 issues the
        // copies.
        constexpr int kBlkPerTile = kBN / kBlock;            // 8
        constexpr int kTilesPerChunk = 32 / kBlkPerTile;     // 4
        auto table_entry = [&](int lb) -> int {             // physical block of logical block lb
            if (lb >= nblk_seq) return -1;                   // past the sequence
            int blk = p.table[lb];
            if ((unsigned)blk >= (unsigned)p.N) {
                flag_status(p.status, PKV_DEV_BAD_BLOCK);
                blk = 0;
            }
            return blk;
        };
        const uint32_t qb = smem_u32(&bars.q_full);
        if (lane == 0) {
            prefetch_tensormap(&tmQ);
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
            mbar_arrive_expect_tx(qb, kQT * kQBytes);
            for (int x = 0; x < kQT; ++x) {
                tma_load_3d(sQ + x * kQBytes, &tmQ, 0, g * p.G, i0 + x * pos_per_tile, qb);
                tma_load_3d(sQ + x * kQBytes + kQBytes / 2, &tmQ, 64, g * p.G, i0 + x * pos_per_tile, qb);
            }
        }
        const int lb0 = t_lo * kBlkPerTile;                  // first logical block of this CTA
        int cur = table_entry(lb0 + lane);                   // chunk 0
        int nxt = table_entry(lb0 + 32 + lane);              // chunk 1
        int issued = 0, issued_k = 0;                        // tiles whose V (K) copies were issued
        for (int t = 0; t < ntiles; ++t) {                   // t counts this CTA's tiles
            const int s = t % kNS;
            if (t > 0 && t % kTilesPerChunk == 0) {
                cur = nxt;
                nxt = table_entry(lb0 + (t / kTilesPerChunk + 1) * 32 + lane);
            }
            int row_of[kBlkPerTile];
#pragma unroll
            for (int kb = 0; kb < kBlkPerTile; ++kb) {
                const int blk = __shfl_sync(0xffffffffu, cur, (t % kTilesPerChunk) * kBlkPerTile + kb);
                // past the sequence: block 0 (in bounds; those keys are masked and their V zeroed)
                row_of[kb] = ((blk < 0 ? 0 : blk) * p.H_kv + g) * kBlock;
            }
            bool go = true;
            if (lane == 0 && t >= kNS)
                go = wait_or_abort(smem_u32(&bars.k_empty[s]), ((t - kNS) / kNS) & 1, &s_abort, p.status, p.wait_cycles);
            if (!__shfl_sync(0xffffffffu, go ? 1 : 0, 0)) break;
            if (lane == 0) {
                const uint32_t fb = smem_u32(&bars.k_full[s]);
                mbar_arrive_expect_tx(fb, kKVBytes);
                if (t != p.hold_tile) {   // test hook: the withheld tile's K bytes never arrive
#pragma unroll
                    for (int kb = 0; kb < kBlkPerTile; ++kb)
#pragma unroll
                        for (int x = 0; x < 2; ++x)
                            tma_load_2d(sK + s * kKVBytes + x * (kKVBytes / 2) + kb * 2048, &tmK, 64 * x, row_of[kb],
                                        fb);
                }
            }
            issued_k = t + 1;
            if (lane == 0 && t >= kNS)
                go = wait_or_abort(smem_u32(&bars.v_empty[s]), ((t - kNS) / kNS) & 1, &s_abort, p.status, p.wait_cycles);
            if (!__shfl_sync(0xffffffffu, go ? 1 : 0, 0)) break;
            if (lane == 0) {
                const uint32_t fb = smem_u32(&bars.v_full[s]);
                mbar_arrive_expect_tx(fb, kKVBytes);
#pragma unroll
                for (int kb = 0; kb < kBlkPerTile; ++kb)
#pragma unroll
                    for (int x = 0; x < 2; ++x)
                        tma_load_2d(sV + s * kKVBytes + x * (kKVBytes / 2) + kb * 2048, &tmV, 64 * x, row_of[kb], fb);
            }
            issued = t + 1;
        }
        // do not leave while copies into this CTA's shared memory may be in flight
        if (lane == 0 && s_abort) {
            for (int t = max(0, issued_k - kNS); t < issued_k; ++t)
                mbar_wait_bounded(smem_u32(&bars.k_full[t % kNS]), (t / kNS) & 1, p.wait_cycles);
            for (int t = max(0, issued - kNS); t < issued; ++t)
                mbar_wait_bounded(smem_u32(&bars.v_full[t % kNS]), (t / kNS) & 1, p.wait_cycles);
            mbar_wait_bounded(qb, 0, p.wait_cycles);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs this loop (every lane waits on the same barriers); one elected
        // lane issues each MMA and commit.
        {
            const uint32_t id_qk = idesc_f16(BF16, false, kBM, kBN);
            const uint32_t id_pv = idesc_f16(BF16, true, kBM, kD);
            // S(x) = Q(x) . K^T of stage s: M = 128 rows, N = 128 keys, 8 steps of K = 16 dims
            auto qk = [&](int x, int s) {
                const uint32_t kbase = sK + s * kKVBytes, qbase = sQ + x * kQBytes;
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * (kQBytes / 2) + (ks & 3) * 32;
                    umma_w(tmem + 256 * x, sdesc_k128(qbase + off), sdesc_k128(kbase + off), id_qk, ks > 0);
                }
            };
            // O(x) += P(x) . V of stage s: A = P from TMEM (per 32 keys: 16 columns of high
            // parts, then for bf16 16 of low parts), B = V as an MN-major operand; 8 steps of 16 keys
            auto pv = [&](int x, int s, bool first) {
                const uint32_t vbase = sV + s * kKVBytes;
#pragma unroll
                for (int ks = 0; ks < kBN / 16; ++ks) {
                    const uint64_t bv = sdesc_mn128(vbase + ks * 2048, kKVBytes / 2);
                    const uint32_t a = tmem + 256 * x + 32 * (ks >> 1) + 8 * (ks & 1);
                    umma_ts_w(tmem + 256 * x + 128, a, bv, id_pv, !(first && ks == 0));
                    if constexpr (BF16) umma_ts_w(tmem + 256 * x + 128, a + 16, bv, id_pv, true);   // low part
                }
            };
            // every lane takes the same branch: a wait's outcome is agreed on by the warp
            auto wait = [&](uint32_t bar, uint32_t parity) {
                return __all_sync(0xffffffffu, wait_or_abort(bar, parity, &s_abort, p.status, p.wait_cycles));
            };
            bool ok = wait(smem_u32(&bars.q_full), 0) && wait(smem_u32(&bars.k_full[0]), 0);
            if (ok) {
                tc_fence_after();
                qk(0, 0);
                umma_commit_w(smem_u32(&bars.s_full[0]));
                qk(1, 0);
                umma_commit_w(smem_u32(&bars.s_full[1]));
                umma_commit_w(smem_u32(&bars.k_empty[0]));
            }
            for (int t = 0; ok && t < ntiles; ++t) {
                const int s = t % kNS, s1 = (t + 1) % kNS;
                const bool more = t + 1 < ntiles;
                // tile A: P . V, then its next scores
                if (!wait(smem_u32(&bars.p_full[0]), t & 1)) break;
                if (!wait(smem_u32(&bars.v_full[s]), (t / kNS) & 1)) break;
                tc_fence_after();
                pv(0, s, t == 0);
                if (more) {
                    if (!wait(smem_u32(&bars.k_full[s1]), ((t + 1) / kNS) & 1)) break;
                    tc_fence_after();
                    qk(0, s1);
                    umma_commit_w(smem_u32(&bars.s_full[0]));
                } else {
                    umma_commit_w(smem_u32(&bars.o_done[0]));
                }
                // tile B
                if (!wait(smem_u32(&bars.p_full[1]), t & 1)) break;
                tc_fence_after();
                pv(1, s, t == 0);
                umma_commit_w(smem_u32(&bars.v_empty[s]));
                if (more) {
                    qk(1, s1);
                    umma_commit_w(smem_u32(&bars.s_full[1]));
                    umma_commit_w(smem_u32(&bars.k_empty[s1]));
                } else {
                    umma_commit_w(smem_u32(&bars.o_done[1]));
                }
            }
            // Every MMA this thread issued, also on an abort, is done before TMEM is freed.
            umma_commit_w(smem_u32(&bars.mma_drain));
            mbar_wait_bounded(smem_u32(&bars.mma_drain), 0, p.wait_cycles);
        }
    } else {
        // ------------------------------------------------------------ softmax
        // Warps 2..5: tile A, warps 6..9: tile B.  quarter = warp % 4 fixes the 32 TMEM lanes
        // (query rows) a warp may touch; one thread per row.
        const int x = (warp - 2) >> 2;
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;                   // query row of this thread in tile x
        const int tile_pos0 = i0 + x * pos_per_tile;
        const int pos = tile_pos0 + r / p.G;
        const int kmax = p.cascade ? p.nkeys : p.P0 + min(pos, p.C - 1) + 1;              // keys < kmax visible
        const int kmin_tile = p.cascade ? p.nkeys : p.P0 + min(tile_pos0, p.C - 1) + 1;   // smallest kmax of tile x
        const uint32_t tS = tmem + ((uint32_t)(quarter * 32) << 16) + 256 * x;
        const uint32_t tO = tS + 128;
        const float sl = p.scale_log2;
        const bool pos_scale = sl > 0.f;
        float m_used = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int t = 0; t < ntiles; ++t) {
            if (!__all_sync(0xffffffffu, wait_or_abort(smem_u32(&bars.s_full[x]), t & 1, &s_abort, p.status, p.wait_cycles))) {
                ok = false;
                break;
            }
            tc_fence_after();
            // pass 1: the row maximum of the tile's 128 scores (64 at a time), in three-input
            // maxima; the scale is applied before the causal mask, so any scale sign works
            const int key0 = (t_lo + t) * kBN;
            const bool need_mask = key0 + kBN > kmin_tile;
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};   // four independent chains
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float v[64];
                tmem_ld32(tS + 64 * hh, *reinterpret_cast<float(*)[32]>(&v[0]));
                tmem_ld32(tS + 64 * hh + 32, *reinterpret_cast<float(*)[32]>(&v[32]));
                tmem_wait_ld();
                if (!pos_scale) {
#pragma unroll
                    for (int j = 0; j < 64; ++j) v[j] *= sl;
                }
                if (need_mask) {
#pragma unroll
                    for (int j = 0; j < 64; ++j)
                        if (key0 + 64 * hh + j >= kmax) v[j] = -INFINITY;
                }
#pragma unroll
                for (int j = 0; j < 64; j += 8)
#pragma unroll
                    for (int k = 0; k < 4; ++k) m4[k] = fmax3(m4[k], v[j + 2 * k], v[j + 2 * k + 1]);
            }
            float mx = fmax3(fmax3(m4[0], m4[1], m4[2]), m4[3], -INFINITY);
            if (pos_scale) mx *= sl;
            float m_new = m_used;
            if (mx > m_used + kRescaleSlack || m_used == -INFINITY) m_new = mx;
            const float alpha = m_used == -INFINITY ? 0.f : ex2(m_used - m_new);
            // P = 2^(scale * score - m), back into the score's columns: keys 32c .. 32c+31 ->
            // columns 32c .. 32c+15 (high part), 32c+16 .. 32c+31 (bf16 only: low part).
            // bf16: the high part is the truncation (upper half of the fp32 word), the low part
            // the truncated remainder, both by byte permutes; fp16: P rounded to fp16.
            // pass 2: reread each 32-key chunk, exponentiate, pack, store over the same columns
            const float mref = m_new == -INFINITY ? 0.f : m_new;
            const float2 sl2 = make_float2(sl, sl), mref2 = make_float2(-mref, -mref);
            float2 sum2 = make_float2(0.f, 0.f);
#pragma unroll 1
            for (int c = 0; c < kBN / 32; ++c) {
                float v[32];
                tmem_ld32(tS + 32 * c, v);
                tmem_wait_ld();
                uint32_t w[32];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float2 a = ffma2(make_float2(v[2 * e], v[2 * e + 1]), sl2, mref2);
                    if (need_mask) {
                        if (key0 + 32 * c + 2 * e >= kmax) a.x = -INFINITY;
                        if (key0 + 32 * c + 2 * e + 1 >= kmax) a.y = -INFINITY;
                    }
                    const float2 pp = make_float2(ex2(a.x), ex2(a.y));
                    if constexpr (BF16) {
                        const uint32_t u0 = __float_as_uint(pp.x), u1 = __float_as_uint(pp.y);
                        w[e] = __byte_perm(u0, u1, 0x7632);
                        const float2 rr = fsub2(pp, make_float2(__uint_as_float(u0 & 0xffff0000u),
                                                                __uint_as_float(u1 & 0xffff0000u)));
                        w[16 + e] = __byte_perm(__float_as_uint(rr.x), __float_as_uint(rr.y), 0x7632);
                    } else {   // fp16 P in one part: 11 bits, relative error <= 2^-12
                        w[e] = pack2<false>(pp.x, pp.y);
                    }
                    sum2 = fadd2(sum2, pp);
                }
                if constexpr (BF16) tmem_st32u(tS + 32 * c, w);
                else tmem_st16u(tS + 32 * c, *reinterpret_cast<const uint32_t(*)[16]>(&w[0]));
            }
            l_run = l_run * alpha + (sum2.x + sum2.y);
            m_used = m_new;
            // the running max moved: rescale this row of O (P . V(t-1) is done: s_full(t) says so)
            if (t > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
                for (int c = 0; c < kD / 32; ++c) {
                    float o[32];
                    tmem_ld32(tO + 32 * c, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] *= alpha;
                    tmem_st32(tO + 32 * c, o);
                }
            }
            // keys past the end of the sequence: zero their V rows (P is 0 there, V may be
            // stale).  Tile A's warps do it before their P . V, which runs before tile B's.
            if (x == 0 && t == ntiles - 1 && key0 + kBN > seq_len) {   // only the last split's last tile
                const int s = t % kNS;
                if (!__all_sync(0xffffffffu, wait_or_abort(smem_u32(&bars.v_full[s]), (t / kNS) & 1, &s_abort, p.status, p.wait_cycles))) {
                    ok = false;
                    break;
                }
                const int first = seq_len - key0;
                const int tid = threadIdx.x - 64;             // 0..127
                for (int i = tid; i < 2 * (kBN - first) * 8; i += 128) {
                    const int x16 = i & 7, rowi = (i >> 3) % (kBN - first), half = (i >> 3) / (kBN - first);
                    const uint32_t a = sV + s * kKVBytes + half * (kKVBytes / 2) + (first + rowi) * 128 + x16 * 16;
                    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
                }
                fence_proxy_async_smem();
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bars.p_full[x]));
        }
        if (ok && __all_sync(0xffffffffu, wait_or_abort(smem_u32(&bars.o_done[x]), 0, &s_abort, p.status, p.wait_cycles))) {
            tc_fence_after();
            const bool valid = pos < p.C;
            const float inv = p.cascade ? 1.f : 1.f / l_run;
            const size_t qrow = (size_t)pos * p.H_q + g * p.G + (r % p.G);
            const size_t slot = qrow * p.slots + blockIdx.z;
            float* orow = p.cascade ? p.ws_o + slot * kD : p.out + qrow * kD;
            if (p.cascade && valid)
                *reinterpret_cast<float2*>(p.ws_ml + slot * 2) = make_float2(m_used, l_run);
#pragma unroll 1
            for (int c = 0; c < kD / 32; ++c) {
                float o[32];
                tmem_ld32(tO + 32 * c, o);
                tmem_wait_ld();
                if (valid) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        *reinterpret_cast<float4*>(orow + 32 * c + i) =
                            make_float4(o[i] * inv, o[i + 1] * inv, o[i + 2] * inv, o[i + 3] * inv);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

}  // namespace

int prefill_tc_key_splits(int C, int G, int H_kv, int nkeys)
{
    const int ctas = (C + kQT * (kBM / G) - 1) / (kQT * (kBM / G)) * H_kv;
    const int tiles = (nkeys + kBN - 1) / kBN;
    int z = num_sms() / (ctas > 0 ? ctas : 1);
    z = z < 1 ? 1 : z;
    return z < tiles ? z : tiles;
}

bool prefill_tc_supported(int d, int G, int kv_dtype)
{
    return d == kD && G >= 1 && G <= kBM && (kBM % G) == 0 && (kv_dtype == PKV_BF16 || kv_dtype == PKV_F16);
}

// Q viewed as [C][H_q][d] with boxes of 64 dims x G heads x 128/G positions.
bool make_q_map(CUtensorMap* map, const void* q, int C, int H_q, int G, PFN_encode enc)
{
    const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)H_q, (cuuint64_t)C};
    const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)H_q * kD * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)G, (cuuint32_t)(kBM / G)};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(q), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int launch_prefill_tc(const PrefillArgs& a, const CUtensorMap* tmq, const CUtensorMap* tmk, const CUtensorMap* tmv,
                      cudaStream_t s)
{
    TcParams p;
    p.table = a.table;
    p.out = a.out;
    p.status = a.status;
    p.P0 = a.P0;
    p.C = a.C;
    p.H_q = a.H_q;
    p.H_kv = a.H_kv;
    p.G = a.G;
    p.N = a.N;
    p.scale_log2 = a.scale * kLog2e;
    p.cascade = a.cascade_nkeys > 0;
    p.nkeys = a.cascade_nkeys;
    p.slots = a.ws_slots;
    p.ws_o = a.ws_o;
    p.ws_ml = a.ws_ml;
    const WaitHook hook = wait_hook();
    p.hold_tile = hook.hold_tile;
    p.wait_cycles = hook.wait_cycles;
    auto kern = a.kv_dtype == PKV_BF16 ? prefill_tc_kernel<true> : prefill_tc_kernel<false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess)
        return PKV_ERR_CUDA;
    const int pos_per_cta = kQT * (kBM / a.G);
    const dim3 grid((a.C + pos_per_cta - 1) / pos_per_cta, a.H_kv, a.cascade_nkeys > 0 ? a.key_splits : 1);
    kern<<<grid, kThreads, kSmem, s>>>(p, *tmq, *tmk, *tmv);
    return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

}  // namespace pkv
