// decode_tc.cu -- paged_decode_attn for wide query groups (64 or 128 query heads per KV head,
// down to multi-query attention) on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// "KV cache, GQA, paging and continuous batching", section "Mechanics": with one KV head
// for many query heads (MQA in the limit) every K/V byte is used by all G query heads, so
// the decode does G multiply-adds per K element and G per V element.  At G = 64 the
// warp-level mma.sync form is bound by its own tensor work, far below the HBM rate; here
// the two contractions run as tcgen05 MMAs with fp32 accumulators in TMEM.
//
// One CTA = (128/G sequences, one KV head, one split-K partition of each of them).  Its 128
// query rows are the G heads of each sequence (rows s*G .. s*G + G-1 belong to sequence s).
// A key tile holds 64 keys, 64/(128/G) consecutive ones from each sequence (whole paged
// blocks of that sequence's table).  S = Q . K^T (M 128, N 64) then has one diagonal block
// per sequence; the softmax keeps each row's own block and writes P = 0 into the others, so
// O += P . V (M 128, N 128, K 64) takes every sequence's rows from its own keys only.  At
// G = 64 half of the tensor work is spent on the zero blocks; the decode is bound by HBM,
// and the tensor pipe has room for that.
//   warp 0      TMA producer of Q (once, 3-D boxes over [sequence][head][dim]) and of the
//               2-stage K ring: per key tile one 16-row box pair per paged block (128-byte
//               swizzle, no multicast); warp 6 does the same for the V ring, so that K
//               tiles, freed as soon as their Q . K^T is done, are not held up behind V
//               tiles, freed only after P . V.  The TMA row of every paged block the CTA
//               reads is looked up once, at the start, into shared memory;
//   warp 1      allocates 256 TMEM columns (S, later P, of even tiles: 0..63, of odd tiles:
//               64..127; O: 128..255) and issues every MMA from one thread, in the order
//               QK(0), QK(1), then per tile t P.V(t), QK(t+2): the scores of tile t+1 are
//               computed while the softmax of tile t runs;
//   warps 2..5  softmax, one thread per query row (= TMEM lane): read the row's own 32 or
//               64 scores, mask what lies past its partition's end, keep the running max
//               lazily (it moves only when the new max exceeds the old by 2^8, then the
//               thread rescales its O row), and store P over the scores: for bf16 pools as
//               a high and a low bf16 part (two MMAs keep P . V at ~16 mantissa bits), for
//               fp16 pools as one fp16 part (11 bits, one MMA).
// Two CTAs fit one SM (99 KiB of shared memory, 256 TMEM columns each).  Partials (o, m, l) of sequences longer
// than one partition go to the decode workspace and are merged by decode_reduce, as in the
// other decode engines.  Every wait is bounded; a timeout sets PKV_DEV_TIMEOUT.
#include "decode_common.cuh"
#include "tcgen05.cuh"

namespace pkv {

namespace {

constexpr int kD = 128;                         // head dim handled here
constexpr int kM = 128;                         // query rows per CTA
constexpr int kBN = 64;                         // keys per tile
constexpr int kNS = 2;                          // ring stages
constexpr int kQBox = kM * 128;                 // one 64-dim box of Q: 128 rows x 128 B
constexpr int kQBytes = 2 * kQBox;              // 32 KiB
constexpr int kKVBox = kBN * 128;               // one 64-dim box of a K (V) tile: 64 rows x 128 B
constexpr int kKVBytes = 2 * kKVBox;            // 16 KiB per K (or V) stage
constexpr int kRowsMax = 4096 / 16;           // paged blocks of one partition (at most 4096 keys)
constexpr int kRowsOff = kQBytes + kNS * 2 * kKVBytes;   // TMA row of every paged block of the CTA
constexpr int kSmem = kRowsOff + 2 * kRowsMax * 4 + 1024;
constexpr uint32_t kTmemCols = 256;             // S / P of even tiles at 0, of odd tiles at 64, O at 128
constexpr int kThreads = 224;                   // K producer, MMA, 4 softmax warps, V producer
constexpr float kRescaleSlack = 8.f;            // log2 units

struct TcDecodeBars {
    uint64_t q_full;
    uint64_t k_full[kNS];
    uint64_t k_empty[kNS];
    uint64_t v_full[kNS];
    uint64_t v_empty[kNS];
    uint64_t s_full[2];   // S(t) is in buffer t % 2 (every MMA issued before it is done too)
    uint64_t p_full[2];   // P(t) stored by the 4 softmax warps (and V rows past an end zeroed)
    uint64_t pv_done;     // completes once per P . V, in order
    uint64_t o_done;      // the last P . V is done
    uint64_t mma_drain;   // every MMA is done (before TMEM is freed)
};

template <bool BF16>
__global__ void __launch_bounds__(kThreads, 2)
decode_tc_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmQ,
                 const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV)
{
    extern __shared__ uint8_t smem_dyn[];
    __shared__ TcDecodeBars bars;
    __shared__ uint32_t s_tmem_base;
    __shared__ volatile int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int part = blockIdx.x, g = blockIdx.y;
    const int G = p.G;
    const int spt = kM / G;                      // sequences per CTA: 2 (G = 64) or 1 (G = 128)
    const int kps = kBN / spt;                   // keys of one sequence per tile: 32 or 64
    const int bps = kps / kBlock;                // its paged blocks per tile: 2 or 4
    const int b0 = blockIdx.z * spt;

    // each sequence's key range in this partition: [lo_s, end_s), lo_s = part * P
    int ctx_s[2] = {0, 0}, end_s[2] = {0, 0};
    int ntiles = 0;
    for (int s = 0; s < spt; ++s) {
        const int b = b0 + s;
        if (b >= p.num_seqs) continue;
        const int ctx = checked_ctx(p, b, threadIdx.x == 0 && part == 0 && g == 0);
        ctx_s[s] = ctx;
        const int lo = part * p.part_tokens;
        end_s[s] = min(ctx, lo + p.part_tokens);
        if (end_s[s] > lo) ntiles = max(ntiles, (end_s[s] - lo + kps - 1) / kps);
    }
    if (ntiles == 0) {   // nothing in this partition; an empty context gets a zero row
        if (part == 0 && p.part_base == 0) {
            for (int s = 0; s < spt; ++s) {
                const int b = b0 + s;
                if (b >= p.num_seqs || ctx_s[s] != 0) continue;
                float* o = p.out + ((size_t)b * p.H_q + (size_t)g * G) * kD;
                for (int i = threadIdx.x; i < G * kD; i += kThreads) o[i] = 0.f;
            }
        }
        return;
    }
    const int tok_lo = part * p.part_tokens;

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    const uint32_t sQ = smem_u32(smem);
    const uint32_t sK = sQ + kQBytes;
    const uint32_t sV = sK + kNS * kKVBytes;

    if (threadIdx.x == 0) {
        s_abort = 0;
        mbar_init(smem_u32(&bars.q_full), 1);
        for (int s = 0; s < kNS; ++s) {
            mbar_init(smem_u32(&bars.k_full[s]), 1);
            mbar_init(smem_u32(&bars.k_empty[s]), 1);
            mbar_init(smem_u32(&bars.v_full[s]), 1);
            mbar_init(smem_u32(&bars.v_empty[s]), 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(smem_u32(&bars.s_full[x]), 1);
            mbar_init(smem_u32(&bars.p_full[x]), 4);
        }
        mbar_init(smem_u32(&bars.pv_done), 1);
        mbar_init(smem_u32(&bars.o_done), 1);
        mbar_init(smem_u32(&bars.mma_drain), 1);
        mbar_fence_init();
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        mbar_arrive_expect_tx(smem_u32(&bars.q_full), kQBytes);
        tma_load_3d(sQ, &tmQ, 0, g * G, b0, smem_u32(&bars.q_full));
        tma_load_3d(sQ + kQBox, &tmQ, 64, g * G, b0, smem_u32(&bars.q_full));
    }
    // TMA row of paged block kb (< 4) of tile t at rows[t * 4 + kb]: sequence kb / bps, its
    // block kb % bps of the tile; block 0 (in bounds) past a sequence's range, where the
    // keys are masked and the V rows zeroed
    int* rows = reinterpret_cast<int*>(smem + kRowsOff);
    for (int i = threadIdx.x; i < ntiles * (kBN / kBlock); i += kThreads) {
        const int t = i >> 2, kb = i & 3;
        const int s = kb / bps, lb = (tok_lo + t * kps) / kBlock + (kb - s * bps);
        int blk = 0;
        if (lb * kBlock < end_s[s]) {
            blk = p.tables[(size_t)(b0 + s) * p.W + lb];
            if ((unsigned)blk >= (unsigned)p.N) {
                flag_status(p.status, PKV_DEV_BAD_BLOCK);
                blk = 0;
            }
        }
        rows[i] = (blk * p.H_kv + g) * kBlock;
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

    if (warp == 0 || warp == 6) {
        // ------------------------------------------------------------ producers (K: warp 0, V: warp 6)
        const bool is_k = warp == 0;
        uint64_t* full = is_k ? bars.k_full : bars.v_full;
        uint64_t* empty = is_k ? bars.k_empty : bars.v_empty;
        const CUtensorMap* tm = is_k ? &tmK : &tmV;
        const uint32_t ring = is_k ? sK : sV;
        int issued = 0;
        if (lane == 0) {
            for (int t = 0; t < ntiles; ++t) {
                const int st = t % kNS;
                if (t >= kNS &&
                    !wait_or_abort(smem_u32(&empty[st]), ((t - kNS) / kNS) & 1, &s_abort, p.status, p.wait_cycles))
                    break;
                const uint32_t fb = smem_u32(&full[st]);
                mbar_arrive_expect_tx(fb, kKVBytes);
                issued = t + 1;
                if (is_k && t == p.hold_tile) continue;   // test hook: the withheld tile's K bytes never arrive
#pragma unroll
                for (int kb = 0; kb < kBN / kBlock; ++kb)
#pragma unroll
                    for (int x = 0; x < 2; ++x) {
                        if constexpr (kHintKV)
                            tma_load_2d_hint(ring + st * kKVBytes + x * kKVBox + kb * 2048, tm, 64 * x, rows[t * 4 + kb],
                                             fb, l2_evict_first());
                        else
                            tma_load_2d(ring + st * kKVBytes + x * kKVBox + kb * 2048, tm, 64 * x, rows[t * 4 + kb], fb);
                    }
            }
            // do not leave while copies into this CTA's shared memory may be in flight
            if (s_abort) {
                for (int t = max(0, issued - kNS); t < issued; ++t)
                    mbar_wait_bounded(smem_u32(&full[t % kNS]), (t / kNS) & 1, p.wait_cycles);
                if (is_k) mbar_wait_bounded(smem_u32(&bars.q_full), 0, p.wait_cycles);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs this loop (every lane waits on the same barriers, and the warp
        // agrees on each outcome); one elected lane issues each MMA and commit.
        {
            auto wait = [&](uint32_t bar, uint32_t parity) {
                return __all_sync(0xffffffffu, wait_or_abort(bar, parity, &s_abort, p.status, p.wait_cycles));
            };
            const uint32_t id_qk = idesc_f16(BF16, false, kM, kBN);
            const uint32_t id_pv = idesc_f16(BF16, true, kM, kD);
            const uint32_t tO = tmem + 128;
            // S(t) = Q . K(t)^T into buffer t % 2: M 128 rows, N 64 keys, 8 steps of K = 16 dims
            auto qk = [&](int t) -> bool {
                const int st = t % kNS;
                if (!wait(smem_u32(&bars.k_full[st]), (t / kNS) & 1))
                    return false;
                tc_fence_after();
                const uint32_t kbase = sK + st * kKVBytes;
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks) {
                    const uint32_t qoff = (ks >> 2) * kQBox + (ks & 3) * 32;
                    const uint32_t koff = (ks >> 2) * kKVBox + (ks & 3) * 32;
                    umma_w(tmem + 64 * (t & 1), sdesc_k128(sQ + qoff), sdesc_k128(kbase + koff), id_qk, ks > 0);
                }
                umma_commit_w(smem_u32(&bars.s_full[t & 1]));
                umma_commit_w(smem_u32(&bars.k_empty[st]));
                return true;
            };
            // Tensor-core order: QK(0), QK(1), then per tile t: P.V(t), QK(t+2) -- QK(t+1) runs
            // while the softmax of tile t does, and QK(t+2) overwrites buffer t % 2 only after
            // P.V(t) has read it (one thread's MMAs execute in order).
            bool ok = wait(smem_u32(&bars.q_full), 0) && qk(0) &&
                      (ntiles < 2 || qk(1));
            for (int t = 0; ok && t < ntiles; ++t) {
                const int st = t % kNS;
                // O += P . V: A = P from TMEM (per 32 keys 16 columns of high parts, then for
                // bf16 16 of low parts), B = V as an MN-major operand, 4 steps of 16 keys
                if (!wait(smem_u32(&bars.p_full[t & 1]), (t >> 1) & 1)) break;
                if (!wait(smem_u32(&bars.v_full[st]), (t / kNS) & 1)) break;
                tc_fence_after();
                const uint32_t vbase = sV + st * kKVBytes;
                const uint32_t tP = tmem + 64 * (t & 1);
#pragma unroll
                for (int ks = 0; ks < kBN / 16; ++ks) {
                    const uint64_t bv = sdesc_mn128(vbase + ks * 2048, kKVBox);
                    const uint32_t a = tP + 32 * (ks >> 1) + 8 * (ks & 1);
                    umma_ts_w(tO, a, bv, id_pv, !(t == 0 && ks == 0));
                    if constexpr (BF16) umma_ts_w(tO, a + 16, bv, id_pv, true);   // low part
                }
                umma_commit_w(smem_u32(&bars.v_empty[st]));
                umma_commit_w(smem_u32(&bars.pv_done));
                if (t + 2 < ntiles && !qk(t + 2)) break;
            }
            umma_commit_w(smem_u32(&bars.o_done));
            // every MMA this thread issued, also on an abort, is done before TMEM is freed
            umma_commit_w(smem_u32(&bars.mma_drain));
            mbar_wait_bounded(smem_u32(&bars.mma_drain), 0, p.wait_cycles);
        }
    } else {
        // ------------------------------------------------------------ softmax
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;           // query row = TMEM lane
        const int s = r / G, h = r - s * G;          // sequence of the CTA, query head in the group
        const int b = b0 + s;
        const uint32_t tL = tmem + ((uint32_t)(quarter * 32) << 16);   // this warp's lane quarter
        const uint32_t tO = tL + 128;
        const float sl = p.scale_log2;
        const int my_end = end_s[s];
        const int my_col = s * kps;                  // this row's keys: columns my_col .. my_col + kps - 1
        float m_used = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int t = 0; t < ntiles; ++t) {
            if (!__all_sync(0xffffffffu, wait_or_abort(smem_u32(&bars.s_full[t & 1]), (t >> 1) & 1, &s_abort, p.status,
                                                        p.wait_cycles))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t tS = tL + 64 * (t & 1);   // this tile's S / P buffer
            const int key0 = tok_lo + t * kps;       // token of this row's first column
            const int nvalid = min(kps, max(0, my_end - key0));
            float v[64];
            tmem_ld32(tS + my_col, *reinterpret_cast<float(*)[32]>(&v[0]));
            if (kps == 64) tmem_ld32(tS + my_col + 32, *reinterpret_cast<float(*)[32]>(&v[32]));
            tmem_wait_ld();
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int j = 0; j < 64; ++j) {
                if (j >= kps) break;
                const float x = j < nvalid ? v[j] * sl : -INFINITY;
                v[j] = x;
                m4[j & 3] = fmaxf(m4[j & 3], x);
            }
            const float mx = fmax3(fmax3(m4[0], m4[1], m4[2]), m4[3], -INFINITY);
            float m_new = m_used;
            if (mx > m_used + kRescaleSlack || m_used == -INFINITY) m_new = mx;
            const float alpha = m_used == -INFINITY ? 0.f : ex2(m_used - m_new);
            const float mref = m_new == -INFINITY ? 0.f : m_new;
            float2 sum2 = make_float2(0.f, 0.f);
            // P for the row's own keys, 32 at a time: columns 32c .. 32c+15 high parts,
            // 32c+16 .. 32c+31 low parts (bf16); the other sequence's columns get zeros
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                if (32 * c >= kps) break;
                uint32_t w[32];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float2 a = make_float2(v[32 * c + 2 * e] - mref, v[32 * c + 2 * e + 1] - mref);
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
                if constexpr (BF16) tmem_st32u(tS + my_col + 32 * c, w);
                else tmem_st16u(tS + my_col + 32 * c, *reinterpret_cast<const uint32_t(*)[16]>(&w[0]));
            }
            if (kps == 32) {   // two sequences: zero P over the other one's keys
                uint32_t z[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) z[e] = 0u;
                tmem_st32u(tS + (32 - my_col), z);
            }
            l_run = l_run * alpha + (sum2.x + sum2.y);
            m_used = m_new;
            // the running max moved: rescale this row of O once P . V(t-1) is done (P . V(t-2)
            // is: QK(t) came after it, and s_full(t) covers every earlier MMA; P . V(t) waits
            // for this tile's P)
            if (t > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                if (!__all_sync(0xffffffffu, wait_or_abort(smem_u32(&bars.pv_done), (t - 1) & 1, &s_abort, p.status,
                                                            p.wait_cycles))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
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
            // keys past a sequence's range in this tile: zero their V rows (P is 0 there, V
            // may be anything, NaN included)
            bool tail = false;
            for (int s2 = 0; s2 < spt; ++s2) tail |= end_s[s2] < key0 + kps;
            if (tail) {
                const int st = t % kNS;
                if (!__all_sync(0xffffffffu, wait_or_abort(smem_u32(&bars.v_full[st]), (t / kNS) & 1, &s_abort, p.status, p.wait_cycles))) {
                    ok = false;
                    break;
                }
                const int tid = threadIdx.x - 64;    // 0..127
                for (int s2 = 0; s2 < spt; ++s2) {
                    const int nv = min(kps, max(0, end_s[s2] - key0));
                    const int nz = kps - nv;          // rows s2*kps + nv .. (s2+1)*kps - 1
                    for (int i = tid; i < 2 * nz * 8; i += 128) {
                        const int x16 = i & 7, rowi = (i >> 3) % nz, half = (i >> 3) / nz;
                        const uint32_t a = sV + st * kKVBytes + half * kKVBox + (s2 * kps + nv + rowi) * 128 + x16 * 16;
                        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
                    }
                }
                fence_proxy_async_smem();   // each warp's zeros reach the MMA through its p_full arrival
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bars.p_full[t & 1]));
        }
        if (ok && __all_sync(0xffffffffu, wait_or_abort(smem_u32(&bars.o_done), 0, &s_abort, p.status, p.wait_cycles))) {
            tc_fence_after();
            const bool has = b < p.num_seqs && my_end > tok_lo;   // this row's sequence has keys here
            const int nparts = (ctx_s[s] + p.part_tokens - 1) / p.part_tokens;
            const bool final_out = nparts == 1 && p.part_base == 0;
            const size_t qrow = (size_t)b * p.H_q + (size_t)g * G + h;
            float* orow = final_out ? p.out + qrow * kD : p.ws_o + ws_slot(p, qrow, part) * kD;
            const float inv = final_out ? 1.f / l_run : 1.f;
            const uint64_t pol = l2_evict_last();   // partials: the merge reads them back soon
            if (has && !final_out) {
                float2* dst = reinterpret_cast<float2*>(p.ws_ml + ws_slot(p, qrow, part) * 2);
                if (kHintPartials) st_hint(dst, make_float2(m_used, l_run), pol);
                else *dst = make_float2(m_used, l_run);
            }
#pragma unroll 1
            for (int c = 0; c < kD / 32; ++c) {
                float o[32];
                tmem_ld32(tO + 32 * c, o);
                tmem_wait_ld();
                if (has) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        float4* dst = reinterpret_cast<float4*>(orow + 32 * c + i);
                        const float4 v = make_float4(o[i] * inv, o[i + 1] * inv, o[i + 2] * inv, o[i + 3] * inv);
                        if (kHintPartials && !final_out) st_hint(dst, v, pol);
                        else *dst = v;
                    }
                }
            }
        }
        if (part == 0 && b < p.num_seqs && ctx_s[s] == 0) {   // an empty context beside a non-empty one
            float* o = p.out + ((size_t)b * p.H_q + (size_t)g * G + h) * kD;
            for (int i = 0; i < kD; i += 4) *reinterpret_cast<float4*>(o + i) = make_float4(0.f, 0.f, 0.f, 0.f);
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

bool decode_tc_supported(int d, int G, int kv_dtype)
{
    return d == kD && (G == 64 || G == 128) && (kv_dtype == PKV_BF16 || kv_dtype == PKV_F16);
}

int launch_decode_tc(const DecodeParams& p, int kv_dtype, const CUtensorMap* tmq, const CUtensorMap* tmk,
                     const CUtensorMap* tmv, cudaStream_t s)
{
    auto kern = kv_dtype == PKV_BF16 ? decode_tc_kernel<true> : decode_tc_kernel<false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess)
        return PKV_ERR_CUDA;
    const int spt = kM / p.G;
    const dim3 grid(p.max_parts, p.H_kv, (p.num_seqs + spt - 1) / spt);
    kern<<<grid, kThreads, kSmem, s>>>(p, *tmq, *tmk, *tmv);
    return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

}  // namespace pkv
