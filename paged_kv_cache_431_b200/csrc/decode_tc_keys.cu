// decode_tc_keys.cu -- paged_decode_attn for groups of 64 query heads per KV head (multi-query
// attention at 64 heads, or GQA with groups that wide) on the 5th-generation tensor cores,
// with the KEYS on the MMA's M side.
//
// "KV cache, GQA, paging and continuous batching", section "Mechanics": with one KV head for
// G query heads every K/V byte meets G heads.  A tcgen05 MMA has M = 128 rows, but one decode
// step of one sequence has only G = 64 query rows, so the two contractions are transposed:
//   S^T  = K . Q^T     M = 128 keys of one sequence, N = 64 heads, K = 128 dims
//   O^T += V^T . P^T   M = 128 dims (the V tile read as an MN-major operand), N = 64 heads,
//                      K = 128 keys (P^T staged in shared memory by the softmax threads)
// and no tensor work goes to another sequence's keys.  The scores land in TMEM one key per
// lane: the softmax thread of key k reads that key's 64 scores, one per head.  The running
// maximum is per head and shared by the 128 key threads, and it moves lazily: every thread
// checks its scores against it, the softmax warps vote, and only a tile with a score
// above max + 8 (log2 units) recomputes the per-head maxima (a reduction across the threads),
// rescales the O^T columns in TMEM and the threads' partial sums.  Each thread keeps the
// partial row sums l of its keys, one per head; they are added across the threads at the end.
//
// One CTA = (split-K partition, KV head, sequence).  Warps:
//   0      TMA producer of Q (once: two 64-dim boxes of the group's 64 heads) and of the
//          2-stage K ring: per 128-key tile, 8 paged blocks x two 64-dim boxes (128-byte
//          swizzle, no multicast).  The TMA row of every paged block of the partition is
//          looked up once, at the start, into shared memory;
//   10     the same for the V ring;
//   1      allocates 256 TMEM columns (S^T of even tiles 0..63, of odd tiles 64..127, O^T
//          128..191) and issues every MMA from one elected lane: QK(0), QK(1), then per tile t
//          P.V(t) and QK(t+2), QK(t+2) first when its K tile has landed: the scores of the
//          next tiles are computed while the softmax runs, and no Q.K^T waits behind a V copy;
//   2..9   softmax, two threads per key (= TMEM lane), 32 heads each, and the epilogue, two
//          threads per dimension (= TMEM lane of O^T).  P^T goes to shared memory in the
//          layout a 128-byte swizzled TMA box of [key][64 heads] would have: for bf16 pools as
//          a high and a low bf16 part (two MMAs keep P . V at ~16 mantissa bits), for fp16
//          pools as one part; two P^T buffers, so the softmax of tile t+1 need not wait for
//          P . V(t).
// 208 KiB of shared memory (Q, 2 K stages, 2 V stages, 2 P^T buffers): one CTA per SM.  Partials (o, m, l) of sequences longer than one
// partition go to the decode workspace and are merged by decode_reduce.  Every wait is
// bounded, the meeting points of the softmax warps included (an mbarrier, not bar.sync);
// a timeout sets PKV_DEV_TIMEOUT and the CTA winds down.
#include "decode_common.cuh"
#include "tcgen05.cuh"

namespace pkv {

namespace {

constexpr int kD = 128;                          // head dim handled here
constexpr int kG = 64;                           // query heads per KV head
constexpr int kBN = 128;                         // keys per tile (the MMA's M)
#ifndef PKV_TCK_VSTAGES
#define PKV_TCK_VSTAGES 2
#endif
#ifndef PKV_TCK_PBUFS
#define PKV_TCK_PBUFS 2
#endif
#ifndef PKV_TCK_KSTAGES
#define PKV_TCK_KSTAGES 2
#endif
constexpr int kNS = PKV_TCK_KSTAGES;             // K ring stages
constexpr int kNSV = PKV_TCK_VSTAGES;            // V ring stages
constexpr int kPB = PKV_TCK_PBUFS;               // P^T buffers (tile t uses t % kPB)
constexpr int kQBox = kG * 128;                  // one 64-dim box of Q: 64 heads x 128 B
constexpr int kQBytes = 2 * kQBox;               // 16 KiB
constexpr int kKVBox = kBN * 128;                // one 64-dim half of a K (V) tile: 16 KiB
constexpr int kKVBytes = 2 * kKVBox;             // 32 KiB per stage
constexpr int kPBytes = kBN * kG * 2;            // one part of P^T (128 keys x 64 heads): 16 KiB
constexpr int kPOff = kQBytes + (kNS + kNSV) * kKVBytes;   // P^T buffers, each a high and a low part
constexpr int kRowsMax = 4096 / 16;              // paged blocks of one partition (at most 4096 keys)
constexpr int kRowsOff = kPOff + kPB * 2 * kPBytes;
constexpr int kSmem = kRowsOff + kRowsMax * 4 + 1024;
static_assert(kSmem <= 225 * 1024, "one CTA's shared memory (plus the static part) must fit 227 KiB");
constexpr uint32_t kTmemCols = 256;              // S^T of even tiles at 0, of odd tiles at 64, O^T at 128
constexpr int kSoftWarps = 8;                    // two per lane quarter: heads 0..31 and 32..63 of a key
constexpr int kHT = kG / 2;                      // heads per softmax thread
constexpr int kThreads = 32 * (3 + kSoftWarps);  // K producer, MMA, 8 softmax warps, V producer
constexpr int kVWarp = 2 + kSoftWarps;           // the V producer
constexpr float kRescaleSlack = 8.f;             // log2 units

struct KeysBars {
    uint64_t q_full;
    uint64_t k_full[kNS];
    uint64_t k_empty[kNS];
    uint64_t v_full[kNSV];
    uint64_t v_empty[kNSV];
    uint64_t s_full[2];   // S^T(t) is in buffer t % 2 (every MMA issued before it is done too)
    uint64_t p_full[2];   // P^T(t) stored by the 8 softmax warps (and V rows past the end zeroed)
    uint64_t pv_done[2];  // P . V(t) is done, barrier t % 2 (then P^T buffer t % kPB may be rewritten)
    uint64_t o_done;      // the last P . V is done
    uint64_t mma_drain;   // every MMA is done (before TMEM is freed)
    uint64_t group;       // meeting point of the 8 softmax warps, one phase per meeting
};

// v[h], h < N (32 or 64), reduced (max or sum) over the warp's 32 lanes by halving exchanges:
// each step a lane keeps one half of its values, receives its partner's copy of that half and
// combines.  Afterwards lane L holds head L in v[0] (N = 32), heads 2L, 2L + 1 in v[0], v[1] (N = 64).
template <int N, bool MAX>
__device__ __forceinline__ void warp_reduce_heads(float (&v)[N], int lane)
{
    static_assert(N == 32 || N == 64, "32 or 64 values per lane");
#pragma unroll
    for (int s = 0; s < 5; ++s) {
        const int half = (N / 2) >> s, off = 16 >> s;
        const bool up = (lane & off) != 0;
#pragma unroll
        for (int j = 0; j < half; ++j) {
            const float keep = up ? v[half + j] : v[j];
            const float give = up ? v[j] : v[half + j];
            const float got = __shfl_xor_sync(0xffffffffu, give, off);
            v[j] = MAX ? fmaxf(keep, got) : keep + got;
        }
    }
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads, 1)
decode_tck_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmQ,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV)
{
    extern __shared__ uint8_t smem_dyn[];
    __shared__ KeysBars bars;
    __shared__ uint32_t s_tmem_base;
    __shared__ volatile int s_abort;
    __shared__ __align__(16) float s_m[kG];    // running max per head (log2 units, scale applied), read as float4
    __shared__ __align__(16) float s_alpha[kG];   // rescale factor of the last recomputation
    __shared__ __align__(16) float s_red[4][kG];   // per-warp reductions
    __shared__ volatile int s_hit[2];          // t + 1: tile t needs the recomputation

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int part = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int ctx = checked_ctx(p, b, threadIdx.x == 0 && part == 0 && g == 0);
    const int tok_lo = part * p.part_tokens;
    const int end = min(ctx, tok_lo + p.part_tokens);
    const int ntiles = end > tok_lo ? (end - tok_lo + kBN - 1) / kBN : 0;
    if (ntiles == 0) {   // nothing in this partition; an empty context gets a zero row
        if (part == 0 && p.part_base == 0 && ctx == 0) {
            float* o = p.out + ((size_t)b * p.H_q + (size_t)g * kG) * kD;
            for (int i = threadIdx.x; i < kG * kD; i += kThreads) o[i] = 0.f;
        }
        return;
    }

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    const uint32_t sQ = smem_u32(smem);
    const uint32_t sK = sQ + kQBytes;
    const uint32_t sV = sK + kNS * kKVBytes;
    const uint32_t sP = sQ + kPOff;

    if (threadIdx.x == 0) {
        s_abort = 0;
        s_hit[0] = 0;
        s_hit[1] = 0;
        mbar_init(smem_u32(&bars.q_full), 1);
        for (int s = 0; s < kNS; ++s) {
            mbar_init(smem_u32(&bars.k_full[s]), 1);
            mbar_init(smem_u32(&bars.k_empty[s]), 1);
        }
        for (int s = 0; s < kNSV; ++s) {
            mbar_init(smem_u32(&bars.v_full[s]), 1);
            mbar_init(smem_u32(&bars.v_empty[s]), 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(smem_u32(&bars.s_full[x]), 1);
            mbar_init(smem_u32(&bars.p_full[x]), kSoftWarps);
        }
        mbar_init(smem_u32(&bars.pv_done[0]), 1);
        mbar_init(smem_u32(&bars.pv_done[1]), 1);
        mbar_init(smem_u32(&bars.o_done), 1);
        mbar_init(smem_u32(&bars.mma_drain), 1);
        mbar_init(smem_u32(&bars.group), kSoftWarps);
        mbar_fence_init();
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        mbar_arrive_expect_tx(smem_u32(&bars.q_full), kQBytes);
        tma_load_3d(sQ, &tmQ, 0, g * kG, b, smem_u32(&bars.q_full));
        tma_load_3d(sQ + kQBox, &tmQ, 64, g * kG, b, smem_u32(&bars.q_full));
    }
    if (threadIdx.x < kG) s_m[threadIdx.x] = -INFINITY;
    // TMA row of paged block kb (< 8) of tile t at rows[t * 8 + kb]; block 0 (in bounds) past
    // the partition's end, where the keys are masked and the V rows zeroed
    int* rows = reinterpret_cast<int*>(smem + kRowsOff);
    for (int i = threadIdx.x; i < ntiles * (kBN / kBlock); i += kThreads) {
        const int lb = tok_lo / kBlock + i;
        int blk = 0;
        if (lb * kBlock < end) {
            blk = p.tables[(size_t)b * p.W + lb];
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

    if (warp == 0 || warp == kVWarp) {
        // ------------------------------------------------------------ producers (K: warp 0, V: warp 10)
        const bool is_k = warp == 0;
        uint64_t* full = is_k ? bars.k_full : bars.v_full;
        uint64_t* empty = is_k ? bars.k_empty : bars.v_empty;
        const CUtensorMap* tm = is_k ? &tmK : &tmV;
        const uint32_t ring = is_k ? sK : sV;
        const int ns = is_k ? kNS : kNSV;
        int issued = 0;
        if (lane == 0) {
            for (int t = 0; t < ntiles; ++t) {
                const int st = t % ns;
                if (t >= ns &&
                    !wait_or_abort(smem_u32(&empty[st]), ((t - ns) / ns) & 1, &s_abort, p.status, p.wait_cycles))
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
                            tma_load_2d_hint(ring + st * kKVBytes + x * kKVBox + kb * 2048, tm, 64 * x, rows[t * 8 + kb],
                                             fb, l2_evict_first());
                        else
                            tma_load_2d(ring + st * kKVBytes + x * kKVBox + kb * 2048, tm, 64 * x, rows[t * 8 + kb], fb);
                    }
            }
            // do not leave while copies into this CTA's shared memory may be in flight
            if (s_abort) {
                for (int t = max(0, issued - ns); t < issued; ++t)
                    mbar_wait_bounded(smem_u32(&full[t % ns]), (t / ns) & 1, p.wait_cycles);
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
            // S^T: A = K tile (keys x dims, K-major), B = Q (heads x dims, K-major)
            const uint32_t id_qk = idesc_f16_ab(BF16, false, false, kBN, kG);
            // O^T: A = V^T (the [key][dim] tile read MN-major), B = P^T ([key][head], MN-major)
            const uint32_t id_pv = idesc_f16_ab(BF16, true, true, kD, kG);
            const uint32_t tO = tmem + 128;
            // S^T(t) = K(t) . Q^T into buffer t % 2: 8 steps of K = 16 dims
            auto qk = [&](int t) -> bool {
                const int st = t % kNS;
                if (!wait(smem_u32(&bars.k_full[st]), (t / kNS) & 1))
                    return false;
                tc_fence_after();
                const uint32_t kbase = sK + st * kKVBytes;
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks) {
                    const uint32_t off_q = (ks >> 2) * kQBox + (ks & 3) * 32;
                    const uint32_t off_k = (ks >> 2) * kKVBox + (ks & 3) * 32;
                    umma_w(tmem + 64 * (t & 1), sdesc_k128(kbase + off_k), sdesc_k128(sQ + off_q), id_qk, ks > 0);
                }
                umma_commit_w(smem_u32(&bars.s_full[t & 1]));
                umma_commit_w(smem_u32(&bars.k_empty[st]));
                return true;
            };
            // Tensor-core order: QK(0), QK(1), then per tile t: P.V(t) and QK(t+2), QK(t+2)
            // first when its K tile has landed already (the next softmax waits on it; P.V(t)
            // first measured slower).  QK(t+2) overwrites S^T buffer t % 2 once the softmax has
            // stored P^T(t) (it read S^T(t) before); P.V(t) reads P^T from shared memory, so
            // neither has to wait for the other's copy.
            bool ok = wait(smem_u32(&bars.q_full), 0) && qk(0) && (ntiles < 2 || qk(1));
            for (int t = 0; ok && t < ntiles; ++t) {
                const int st = t % kNSV;
                if (!wait(smem_u32(&bars.p_full[t & 1]), (t >> 1) & 1)) break;
                bool qk_next = t + 2 < ntiles;
                if (qk_next) {
                    const bool landed = __shfl_sync(
                        0xffffffffu, mbar_try_wait(smem_u32(&bars.k_full[(t + 2) % kNS]), ((t + 2) / kNS) & 1) ? 1 : 0, 0);
                    if (landed) {
                        if (!qk(t + 2)) break;
                        qk_next = false;
                    }
                }
                if (!wait(smem_u32(&bars.v_full[st]), (t / kNSV) & 1)) break;
                tc_fence_after();
                const uint32_t vbase = sV + st * kKVBytes;
                const uint32_t pbase = sP + (t % kPB) * 2 * kPBytes;
                // O^T += V^T . P^T: 8 steps of K = 16 keys (2048 bytes of each operand)
#pragma unroll
                for (int ks = 0; ks < kBN / 16; ++ks) {
                    const uint64_t av = sdesc_mn128(vbase + ks * 2048, kKVBox);
                    umma_w(tO, av, sdesc_mn128(pbase + ks * 2048, kPBytes), id_pv, !(t == 0 && ks == 0));
                    if constexpr (BF16)   // low part of P
                        umma_w(tO, av, sdesc_mn128(pbase + kPBytes + ks * 2048, kPBytes), id_pv, true);
                }
                umma_commit_w(smem_u32(&bars.v_empty[st]));
                umma_commit_w(smem_u32(&bars.pv_done[t & 1]));
                if (qk_next && !qk(t + 2)) break;
            }
            umma_commit_w(smem_u32(&bars.o_done));
            // every MMA this thread issued, also on an abort, is done before TMEM is freed
            umma_commit_w(smem_u32(&bars.mma_drain));
            mbar_wait_bounded(smem_u32(&bars.mma_drain), 0, p.wait_cycles);
        }
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        // warps 2..5 take heads 0..31 of each key, warps 6..9 heads 32..63; quarter = warp % 4
        // fixes the 32 TMEM lanes (keys; dims of O^T in the epilogue) a warp may touch
        const int quarter = warp & 3;
        const int hb = warp < 6 ? 0 : kHT;           // this thread's first head
        const int sid = threadIdx.x - 64;            // 0 .. 255 over the softmax warps
        const int k = quarter * 32 + lane;           // key of the tile (= TMEM lane); dim of O^T later
        const uint32_t tL = tmem + ((uint32_t)(quarter * 32) << 16) + hb;   // lane quarter, own columns
        const uint32_t tO = tL + 128;
        const float sl = p.scale_log2;
        float l_part[kHT];                           // sum over this thread's keys of P, per head
#pragma unroll
        for (int h = 0; h < kHT; ++h) l_part[h] = 0.f;
        int meetings = 0;
        // the softmax warps meet (bounded: a warp that gave up leaves the others to time out)
        auto meet = [&]() -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bars.group));
            const bool r = __all_sync(0xffffffffu, wait_or_abort(smem_u32(&bars.group), meetings & 1, &s_abort,
                                                                  p.status, p.wait_cycles));
            ++meetings;
            return r;
        };
        auto load_scores = [&](uint32_t tS, float (&v)[kHT]) {
            tmem_ld32(tS, v);
            tmem_wait_ld();
        };
        bool ok = true;
        for (int t = 0; t < ntiles; ++t) {
            if (!__all_sync(0xffffffffu, wait_or_abort(smem_u32(&bars.s_full[t & 1]), (t >> 1) & 1, &s_abort, p.status,
                                                        p.wait_cycles))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t tS = tL + 64 * (t & 1);   // this tile's S^T buffer, own heads
            const bool valid = tok_lo + t * kBN + k < end;
            // x[h] = scale * s[h] - m[h] (log2 units); the tile needs a new max where it exceeds 8
            float x[kHT];
            load_scores(tS, x);
            float mx = -INFINITY;
#pragma unroll
            for (int h = 0; h < kHT; h += 4) {
                const float4 m4 = *reinterpret_cast<const float4*>(&s_m[hb + h]);
                const float2 a = ffma2(make_float2(x[h], x[h + 1]), make_float2(sl, sl), make_float2(-m4.x, -m4.y));
                const float2 c = ffma2(make_float2(x[h + 2], x[h + 3]), make_float2(sl, sl), make_float2(-m4.z, -m4.w));
                x[h] = a.x;
                x[h + 1] = a.y;
                x[h + 2] = c.x;
                x[h + 3] = c.y;
                mx = fmax3(mx, fmax3(a.x, a.y, c.x), c.y);
            }
            if (__any_sync(0xffffffffu, valid && !(mx <= kRescaleSlack)) && lane == 0) s_hit[t & 1] = t + 1;
            if (!meet()) {
                ok = false;
                break;
            }
            if (s_hit[t & 1] == t + 1) {
                // new per-head maxima: this tile's, over the valid keys of the four lane quarters
                load_scores(tS, x);
#pragma unroll
                for (int h = 0; h < kHT; ++h) x[h] = valid ? x[h] * sl : -INFINITY;
                warp_reduce_heads<kHT, true>(x, lane);   // lane L: head hb + L
                s_red[quarter][hb + lane] = x[0];
                if (!meet()) {
                    ok = false;
                    break;
                }
                if (sid < kG) {
                    const float tm = fmaxf(fmaxf(s_red[0][sid], s_red[1][sid]), fmaxf(s_red[2][sid], s_red[3][sid]));
                    const float mo = s_m[sid];
                    const float mn = (mo == -INFINITY || tm > mo + kRescaleSlack) ? tm : mo;
                    s_alpha[sid] = mo == -INFINITY ? 0.f : ex2(mo - mn);
                    s_m[sid] = mn;
                }
                if (!meet()) {
                    ok = false;
                    break;
                }
                bool moved = false;   // one of this warp's heads moved (the same for its lanes)
#pragma unroll
                for (int h = 0; h < kHT; ++h) {
                    const float a = s_alpha[hb + h];
                    l_part[h] *= a;
                    moved |= a != 1.f;
                }
                // rescale this thread's columns of O^T (lane = dim k) once P . V(t-1) is done;
                // P . V(t) waits for this tile's P
                if (t > 0 && moved) {
                    if (!__all_sync(0xffffffffu, wait_or_abort(smem_u32(&bars.pv_done[(t - 1) & 1]), ((t - 1) >> 1) & 1,
                                                                &s_abort, p.status, p.wait_cycles))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    float o[32];
                    tmem_ld32(tO, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] *= s_alpha[hb + i];
                    tmem_st32(tO, o);
                    tmem_wait_st();
                }
                load_scores(tS, x);
#pragma unroll
                for (int h = 0; h < kHT; ++h) x[h] = x[h] * sl - (s_m[hb + h] == -INFINITY ? 0.f : s_m[hb + h]);
            }
            // P for this thread's 32 heads, packed: for bf16 pools a high part (truncation) and a
            // low part (the truncated remainder), for fp16 pools one part (11 bits, relative
            // error <= 2^-12); keys past the end get P = 0
            uint32_t hi[kHT / 2], lo[kHT / 2];
#pragma unroll
            for (int e = 0; e < kHT / 2; ++e) {
                const float2 pp = valid ? make_float2(ex2(x[2 * e]), ex2(x[2 * e + 1])) : make_float2(0.f, 0.f);
                l_part[2 * e] += pp.x;
                l_part[2 * e + 1] += pp.y;
                if constexpr (BF16) {
                    const uint32_t u0 = __float_as_uint(pp.x), u1 = __float_as_uint(pp.y);
                    hi[e] = __byte_perm(u0, u1, 0x7632);
                    const float2 rr = fsub2(pp, make_float2(__uint_as_float(u0 & 0xffff0000u),
                                                            __uint_as_float(u1 & 0xffff0000u)));
                    lo[e] = __byte_perm(__float_as_uint(rr.x), __float_as_uint(rr.y), 0x7632);
                } else {
                    hi[e] = pack2<false>(pp.x, pp.y);
                    lo[e] = 0u;
                }
            }
            // P^T buffer t % kPB is free once P . V(t - kPB) is done
            if (t >= kPB && !__all_sync(0xffffffffu, wait_or_abort(smem_u32(&bars.pv_done[(t - kPB) & 1]),
                                                                    ((t - kPB) >> 1) & 1, &s_abort, p.status,
                                                                    p.wait_cycles))) {
                ok = false;
                break;
            }
            // this thread's part of the key's P^T row in buffer t % kPB: heads hb .. hb + 31, 8
            // (16 bytes) at a time at chunk c ^ (k % 8) of the key's 128-byte row
            const uint32_t prow = sP + (t % kPB) * 2 * kPBytes + k * 128;
#pragma unroll
            for (int cc = 0; cc < kHT / 8; ++cc) {
                const uint32_t off = (uint32_t)(((hb / 8 + cc) ^ (k & 7)) << 4);
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(prow + off), "r"(hi[4 * cc]),
                             "r"(hi[4 * cc + 1]), "r"(hi[4 * cc + 2]), "r"(hi[4 * cc + 3])
                             : "memory");
                if constexpr (BF16)
                    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(prow + kPBytes + off),
                                 "r"(lo[4 * cc]), "r"(lo[4 * cc + 1]), "r"(lo[4 * cc + 2]), "r"(lo[4 * cc + 3])
                                 : "memory");
            }
            // keys past the end in this tile: zero their V rows (P is 0 there, V may be
            // anything, NaN included); the thread of heads 0..31 zeroes dims 0..63, the other 64..127
            if (tok_lo + (t + 1) * kBN > end) {
                const int st = t % kNSV;
                if (!__all_sync(0xffffffffu, wait_or_abort(smem_u32(&bars.v_full[st]), (t / kNSV) & 1, &s_abort,
                                                            p.status, p.wait_cycles))) {
                    ok = false;
                    break;
                }
                if (!valid) {
                    const uint32_t vrow = sV + st * kKVBytes + (hb ? kKVBox : 0) + k * 128;
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(vrow + 16 * i), "r"(0u) : "memory");
                }
            }
            fence_proxy_async_smem();   // P^T (and zeroed V rows) reach the MMA through p_full
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bars.p_full[t & 1]));
        }
        if (ok && __all_sync(0xffffffffu, wait_or_abort(smem_u32(&bars.o_done), 0, &s_abort, p.status, p.wait_cycles))) {
            tc_fence_after();
            // l per head: the partial sums of the 128 key threads added up
            warp_reduce_heads<kHT, false>(l_part, lane);
            s_red[quarter][hb + lane] = l_part[0];
            const bool final_out = part_count(p, ctx) == 1 && p.part_base == 0;
            if (meet()) {
                if (sid < kG) {   // per head: 1 / l for the final row, or the partial's (m, l)
                    const float l = s_red[0][sid] + s_red[1][sid] + s_red[2][sid] + s_red[3][sid];
                    s_alpha[sid] = final_out ? 1.f / l : 1.f;
                    if (!final_out) {
                        const size_t qrow = (size_t)b * p.H_q + (size_t)g * kG + sid;
                        float2* dst = reinterpret_cast<float2*>(p.ws_ml + ws_slot(p, qrow, part) * 2);
                        if (kHintPartials) st_hint(dst, make_float2(s_m[sid], l), l2_evict_last());
                        else *dst = make_float2(s_m[sid], l);
                    }
                }
            }
            if (meet()) {
                // O^T lane k = dim k of this thread's 32 heads' output rows: 128 threads write
                // 128 consecutive floats per head
                const size_t row0 = (size_t)b * p.H_q + (size_t)g * kG + hb;
                float* base = final_out ? p.out + row0 * kD + k : p.ws_o + ws_slot(p, row0, part) * kD + k;
                const size_t stride = final_out ? (size_t)kD : (size_t)p.slots * kD;   // next head's row
                float o[32];
                tmem_ld32(tO, o);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) base[(size_t)i * stride] = o[i] * s_alpha[hb + i];
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

bool decode_tck_supported(int d, int G, int kv_dtype)
{
    return d == kD && G == kG && (kv_dtype == PKV_BF16 || kv_dtype == PKV_F16);
}

// q viewed as [B][H_q][d] with boxes of 64 dims x 64 heads x 1 sequence.
bool make_q_map_seq(CUtensorMap* map, const void* q, int B, int H_q, PFN_encode enc)
{
    const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)H_q, (cuuint64_t)B};
    const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)H_q * kD * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)kG, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(q), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int launch_decode_tck(const DecodeParams& p, int kv_dtype, const CUtensorMap* tmq, const CUtensorMap* tmk,
                      const CUtensorMap* tmv, cudaStream_t s)
{
    if (p.part_tokens > kRowsMax * kBlock) return PKV_ERR_ARG;
    auto kern = kv_dtype == PKV_BF16 ? decode_tck_kernel<true> : decode_tck_kernel<false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess)
        return PKV_ERR_CUDA;
    const dim3 grid(p.max_parts, p.H_kv, p.num_seqs);
    kern<<<grid, kThreads, kSmem, s>>>(p, *tmq, *tmk, *tmv);
    return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

}  // namespace pkv
