// decode_tc_fp8.cu -- paged_decode_attn for fp8 (e4m3) pools with 8 query heads per KV head on
// the 5th-generation tensor cores, keys on the MMA's M side, the stored codes fed to the MMA as
// they are.
//
// "LLM Inference ...", section "KV-cache quantization": the pool holds e4m3 codes with one fp32
// scale per (block, KV head), and attention uses code * scale.  Neither K nor V is converted
// here: tcgen05.mma kind::f8f6f4 multiplies e4m3 codes, and the scales, constant over a key's
// row, are applied per key (= per TMEM lane) outside the MMA:
//   S^T  = Kc . Qd^T    M = 128 keys, N = 8 heads, K = 128 dims; once per digit d of q
//   O^T += Vc^T . Pd^T  M = 128 dims (the V tile read MN-major), N = 8 heads, K = 128 keys;
//                       once per digit d of P'
// q is not an e4m3 number, so it enters as three e4m3 digits: scaled per head by a power of
// two that brings max |q| into [128, 256), q = d1 + d2 + d3 + r with d1 = e4m3(q),
// d2 = e4m3(q - d1), d3 = e4m3(q - d1 - d2); each digit carries 4 significant bits, so
// |r| <= 2^-12 |q| down to e4m3's subnormal step.  P' = p * v_scale(key) * 2^ev, with 2^ev a
// power of two for the CTA that puts the largest P' in [64, 256), enters as three digits the
// same way (the running max moves when a score exceeds it by 1, so p <= 2).  A product
// of two e4m3 numbers is exact; the tensor cores accumulate in fp32.  Then
//   score(key, h) = S^T[key][h] * k_scale(key) * 2^-eq(h) * scale,   O(h) = O^T[:, h] * 2^-ev / l(h).
//
// One CTA = (split-K partition, KV head, sequence), 128-key tiles.  Warps:
//   0      TMA producer of the K ring (3 stages of 128 keys x 128 code bytes: one 16-row box
//          per paged block, 128-byte swizzle, no multicast); 6 the same for the V ring;
//   1      allocates 32 TMEM columns (S^T of even tiles 0..7, of odd tiles 8..15, O^T
//          16..23) and issues every MMA from one elected lane: QK(0), QK(1), then per tile t
//          P.V(t) and QK(t+2), QK(t+2) first when its K tile has landed;
//   2..5   setup (q's digits, the partition's scales), then the softmax, one thread per key
//          (= TMEM lane, 8 heads), and the epilogue, one thread per dimension (= TMEM lane
//          of O^T).  The running max is per head and shared by the key threads; it moves
//          lazily (a tile with a score above max + 1, log2 units, recomputes it by a
//          reduction across the threads and rescales O^T and the partial sums).
// 108 KiB of shared memory: two CTAs per SM.  Every wait is bounded, the softmax warps'
// meetings included; a timeout sets PKV_DEV_TIMEOUT and the CTA winds down.
#include <cuda_fp8.h>

#include "decode_common.cuh"
#include "tcgen05.cuh"

namespace pkv {

namespace {

constexpr int kD = 128;                          // head dim handled here (one 128-byte code row)
constexpr int kG = 8;                            // query heads per KV head
constexpr int kBN = 128;                         // keys per tile (the MMA's M)
constexpr int kNS = 3;                           // stages of each of the K and V rings
constexpr int kDig = 3;                          // e4m3 digits of q and of P'
constexpr int kTile = kBN * kD;                  // one K (V) tile: 16 KiB of codes
constexpr int kQDig = kG * kD;                   // one digit of q: 8 heads x 128 bytes (one swizzle atom)
constexpr int kPDig = kG * kBN;                  // one digit of P'^T: 8 heads x 128 keys
constexpr int kQOff = 0;
constexpr int kKOff = kQOff + kDig * kQDig;      // 3 KiB
constexpr int kVOff = kKOff + kNS * kTile;
constexpr int kPOff = kVOff + kNS * kTile;       // P'^T digits of even / odd tiles
constexpr int kRowsMax = 4096 / 16;              // paged blocks of one partition (at most 4096 keys)
constexpr int kRowsOff = kPOff + 2 * kDig * kPDig;
constexpr int kScOff = kRowsOff + kRowsMax * 4;  // (k_scale, v_scale) per paged block
constexpr int kSmem = kScOff + kRowsMax * 8 + 1024;
static_assert(kSmem <= 110 * 1024, "two CTAs per SM");
constexpr uint32_t kTmemCols = 32;               // S^T even 0..7, odd 8..15, O^T 16..23
constexpr int kThreads = 224;                    // K producer, MMA, 4 softmax warps, V producer
// log2 units: P = 2^(s - m) stays <= 2, so that P' = P * v_scale * 2^ev can be scaled up to
// [0, 256): its three e4m3 digits then keep ~12 bits relative to the largest P' (e4m3's
// smallest step, 2^-9, would cost relative precision at P' ~ 1)
constexpr float kRescaleSlack = 1.f;

struct Fp8Bars {
    uint64_t k_full[kNS];
    uint64_t k_empty[kNS];
    uint64_t v_full[kNS];
    uint64_t v_empty[kNS];
    uint64_t s_full[2];   // S^T(t) is in buffer t % 2 (every MMA issued before it is done too)
    uint64_t p_full[2];   // P'^T(t) stored by the 4 softmax warps (and V rows past the end zeroed)
    uint64_t pv_done[2];  // P . V(t) is done, barrier t % 2 (then P'^T buffer t % 2 may be rewritten)
    uint64_t o_done;      // the last P . V is done
    uint64_t mma_drain;   // every MMA is done (before TMEM is freed)
    uint64_t group;       // meeting point of the 4 softmax warps, one phase per meeting
};

// Instruction descriptor of kind::f8f6f4: A and B e4m3, fp32 accumulation, A K-major or MN-major,
// B K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_e4m3(bool a_mn_major, int M, int N)
{
    return (1u << 4) | ((a_mn_major ? 1u : 0u) << 15) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D (TMEM) += A . B, e4m3 operands from shared memory, issued by one elected lane of the warp.
__device__ __forceinline__ void umma_e4m3_w(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, bool accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(accumulate ? 1u : 0u)
        : "memory");
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8])
{
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float (&v)[8])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
                 ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
                   "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
                   "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
                 : "memory");
}

// Two floats -> their e4m3 digits (low byte: a), and the remainders a - e4m3(a), b - e4m3(b).
__device__ __forceinline__ uint32_t e4m3_digit2(float& a, float& b)
{
    const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(c, __NV_E4M3);
    a -= __half2float(__ushort_as_half(h.x));   // exact: the digit is 0 or within a factor of 2 of a
    b -= __half2float(__ushort_as_half(h.y));
    return (uint32_t)c;
}

// Byte offset of (row r < 8, column c < 128) in a 128-byte-swizzled 8-row atom.
__device__ __forceinline__ uint32_t swz_byte(int r, int c)
{
    return (uint32_t)(r * 128 + ((((c >> 4) ^ r) & 7) << 4) + (c & 15));
}

__device__ __forceinline__ float pow2i(int e)
{
    return __int_as_float((127 + e) << 23);
}

__global__ void __launch_bounds__(kThreads, 2)
decode_tc_fp8_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV)
{
    extern __shared__ uint8_t smem_dyn[];
    __shared__ Fp8Bars bars;
    __shared__ uint32_t s_tmem_base;
    __shared__ volatile int s_abort;
    __shared__ float s_m[kG];                  // running max per head (log2 units, scale applied)
    __shared__ float s_alpha[kG];              // rescale factor of the last recomputation / 1 / l
    __shared__ float s_fq[kG];                 // scale * log2(e) * 2^-eq(h)
    __shared__ float s_red[4][kG];             // per-warp reductions
    __shared__ float s_vmax[4];                // largest V scale of the partition, per warp
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
    const int nblk = (end - tok_lo + kBlock - 1) / kBlock;   // paged blocks with keys in range

    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    const uint32_t s0 = smem_u32(smem);
    const uint32_t sQ = s0 + kQOff, sK = s0 + kKOff, sV = s0 + kVOff, sP = s0 + kPOff;
    int* rows = reinterpret_cast<int*>(smem + kRowsOff);
    float2* scl = reinterpret_cast<float2*>(smem + kScOff);

    if (threadIdx.x == 0) {
        s_abort = 0;
        s_hit[0] = 0;
        s_hit[1] = 0;
        for (int s = 0; s < kNS; ++s) {
            mbar_init(smem_u32(&bars.k_full[s]), 1);
            mbar_init(smem_u32(&bars.k_empty[s]), 1);
            mbar_init(smem_u32(&bars.v_full[s]), 1);
            mbar_init(smem_u32(&bars.v_empty[s]), 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(smem_u32(&bars.s_full[x]), 1);
            mbar_init(smem_u32(&bars.p_full[x]), 4);
            mbar_init(smem_u32(&bars.pv_done[x]), 1);
        }
        mbar_init(smem_u32(&bars.o_done), 1);
        mbar_init(smem_u32(&bars.mma_drain), 1);
        mbar_init(smem_u32(&bars.group), 4);
        mbar_fence_init();
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    if (threadIdx.x < kG) s_m[threadIdx.x] = -INFINITY;
    // TMA row and (k_scale, v_scale) of every paged block of the partition; block 0 (in bounds,
    // scales 0) past the partition's end, where the keys are masked and the V rows zeroed
    for (int i = threadIdx.x; i < ntiles * (kBN / kBlock); i += kThreads) {
        int blk = 0;
        float2 sc = make_float2(0.f, 0.f);
        if (i < nblk) {
            blk = p.tables[(size_t)b * p.W + tok_lo / kBlock + i];
            if ((unsigned)blk >= (unsigned)p.N) {
                flag_status(p.status, PKV_DEV_BAD_BLOCK);
                blk = 0;
            }
            const size_t si = (size_t)blk * p.H_kv + g;
            sc = make_float2(p.k_scale[si], p.v_scale[si]);
        }
        rows[i] = (blk * p.H_kv + g) * kBlock;
        scl[i] = sc;
    }
    if (warp >= 2 && warp < 6) {
        // q's digits: thread i of the 128 takes head i / 16, dims 8 (i % 16) .. + 7
        const int i = threadIdx.x - 64, h = i >> 4, d0 = (i & 15) * 8;
        const uint16_t* qh = static_cast<const uint16_t*>(p.q) + ((size_t)b * p.H_q + (size_t)g * kG + h) * kD + d0;
        const uint4 raw = *reinterpret_cast<const uint4*>(qh);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
        float q[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = p.q_bf16 ? unpack2<true>(w[j]) : unpack2<false>(w[j]);
            q[2 * j] = f.x;
            q[2 * j + 1] = f.y;
        }
        float amax = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(q[j]));
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        // 2^eq brings max |q| into [128, 256); eq in [-100, 100] keeps every factor finite
        const int ex = (int)((__float_as_uint(amax) >> 23) & 0xffu) - 127;
        const int eq = amax > 0.f ? max(-100, min(100, 7 - ex)) : 0;
        const float up = pow2i(eq);
#pragma unroll
        for (int j = 0; j < 8; ++j) q[j] *= up;
        if ((i & 15) == 0) s_fq[h] = p.scale_log2 * pow2i(-eq);
#pragma unroll
        for (int dg = 0; dg < kDig; ++dg) {
            uint32_t lo = 0, hi = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t c = e4m3_digit2(q[2 * j], q[2 * j + 1]);
                if (j < 2) lo |= c << (16 * j);
                else hi |= c << (16 * (j - 2));
            }
            const uint32_t a = sQ + dg * kQDig + swz_byte(h, d0);
            asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(a), "r"(lo), "r"(hi) : "memory");
        }
        fence_proxy_async_smem();   // the digits are read by the tensor cores
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

    if ((warp == 0 || warp == 6) && lane != 0) {
        // the producers' other lanes only meet the CTA at the end
    } else if (warp == 0 || warp == 6) {
        // ------------------------------------------------------------ producers (K: warp 0, V: warp 6)
        const bool is_k = warp == 0;
        uint64_t* full = is_k ? bars.k_full : bars.v_full;
        uint64_t* empty = is_k ? bars.k_empty : bars.v_empty;
        const CUtensorMap* tm = is_k ? &tmK : &tmV;
        const uint32_t ring = is_k ? sK : sV;
        int issued = 0;
        for (int t = 0; t < ntiles; ++t) {
            const int st = t % kNS;
            if (t >= kNS &&
                !wait_or_abort(smem_u32(&empty[st]), ((t - kNS) / kNS) & 1, &s_abort, p.status, p.wait_cycles))
                break;
            const uint32_t fb = smem_u32(&full[st]);
            mbar_arrive_expect_tx(fb, kTile);
            issued = t + 1;
            if (is_k && t == p.hold_tile) continue;   // test hook: the withheld tile's K bytes never arrive
#pragma unroll
            for (int kb = 0; kb < kBN / kBlock; ++kb) {
                const uint32_t dst = ring + st * kTile + kb * (kBlock * kD);
                if constexpr (kHintKV) tma_load_2d_hint(dst, tm, 0, rows[t * 8 + kb], fb, l2_evict_first());
                else tma_load_2d(dst, tm, 0, rows[t * 8 + kb], fb);
            }
        }
        // do not leave while copies into this CTA's shared memory may be in flight
        if (s_abort) {
            for (int t = max(0, issued - kNS); t < issued; ++t)
                mbar_wait_bounded(smem_u32(&full[t % kNS]), (t / kNS) & 1, p.wait_cycles);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        {
            auto wait = [&](uint32_t bar, uint32_t parity) {
                return __all_sync(0xffffffffu, wait_or_abort(bar, parity, &s_abort, p.status, p.wait_cycles));
            };
            // S^T: A = K codes (keys x dims, K-major), B = a digit of q (heads x dims, K-major)
            const uint32_t id_qk = idesc_e4m3(false, kBN, kG);
            // O^T: A = V^T (the [key][dim] code tile read MN-major), B = a digit of P'^T (heads x keys, K-major)
            const uint32_t id_pv = idesc_e4m3(true, kD, kG);
            const uint32_t tO = tmem + 16;
            // S^T(t) = K(t) . (d1 + d2 + d3)^T into buffer t % 2: per digit 4 steps of K = 32 dims
            auto qk = [&](int t) -> bool {
                const int st = t % kNS;
                if (!wait(smem_u32(&bars.k_full[st]), (t / kNS) & 1))
                    return false;
                tc_fence_after();
                const uint32_t kbase = sK + st * kTile;
#pragma unroll
                for (int dg = 0; dg < kDig; ++dg)
#pragma unroll
                    for (int ks = 0; ks < kD / 32; ++ks)
                        umma_e4m3_w(tmem + 8 * (t & 1), sdesc_k128(kbase + 32 * ks), sdesc_k128(sQ + dg * kQDig + 32 * ks),
                                    id_qk, dg > 0 || ks > 0);
                umma_commit_w(smem_u32(&bars.s_full[t & 1]));
                umma_commit_w(smem_u32(&bars.k_empty[st]));
                return true;
            };
            bool ok = qk(0) && (ntiles < 2 || qk(1));
            for (int t = 0; ok && t < ntiles; ++t) {
                const int st = t % kNS;
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
                if (!wait(smem_u32(&bars.v_full[st]), (t / kNS) & 1)) break;
                tc_fence_after();
                const uint32_t vbase = sV + st * kTile;
                const uint32_t pbase = sP + (t & 1) * kDig * kPDig;
                // O^T += V^T . (d1 + d2 + d3)^T: per digit 4 steps of K = 32 keys (32 code rows)
#pragma unroll
                for (int dg = 0; dg < kDig; ++dg)
#pragma unroll
                    for (int ks = 0; ks < kBN / 32; ++ks)
                        umma_e4m3_w(tO, sdesc_mn128(vbase + ks * 4096, kTile), sdesc_k128(pbase + dg * kPDig + 32 * ks),
                                    id_pv, !(t == 0 && dg == 0 && ks == 0));
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
        const int quarter = warp & 3;
        const int k = quarter * 32 + lane;           // key of the tile (= TMEM lane); dim of O^T later
        const uint32_t tL = tmem + ((uint32_t)(quarter * 32) << 16);
        const uint32_t tO = tL + 16;
        // 2^ev keeps P' = p * v_scale * 2^ev <= 256 (p <= 2^8 under the lazy max)
        float vm = 0.f;
        for (int j = k; j < nblk; j += 128) vm = fmaxf(vm, scl[j].y);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) vm = fmaxf(vm, __shfl_xor_sync(0xffffffffu, vm, o));
        if (lane == 0) s_vmax[quarter] = vm;
        float fq[kG];
#pragma unroll
        for (int h = 0; h < kG; ++h) fq[h] = s_fq[h];
        float l_part[kG];
#pragma unroll
        for (int h = 0; h < kG; ++h) l_part[h] = 0.f;
        int meetings = 0;
        auto meet = [&]() -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bars.group));
            const bool r = __all_sync(0xffffffffu, wait_or_abort(smem_u32(&bars.group), meetings & 1, &s_abort,
                                                                  p.status, p.wait_cycles));
            ++meetings;
            return r;
        };
        bool ok = meet();
        // 2^ev: the largest V scale times 2^ev lies in [64, 128), so P' < 256 (e4m3 reaches 448)
        const float vmax = fmaxf(fmaxf(s_vmax[0], s_vmax[1]), fmaxf(s_vmax[2], s_vmax[3]));
        const int ev_exp = (int)((__float_as_uint(vmax) >> 23) & 0xffu) - 127;   // vmax in [2^e, 2^(e+1))
        const int ev = vmax > 0.f ? max(-100, min(100, 6 - ev_exp)) : 0;
        const float vup = pow2i(ev);
        for (int t = 0; ok && t < ntiles; ++t) {
            if (!__all_sync(0xffffffffu, wait_or_abort(smem_u32(&bars.s_full[t & 1]), (t >> 1) & 1, &s_abort, p.status,
                                                        p.wait_cycles))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t tS = tL + 8 * (t & 1);
            const int key = tok_lo + t * kBN + k;
            const bool valid = key < end;
            const float2 sc = scl[t * 8 + (k >> 4)];   // this key's block: (k_scale, v_scale)
            float x[kG];
            tmem_ld8(tS, x);
            tmem_wait_ld();
            float mx = -INFINITY;
#pragma unroll
            for (int h = 0; h < kG; ++h) {
                x[h] = x[h] * (sc.x * fq[h]) - s_m[h];
                mx = fmaxf(mx, x[h]);
            }
            if (__any_sync(0xffffffffu, valid && !(mx <= kRescaleSlack)) && lane == 0) s_hit[t & 1] = t + 1;
            if (!meet()) {
                ok = false;
                break;
            }
            if (s_hit[t & 1] == t + 1) {
                // new per-head maxima: this tile's, over the valid keys of the four warps
                tmem_ld8(tS, x);
                tmem_wait_ld();
#pragma unroll
                for (int h = 0; h < kG; ++h) {
                    float v = valid ? x[h] * (sc.x * fq[h]) : -INFINITY;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
                    if (lane == h) s_red[quarter][h] = v;
                }
                if (!meet()) {
                    ok = false;
                    break;
                }
                if (k < kG) {
                    const float tm = fmaxf(fmaxf(s_red[0][k], s_red[1][k]), fmaxf(s_red[2][k], s_red[3][k]));
                    const float mo = s_m[k];
                    const float mn = (mo == -INFINITY || tm > mo + kRescaleSlack) ? tm : mo;
                    s_alpha[k] = mo == -INFINITY ? 0.f : ex2(mo - mn);
                    s_m[k] = mn;
                }
                if (!meet()) {
                    ok = false;
                    break;
                }
                bool moved = false;
                float al[kG];
#pragma unroll
                for (int h = 0; h < kG; ++h) {
                    al[h] = s_alpha[h];
                    l_part[h] *= al[h];
                    moved |= al[h] != 1.f;
                }
                // rescale O^T (lane = dim k, one column per head) once P . V(t-1) is done
                if (t > 0 && moved) {
                    if (!__all_sync(0xffffffffu, wait_or_abort(smem_u32(&bars.pv_done[(t - 1) & 1]), ((t - 1) >> 1) & 1,
                                                                &s_abort, p.status, p.wait_cycles))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    float o[8];
                    tmem_ld8(tO, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int h = 0; h < kG; ++h) o[h] *= al[h];
                    tmem_st8(tO, o);
                    tmem_wait_st();
                }
                tmem_ld8(tS, x);
                tmem_wait_ld();
#pragma unroll
                for (int h = 0; h < kG; ++h) x[h] = x[h] * (sc.x * fq[h]) - (s_m[h] == -INFINITY ? 0.f : s_m[h]);
            }
            // P' = 2^x * v_scale * 2^ev (keys past the end: 0) as three e4m3 digits
            const float vs = sc.y * vup;
            float pp[kG];
#pragma unroll
            for (int h = 0; h < kG; ++h) {
                const float e = valid ? ex2(x[h]) : 0.f;
                l_part[h] += e;
                pp[h] = e * vs;
            }
            uint32_t dig[kDig][kG / 2];
#pragma unroll
            for (int dg = 0; dg < kDig; ++dg)
#pragma unroll
                for (int j = 0; j < kG / 2; ++j) dig[dg][j] = e4m3_digit2(pp[2 * j], pp[2 * j + 1]);
            // P'^T buffer t % 2 is free once P . V(t - 2) is done
            if (t >= 2 && !__all_sync(0xffffffffu, wait_or_abort(smem_u32(&bars.pv_done[t & 1]), ((t - 2) >> 1) & 1,
                                                                  &s_abort, p.status, p.wait_cycles))) {
                ok = false;
                break;
            }
            // digit dg, head h, key k: byte (h, k) of the digit's 8-row, 128-byte swizzled atom
            const uint32_t pbase = sP + (t & 1) * kDig * kPDig;
#pragma unroll
            for (int dg = 0; dg < kDig; ++dg)
#pragma unroll
                for (int h = 0; h < kG; ++h) {
                    const uint32_t byte = (dig[dg][h >> 1] >> (8 * (h & 1))) & 0xffu;
                    asm volatile("st.shared.u8 [%0], %1;" ::"r"(pbase + dg * kPDig + swz_byte(h, k)), "r"(byte) : "memory");
                }
            // keys past the end in this tile: zero their V code rows (P' is 0 there, a code may
            // be NaN)
            if (tok_lo + (t + 1) * kBN > end) {
                const int st = t % kNS;
                if (!__all_sync(0xffffffffu, wait_or_abort(smem_u32(&bars.v_full[st]), (t / kNS) & 1, &s_abort,
                                                            p.status, p.wait_cycles))) {
                    ok = false;
                    break;
                }
                if (!valid) {
                    const uint32_t vrow = sV + st * kTile + k * 128;
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(vrow + 16 * i), "r"(0u) : "memory");
                }
            }
            fence_proxy_async_smem();   // the digits (and zeroed V rows) reach the MMA through p_full
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bars.p_full[t & 1]));
        }
        if (ok && __all_sync(0xffffffffu, wait_or_abort(smem_u32(&bars.o_done), 0, &s_abort, p.status, p.wait_cycles))) {
            tc_fence_after();
            // l per head: the partial sums of the 128 key threads added up
#pragma unroll
            for (int h = 0; h < kG; ++h) {
                float v = l_part[h];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == h) s_red[quarter][h] = v;
            }
            const bool final_out = part_count(p, ctx) == 1 && p.part_base == 0;
            if (meet()) {
                if (k < kG) {   // per head: 2^-ev / l for the final row, 2^-ev and the partial's (m, l) otherwise
                    const float l = s_red[0][k] + s_red[1][k] + s_red[2][k] + s_red[3][k];
                    s_alpha[k] = final_out ? pow2i(-ev) / l : pow2i(-ev);
                    if (!final_out) {
                        const size_t qrow = (size_t)b * p.H_q + (size_t)g * kG + k;
                        float2* dst = reinterpret_cast<float2*>(p.ws_ml + ws_slot(p, qrow, part) * 2);
                        if (kHintPartials) st_hint(dst, make_float2(s_m[k], l), l2_evict_last());
                        else *dst = make_float2(s_m[k], l);
                    }
                }
            }
            if (meet()) {
                // O^T lane k = dim k of every head's output row
                const size_t row0 = (size_t)b * p.H_q + (size_t)g * kG;
                float* base = final_out ? p.out + row0 * kD + k : p.ws_o + ws_slot(p, row0, part) * kD + k;
                const size_t stride = final_out ? (size_t)kD : (size_t)p.slots * kD;
                float o[8];
                tmem_ld8(tO, o);
                tmem_wait_ld();
#pragma unroll
                for (int h = 0; h < kG; ++h) base[(size_t)h * stride] = o[h] * s_alpha[h];
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

bool decode_tc_fp8_supported(int d, int G, int kv_dtype)
{
    return d == kD && G == kG && kv_dtype == PKV_FP8E4M3;
}

int launch_decode_tc_fp8(const DecodeParams& p, const CUtensorMap* tmk, const CUtensorMap* tmv, cudaStream_t s)
{
    if (p.part_tokens > kRowsMax * kBlock) return PKV_ERR_ARG;
    auto kern = decode_tc_fp8_kernel;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess)
        return PKV_ERR_CUDA;
    const dim3 grid(p.max_parts, p.H_kv, p.num_seqs);
    kern<<<grid, kThreads, kSmem, s>>>(p, *tmk, *tmv);
    return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

}  // namespace pkv
