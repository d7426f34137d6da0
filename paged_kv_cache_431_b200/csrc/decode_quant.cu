// decode_quant.cu -- paged_decode_attn over quantized pools (int8, fp8 e4m3, int4).
//
// Inference guide a2-inf-2, section "KV-cache quantization": keys and values stored as
// 8- or 4-bit codes sharing one scale; "KV cache, continuous batching and paged
// attention", section "The KV cache": an fp8 or int8 cache.  Here every (block, KV
// head) tile carries one fp32 scale for K and one for V, and a value is code * scale.
//
// Same structure as the 16-bit kernel (one warp per partition x KV head x sequence,
// TMA ring of K/V code tiles, online softmax, split-K partials), with dequantization
// fused into the fragment loads:
//   * int8 K codes go to the signed 8-bit mma.sync m16n8k32 as they are (exact int32
//     sums), against q split into two signed 8-bit digits per element (q scaled per query
//     head by a power of two and rounded);
//   * the other codes are converted to fp16 in registers and fed to mma.sync m16n8k16 (f16
//     in, fp32 accumulate); q is scaled by a power of two chosen per CTA (its largest |q|
//     brought near 2^14, exact, undone in the score) and converted to fp16 once per warp,
//     so a bf16 q keeps its range:
//       - int4 K codes: the code plus its offset (c + 8) is moved into the significand of
//         an fp16 subnormal (one logic op per pair, exact); the offset's share of every
//         score, 8 * sum(q), is subtracted once per score, and q is pre-scaled by a power
//         of two so that its products with the subnormals stay well inside the
//         accumulator's range;
//       - integer V codes: the exponent trick (code + offset placed in the significand of
//         1024.0, then 1024 + offset subtracted: exact) -- V meets the two-part P, whose
//         low part times a subnormal loses precision in the tensor cores;
//       - fp8 e4m3: the hardware e4m3x2 -> f16x2 conversion (exact);
//   * the K scale of a tile multiplies that tile's scores, the V scale multiplies P
//     before P . V, so the MMAs see plain integer-valued or fp8-valued operands;
//   * which physical head dims feed which MMA k-slot is chosen so that every lane
//     reads contiguous code bytes (a dot product does not depend on the order of its
//     terms); q's fragments use the same assignment.  Output dims are mapped back in
//     the epilogue.
#include <cuda_fp8.h>

#include "decode_common.cuh"

namespace pkv {

namespace {

template <int DT, int D>
struct QCfg {
    static constexpr int ROW = DT == PKV_INT4 ? D / 2 : D;     // bytes per token row
    static constexpr int TILE = 16 * ROW;                      // one (block, head) tile
    static constexpr int STAGE = 2 * TILE;                     // K and V
    static constexpr int STAGES = DT == PKV_INT4 ? 3 : 2;
    static constexpr int RING = STAGES * STAGE;
    static constexpr int STAGING = 16 * (D + 4) * 4;           // epilogue: 16 O rows, fp32
    static constexpr int BODY = RING > STAGING ? RING : STAGING;   // the epilogue reuses the ring
    static constexpr int SWZ = ROW == 128 ? 7 : ROW == 64 ? 3 : 1;   // TMA 128/64/32-byte swizzle
    static constexpr int KRUN = ROW / 4;                       // K bytes per lane per token
    static constexpr int VRUN = ROW / 8;                       // V bytes per lane per row
    static constexpr int KS = D / 16;                          // MMA k-steps of Q.K^T
    static constexpr int MT = D / 16;                          // MMA m-tiles of O^T
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
};

// Address of byte `off` (< ROW) of row `t` of a tile written by TMA with the swizzle that
// XORs the 16-byte chunk index with address bits 7.. of the row start.
template <int ROW, int SWZ>
__device__ __forceinline__ uint32_t qaddr(uint32_t tile, int t, int off)
{
    const int base = t * ROW;
    return tile + (uint32_t)(base + ((((off >> 4) ^ ((base >> 7) & SWZ)) << 4) | (off & 15)));
}

template <int N>
__device__ __forceinline__ void lds_words(uint32_t (&w)[N], uint32_t addr);

template <>
__device__ __forceinline__ void lds_words<4>(uint32_t (&w)[4], uint32_t addr)
{
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(addr));
}
template <>
__device__ __forceinline__ void lds_words<2>(uint32_t (&w)[2], uint32_t addr)
{
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w[0]), "=r"(w[1]) : "r"(addr));
}
template <>
__device__ __forceinline__ void lds_words<1>(uint32_t (&w)[1], uint32_t addr)
{
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w[0]) : "r"(addr));
}

// `bytes` code bytes from row t at byte `off` (16-byte pieces are swizzled separately).
template <int ROW, int SWZ, int BYTES>
__device__ __forceinline__ void load_run(uint32_t (&w)[BYTES / 4], uint32_t tile, int t, int off)
{
    if constexpr (BYTES >= 16) {
#pragma unroll
        for (int c = 0; c < BYTES / 16; ++c) {
            uint32_t q[4];
            lds_words<4>(q, qaddr<ROW, SWZ>(tile, t, off + 16 * c));
#pragma unroll
            for (int i = 0; i < 4; ++i) w[4 * c + i] = q[i];
        }
    } else {
        lds_words<BYTES / 4>(w, qaddr<ROW, SWZ>(tile, t, off));
    }
}

// int4 K codes become fp16 SUBNORMALS: a half whose exponent field is 0 and whose
// significand field holds the integer u has the value u * 2^-24, exactly.  So a K code needs
// only to be moved into the low bits of a half; the offset that makes it non-negative
// (u = c + 8) is removed once per score (see the kernel) instead of once per element.
//
// 2^e as a float, e in [-126, 127].
__device__ __forceinline__ float pow2f(int e)
{
    return __int_as_float((127 + e) << 23);
}

// Shift e in [-100, 100] that brings x > 0 into [2^13, 2^14) as x * 2^e (100 for x = 0 or a
// subnormal x).  The bound keeps 2^e, 2^-e and 2^(24 - e) finite floats; it covers every
// |q| below 2^114.
__device__ __forceinline__ int pow2_shift(float x)
{
    const int ex = (int)((__float_as_uint(x) >> 23) & 0xffu) - 127;   // x in [2^ex, 2^(ex+1)) if normal
    return max(-100, min(100, 13 - ex));
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// int4 codes as stored (two's complement nibbles): nibble s (0..3) of each 16-bit half
// -> two halves.  Even nibbles land in bits 0..3 (u * 2^-24), odd nibbles stay in bits
// 4..7 (16 u * 2^-24); the XOR that turns c into u = c + 8 rides in the same logic op.
__device__ __forceinline__ uint32_t u4x2(uint32_t w, int s)
{
    const uint32_t x = (s & 2) ? (w >> 8) : w;
    return (s & 1) ? ((x & 0x00f000f0u) ^ 0x00800080u) : ((x & 0x000f000fu) ^ 0x00080008u);
}

__device__ __forceinline__ uint32_t h2_sub(uint32_t a, float c)
{
    __half2 r = __hsub2(*reinterpret_cast<__half2*>(&a), __float2half2_rn(c));
    return *reinterpret_cast<uint32_t*>(&r);
}

__device__ __forceinline__ uint32_t h2_fma(uint32_t a, float m, float c)
{
    __half2 r = __hfma2(*reinterpret_cast<__half2*>(&a), __float2half2_rn(m), __float2half2_rn(c));
    return *reinterpret_cast<uint32_t*>(&r);
}

// V codes become NORMAL fp16 integers c: 0x64XX is 1024 + XX, minus 1024 + the offset
// (exact).  P . V keeps these: P is split into two fp16 parts, and the low part's
// products with subnormal V codes were measured to lose precision in the tensor cores.
__device__ __forceinline__ uint32_t i8x2(uint32_t wx, uint32_t sel)
{
    return h2_sub(__byte_perm(wx, 0x64646464u, sel), 1152.f);
}

__device__ __forceinline__ uint32_t i4x2(uint32_t w, int s)
{
    const uint32_t x = (s & 2) ? (w >> 8) : w;
    if (s & 1) return h2_fma(((x & 0x00f000f0u) ^ 0x00800080u) | 0x64006400u, 0.0625f, -72.f);
    return h2_sub(((x & 0x000f000fu) ^ 0x00080008u) | 0x64006400u, 1032.f);
}

// e4m3 pair (low byte -> low half) -> fp16 pair.
__device__ __forceinline__ uint32_t e4m3x2(uint32_t w16)
{
    __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w16 & 0xffffu), __NV_E4M3);
    return (uint32_t)h.x | ((uint32_t)h.y << 16);
}

// D += A * B, m16n8k32, signed 8-bit A (row-major, 4 regs) and B (column-major, 2 regs), int32
// accumulate (exact).
__device__ __forceinline__ void mma_s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
                 "{%0, %1, %2, %3};"
                 : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Physical head dim that feeds MMA k-slot e (0..3: logical 2qd, 2qd+1, 2qd+8, 2qd+9)
// of k-step ks for lane group qd.
template <int DT, int D>
__device__ __forceinline__ int kdim(int ks, int qd, int e)
{
    using C = QCfg<DT, D>;
    if constexpr (DT == PKV_INT4) {
        const int i = (ks & 1) * 2 + (e >> 1) + (e & 1) * 4;   // nibble of the word
        return qd * 2 * C::KRUN + 8 * (ks >> 1) + i;
    } else {
        return qd * C::KRUN + 4 * ks + e;
    }
}

// B fragment (K^T) of k-step ks from the lane's K code run.
template <int DT, int NW>
__device__ __forceinline__ void kfrag(const uint32_t (&kw)[NW], int ks, uint32_t& b0, uint32_t& b1)
{
    static_assert(DT != PKV_INT8, "int8 K codes go to the 8-bit MMA unconverted");
    if constexpr (DT == PKV_FP8E4M3) {
        b0 = e4m3x2(kw[ks]);
        b1 = e4m3x2(kw[ks] >> 16);
    } else {
        b0 = u4x2(kw[ks >> 1], (ks & 1) * 2);
        b1 = u4x2(kw[ks >> 1], (ks & 1) * 2 + 1);
    }
}

// A fragments (V^T) for the m-tiles one word of the lane's V run covers.  ab / cd are
// the words of token rows (2qd, 2qd+1) and (2qd+8, 2qd+9); va[j] gets m-tile j of the word.
template <int DT>
__device__ __forceinline__ void vfrags(uint32_t a, uint32_t b, uint32_t c, uint32_t d, uint32_t (&va)[4][4])
{
    if constexpr (DT == PKV_INT4) {
        const uint32_t ab0 = __byte_perm(a, b, 0x5410), ab1 = __byte_perm(a, b, 0x7632);
        const uint32_t cd0 = __byte_perm(c, d, 0x5410), cd1 = __byte_perm(c, d, 0x7632);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t ab = j < 2 ? ab0 : ab1, cd = j < 2 ? cd0 : cd1;
            const int s = (j & 1) * 2;
            va[j][0] = i4x2(ab, s);
            va[j][1] = i4x2(ab, s + 1);
            va[j][2] = i4x2(cd, s);
            va[j][3] = i4x2(cd, s + 1);
        }
    } else {
        const uint32_t ab_lo = __byte_perm(a, b, 0x5140), ab_hi = __byte_perm(a, b, 0x7362);
        const uint32_t cd_lo = __byte_perm(c, d, 0x5140), cd_hi = __byte_perm(c, d, 0x7362);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const uint32_t ab = j ? ab_hi : ab_lo, cd = j ? cd_hi : cd_lo;
            if constexpr (DT == PKV_INT8) {
                va[j][0] = i8x2(ab ^ 0x80808080u, 0x4140);
                va[j][1] = i8x2(ab ^ 0x80808080u, 0x4342);
                va[j][2] = i8x2(cd ^ 0x80808080u, 0x4140);
                va[j][3] = i8x2(cd ^ 0x80808080u, 0x4342);
            } else {
                va[j][0] = e4m3x2(ab);
                va[j][1] = e4m3x2(ab >> 16);
                va[j][2] = e4m3x2(cd);
                va[j][3] = e4m3x2(cd >> 16);
            }
        }
    }
}

template <int DT, int D, int NHT>
__global__ void __launch_bounds__(32)
decode_mmaq_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV)
{
    using Cfg = QCfg<DT, D>;
    constexpr int STAGES = Cfg::STAGES;
    constexpr int ROW = Cfg::ROW, SWZ = Cfg::SWZ;
    // int4 K codes enter Q . K^T as subnormals u * 2^-24 with u = c + OFF; odd nibbles enter
    // as 16 u, and their q is pre-divided by 16.  q is pre-scaled by a power of two chosen
    // per CTA (largest |q| brought near 2^14): for int4 the products then stay well clear of
    // the bottom of the accumulator's range, and for fp8 a bf16 q of any magnitude up to
    // 2^113 fits fp16 (a bf16 q above 65504 would otherwise become inf).  The scaling is
    // exact and is undone, with the offset, in the score.
    constexpr bool SUBN = DT == PKV_INT4;
    // int8 K codes enter Q . K^T as they are, through the signed 8-bit MMA (m16n8k32, exact
    // int32 sums): q times 2^e_h, a power of two chosen per query head h (its largest |q|
    // brought to [2^13, 2^14)), is rounded to an integer Q and split into two signed 8-bit
    // digits, Q = 256 d1 + d0 with d0 in [-128, 127] and |d1| <= 64, each with its own
    // accumulator; the score is (256 acc1 + acc0) * 2^-e_h (the int32 sum is exact).  A scale
    // per head keeps a head with small q as precise as one with large q.
    constexpr bool KI8 = DT == PKV_INT8;
    // L2 hints (evict_first on the K/V stream, evict_last on the partials): measured faster for
    // int8 (475 -> 468 us per long-context call) and equal for fp8, but slower for int4 (527 ->
    // 549 us), which keeps the default policy
    constexpr bool HINT = kHintKV && DT != PKV_INT4, HINTP = kHintPartials && DT != PKV_INT4;
    constexpr float OFF = 8.f;                               // int4 code offset
    constexpr float ODD = DT == PKV_INT4 ? 0.0625f : 1.f;   // q factor on k-slots 8..15
    extern __shared__ uint8_t smem_dyn[];
    __shared__ __align__(8) uint64_t bars[STAGES];

    pdl_launch_dependents();   // the split-K merge may be scheduled behind the last wave
    const int lane = threadIdx.x;
    const int part = blockIdx.x, b = blockIdx.z;
    const int g = blockIdx.y / p.hgroups, hg = blockIdx.y - g * p.hgroups;   // KV head, group of 16 heads
    const int GC = min(16, p.G - 16 * hg);                                   // query heads of this CTA
    const int r = lane >> 2, qd = lane & 3;
    const int hbase = g * p.G + 16 * hg;

    const int ctx = checked_ctx(p, b, lane == 0 && part == 0 && g == 0);
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

    // dynamic shared memory: [K/V ring, reused by the epilogue][(K scale, V scale) per
    // tile][block id per tile]
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
    float2* tsc = reinterpret_cast<float2*>(smem + Cfg::BODY);
    int* tbl = reinterpret_cast<int*>(tsc + p.part_tokens / kBlock);
    const int32_t* trow = p.tables + (size_t)b * p.W + tok0 / kBlock;
    for (int j = lane; j < ntiles; j += 32) {
        int blk = trow[j];
        if ((unsigned)blk >= (unsigned)p.N) {
            flag_status(p.status, PKV_DEV_BAD_BLOCK);
            blk = 0;
        }
        tbl[j] = blk;
        const size_t si = (size_t)blk * p.H_kv + g;
        tsc[j] = make_float2(p.k_scale[si], p.v_scale[si]);
    }
    if (lane == 0) {
        for (int s = 0; s < STAGES; ++s) mbar_init(smem_u32(&bars[s]), 1);
        mbar_fence_init();
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    __syncwarp();

    auto issue = [&](int j) {
        const int s = j % STAGES;
        const uint32_t bar = smem_u32(&bars[s]);
        const uint32_t kdst = smem_u32(smem + s * Cfg::STAGE);
        const int row = (tbl[j] * p.H_kv + g) * kBlock;
        mbar_arrive_expect_tx(bar, Cfg::STAGE);
        if (j == p.hold_tile) return;   // test hook: the stage's bytes never arrive
        if constexpr (HINT) {   // the K/V stream is read once: first out of L2
            const uint64_t pol = l2_evict_first();
            tma_load_2d_hint(kdst, &tmK, 0, row, bar, pol);
            tma_load_2d_hint(kdst + Cfg::TILE, &tmV, 0, row, bar, pol);
        } else {
            tma_load_2d(kdst, &tmK, 0, row, bar);
            tma_load_2d(kdst + Cfg::TILE, &tmV, 0, row, bar);
        }
    };
    if (lane == 0) {
        for (int j = 0; j < min(STAGES, ntiles); ++j) issue(j);
    }

    // q as fp16 A fragments (int4, fp8), k-slots assigned to physical dims by kdim(); for
    // int4 also -OFF * (sum of the fragments' q over d, odd slots counted times 16) per head
    // row r, r + 8: the part of 2^24 * (q . k) that the code offset adds
    uint32_t qa[KI8 ? 1 : Cfg::KS][4];
    // int8: MMA k-slot (ks, half, j) of lane group qd holds head dim qd * (D/4) + 8 ks + 4 half
    // + j, so every lane's B fragments are D/4 contiguous code bytes of a K row
    constexpr int KS8 = D / 32;
    uint32_t qa8[KI8 ? 2 : 1][KI8 ? KS8 : 1][4];
    float qoff[2] = {0.f, 0.f};
    int eq = 0;   // q is multiplied by 2^eq, which brings max |q| to [2^13, 2^14)
    int eqr[2] = {0, 0};   // int8: the same per query row (rows r and r + 8)
    {
        const bool bf = p.q_bf16;
        const uint16_t* qh = static_cast<const uint16_t*>(p.q) + ((size_t)b * p.H_q + hbase) * D;
        auto qv = [&](int row, int dim) -> float {
            const uint16_t u = __ldg(qh + row * D + dim);
            return bf ? __uint_as_float((uint32_t)u << 16) : __half2float(__ushort_as_half(u));
        };
        const bool r0 = r < GC, r1 = (NHT == 2) && (r + 8 < GC);
        float qmax = 0.f;
        for (int i = lane; i < GC * D; i += 32) qmax = fmaxf(qmax, fabsf(qv(0, i)));
        eq = pow2_shift(warp_max(qmax));
        const float qs = pow2f(eq), qo = qs * ODD;
        if constexpr (KI8) {
            // the largest |q| of rows r and r + 8: this lane's share of their dims, then the quad's
            float rm[2] = {0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < KS8; ++ks)
#pragma unroll
                for (int reg = 0; reg < 4; ++reg) {
                    const int row = r + 8 * (reg & 1);
                    const bool live = (reg & 1) ? (NHT == 2 && r + 8 < GC) : (r < GC);
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj)
                        if (live) rm[reg & 1] = fmaxf(rm[reg & 1], fabsf(qv(row, qd * (D / 4) + 8 * ks + 4 * (reg >> 1) + jj)));
                }
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                rm[hr] = fmaxf(rm[hr], __shfl_xor_sync(0xffffffffu, rm[hr], 1));
                rm[hr] = fmaxf(rm[hr], __shfl_xor_sync(0xffffffffu, rm[hr], 2));
                eqr[hr] = pow2_shift(rm[hr]);
            }
#pragma unroll
            for (int ks = 0; ks < KS8; ++ks)
#pragma unroll
                for (int reg = 0; reg < 4; ++reg) {   // a0: row r, dims +0; a1: r+8, +0; a2: r, +4; a3: r+8, +4
                    const int row = r + 8 * (reg & 1);
                    const bool live = (reg & 1) ? (NHT == 2 && r + 8 < GC) : (r < GC);
                    uint32_t w0 = 0u, w1 = 0u;
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const int Q = live ? __float2int_rn(qv(row, qd * (D / 4) + 8 * ks + 4 * (reg >> 1) + jj) *
                                                            pow2f(eqr[reg & 1]))
                                           : 0;
                        const int d1 = (Q + 128) >> 8;
                        w1 |= (uint32_t)(d1 & 0xff) << (8 * jj);
                        w0 |= (uint32_t)((Q - 256 * d1) & 0xff) << (8 * jj);
                    }
                    qa8[0][ks][reg] = w0;
                    qa8[1][ks][reg] = w1;
                }
        }
#pragma unroll
        for (int ks = 0; ks < (KI8 ? 0 : Cfg::KS); ++ks) {
            const int d0 = kdim<DT, D>(ks, qd, 0), d1 = kdim<DT, D>(ks, qd, 1);
            const int d2 = kdim<DT, D>(ks, qd, 2), d3 = kdim<DT, D>(ks, qd, 3);
            qa[ks][0] = r0 ? pack2<false>(qv(r, d0) * qs, qv(r, d1) * qs) : 0u;
            qa[ks][2] = r0 ? pack2<false>(qv(r, d2) * qo, qv(r, d3) * qo) : 0u;
            qa[ks][1] = r1 ? pack2<false>(qv(r + 8, d0) * qs, qv(r + 8, d1) * qs) : 0u;
            qa[ks][3] = r1 ? pack2<false>(qv(r + 8, d2) * qo, qv(r + 8, d3) * qo) : 0u;
        }
        if constexpr (SUBN) {
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                float even = 0.f, odd = 0.f;
#pragma unroll
                for (int ks = 0; ks < Cfg::KS; ++ks) {
                    const float2 e = unpack2<false>(qa[ks][hr]), o = unpack2<false>(qa[ks][2 + hr]);
                    even += e.x + e.y;
                    odd += o.x + o.y;
                }
                qoff[hr] = -OFF * pow2f(-eq) * warp_sum_quad(even + odd * (1.f / ODD));
            }
        }
    }
    // log2-domain score = (acc * 2^(24-eq) + qoff) * sl for int4, acc * 2^-eq * sl for int8 / fp8
    float kq[2];   // per query row r (hr 0) and r + 8 (hr 1)
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) kq[hr] = KI8 ? pow2f(-eqr[hr]) : pow2f(SUBN ? 24 - eq : -eq);

    float o[Cfg::MT][NHT][4];
#pragma unroll
    for (int mt = 0; mt < Cfg::MT; ++mt)
#pragma unroll
        for (int hn = 0; hn < NHT; ++hn)
#pragma unroll
            for (int c = 0; c < 4; ++c) o[mt][hn][c] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};

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
        const bool whole = nv == kBlock && nlo <= 0;   // every token of the tile visible (warp-uniform)
        // int8 / fp8 skip the score mask on whole tiles; int4 keeps one masked path (its
        // compiled schedule measured faster that way)
        constexpr bool SKIP_MASK = DT != PKV_INT4;
        const float2 sc_kv = tsc[j];

        // S = Q . K^T, token 8 nt + r of the tile in n-tile nt
        float sc[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int c = 0; c < 4; ++c) sc[nt][c] = 0.f;
            uint32_t kw[Cfg::KRUN / 4];
            load_run<ROW, SWZ, Cfg::KRUN>(kw, kb, nt * 8 + r, qd * Cfg::KRUN);
            if constexpr (KI8) {
                int a0[4] = {0, 0, 0, 0}, a1[4] = {0, 0, 0, 0};
#pragma unroll
                for (int ks = 0; ks < KS8; ++ks) {
                    mma_s8(a0, qa8[0][ks], kw[2 * ks], kw[2 * ks + 1]);
                    mma_s8(a1, qa8[1][ks], kw[2 * ks], kw[2 * ks + 1]);
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) sc[nt][c] = (float)(256 * a1[c] + a0[c]);
            } else {
#pragma unroll
                for (int ks = 0; ks < Cfg::KS; ++ks) {
                    uint32_t b0, b1;
                    kfrag<DT>(kw, ks, b0, b1);
                    mma16816<false>(sc[nt], qa[ks], b0, b1);
                }
            }
        }

        const float sl = p.scale_log2 * sc_kv.x;
        float pr[2][4];
        float alpha[2];
#pragma unroll
        for (int hr = 0; hr < NHT; ++hr) {
            float x[2][2];
            float mx = -INFINITY;
            const float cb = SUBN ? qoff[hr] * sl : 0.f;
            const float slk = sl * kq[hr];
            if (SKIP_MASK && whole) {
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        x[nt][e] = fmaf(sc[nt][2 * hr + e], slk, cb);
                        mx = fmaxf(mx, x[nt][e]);
                    }
            } else {
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int tok = nt * 8 + 2 * qd + e;
                        x[nt][e] = (tok < nv && tok >= nlo) ? fmaf(sc[nt][2 * hr + e], slk, cb) : -INFINITY;
                        mx = fmaxf(mx, x[nt][e]);
                    }
            }
            mx = warp_max_quad(mx);
            const float mn = fmaxf(m_run[hr], mx);
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
        const bool moved = (alpha[0] != 1.f) || (NHT == 2 && alpha[1] != 1.f);
        if (__any_sync(0xffffffffu, moved)) {
#pragma unroll
            for (int hn = 0; hn < NHT; ++hn) {
                const float a_lo = __shfl_sync(0xffffffffu, alpha[hn], 8 * qd);
                const float a_hi = __shfl_sync(0xffffffffu, alpha[hn], 8 * qd + 4);
#pragma unroll
                for (int mt = 0; mt < Cfg::MT; ++mt) {
                    o[mt][hn][0] *= a_lo;
                    o[mt][hn][1] *= a_hi;
                    o[mt][hn][2] *= a_lo;
                    o[mt][hn][3] *= a_hi;
                }
            }
        }

        // P^T (times the tile's V scale) as fp16 hi + lo B fragments
        uint32_t bh[NHT][2], bl[NHT][2];
#pragma unroll
        for (int hn = 0; hn < NHT; ++hn)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const float p0 = pr[nt][2 * hn] * sc_kv.y, p1 = pr[nt][2 * hn + 1] * sc_kv.y;
                bh[hn][nt] = pack2<false>(p0, p1);
                const float2 back = unpack2<false>(bh[hn][nt]);
                bl[hn][nt] = pack2<false>(p0 - back.x, p1 - back.y);
            }

        uint32_t keep01 = 0xffffffffu, keep23 = 0xffffffffu;
        const bool partial = !whole;
        if (partial) {   // zero V outside [nlo, nv): P is 0 there, V may be stale
            auto in = [&](int t) { return t >= nlo && t < nv; };
            keep01 = (in(2 * qd) ? 0x0000ffffu : 0u) | (in(2 * qd + 1) ? 0xffff0000u : 0u);
            keep23 = (in(8 + 2 * qd) ? 0x0000ffffu : 0u) | (in(9 + 2 * qd) ? 0xffff0000u : 0u);
        }
        uint32_t wa[Cfg::VRUN / 4], wb[Cfg::VRUN / 4], wc[Cfg::VRUN / 4], wd[Cfg::VRUN / 4];
        load_run<ROW, SWZ, Cfg::VRUN>(wa, vb, 2 * qd, r * Cfg::VRUN);
        load_run<ROW, SWZ, Cfg::VRUN>(wb, vb, 2 * qd + 1, r * Cfg::VRUN);
        load_run<ROW, SWZ, Cfg::VRUN>(wc, vb, 2 * qd + 8, r * Cfg::VRUN);
        load_run<ROW, SWZ, Cfg::VRUN>(wd, vb, 2 * qd + 9, r * Cfg::VRUN);
        constexpr int MT_PER_WORD = DT == PKV_INT4 ? 4 : 2;
#pragma unroll
        for (int k = 0; k < Cfg::VRUN / 4; ++k) {
            uint32_t va[4][4];
            vfrags<DT>(wa[k], wb[k], wc[k], wd[k], va);
#pragma unroll
            for (int jj = 0; jj < MT_PER_WORD; ++jj) {
                const int mt = k * MT_PER_WORD + jj;
                if (partial) {   // zero V outside the visible tokens
                    va[jj][0] &= keep01;
                    va[jj][1] &= keep01;
                    va[jj][2] &= keep23;
                    va[jj][3] &= keep23;
                }
#pragma unroll
                for (int hn = 0; hn < NHT; ++hn) {
                    mma16816<false>(o[mt][hn], va[jj], bh[hn][0], bh[hn][1]);
                    mma16816<false>(o[mt][hn], va[jj], bl[hn][0], bl[hn][1]);
                }
            }
        }

        __syncwarp();
        if (lane == 0 && j + STAGES < ntiles) {
            fence_proxy_async_smem();
            issue(j + STAGES);
        }
    }

    if (!ok) {   // no copy may still be landing in this CTA's shared memory when it exits
        if (lane == 0) flag_status(p.status, PKV_DEV_TIMEOUT);
        for (int jj = j; jj < min(ntiles, j + STAGES); ++jj)
            mbar_wait_bounded(smem_u32(&bars[jj % STAGES]), (jj / STAGES) & 1, p.wait_cycles);
        return;
    }

    // ---- epilogue: O^T row (D/8) r + 2 mt (+1 for the second half) -> [head][dim]
#pragma unroll
    for (int hr = 0; hr < NHT; ++hr) l_run[hr] = warp_sum_quad(l_run[hr]);
    const bool final_out = (p.part_base == 0 && nparts == 1);
    float* so = reinterpret_cast<float*>(smem);
    constexpr int SR = D + 4;
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
        for (int mt = 0; mt < Cfg::MT; ++mt) {
            const int d0 = (D / 8) * r + 2 * mt;
            so[h0 * SR + d0] = o[mt][hn][0] * inv_lo;
            so[(h0 + 1) * SR + d0] = o[mt][hn][1] * inv_hi;
            so[h0 * SR + d0 + 1] = o[mt][hn][2] * inv_lo;
            so[(h0 + 1) * SR + d0 + 1] = o[mt][hn][3] * inv_hi;
        }
    }
    __syncwarp();
    const size_t row0 = (size_t)b * p.H_q + hbase;
    float* dst = final_out ? p.out : p.ws_o;
    for (int i = lane; i < GC * (D / 4); i += 32) {
        const int h = i / (D / 4), c4 = i % (D / 4);
        const float4 v = *reinterpret_cast<const float4*>(&so[h * SR + 4 * c4]);
        const size_t off = final_out ? (row0 + h) * D : ws_slot(p, row0 + h, part) * D;
        float4* at = reinterpret_cast<float4*>(dst + off + 4 * c4);
        if (HINTP && !final_out) st_hint(at, v, l2_evict_last());   // the merge reads it back soon
        else *at = v;
    }
    if (!final_out && qd == 0) {
#pragma unroll
        for (int hr = 0; hr < NHT; ++hr) {
            const int h = r + 8 * hr;
            if (h < GC) {
                float2* at = reinterpret_cast<float2*>(p.ws_ml + ws_slot(p, row0 + h, part) * 2);
                if (HINTP) st_hint(at, make_float2(m_run[hr], l_run[hr]), l2_evict_last());
                else *at = make_float2(m_run[hr], l_run[hr]);
            }
        }
    }
}

template <int DT, int D>
int launch_q(const DecodeParams& p, int nht, dim3 grid, cudaStream_t s, const CUtensorMap* tmk, const CUtensorMap* tmv)
{
    const int smem = QCfg<DT, D>::BODY + 1024 + (p.part_tokens / kBlock) * (int)(sizeof(float2) + sizeof(int));
    auto k1 = decode_mmaq_kernel<DT, D, 1>;
    auto k2 = decode_mmaq_kernel<DT, D, 2>;
    auto kern = nht == 1 ? k1 : k2;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return PKV_ERR_CUDA;
    kern<<<grid, 32, smem, s>>>(p, *tmk, *tmv);
    return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

}  // namespace

int launch_decode_quant(const DecodeParams& p, int kv_dtype, int d, int nht, dim3 grid, cudaStream_t s,
                        const CUtensorMap* tmk, const CUtensorMap* tmv)
{
    switch (kv_dtype * 1000 + d) {
    case PKV_INT8 * 1000 + 128: return launch_q<PKV_INT8, 128>(p, nht, grid, s, tmk, tmv);
    case PKV_INT8 * 1000 + 64: return launch_q<PKV_INT8, 64>(p, nht, grid, s, tmk, tmv);
    case PKV_FP8E4M3 * 1000 + 128: return launch_q<PKV_FP8E4M3, 128>(p, nht, grid, s, tmk, tmv);
    case PKV_FP8E4M3 * 1000 + 64: return launch_q<PKV_FP8E4M3, 64>(p, nht, grid, s, tmk, tmv);
    case PKV_INT4 * 1000 + 128: return launch_q<PKV_INT4, 128>(p, nht, grid, s, tmk, tmv);
    case PKV_INT4 * 1000 + 64: return launch_q<PKV_INT4, 64>(p, nht, grid, s, tmk, tmv);
    default: return PKV_ERR_UNSUPPORTED;
    }
}

}  // namespace pkv
