// decode_simt.cu -- paged_decode_attn on the CUDA cores (FP32 FMA), 16-bit pools.
//
// The FP32-pipe form of the decode ("KV cache, continuous batching and paged attention",
// section "Paged attention"; "KV cache, GQA, paging and continuous batching", section
// "Mechanics": G query heads per KV head).  It is the engine selected by
// pkv_decode_opts.engine = 2 and exists to be measured against the tensor-core engine:
// at G = 8 it issues 2 G d FMAs per (token, KV head), 8 flop per K/V byte.
//
// Same staging as the tensor-core kernel (one warp per partition x KV head x sequence,
// swizzled TMA ring of K/V tiles).  Per 16-token tile:
//   scores   lane = (dim group dg of 8 dims, token half tg); every lane multiplies its 8
//            dims of q (all G heads, kept in registers) with 8 tokens of K, then a
//            transpose-reduction over the 16 dim groups (shuffles that halve the value
//            set at each level) leaves each lane G/2 complete scores of one head;
//   softmax  row max / sum over the lanes that share a head (shuffles);
//   P . V    P goes through shared memory (duplicated, so it can feed packed FMAs);
//            lane = 4 output dims of all G heads, V read straight from the staged tile.
// With F2 the products use packed fp32x2 FMA (fma.rn.f32x2, sm_100): q . K pairs two
// heads, P . V pairs two dims, halving the FMA instructions.
#include "decode_common.cuh"

namespace pkv {

namespace {

template <bool BF16>
__device__ __forceinline__ void cvt8(const uint32_t (&w)[4], float (&f)[8])
{
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 t = unpack2<BF16>(w[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c)
{
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;"
        : "=l"(d)
        : "l"(*reinterpret_cast<unsigned long long*>(&a)), "l"(*reinterpret_cast<unsigned long long*>(&b)),
          "l"(*reinterpret_cast<unsigned long long*>(&c)));
    return *reinterpret_cast<float2*>(&d);
}

template <int D, int STAGES>
struct SimtCfg {
    static constexpr int TILE = 16 * 2 * D;
    static constexpr int NBOX = D / 64;
    static constexpr int STAGE = 2 * TILE;
    static constexpr int SMEM = STAGES * STAGE + 1024;
};

template <int G, bool BF16, bool F2, int STAGES>
__global__ void __launch_bounds__(32)
decode_simt_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV)
{
    constexpr int D = 128;
    constexpr int NF = G / 2;               // scores per lane after the reduction
    constexpr int LPH = 16 / G;             // lanes of one token half per head
    static_assert(G == 4 || G == 8, "G 4 or 8");
    using Cfg = SimtCfg<D, STAGES>;
    extern __shared__ uint8_t smem_dyn[];
    __shared__ __align__(8) uint64_t bars[STAGES];
    __shared__ int tbl[kMaxPartTiles];
    __shared__ __align__(16) float p_s[G][32];   // P of the tile, each value twice
    __shared__ float a_s[G], m_s[G], l_s[G];

    pdl_launch_dependents();   // the split-K merge may be scheduled behind the last wave
    const int lane = threadIdx.x;
    const int part = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int dg = lane & 15, tg = lane >> 4;
    const int hh = dg / LPH;                // head of this lane's scores
    const int hbase = g * G;

    const int ctx = checked_ctx(p, b, lane == 0 && part == 0 && g == 0);
    const int nparts = part_count(p, ctx);
    const int tok0 = seq_base(p, ctx) + part * p.part_tokens;
    const int lo = visible_lo(p, ctx);   // tokens before lo are outside the window
    if (tok0 >= ctx) {
        if (part == 0 && p.part_base == 0) {   // empty context: a zero row
            float* o = p.out + ((size_t)b * p.H_q + hbase) * D;
            for (int i = lane; i < G * D; i += 32) o[i] = 0.f;
        }
        return;
    }
    const int ntok = min(p.part_tokens, ctx - tok0);
    const int ntiles = (ntok + kBlock - 1) / kBlock;
    const int32_t* trow = p.tables + (size_t)b * p.W + tok0 / kBlock;
    for (int j = lane; j < ntiles; j += 32) {
        int blk = trow[j];
        if ((unsigned)blk >= (unsigned)p.N) {
            flag_status(p.status, PKV_DEV_BAD_BLOCK);
            blk = 0;
        }
        tbl[j] = blk;
    }
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
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
#pragma unroll
        for (int x = 0; x < Cfg::NBOX; ++x) tma_load_2d(kdst + x * 2048, &tmK, x * 64, row, bar);
#pragma unroll
        for (int x = 0; x < Cfg::NBOX; ++x) tma_load_2d(kdst + Cfg::TILE + x * 2048, &tmV, x * 64, row, bar);
    };
    if (lane == 0) {
        for (int j = 0; j < min(STAGES, ntiles); ++j) issue(j);
    }

    // q: this lane's 8 dims of every head; F2 keeps head pairs together
    float qf[G][8];
    {
        const uint16_t* qh = static_cast<const uint16_t*>(p.q) + ((size_t)b * p.H_q + hbase) * D + 8 * dg;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const uint4 u = __ldg(reinterpret_cast<const uint4*>(qh + h * D));
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
            cvt8<BF16>(w, qf[h]);
        }
    }
    float o[G][4];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int k = 0; k < 4; ++k) o[h][k] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;
    const float sl = p.scale_log2;

    int j = 0;
    bool ok = true;
    for (; j < ntiles; ++j) {
        const int s = j % STAGES;
        // the whole warp gives up together (its shuffles need every lane)
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&bars[s]), (j / STAGES) & 1, p.wait_cycles))) {
            ok = false;
            break;
        }
        const uint32_t kb = smem_u32(smem + s * Cfg::STAGE);
        const uint32_t vb = kb + Cfg::TILE;
        const int nv = min(kBlock, ntok - j * kBlock);
        const int nlo = lo - (tok0 + j * kBlock);   // tokens of this tile before the window: < nlo

        // partial scores: this lane's 8 dims, 8 tokens, G heads
        float acc[G * 8];
#pragma unroll
        for (int i = 0; i < G * 8; ++i) acc[i] = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            uint32_t w[4];
            lds128(w, swz128(kb, 8 * tg + i, dg));
            float kf[8];
            cvt8<BF16>(w, kf);
            if constexpr (F2) {
#pragma unroll
                for (int h = 0; h < G; h += 2) {
                    float2 a2 = make_float2(acc[h * 8 + i], acc[(h + 1) * 8 + i]);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        a2 = ffma2(make_float2(qf[h][e], qf[h + 1][e]), make_float2(kf[e], kf[e]), a2);
                    acc[h * 8 + i] = a2.x;
                    acc[(h + 1) * 8 + i] = a2.y;
                }
            } else {
#pragma unroll
                for (int h = 0; h < G; ++h)
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[h * 8 + i] = fmaf(qf[h][e], kf[e], acc[h * 8 + i]);
            }
        }
        // transpose-reduction over the 16 dim groups: each level keeps half of the values
#pragma unroll
        for (int lvl = 0; lvl < 4; ++lvl) {
            const int m = 8 >> lvl;
            const int n = (G * 8) >> lvl, half = n >> 1;
            const bool upper = (dg & m) != 0;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                if (i < half) {
                    const float send = upper ? acc[i] : acc[i + half];
                    const float keep = upper ? acc[i + half] : acc[i];
                    acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                }
            }
        }
        // this lane: scores of head hh, tokens 8 tg + NF (dg % LPH) + f
        const int t0 = 8 * tg + NF * (dg % LPH);
        float x[NF];
        float mx = -INFINITY;
#pragma unroll
        for (int f = 0; f < NF; ++f) {
            x[f] = (t0 + f < nv && t0 + f >= nlo) ? acc[f] * sl : -INFINITY;
            mx = fmaxf(mx, x[f]);
        }
#pragma unroll
        for (int msk = 1; msk < LPH; msk <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, msk));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float mn = fmaxf(m_run, mx);
        const float alpha = ex2(m_run - mn);
        float sum = 0.f;
#pragma unroll
        for (int f = 0; f < NF; ++f) {
            const float pv = ex2(x[f] - mn);
            sum += pv;
            p_s[hh][2 * (t0 + f)] = pv;
            p_s[hh][2 * (t0 + f) + 1] = pv;
        }
        l_run = l_run * alpha + sum;
        m_run = mn;
        if ((dg % LPH) == 0 && tg == 0) a_s[hh] = alpha;
        __syncwarp();

        // O[h][4 lane .. 4 lane + 3] = O * alpha + sum_t P[h][t] V[t]
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float a = a_s[h];
#pragma unroll
            for (int k = 0; k < 4; ++k) o[h][k] *= a;
        }
        const uint32_t vaddr_off = (uint32_t)((lane & 1) * 8);
        for (int t = max(nlo, 0); t < nv; ++t) {
            uint32_t w0, w1;
            asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w0), "=r"(w1) : "r"(swz128(vb, t, lane >> 1) + vaddr_off));
            const float2 v01 = unpack2<BF16>(w0), v23 = unpack2<BF16>(w1);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float2 pp = *reinterpret_cast<const float2*>(&p_s[h][2 * t]);
                if constexpr (F2) {
                    float2 o01 = ffma2(pp, v01, make_float2(o[h][0], o[h][1]));
                    float2 o23 = ffma2(pp, v23, make_float2(o[h][2], o[h][3]));
                    o[h][0] = o01.x;
                    o[h][1] = o01.y;
                    o[h][2] = o23.x;
                    o[h][3] = o23.y;
                } else {
                    o[h][0] = fmaf(pp.x, v01.x, o[h][0]);
                    o[h][1] = fmaf(pp.x, v01.y, o[h][1]);
                    o[h][2] = fmaf(pp.x, v23.x, o[h][2]);
                    o[h][3] = fmaf(pp.x, v23.y, o[h][3]);
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

    // row sums over the lanes of each head, then this lane's 4 dims of every head
#pragma unroll
    for (int msk = 1; msk < LPH; msk <<= 1) l_run += __shfl_xor_sync(0xffffffffu, l_run, msk);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 16);
    if ((dg % LPH) == 0 && tg == 0) {
        l_s[hh] = l_run;
        m_s[hh] = m_run;
    }
    __syncwarp();
    const size_t row0 = (size_t)b * p.H_q + hbase;
    const bool final_out = (p.part_base == 0 && nparts == 1);
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const float inv = final_out ? 1.f / l_s[h] : 1.f;
        const float4 v = make_float4(o[h][0] * inv, o[h][1] * inv, o[h][2] * inv, o[h][3] * inv);
        if (final_out) {
            *reinterpret_cast<float4*>(p.out + (row0 + h) * D + 4 * lane) = v;
        } else {
            *reinterpret_cast<float4*>(p.ws_o + ws_slot(p, row0 + h, part) * D + 4 * lane) = v;
        }
    }
    if (!final_out && lane < G)
        *reinterpret_cast<float2*>(p.ws_ml + ws_slot(p, row0 + lane, part) * 2) = make_float2(m_s[lane], l_s[lane]);
}

template <int G, bool BF16>
int launch_simt_g(const DecodeParams& p, dim3 grid, cudaStream_t s, const CUtensorMap* tmk, const CUtensorMap* tmv,
                  bool f2)
{
    constexpr int kStages = 4;
    constexpr int smem = SimtCfg<128, kStages>::SMEM;
    auto kern = f2 ? decode_simt_kernel<G, BF16, true, kStages> : decode_simt_kernel<G, BF16, false, kStages>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return PKV_ERR_CUDA;
    kern<<<grid, 32, smem, s>>>(p, *tmk, *tmv);
    return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

}  // namespace

bool decode_simt_supported(int d, int G, int kv_dtype)
{
    return d == 128 && (G == 4 || G == 8) && (kv_dtype == PKV_BF16 || kv_dtype == PKV_F16);
}

int launch_decode_simt(const DecodeParams& p, int kv_dtype, int G, bool f2, dim3 grid, cudaStream_t s,
                       const CUtensorMap* tmk, const CUtensorMap* tmv)
{
    const bool bf = kv_dtype == PKV_BF16;
    if (G == 8) return bf ? launch_simt_g<8, true>(p, grid, s, tmk, tmv, f2) : launch_simt_g<8, false>(p, grid, s, tmk, tmv, f2);
    return bf ? launch_simt_g<4, true>(p, grid, s, tmk, tmv, f2) : launch_simt_g<4, false>(p, grid, s, tmk, tmv, f2);
}

}  // namespace pkv
