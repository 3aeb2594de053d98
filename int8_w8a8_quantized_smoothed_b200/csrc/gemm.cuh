// INT8 x INT8 -> INT32 GEMM on the 5th-generation tensor cores (tcgen05.mma kind::i8) with
// the dequantization epilogue y = bf16((float(acc) * s_tok[m]) * s_ch[n]) fused.
//
// Both kernels are warp-specialized, 192 threads:
//   warp 0      TMA producer: one thread streams K-slices (128 bytes wide, 128B-swizzled)
//               of both operands into a ring of shared-memory stages (mbarrier full/empty);
//   warp 1      TMEM allocator + MMA issuer: one thread issues tcgen05.mma (K = 32 per
//               instruction, 4 per stage) into an int32 accumulator in tensor memory and
//               releases each stage with tcgen05.commit;
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (warp w reads TMEM lanes
//               32*(w%4) .. +31), dequantization in binary32, bf16 stores.
//
// prefill kernel: persistent over 128 x BN output tiles (BN = 128 or 256), two TMEM
//   accumulators so the epilogue of tile t overlaps the MMAs of tile t+1.
// decode kernel: swap-AB (D^T = W X^T: the weight fills the MMA's 128-row side, the <= 256
//   tokens its N side), persistent stream-K: each CTA streams an equal contiguous share of
//   the (channel block, k-block) units, several k-blocks per pipeline stage; blocks split
//   between CTAs are summed exactly in int32 by the block's owner (see below).
#pragma once

#include "ptx.cuh"

namespace w8a8 {

constexpr int kGemmThreads = 192;
constexpr int kBM = 128;  // MMA M: TMEM lanes
constexpr int kBK = 128;  // bytes of K per pipeline stage (one 128B swizzle row)
constexpr int kUmmaK = 32; // K of one kind::i8 MMA

// ---------------------------------------------------------------- prefill (persistent)

template <int BN, int STAGES> struct PrefillCfg {
    static constexpr int kABytes = kBM * kBK;
    static constexpr int kBBytes = BN * kBK;
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kBarOff = STAGES * kStageBytes;
    // full[S], empty[S], tmem_full[2], tmem_empty[2], tmem slot
    static constexpr int kSmemBytes = kBarOff + (2 * STAGES + 4) * 8 + 16 + 1024;
    static constexpr int kTmemCols = 2 * BN;
    static_assert(kTmemCols <= 512, "two accumulators must fit TMEM");
};

// Tile order: groups of kGroupM row-tiles, column-major inside a group, so CTAs running
// at the same time share A row-panels and B column-panels in L2.
constexpr int kGroupM = 16;

__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int &mb, int &nb)
{
    const int per_group = kGroupM * num_n;
    const int group = tile / per_group;
    const int first_m = group * kGroupM;
    const int gm = min(kGroupM, num_m - first_m);
    const int local = tile - group * per_group;
    mb = first_m + local % gm;
    nb = local / gm;
}

template <int BN, int STAGES>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_prefill_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB, const float *__restrict__ s_tok,
                        const float *__restrict__ s_ch, int M, int N, int K,
                        uint16_t *__restrict__ y, int32_t *__restrict__ acc_out,
                        unsigned long long limit_ns)
{
    using Cfg = PrefillCfg<BN, STAGES>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sA = sbase;
    const uint32_t sB = sbase + STAGES * Cfg::kABytes;
    const uint32_t bar_full = sbase + Cfg::kBarOff;
    const uint32_t bar_empty = bar_full + 8 * STAGES;
    const uint32_t bar_tfull = bar_empty + 8 * STAGES;
    const uint32_t bar_tempty = bar_tfull + 16;
    const uint32_t tslot = bar_tempty + 16;
    uint32_t *tslot_ptr = reinterpret_cast<uint32_t *>(smem + Cfg::kBarOff + (2 * STAGES + 4) * 8);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_m = (M + kBM - 1) / kBM;
    const int num_n = (N + BN - 1) / BN;
    const int tiles = num_m * num_n;
    const int kblocks = (K + kBK - 1) / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_tfull + 8 * b, 1);
            mbar_init(bar_tempty + 8 * b, 4);
        }
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tslot, Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t *>(tslot_ptr);

    if (warp == 0) {
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
                int mb, nb;
                tile_coords(tile, num_m, num_n, mb, nb);
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const uint32_t s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1u;
                    if (!mbar_wait(bar_empty + 8 * s, ph ^ 1u, limit_ns)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(bar_full + 8 * s, Cfg::kStageBytes);
                    tma_load_2d(sA + s * Cfg::kABytes, &tmA, bar_full + 8 * s, kb * kBK, mb * kBM);
                    tma_load_2d(sB + s * Cfg::kBBytes, &tmB, bar_full + 8 * s, kb * kBK, nb * BN);
                }
            }
            // Wait until the loads still in the ring have landed before the CTA may exit.
            if (ok) {
                const uint32_t n_issued = it;
                for (uint32_t j = (n_issued > STAGES ? n_issued - STAGES : 0); j < n_issued; ++j)
                    mbar_wait(bar_full + 8 * (j % STAGES), (j / STAGES) & 1u, limit_ns);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_i8(kBM, BN);
            uint32_t it = 0, t = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++t) {
                const uint32_t buf = t & 1u;
                const uint32_t aph = (t >> 1) & 1u;
                if (!mbar_wait(bar_tempty + 8 * buf, aph ^ 1u, limit_ns))
                    break;
                tc_fence_after();
                const uint32_t d = tmem_base + buf * BN;
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const uint32_t s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1u;
                    if (!mbar_wait(bar_full + 8 * s, ph, limit_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = sA + s * Cfg::kABytes;
                    const uint32_t b0 = sB + s * Cfg::kBBytes;
#pragma unroll
                    for (int k = 0; k < kBK / kUmmaK; ++k)
                        umma_i8(d, sw128_kmajor_desc(a0 + k * kUmmaK),
                                sw128_kmajor_desc(b0 + k * kUmmaK), idesc,
                                (kb > 0 || k > 0) ? 1u : 0u);
                    umma_commit(bar_empty + 8 * s);
                }
                if (ok)
                    umma_commit(bar_tfull + 8 * buf);
            }
        }
    } else {
        // epilogue warps 2..5 -> TMEM lane quarters 2, 3, 0, 1
        const int quarter = warp & 3;
        uint32_t t = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++t) {
            int mb, nb;
            tile_coords(tile, num_m, num_n, mb, nb);
            const uint32_t buf = t & 1u;
            const uint32_t aph = (t >> 1) & 1u;
            if (!mbar_wait(bar_tfull + 8 * buf, aph, limit_ns))
                break;
            tc_fence_after();
            const int row = mb * kBM + quarter * 32 + lane;
            const bool row_ok = row < M;
            const float st = row_ok ? __ldg(s_tok + row) : 0.0f;
            const uint32_t tbase = tmem_base + buf * BN + (static_cast<uint32_t>(quarter * 32) << 16);
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tbase + c * 32, r);
                tmem_ld_wait();
                const int n0 = nb * BN + c * 32;
                if (row_ok) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const int n = n0 + 8 * g;
                        if (n < N) {
                            const float4 c0 = __ldg(reinterpret_cast<const float4 *>(s_ch + n));
                            const float4 c1 = __ldg(reinterpret_cast<const float4 *>(s_ch + n) + 1);
                            const float sc[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                            float f[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                f[i] = dequant_f32(static_cast<int32_t>(r[8 * g + i]), st, sc[i]);
                            uint4 o;
                            o.x = pack_bf16x2(f[0], f[1]);
                            o.y = pack_bf16x2(f[2], f[3]);
                            o.z = pack_bf16x2(f[4], f[5]);
                            o.w = pack_bf16x2(f[6], f[7]);
                            *reinterpret_cast<uint4 *>(y + static_cast<int64_t>(row) * N + n) = o;
                            if (acc_out) {
                                int4 *ap = reinterpret_cast<int4 *>(acc_out + static_cast<int64_t>(row) * N + n);
                                ap[0] = make_int4(r[8 * g + 0], r[8 * g + 1], r[8 * g + 2], r[8 * g + 3]);
                                ap[1] = make_int4(r[8 * g + 4], r[8 * g + 5], r[8 * g + 6], r[8 * g + 7]);
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar_tempty + 8 * buf);
        }
    }
    __syncwarp();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::kTmemCols);
    }
}

// ---------------------------------------------------------------- decode (swap-AB stream-K)
//
// Work units are (channel block t, k-block kb) pairs in tile-major order, U = NB * KB of
// them. CTA g of G (one per SM, persistent) takes the contiguous range
// [floor(g U / G), floor((g+1) U / G)), so every SM streams the same number of weight bytes.
// A range is cut into segments at channel-block boundaries. A segment covering a whole block
// is dequantized and stored directly. A block split between CTAs has one owner, the segment
// holding k-block 0 (the last segment of its CTA, so it finishes last); every other segment
// of that block (the first segment of a later CTA) stores its int32 partial in the CTA's own
// workspace slot and raises the CTA's flag; the owner waits for the flags of the later CTAs
// that share its block, adds their partials (exact int32), dequantizes, stores, and lowers
// the flags again so the workspace is zero between calls.

template <int NT, int STAGES, int KPS> struct DecodeCfg {
    static constexpr int kWBytes = kBM * kBK;           // one k-block of 128 weight rows
    static constexpr int kXBytes = NT * kBK;            // one k-block of NT token rows
    static constexpr int kStageBytes = KPS * (kWBytes + kXBytes);
    static constexpr int kBarOff = STAGES * kStageBytes;
    // full[S], empty[S], tmem_full[2], tmem_empty[2], tmem slot, flag word
    static constexpr int kSmemBytes = kBarOff + (2 * STAGES + 4) * 8 + 32 + 1024;
    static constexpr int kTmemCols = 2 * NT < 32 ? 32 : 2 * NT;
    static_assert(kXBytes % 1024 == 0, "token tile must keep stages 1024-byte aligned");
    static_assert(kTmemCols <= 512, "two accumulators must fit TMEM");
};

// CTA holding unit v under the even split of U units over G CTAs.
__host__ __device__ __forceinline__ int64_t sk_owner_of(int64_t v, int64_t U, int64_t G)
{
    int64_t c = (v * G) / U;
    while (c + 1 < G && ((c + 1) * U) / G <= v)
        ++c;
    while (c > 0 && (c * U) / G > v)
        --c;
    return c;
}

struct SkSegment {
    int64_t t;   // channel block
    int kb0, kb1; // k-block range [kb0, kb1)
};

// Segment iterator over [u, u1): next segment starting at u.
__device__ __forceinline__ SkSegment sk_segment(int64_t u, int64_t u1, int KB)
{
    SkSegment sg;
    sg.t = u / KB;
    sg.kb0 = static_cast<int>(u - sg.t * KB);
    const int64_t left = u1 - u;
    sg.kb1 = static_cast<int>(min(static_cast<int64_t>(KB), sg.kb0 + left));
    return sg;
}

template <int NT, int STAGES, int KPS>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_decode_kernel(const __grid_constant__ CUtensorMap tmW,
                       const __grid_constant__ CUtensorMap tmX, const float *__restrict__ s_tok,
                       const float *__restrict__ s_ch, int M, int N, int K,
                       uint16_t *__restrict__ y, int32_t *__restrict__ acc_out,
                       int32_t *__restrict__ ws_part, unsigned int *__restrict__ ws_flag,
                       unsigned long long limit_ns)
{
    using Cfg = DecodeCfg<NT, STAGES, KPS>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sW = sbase;                               // [STAGES][KPS][128 x 128 B]
    const uint32_t sX = sbase + STAGES * KPS * Cfg::kWBytes; // [STAGES][KPS][NT x 128 B]
    const uint32_t bar_full = sbase + Cfg::kBarOff;
    const uint32_t bar_empty = bar_full + 8 * STAGES;
    const uint32_t bar_tfull = bar_empty + 8 * STAGES;
    const uint32_t bar_tempty = bar_tfull + 16;
    const uint32_t tslot = bar_tempty + 16;
    uint32_t *tslot_ptr = reinterpret_cast<uint32_t *>(smem + Cfg::kBarOff + (2 * STAGES + 4) * 8);
    volatile uint32_t *sh_word = tslot_ptr + 4;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int KB = (K + kBK - 1) / kBK;
    const int64_t NB = (N + kBM - 1) / kBM;
    const int64_t U = NB * KB;
    const int64_t G = gridDim.x;
    const int64_t g = blockIdx.x;
    const int64_t u_begin = (g * U) / G;
    const int64_t u_end = ((g + 1) * U) / G;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_tfull + 8 * b, 1);
            mbar_init(bar_tempty + 8 * b, 4);
        }
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmW);
        tma_prefetch_desc(&tmX);
    }
    if (warp == 1) {
        tmem_alloc(tslot, Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t *>(tslot_ptr);

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first(); // weights are streamed once
            uint32_t it = 0;
            bool ok = true;
            for (int64_t u = u_begin; u < u_end && ok;) {
                const SkSegment sg = sk_segment(u, u_end, KB);
                for (int kb = sg.kb0; kb < sg.kb1; kb += KPS, ++it) {
                    const int nk = min(KPS, sg.kb1 - kb);
                    const uint32_t s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1u;
                    if (!mbar_wait(bar_empty + 8 * s, ph ^ 1u, limit_ns)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(bar_full + 8 * s, nk * (Cfg::kWBytes + Cfg::kXBytes));
                    for (int j = 0; j < nk; ++j) {
                        tma_load_2d_hint(sW + (s * KPS + j) * Cfg::kWBytes, &tmW, bar_full + 8 * s,
                                         (kb + j) * kBK, static_cast<int32_t>(sg.t * kBM), pol_w);
                        tma_load_2d(sX + (s * KPS + j) * Cfg::kXBytes, &tmX, bar_full + 8 * s,
                                    (kb + j) * kBK, 0);
                    }
                }
                u += sg.kb1 - sg.kb0;
            }
            if (ok) {
                for (uint32_t j = (it > STAGES ? it - STAGES : 0); j < it; ++j)
                    mbar_wait(bar_full + 8 * (j % STAGES), (j / STAGES) & 1u, limit_ns);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_i8(kBM, NT);
            uint32_t it = 0, seg = 0;
            bool ok = true;
            for (int64_t u = u_begin; u < u_end && ok; ++seg) {
                const SkSegment sg = sk_segment(u, u_end, KB);
                const uint32_t buf = seg & 1u;
                const uint32_t aph = (seg >> 1) & 1u;
                if (!mbar_wait(bar_tempty + 8 * buf, aph ^ 1u, limit_ns))
                    break;
                tc_fence_after();
                const uint32_t d = tmem_base + buf * NT;
                for (int kb = sg.kb0; kb < sg.kb1; kb += KPS, ++it) {
                    const int nk = min(KPS, sg.kb1 - kb);
                    const uint32_t s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1u;
                    if (!mbar_wait(bar_full + 8 * s, ph, limit_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int j = 0; j < nk; ++j) {
                        const uint32_t w0 = sW + (s * KPS + j) * Cfg::kWBytes;
                        const uint32_t x0 = sX + (s * KPS + j) * Cfg::kXBytes;
#pragma unroll
                        for (int k = 0; k < kBK / kUmmaK; ++k)
                            umma_i8(d, sw128_kmajor_desc(w0 + k * kUmmaK),
                                    sw128_kmajor_desc(x0 + k * kUmmaK), idesc,
                                    (kb > sg.kb0 || j > 0 || k > 0) ? 1u : 0u);
                    }
                    umma_commit(bar_empty + 8 * s);
                }
                if (ok)
                    umma_commit(bar_tfull + 8 * buf);
                u += sg.kb1 - sg.kb0;
            }
        }
    } else {
        // Epilogue: warp w reads TMEM lanes 32*(w%4)..+31 = channels of the block.
        const int quarter = warp & 3;
        const int etid = threadIdx.x - 64; // 0..127
        const int r = quarter * 32 + lane; // channel within the block
        constexpr int kChunk = NT < 32 ? NT : 32;
        uint32_t seg = 0;
        bool ok = true;
        for (int64_t u = u_begin; u < u_end && ok; ++seg) {
            const SkSegment sg = sk_segment(u, u_end, KB);
            u += sg.kb1 - sg.kb0;
            const uint32_t buf = seg & 1u;
            const uint32_t aph = (seg >> 1) & 1u;
            const bool whole = (sg.kb0 == 0 && sg.kb1 == KB);
            const bool owner = (sg.kb0 == 0 && !whole);
            const int n = static_cast<int>(sg.t * kBM) + r;
            const bool n_ok = n < N;
            const float sc = n_ok ? __ldg(s_ch + n) : 0.0f;
            // contributors to an owned block: the later CTAs whose ranges reach into it
            int64_t g_last = g;
            if (owner) {
                g_last = sk_owner_of(sg.t * KB + KB - 1, U, G);
                if (etid == 0) {
                    bool all = true;
                    for (int64_t c = g + 1; c <= g_last && all; ++c) {
                        const volatile unsigned int *f = ws_flag + c;
                        if (*f == 0u) {
                            const uint64_t t0 = globaltimer_ns();
                            while (*f == 0u) {
                                if (globaltimer_ns() - t0 > limit_ns) {
                                    flag_timeout();
                                    all = false;
                                    break;
                                }
                            }
                        }
                    }
                    *sh_word = all ? 1u : 0u;
                }
                named_bar_sync(1, 128);
                if (*sh_word == 0u)
                    ok = false;
                __threadfence();
            }
            if (!mbar_wait(bar_tfull + 8 * buf, aph, limit_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t tbase = tmem_base + buf * NT + (static_cast<uint32_t>(quarter * 32) << 16);
#pragma unroll 1
            for (int c0 = 0; c0 < NT && c0 < M; c0 += kChunk) {
                uint32_t a[32];
                if constexpr (kChunk == 32) {
                    tmem_ld_32x32b_x32(tbase + c0, a);
                } else {
                    uint32_t a16[16];
                    tmem_ld_32x32b_x16(tbase + c0, a16);
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        a[i] = a16[i];
                }
                tmem_ld_wait();
                if (!whole && !owner) {
                    // contributor: partial sums to this CTA's slot, [m][128] int32
#pragma unroll
                    for (int j = 0; j < kChunk; ++j) {
                        const int m = c0 + j;
                        if (m < M)
                            __stcg(ws_part + (g * M + m) * kBM + r, static_cast<int32_t>(a[j]));
                    }
                    continue;
                }
                if (owner) {
                    for (int64_t c = g + 1; c <= g_last; ++c) {
#pragma unroll
                        for (int j = 0; j < kChunk; ++j) {
                            const int m = c0 + j;
                            if (m < M) {
                                int32_t *pp = ws_part + (c * M + m) * kBM + r;
                                a[j] = static_cast<uint32_t>(static_cast<int32_t>(a[j]) + __ldcg(pp));
                                __stcg(pp, 0); // the workspace is zero again after the call
                            }
                        }
                    }
                }
                if (n_ok) {
#pragma unroll
                    for (int j = 0; j < kChunk; ++j) {
                        const int m = c0 + j;
                        if (m < M) {
                            const int32_t v = static_cast<int32_t>(a[j]);
                            const int64_t off = static_cast<int64_t>(m) * N + n;
                            y[off] = static_cast<uint16_t>(bf16_bits(dequant_f32(v, __ldg(s_tok + m), sc)));
                            if (acc_out)
                                acc_out[off] = v;
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar_tempty + 8 * buf);
            if (!whole && !owner) {
                // publish the partial: every thread's stores, then one flag write
                __threadfence();
                named_bar_sync(1, 128);
                if (etid == 0)
                    atomicExch(ws_flag + g, 1u);
            } else if (owner) {
                named_bar_sync(1, 128);
                if (etid == 0)
                    for (int64_t c = g + 1; c <= g_last; ++c)
                        atomicExch(ws_flag + c, 0u);
            }
        }
    }
    __syncwarp();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::kTmemCols);
    }
}

} // namespace w8a8
