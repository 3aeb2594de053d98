// The decoder block's linear path at decode sizes (M <= 64 tokens) as ONE persistent kernel.
//
// Phases, in the order of a Llama decoder block:
//   R0  q1, s1 = smoothed RMSNorm + quant of x                 (gamma1' carries the smoothing)
//   G0  qkv   = GEMM(q1, s1, W_qkv)                            bf16 [M, QKV]
//   R1  q2, s2 = quantize_rows(attn, sinv_o)                   (attention stand-in input)
//   G1  o     = GEMM(q2, s2, W_o)                              bf16 [M, H]
//   R2  h = bf16(o + x); q3, s3 = smoothed RMSNorm + quant of h
//   G2  a     = SiLU(gate) * up from GEMM(q3, s3, W_gate|up)   fp32 [M, I] (interleaved rows)
//   R3  q4, s4 = quant of a (spread over the grid; the per-token maxima come from G2's
//       epilogues)
//   G3  y     = GEMM(q4, s4, W_down)                           bf16 [M, H]
// with a grid-wide barrier after every phase (B0..B6). Each phase computes exactly what the
// separate kernels compute (the same per-element arithmetic); only the binary64 order of the
// RMSNorm sums differs, which the method leaves free.
//
// Why one kernel: at decode sizes every GEMM is a weight stream of a few to ~100 MB, and a
// kernel boundary costs several microseconds of ramp (launch, prologue, pipeline fill) and
// tail (last MMAs, split-K reduction, epilogue) during which HBM idles. Here the producer warp
// runs ahead through ALL four GEMMs' weight tiles (static data, no dependency), holding back
// only the activation tiles of a GEMM until the barrier that makes them ready; the shared-
// memory ring therefore keeps filling with the next GEMM's weights while the current GEMM's
// tail, the barriers and the row phases run, and the weight stream is continuous.
//
// Roles (192 threads, one CTA per SM, all CTAs co-resident: cooperative launch):
//   warp 0      TMA producer: for every GEMM phase, this CTA's stream-K share of the
//               (channel block, k-block) units, weights and token tiles into the stage ring
//   warp 1      TMEM allocator + MMA issuer (tcgen05.mma kind::i8), two accumulators
//   warps 2..5  row phases and the GEMM epilogues (a block split between CTAs is summed in a
//               per-phase workspace and finished by whichever piece arrives last), and the
//               grid barriers
// Barrier counter: one 64-bit word that only grows; a launch performs 7 * G arrivals, and
// every CTA derives the launch's base as the counter rounded down to a multiple of 7 * G (no
// CTA can pass B0 before all have read it).
#pragma once

#include "gemm.cuh"
#include "rowquant.cuh"

namespace w8a8 {

constexpr int kBlockPhases = 4;   // GEMM phases
constexpr int kBlockBarriers = 7; // grid barriers per launch

struct BlockGemm {
    const float *s_ch;  // channel scales [N] (interleaved like the weight for the SiLU phase)
    uint16_t *y;        // bf16 output [M, N]; null for the SiLU phase
    int N, K;
    // split blocks: every piece adds its int32 partial into acc [block][Mp/4][128][4] (bulk
    // reduction, exact and order-free) and counts itself in cnt[block]; the piece that arrives
    // last reads the sum, finishes the block and clears both for the next launch
    int32_t *ws_part;
    unsigned int *ws_flag;
};

struct BlockArgs {
    int M, H, I;
    float eps;
    const uint16_t *x;      // [M, H] block input (also the residual of R2)
    const uint16_t *attn;   // [M, H] attention stand-in, input of the o projection
    const float *g1;        // gamma1' [H]
    const float *sinv_o;    // smoothing inverse of the o projection's input [H]
    const float *g2;        // gamma2' [H]
    int8_t *q[4];           // q1..q4: [M, H], [M, H], [M, H], [M, I]
    float *s[4];            // s1..s4: [M]
    uint16_t *h;            // [M, H]
    float *a;               // [M, I]
    unsigned int *amax_w;   // [M] per-token max |a| (bits), zeroed in R0
    BlockGemm g[kBlockPhases];
    unsigned long long *bar;
    unsigned long long limit_ns;
};

struct alignas(64) BlockMaps {
    CUtensorMap w[kBlockPhases]; // weights [N, K]
    CUtensorMap x[kBlockPhases]; // token codes [M, K] (box NT rows)
};

__device__ __forceinline__ unsigned long long ld_acquire_gpu_u64(const unsigned long long *p)
{
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// Bulk reduction (TMA engine): global[dst .. +bytes) += shared[src ..] as int32, tracked by
// this thread's bulk async-group.
__device__ __forceinline__ void bulk_reduce_add_s32_global(int32_t *dst, uint32_t src, uint32_t bytes)
{
    asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.s32 [%0], [%1], %2;" ::"l"(dst),
                 "r"(src), "r"(bytes)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

__device__ __forceinline__ void bulk_wait_all()
{
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_shared()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_cta_shared(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_cta_shared(uint32_t *p, uint32_t v)
{
    asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}


// Waits (bounded) until the barrier counter reaches target; false if the wait ran out.
__device__ __forceinline__ bool grid_wait(const unsigned long long *bar, unsigned long long target,
                                          unsigned long long limit_ns)
{
    if (ld_acquire_gpu_u64(bar) >= target)
        return true;
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_gpu_u64(bar) < target) {
        if (globaltimer_ns() - t0 > limit_ns) {
            flag_timeout();
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ void load8_f32(const float *p, float (&v)[8])
{
    const float4 lo = __ldcg(reinterpret_cast<const float4 *>(p));
    const float4 hi = __ldcg(reinterpret_cast<const float4 *>(p) + 1);
    v[0] = lo.x; v[1] = lo.y; v[2] = lo.z; v[3] = lo.w;
    v[4] = hi.x; v[5] = hi.y; v[6] = hi.z; v[7] = hi.w;
}

// quantize_rows of one bf16 row (y = x * sinv) by the 128-thread group, row in registers.
template <int NV>
__device__ __forceinline__ void row_quant_bf16(const uint16_t *xin, const float *sinv, int K,
                                               int8_t *qrow, float *s_out, int etid, float *shf)
{
    const int nvec = K >> 3;
    uint4 raw[NV];
    float sv[NV][8];
#pragma unroll
    for (int c = 0; c < NV; ++c) {
        const int v = c * 128 + etid;
        raw[c] = v < nvec ? ldg_nc_v4(reinterpret_cast<const uint4 *>(xin) + v)
                          : make_uint4(0u, 0u, 0u, 0u);
        if (v < nvec)
            load8_gamma(sinv + 8 * v, sv[c]);
    }
    float f[NV][8];
    float amax = 0.0f;
#pragma unroll
    for (int c = 0; c < NV; ++c) {
        const int v = c * 128 + etid;
        unpack8(raw[c], f[c]);
        if (v < nvec) {
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                const float2 p = mul2(make_float2(f[c][i], f[c][i + 1]), make_float2(sv[c][i], sv[c][i + 1]));
                f[c][i] = p.x;
                f[c][i + 1] = p.y;
                amax = fmaxf(amax, fmaxf(fabsf(p.x), fabsf(p.y)));
            }
        }
    }
    amax = group_max(amax, shf, etid);
    const float s = __fdiv_rn(amax, 127.0f);
    if (etid == 0)
        *s_out = s;
    const bool by_product = s >= 7.888609052210118e-31f;
    const float r = by_product ? __frcp_rn(s) : 0.0f;
#pragma unroll
    for (int c = 0; c < NV; ++c) {
        const int v = c * 128 + etid;
        if (v < nvec)
            reinterpret_cast<uint2 *>(qrow)[v] = quant8_int8(f[c], s, r, by_product, amax);
    }
}

// The quantization of a (binary32 [M, I], written in this launch) spread over the whole grid:
// token m's scale is amax[m] / 127 with amax[m] the max |a| of the row, raised by the SiLU
// epilogues (atomicMax on the bits of non-negative floats orders like the floats). CTA g
// codes the 8-value vectors [g V / G, (g+1) V / G) of the flattened rows; CTA 0 writes s.
__device__ __forceinline__ void grid_quant_f32(const float *a, const unsigned int *amax_w, int M,
                                               int I, int8_t *q, float *s_out, int64_t g,
                                               int64_t G, int etid)
{
    const int64_t nv_row = I >> 3;
    const int64_t V = static_cast<int64_t>(M) * nv_row;
    const int64_t v0 = (g * V) / G, v1 = ((g + 1) * V) / G;
    for (int64_t v = v0 + etid; v < v1; v += 128) {
        const int m = static_cast<int>(v / nv_row);
        const float amax = __uint_as_float(__ldcg(amax_w + m));
        const float s = __fdiv_rn(amax, 127.0f);
        const bool by_product = s >= 7.888609052210118e-31f;
        const float r = by_product ? __frcp_rn(s) : 0.0f;
        float y[8];
        load8_f32(a + 8 * v, y);
        reinterpret_cast<uint2 *>(q)[v] = quant8_int8(y, s, r, by_product, amax);
    }
    if (g == 0)
        for (int m = etid; m < M; m += 128)
            s_out[m] = __fdiv_rn(__uint_as_float(__ldcg(amax_w + m)), 127.0f);
}

// The SiLU*up form of a block's final step with the per-token maxima: as silu_block_rows, and
// every token's max |a| over the block's 64 channels (8 consecutive lanes hold one token's 8
// vectors) raised into amax_w[m] with atomicMax on its bits. All 128 threads call it.
template <typename GateUp>
__device__ __forceinline__ void silu_block_rows_max(int mt, int t, int etid, const SiluOut &so,
                                                    unsigned int *amax_w, GateUp gate_up)
{
    const int lane = etid & 31;
    for (int base = 0; base < mt * 8; base += 128) {
        const int v = base + etid;
        const bool act = v < mt * 8;
        const int m = v >> 3, j0 = (v & 7) * 8;
        float mx = 0.0f;
        if (act) {
            float g[8], u[8], a[8];
            gate_up(m, j0, g, u);
            silu_mul8(g, u, a);
#pragma unroll
            for (int i = 0; i < 8; ++i)
                mx = fmaxf(mx, fabsf(a[i]));
            float *dst = so.a + static_cast<int64_t>(m) * so.I + static_cast<int64_t>(t) * 64 + j0;
            reinterpret_cast<float4 *>(dst)[0] = make_float4(a[0], a[1], a[2], a[3]);
            reinterpret_cast<float4 *>(dst)[1] = make_float4(a[4], a[5], a[6], a[7]);
        }
#pragma unroll
        for (int o = 1; o < 8; o <<= 1)
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (act && (lane & 7) == 0)
            atomicMax(amax_w + m, __float_as_uint(mx));
    }
}

template <int NT, int STAGES, int KPS> struct BlockCfg {
    static constexpr int kWBytes = kBM * kBK;
    static constexpr int kXBytes = NT * kBK;
    static constexpr int kStageBytes = KPS * (kWBytes + kXBytes);
    // staged output tile: bf16 [NT][128] for whole / owned blocks, or a contribution's int32
    // partial [NT/4][128][4] for the bulk reduction
    static constexpr int kYOff = STAGES * kStageBytes;
    static constexpr int kStokOff = kYOff + NT * kBM * 4;        // token scales [NT]
    static constexpr int kRedOff = kStokOff + NT * 4;            // reductions: 4 double + 4 float
    static constexpr int kBarOff = kRedOff + 64;
    static constexpr int kSmemBytes = kBarOff + (2 * STAGES + 4) * 8 + 32 + 1024;
    static constexpr int kTmemCols = 2 * NT < 32 ? 32 : 2 * NT;
    static_assert(kXBytes % 1024 == 0, "token tile must keep stages 1024-byte aligned");
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

template <int NT, int STAGES, int KPS, int NV>
__global__ void __launch_bounds__(kGemmThreads, 1)
    block_decode_kernel(const __grid_constant__ BlockMaps maps, const __grid_constant__ BlockArgs A)
{
    using Cfg = BlockCfg<NT, STAGES, KPS>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sW = sbase;
    const uint32_t sX = sbase + STAGES * KPS * Cfg::kWBytes;
    uint16_t *ysm = reinterpret_cast<uint16_t *>(smem + Cfg::kYOff);
    float *sh_stok = reinterpret_cast<float *>(smem + Cfg::kStokOff);
    double *shd = reinterpret_cast<double *>(smem + Cfg::kRedOff);
    float *shf = reinterpret_cast<float *>(smem + Cfg::kRedOff + 32);
    const uint32_t bar_full = sbase + Cfg::kBarOff;
    const uint32_t bar_empty = bar_full + 8 * STAGES;
    const uint32_t bar_tfull = bar_empty + 8 * STAGES;
    const uint32_t bar_tempty = bar_tfull + 16;
    const uint32_t tslot = bar_tempty + 16;
    uint32_t *tslot_ptr = reinterpret_cast<uint32_t *>(smem + Cfg::kBarOff + (2 * STAGES + 4) * 8);
    volatile uint32_t *sh_word = tslot_ptr + 4;
    // phases whose token codes are ready (count), published by the epilogue group when it
    // passes the barrier that orders them; read by the producer
    uint32_t *sh_xready = tslot_ptr + 5;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int M = A.M;
    const int64_t G = gridDim.x;
    const int64_t g = blockIdx.x;
    const unsigned long long per_launch = static_cast<unsigned long long>(kBlockBarriers) * G;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_tfull + 8 * b, 1);
            mbar_init(bar_tempty + 8 * b, 4);
        }
        *sh_xready = 0u;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        for (int p = 0; p < kBlockPhases; ++p) {
            tma_prefetch_desc(&maps.w[p]);
            tma_prefetch_desc(&maps.x[p]);
        }
    }
    if (warp == 1)
        tmem_alloc(tslot, Cfg::kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t *>(tslot_ptr);

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first();
            // token-tile loads held back until their phase's inputs are ready: a FIFO of the
            // most recent stages (at most STAGES), oldest at head
            struct Pending {
                uint32_t s;
                int kb, nk, p;
            };
            Pending pend[STAGES];
            int head = 0, npend = 0, p_ready = -1; // phases whose codes are ready: 0 .. p_ready
            bool ok = true;
            const volatile uint32_t *xr = sh_xready;
            auto issue_x = [&](const Pending &e) {
                for (int j = 0; j < e.nk; ++j)
                    tma_load_2d(sX + (e.s * KPS + j) * Cfg::kXBytes, &maps.x[e.p], bar_full + 8 * e.s,
                                (e.kb + j) * kBK, 0);
            };
            // issue the pending token loads whose phases are ready (in order); with wait, first
            // block (bounded) until the oldest one's phase is ready
            auto flush = [&](bool wait) {
                while (npend > 0) {
                    const Pending &e = pend[head];
                    if (e.p > p_ready) {
                        if (static_cast<int>(*xr) <= e.p) { // cheap check first
                            if (!wait)
                                return;
                            const uint64_t t0 = globaltimer_ns();
                            while (static_cast<int>(*xr) <= e.p) {
                                if (globaltimer_ns() - t0 > A.limit_ns) {
                                    flag_timeout();
                                    ok = false;
                                    return;
                                }
                            }
                        }
                        p_ready = static_cast<int>(ld_acquire_cta_shared(sh_xready)) - 1;
                        fence_proxy_async_global(); // the codes were written by the generic proxy
                    }
                    issue_x(e);
                    head = head + 1 == STAGES ? 0 : head + 1;
                    --npend;
                }
            };
            uint32_t it = 0;
            for (int p = 0; p < kBlockPhases && ok; ++p) {
                const int KB = (A.g[p].K + kBK - 1) / kBK;
                const int64_t U = static_cast<int64_t>((A.g[p].N + kBM - 1) / kBM) * KB;
                const int64_t u_begin = (g * U) / G, u_end = ((g + 1) * U) / G;
                for (int64_t u = u_begin; u < u_end && ok;) {
                    const SkSegment sg = sk_segment(u, u_end, KB);
                    for (int kb = sg.kb0; kb < sg.kb1 && ok; kb += KPS, ++it) {
                        const int nk = min(KPS, sg.kb1 - kb);
                        const uint32_t s = it % STAGES;
                        const uint32_t ph = (it / STAGES) & 1u;
                        if (npend == STAGES)
                            flush(true); // the stage to reuse is waiting for its token tile
                        if (!ok)
                            break;
                        if (!mbar_wait(bar_empty + 8 * s, ph ^ 1u, A.limit_ns)) {
                            ok = false;
                            break;
                        }
                        mbar_expect_tx(bar_full + 8 * s, nk * (Cfg::kWBytes + Cfg::kXBytes));
                        for (int j = 0; j < nk; ++j)
                            tma_load_2d_hint(sW + (s * KPS + j) * Cfg::kWBytes, &maps.w[p],
                                             bar_full + 8 * s, (kb + j) * kBK,
                                             static_cast<int32_t>(sg.t * kBM), pol_w);
                        int tail = head + npend;
                        tail = tail >= STAGES ? tail - STAGES : tail;
                        pend[tail] = Pending{s, kb, nk, p};
                        ++npend;
                        flush(false);
                    }
                    u += sg.kb1 - sg.kb0;
                }
            }
            while (ok && npend > 0)
                flush(true);
            if (ok)
                drain_ring(bar_empty, it, STAGES, A.limit_ns);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_i8(kBM, NT);
            uint32_t it = 0, seg = 0;
            bool ok = true;
            for (int p = 0; p < kBlockPhases && ok; ++p) {
                const int KB = (A.g[p].K + kBK - 1) / kBK;
                const int64_t U = static_cast<int64_t>((A.g[p].N + kBM - 1) / kBM) * KB;
                const int64_t u_begin = (g * U) / G, u_end = ((g + 1) * U) / G;
                for (int64_t u = u_begin; u < u_end && ok; ++seg) {
                    const SkSegment sg = sk_segment(u, u_end, KB);
                    const uint32_t buf = seg & 1u;
                    const uint32_t aph = (seg >> 1) & 1u;
                    if (!mbar_wait(bar_tempty + 8 * buf, aph ^ 1u, A.limit_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d = tmem_base + buf * NT;
                    for (int kb = sg.kb0; kb < sg.kb1; kb += KPS, ++it) {
                        const int nk = min(KPS, sg.kb1 - kb);
                        const uint32_t s = it % STAGES;
                        const uint32_t ph = (it / STAGES) & 1u;
                        if (!mbar_wait(bar_full + 8 * s, ph, A.limit_ns)) {
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
        }
    } else {
        const int etid = threadIdx.x - 64; // 0..127
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane; // channel within a block
        unsigned long long base = 0;
        if (etid == 0)
            *sh_word = 0u;
        named_bar_sync(1, 128);
        if (etid == 0) {
            const unsigned long long b = ld_acquire_gpu_u64(A.bar);
            base = (b / per_launch) * per_launch;
            reinterpret_cast<volatile unsigned long long *>(shd)[0] = base;
        }
        named_bar_sync(1, 128);
        base = reinterpret_cast<volatile unsigned long long *>(shd)[0];
        named_bar_sync(1, 128);
        bool ok = true;
        int nbar = 0;
        // arrive at the next barrier (every thread's stores of the phase are done) and wait
        auto barrier = [&]() {
            named_bar_sync(1, 128);
            if (etid == 0) {
                __threadfence();
                atomicAdd(A.bar, 1ull);
                const bool w = ok && grid_wait(A.bar, base + (nbar + 1) * G, A.limit_ns);
                *sh_word = w ? 0u : 1u;
                if (w && (nbar & 1) == 0) // B0, B2, B4, B6: GEMM nbar / 2 may load its codes
                    st_release_cta_shared(sh_xready, static_cast<uint32_t>(nbar / 2 + 1));
            }
            named_bar_sync(1, 128);
            if (*sh_word != 0u)
                ok = false;
            ++nbar;
        };
        // ---- R0 (and the maxima words of the SiLU phase cleared for this launch)
        if (g == 0)
            for (int m = etid; m < M; m += 128)
                A.amax_w[m] = 0u;
        for (int m = static_cast<int>(g); m < M; m += static_cast<int>(G))
            row_rmsnorm<NV>(A.x + static_cast<int64_t>(m) * A.H, false, nullptr, nullptr, A.g1,
                            A.eps, A.H, A.q[0] + static_cast<int64_t>(m) * A.H, A.s[0] + m, etid,
                            shd, shf);
        barrier(); // B0
        uint32_t seg = 0;
        const int Mp = (M + 3) & ~3;
        for (int p = 0; p < kBlockPhases && ok; ++p) {
            const BlockGemm &P = A.g[p];
            const int N = P.N;
            const int KB = (P.K + kBK - 1) / kBK;
            const int64_t U = static_cast<int64_t>((N + kBM - 1) / kBM) * KB;
            const int64_t u_begin = (g * U) / G, u_end = ((g + 1) * U) / G;
            const float *s_tok = A.s[p];
            for (int i = etid; i < M; i += 128)
                sh_stok[i] = __ldcg(s_tok + i);
            named_bar_sync(1, 128);
            const int Q4 = Mp >> 2; // token quads per block in the accumulation buffer
            int4 *acc_all = reinterpret_cast<int4 *>(P.ws_part);
            for (int64_t u = u_begin; u < u_end && ok; ++seg) {
                const SkSegment sg = sk_segment(u, u_end, KB);
                u += sg.kb1 - sg.kb0;
                const uint32_t buf = seg & 1u;
                const uint32_t aph = (seg >> 1) & 1u;
                // a piece of a block split between CTAs, or a whole block
                const bool split = sg.kb0 > 0 || sg.kb1 < KB;
                const int64_t tch = sg.t;
                const int n = static_cast<int>(tch * kBM) + r;
                const float sc = n < N ? __ldg(P.s_ch + n) : 0.0f;
                if (!mbar_wait(bar_tfull + 8 * buf, aph, A.limit_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t tbase = tmem_base + buf * NT + (static_cast<uint32_t>(quarter * 32) << 16);
#pragma unroll
                for (int c0 = 0; c0 < NT; c0 += 16) {
                    if (c0 < M) {
                        uint32_t acc[16];
                        tmem_ld_32x32b_x16(tbase + c0, acc);
                        tmem_ld_wait();
                        if (split) {
                            // int32 partial [Mp/4][128][4]; tokens M .. Mp-1 hold zeros (their
                            // rows of the token tile were zero-filled)
                            int32_t *stg = reinterpret_cast<int32_t *>(ysm) + ((c0 >> 2) * kBM + r) * 4;
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                if (c0 + j < Mp)
                                    stg[(j >> 2) * kBM * 4 + (j & 3)] = static_cast<int32_t>(acc[j]);
                        } else {
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                if (c0 + j < M)
                                    ysm[(c0 + j) * kBM + r] = static_cast<uint16_t>(bf16_bits(
                                        dequant_f32(static_cast<int32_t>(acc[j]), sh_stok[c0 + j], sc)));
                        }
                    }
                }
                if (split)
                    fence_proxy_async_shared(); // staged partial, before the bulk read
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(bar_tempty + 8 * buf);
                named_bar_sync(1, 128);
                if (split) {
                    // add the piece into the block's sum and count it; the piece that arrives
                    // last finishes the block (reads the sum, dequantizes, stores) and clears
                    // the sum and the count for the next launch
                    if (etid == 0) {
                        bulk_reduce_add_s32_global(P.ws_part + tch * Q4 * kBM * 4, smem_u32(ysm),
                                                   static_cast<uint32_t>(Q4) * kBM * 16u);
                        bulk_wait_all();
                        fence_proxy_async_global();
                        const unsigned int prev = atom_add_acq_rel_gpu(P.ws_flag + tch, 1u);
                        const int64_t pieces =
                            sk_owner_of(tch * KB + KB - 1, U, G) - sk_owner_of(tch * KB, U, G) + 1;
                        const bool last = static_cast<int64_t>(prev) + 1 == pieces;
                        if (last)
                            st_relaxed_gpu(P.ws_flag + tch, 0u);
                        *sh_word = last ? 1u : 0u;
                    }
                    named_bar_sync(1, 128);
                    if (*sh_word == 0u)
                        continue; // another piece finishes the block
                    int4 *acc4 = acc_all + tch * Q4 * kBM + r;
                    int4 vq[NT / 4]; // every load issued before any store (they cannot overlap)
#pragma unroll
                    for (int q = 0; q < NT / 4; ++q)
                        vq[q] = q < Q4 ? __ldcg(acc4 + q * kBM) : make_int4(0, 0, 0, 0);
#pragma unroll
                    for (int q = 0; q < NT / 4; ++q)
                        if (q < Q4)
                            __stcg(acc4 + q * kBM, make_int4(0, 0, 0, 0));
#pragma unroll
                    for (int q = 0; q < NT / 4; ++q) {
                        const int vv[4] = {vq[q].x, vq[q].y, vq[q].z, vq[q].w};
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            if (4 * q + e < M)
                                ysm[(4 * q + e) * kBM + r] = static_cast<uint16_t>(
                                    bf16_bits(dequant_f32(vv[e], sh_stok[4 * q + e], sc)));
                    }
                    named_bar_sync(1, 128);
                }
                // the block's bf16 tile is complete in ysm: store it (or form SiLU*up)
                if (P.y == nullptr) {
                    const SiluOut so{A.a, A.I};
                    silu_block_rows_max(M, static_cast<int>(tch), etid, so, A.amax_w,
                                        [&](int m, int j0, float (&gg)[8], float (&uu)[8]) {
                                            const uint16_t *row = ysm + m * kBM;
                                            unpack8(*reinterpret_cast<const uint4 *>(row + j0), gg);
                                            unpack8(*reinterpret_cast<const uint4 *>(row + 64 + j0), uu);
                                        });
                } else {
                    const int nvalid = min(kBM, N - static_cast<int>(tch * kBM));
                    for (int v = etid; v < M * 16; v += 128) {
                        const int m = v >> 4, cv = v & 15;
                        if (cv * 8 < nvalid)
                            *reinterpret_cast<uint4 *>(P.y + static_cast<int64_t>(m) * N +
                                                       tch * kBM + cv * 8) =
                                *reinterpret_cast<const uint4 *>(ysm + m * kBM + cv * 8);
                    }
                }
                named_bar_sync(1, 128);
            }
            if (p == kBlockPhases - 1)
                break; // the block's output is complete; nothing in this launch reads it
            barrier(); // B1, B3, B5: the GEMM's outputs are complete
            if (!ok)
                break;
            // ---- the row phase feeding GEMM p + 1
            if (p == 2) { // R3, spread over the grid
                grid_quant_f32(A.a, A.amax_w, M, A.I, A.q[3], A.s[3], g, G, etid);
            } else {
                for (int m = static_cast<int>(g); m < M; m += static_cast<int>(G)) {
                    if (p == 0) // R1
                        row_quant_bf16<NV>(A.attn + static_cast<int64_t>(m) * A.H, A.sinv_o, A.H,
                                           A.q[1] + static_cast<int64_t>(m) * A.H, A.s[1] + m,
                                           etid, shf);
                    else // R2: h = bf16(o + x), smoothed RMSNorm + quant
                        row_rmsnorm<NV>(A.g[1].y + static_cast<int64_t>(m) * A.H, true,
                                        A.x + static_cast<int64_t>(m) * A.H,
                                        A.h + static_cast<int64_t>(m) * A.H, A.g2, A.eps, A.H,
                                        A.q[2] + static_cast<int64_t>(m) * A.H, A.s[2] + m, etid,
                                        shd, shf);
                }
            }
            barrier(); // B2, B4, B6
        }
        // a CTA that gave up still arrives at the barriers it skipped, so no other CTA waits
        // for it in vain
        if (etid == 0)
            while (nbar < kBlockBarriers) {
                atomicAdd(A.bar, 1ull);
                ++nbar;
            }
    }
    __syncwarp();
    if (warp == 1)
        tmem_relinquish();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::kTmemCols);
    }
}

} // namespace w8a8
