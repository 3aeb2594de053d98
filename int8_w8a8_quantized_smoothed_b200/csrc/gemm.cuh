// INT8 x INT8 -> INT32 GEMM on the 5th-generation tensor cores (tcgen05.mma kind::i8) with
// the dequantization epilogue y = bf16((float(acc) * s_tok[m]) * s_ch[n]) fused; with the
// template flag F8 the same kernels run the FP8 variant, E4M3 x E4M3 -> binary32
// (kind::f8f6f4), the epilogue then scaling the binary32 accumulator.
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
//
// Fused SiLU(gate)*up epilogue (template flag SILU), for the gate|up projection of a Llama
// MLP: the weight's rows are interleaved in blocks of 64 (gate channels 64b..64b+63, then up
// channels 64b..64b+63), so every 128-row group of weight rows holds the gate and up rows of
// the same 64 output channels. The epilogue rounds both dequantized values to bf16 (exactly
// what the plain epilogue stores), forms a = silu(g) * u in binary32 as the SiLU*up row
// kernel does, and stores a; a following row pass takes each token's max |a| and quantizes
// (to int8, or to E4M3 for FP8 operands; the FP8 form has no cluster split-K variant).
#pragma once

#include "ptx.cuh"
#include "rowquant.cuh"
#include "rowpass.cuh"

namespace w8a8 {

constexpr int kGemmThreads = 192;
constexpr int kMaxClusterSize = 8; // portable thread-block cluster size
constexpr int kBM = 128;  // MMA M: TMEM lanes
constexpr int kBK = 128;  // bytes of K per pipeline stage (one 128B swizzle row)
constexpr int kUmmaK = 32; // K of one kind::i8 MMA

// Output of the fused SiLU*up epilogue: a [M, I] binary32. With amax non-null (the small-M
// kernels), also the max |a| of every (token, group of 64 output channels): amax[m * (I / 64)
// + group], from which the quantization pass takes each token's scale without re-reading
// the row.
struct SiluOut {
    float *a;
    int I;
    float *amax = nullptr;
};

// The residual RMSNorm tail of the decode GEMM (cluster split-K): with y [M, N] the GEMM's
// output, h = bf16(y + res) (written to h, which may alias res), then the smoothed RMSNorm of
// h with gamma' (gamma divided by the next layer's smoothing factors) quantized per token
// into q [M, N], s [M]. bar: two zero-initialized counter words (tickets, then departures).
struct RowNormOut {
    const uint16_t *res = nullptr;
    uint16_t *h = nullptr;
    const float *gamma = nullptr;
    float eps = 0.0f;
    int8_t *q = nullptr;
    float *s = nullptr;
    unsigned int *bar = nullptr;
};

__device__ __forceinline__ float bf16_round(float f)
{
    return __uint_as_float(bf16_bits(f) << 16);
}

// One thread's row: 32 gate columns (rg, channel scales scg) and the 32 up columns of the
// same output channels (ru, scu) -> a = silu(bf16(g)) * bf16(u), stored at dst (32 floats,
// 16-byte stores).
template <bool F8 = false>
__device__ __forceinline__ void silu_row_chunk(const uint32_t (&rg)[32], const uint32_t (&ru)[32],
                                                float st, const float *scg, const float *scu,
                                                float *__restrict__ dst)
{
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float g[8], u[8], a[8];
        const float4 g0 = reinterpret_cast<const float4 *>(scg)[2 * e];
        const float4 g1 = reinterpret_cast<const float4 *>(scg)[2 * e + 1];
        const float4 u0 = reinterpret_cast<const float4 *>(scu)[2 * e];
        const float4 u1 = reinterpret_cast<const float4 *>(scu)[2 * e + 1];
        const float cg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
        const float cu[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            g[i] = dequant_acc<F8>(rg[8 * e + i], st, cg[i]);
            u[i] = dequant_acc<F8>(ru[8 * e + i], st, cu[i]);
        }
#pragma unroll
        for (int i = 0; i < 8; i += 2) { // to bf16 and back, two values per conversion
            bf16_round2(g[i], g[i + 1]);
            bf16_round2(u[i], u[i + 1]);
        }
        silu_mul8(g, u, a);
        reinterpret_cast<float4 *>(dst)[2 * e] = make_float4(a[0], a[1], a[2], a[3]);
        reinterpret_cast<float4 *>(dst)[2 * e + 1] = make_float4(a[4], a[5], a[6], a[7]);
    }
}

// silu_row_chunk's 32 values of a, as 8 16-byte words instead of stores.
template <bool F8 = false>
__device__ __forceinline__ void silu_row_chunk_regs(const uint32_t (&rg)[32],
                                                    const uint32_t (&ru)[32], float st,
                                                    const float *scg, const float *scu,
                                                    uint4 (&out)[8])
{
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float g[8], u[8], a[8];
        const float4 g0 = reinterpret_cast<const float4 *>(scg)[2 * e];
        const float4 g1 = reinterpret_cast<const float4 *>(scg)[2 * e + 1];
        const float4 u0 = reinterpret_cast<const float4 *>(scu)[2 * e];
        const float4 u1 = reinterpret_cast<const float4 *>(scu)[2 * e + 1];
        const float cg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
        const float cu[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            g[i] = dequant_acc<F8>(rg[8 * e + i], st, cg[i]);
            u[i] = dequant_acc<F8>(ru[8 * e + i], st, cu[i]);
        }
#pragma unroll
        for (int i = 0; i < 8; i += 2) { // to bf16 and back, two values per conversion
            bf16_round2(g[i], g[i + 1]);
            bf16_round2(u[i], u[i + 1]);
        }
        silu_mul8(g, u, a);
        out[2 * e] = make_uint4(__float_as_uint(a[0]), __float_as_uint(a[1]),
                                __float_as_uint(a[2]), __float_as_uint(a[3]));
        out[2 * e + 1] = make_uint4(__float_as_uint(a[4]), __float_as_uint(a[5]),
                                    __float_as_uint(a[6]), __float_as_uint(a[7]));
    }
}

// Producer tail of an mbarrier ring: waits until the consumer has released the last
// min(issued, stages) stages, i.e. until the empty-barrier phase that each of the last
// issued iterations j completes (parity (j / stages) & 1) has completed.
__device__ __forceinline__ void drain_ring(uint32_t bar_empty, uint32_t issued, uint32_t stages,
                                           unsigned long long limit_ns)
{
    for (uint32_t j = (issued > stages ? issued - stages : 0); j < issued; ++j)
        if (!mbar_wait(bar_empty + 8 * (j % stages), (j / stages) & 1u, limit_ns))
            return;
}

// ---------------------------------------------------------------- prefill (persistent)
//
// gemm_prefill_kernel: one CTA per 128 x BN output tile (BN = 128 or 256), two TMEM
// accumulators so the epilogue of tile t overlaps the MMAs of tile t+1.
//
// gemm_prefill_pair_kernel: a cluster of two CTAs per 256 x 256 tile with the 2-SM MMA
// (cta_group::2). Each CTA loads only its 128-row halves of A and B, and the pair's tensor
// cores share them, so per SM the shared-memory traffic (TMA writes plus operand reads) is
// two thirds of a one-CTA 128 x 256 tile's for the same MACs: the one-CTA kernel is bound by
// that traffic, not by DRAM or the tensor pipe.

template <int BN, int STAGES> struct PrefillCfg {
    static constexpr int kABytes = kBM * kBK;
    static constexpr int kBBytes = BN * kBK;
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kBarOff = STAGES * kStageBytes;
    // full[S], empty[S], tmem_full[2], tmem_empty[2], tmem slot; then each epilogue warp's
    // channel scales of two tiles [4][2][BN]
    static constexpr int kSchOff = (kBarOff + (2 * STAGES + 4) * 8 + 16 + 15) & ~15;
    static constexpr int kSmemBytes = kSchOff + 4 * 2 * BN * 4 + 1024;
    static constexpr int kTmemCols = 2 * BN;
    static_assert(kTmemCols <= 512, "two accumulators must fit TMEM");
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

// Tile order: groups of kGroupM row-tiles, column-major inside a group, so CTAs running
// at the same time share A row-panels and B column-panels in L2.
constexpr int kGroupM = 16;

__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int group_m, int &mb,
                                            int &nb)
{
    const int per_group = group_m * num_n;
    const int group = tile / per_group;
    const int first_m = group * group_m;
    const int gm = min(group_m, num_m - first_m);
    const int local = tile - group * per_group;
    mb = first_m + local % gm;
    nb = local / gm;
}

__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int &mb, int &nb)
{
    tile_coords(tile, num_m, num_n, kGroupM, mb, nb);
}

// Dequantizes 32 accumulator columns of one output row and stores them as bf16 (16-byte
// stores); also the raw accumulator words when acc_out is given. sc: the 32 channel scales of
// these columns, in shared memory.
template <bool F8>
__device__ __forceinline__ void store_row_chunk(const uint32_t (&r)[32], int row, int n0, int N,
                                                float st, const float *sc,
                                                uint16_t *__restrict__ y,
                                                int32_t *__restrict__ acc_out)
{
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        const int n = n0 + 8 * g;
        if (n < N) {
            const float4 c0 = reinterpret_cast<const float4 *>(sc)[2 * g];
            const float4 c1 = reinterpret_cast<const float4 *>(sc)[2 * g + 1];
            const float cs[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
            float f[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                f[i] = dequant_acc<F8>(r[8 * g + i], st, cs[i]);
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

// The bf16 words of 32 dequantized accumulator columns of one output row (4 x 16 bytes).
template <bool F8>
__device__ __forceinline__ void dequant_chunk_bf16(const uint32_t (&r)[32], float st,
                                                   const float *sc, uint4 *o)
{
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        const float4 c0 = reinterpret_cast<const float4 *>(sc)[2 * g];
        const float4 c1 = reinterpret_cast<const float4 *>(sc)[2 * g + 1];
        const float cs[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        float f[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            f[i] = dequant_acc<F8>(r[8 * g + i], st, cs[i]);
        o[g] = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                          pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
    }
}

// The int32 accumulators of 32 columns of one output row, written as they are (the check
// output): columns at or past N are skipped in groups of 8 (N % 8 == 0).
__device__ __forceinline__ void store_acc_chunk(const uint32_t (&r)[32], int row, int n0, int N,
                                                int32_t *__restrict__ acc_out)
{
#pragma unroll
    for (int g = 0; g < 4; ++g)
        if (n0 + 8 * g < N) {
            int4 *ap = reinterpret_cast<int4 *>(acc_out + static_cast<int64_t>(row) * N + n0 + 8 * g);
            ap[0] = make_int4(r[8 * g + 0], r[8 * g + 1], r[8 * g + 2], r[8 * g + 3]);
            ap[1] = make_int4(r[8 * g + 4], r[8 * g + 5], r[8 * g + 6], r[8 * g + 7]);
        }
}

// One warp's 32 output rows of 128 bytes each (lane l holds row l's 8 16-byte chunks in v),
// stored so that every store instruction writes 4 rows x 128 contiguous bytes instead of 32
// rows x 16: the chunks pass through the warp's 4 KB shared buffer, their slots XOR-swizzled
// by row so that neither the writes nor the reads conflict. dst: row 0's first byte; stride:
// bytes from row to row; rows at or past rows_valid and bytes at or past bytes_valid (a
// multiple of 16) of a row are not written.
__device__ __forceinline__ void warp_store_rows(uint4 *stage, const uint4 (&v)[8], int lane,
                                                char *dst, int64_t stride, int rows_valid,
                                                int bytes_valid)
{
#pragma unroll
    for (int j = 0; j < 8; ++j)
        stage[lane * 8 + (j ^ (lane & 7))] = v[j];
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int r = i * 4 + (lane >> 3), j = lane & 7;
        if (r < rows_valid && j * 16 < bytes_valid)
            *reinterpret_cast<uint4 *>(dst + r * stride + j * 16) = stage[r * 8 + (j ^ (r & 7))];
    }
    __syncwarp();
}

// Scales of one output tile for the prefill epilogues, fetched one tile ahead by each
// epilogue warp so that their global-memory latency overlaps the current tile's work: the BN
// channel scales (BN / 32 per lane, published to the warp's own shared-memory copy) and the
// token scale of the lane's own row. Warp-private, so no barrier beyond __syncwarp is needed.
template <int BN> struct TileScales {
    float sc[BN / 32];
    float st;
    __device__ __forceinline__ void fetch(const float *__restrict__ s_ch,
                                          const float *__restrict__ s_tok, int n0, int N, int row,
                                          int M, int lane)
    {
#pragma unroll
        for (int j = 0; j < BN / 32; ++j) {
            const int n = n0 + lane + 32 * j;
            sc[j] = n < N ? __ldg(s_ch + n) : 0.0f;
        }
        st = row < M ? __ldg(s_tok + row) : 0.0f;
    }
    __device__ __forceinline__ void publish(float *sh, int lane) const
    {
#pragma unroll
        for (int j = 0; j < BN / 32; ++j)
            sh[lane + 32 * j] = sc[j];
        __syncwarp();
    }
};

template <int BN, int STAGES, bool SILU = false, bool F8 = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_prefill_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB, const float *__restrict__ s_tok,
                        const float *__restrict__ s_ch, int M, int N, int K,
                        uint16_t *__restrict__ y, int32_t *__restrict__ acc_out, SiluOut so,
                        int prefetch_static, unsigned long long limit_ns)
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
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t *>(tslot_ptr);

    if (warp == 0) {
        if (lane == 0) {
            // With prefetch_static the weight (B) tiles of the first ring of stages are
            // requested before waiting for the previous kernel: the caller guarantees no
            // kernel still in flight writes the weights. Activations always come after.
            uint32_t npre = 0;
            if (prefetch_static) {
                for (int tile = blockIdx.x; tile < tiles && npre < STAGES; tile += gridDim.x) {
                    int mb, nb;
                    tile_coords(tile, num_m, num_n, mb, nb);
                    for (int kb = 0; kb < kblocks && npre < STAGES; ++kb, ++npre) {
                        mbar_expect_tx(bar_full + 8 * npre, Cfg::kStageBytes);
                        tma_load_2d(sB + npre * Cfg::kBBytes, &tmB, bar_full + 8 * npre, kb * kBK,
                                    nb * BN);
                    }
                }
            }
            pdl_wait();
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
                int mb, nb;
                tile_coords(tile, num_m, num_n, mb, nb);
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const uint32_t s = it % STAGES;
                    if (it < npre) { // weights already requested; add the activation tile
                        tma_load_2d(sA + s * Cfg::kABytes, &tmA, bar_full + 8 * s, kb * kBK,
                                    mb * kBM);
                        continue;
                    }
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
            // Producer tail: wait until the MMA warp has released the last ring of stages,
            // so no load and no tcgen05.commit arrival is still in flight when the CTA exits.
            if (ok)
                drain_ring(bar_empty, it, STAGES, limit_ns);
            // every stage consumed: the next kernel in the stream may launch now
            pdl_launch_dependents();
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_8bit<F8>(kBM, BN);
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
                        umma_8bit<F8>(d, sw128_kmajor_desc(a0 + k * kUmmaK),
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
        pdl_wait(); // s_tok comes from the previous kernel; y may still be read by it
        const int quarter = warp & 3;
        float *sh_sch = reinterpret_cast<float *>(smem + Cfg::kSchOff) + (warp - 2) * 2 * BN;
        TileScales<BN> nxt;
        auto fetch = [&](int tile) {
            int mb, nb;
            tile_coords(tile, num_m, num_n, mb, nb);
            nxt.fetch(s_ch, s_tok, nb * BN, N, mb * kBM + quarter * 32 + lane, M, lane);
        };
        if (static_cast<int>(blockIdx.x) < tiles)
            fetch(blockIdx.x);
        uint32_t t = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++t) {
            int mb, nb;
            tile_coords(tile, num_m, num_n, mb, nb);
            const uint32_t buf = t & 1u;
            const uint32_t aph = (t >> 1) & 1u;
            // this tile's scales to the warp's shared memory (the buffer of tile t-2 is free:
            // the warp synchronized after it), the next tile's requested
            nxt.publish(sh_sch + buf * BN, lane);
            const float st = nxt.st;
            if (tile + static_cast<int>(gridDim.x) < tiles)
                fetch(tile + gridDim.x);
            if (!mbar_wait(bar_tfull + 8 * buf, aph, limit_ns))
                break;
            tc_fence_after();
            const int row = mb * kBM + quarter * 32 + lane;
            const bool row_ok = row < M;
            const uint32_t tbase = tmem_base + buf * BN + (static_cast<uint32_t>(quarter * 32) << 16);
            if constexpr (SILU) {
                // gate chunk cg and up chunk cg + 2 hold the same 32 output channels
#pragma unroll 1
                for (int p = 0; p < BN / 64; ++p) {
                    const int cg = (p >> 1) * 4 + (p & 1);
                    const int ch0 = nb * (BN / 2) + (p >> 1) * 64 + (p & 1) * 32;
                    uint32_t rg[32], ru[32];
                    tmem_ld_32x32b_x32(tbase + cg * 32, rg);
                    tmem_ld_32x32b_x32(tbase + (cg + 2) * 32, ru);
                    tmem_ld_wait();
                    if (row_ok && ch0 < so.I)
                        silu_row_chunk<F8>(rg, ru, st, sh_sch + buf * BN + cg * 32,
                                       sh_sch + buf * BN + (cg + 2) * 32,
                                       so.a + static_cast<int64_t>(row) * so.I + ch0);
                }
            } else {
#pragma unroll 1
                for (int c = 0; c < BN / 32; c += 2) {
                    // two chunks requested together: one wait for their latency
                    uint32_t r[32], r2[32];
                    tmem_ld_32x32b_x32(tbase + c * 32, r);
                    tmem_ld_32x32b_x32(tbase + (c + 1) * 32, r2);
                    tmem_ld_wait();
                    if (row_ok)
                        store_row_chunk<F8>(r2, row, nb * BN + (c + 1) * 32, N, st,
                                            sh_sch + buf * BN + (c + 1) * 32, y, acc_out);
                    if (row_ok)
                        store_row_chunk<F8>(r, row, nb * BN + c * 32, N, st,
                                        sh_sch + buf * BN + c * 32, y, acc_out);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar_tempty + 8 * buf);
        }
    }
    __syncwarp();
    if (warp == 1)
        tmem_relinquish(); // after the work, as the allocator's permit protocol expects
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::kTmemCols);
    }
}

// ---------------------------------------------------------------- prefill, CTA pairs

// ---- stream-K: U units split evenly over G workers, worker g taking [g U / G, (g+1) U / G)

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
    int64_t t;    // block (decode: channel block t / tiles, token tile t % tiles) or tile
    int kb0, kb1; // k-block range [kb0, kb1)
};

// The segment of [u, u1) that starts at u.
__device__ __forceinline__ SkSegment sk_segment(int64_t u, int64_t u1, int KB)
{
    SkSegment sg;
    sg.t = u / KB;
    sg.kb0 = static_cast<int>(u - sg.t * KB);
    const int64_t left = u1 - u;
    sg.kb1 = static_cast<int>(min(static_cast<int64_t>(KB), sg.kb0 + left));
    return sg;
}

template <int STAGES> struct PairCfg {
    static constexpr int kHalf = 128;             // rows of A and of B per CTA
    static constexpr int kABytes = kHalf * kBK;   // 16 KB
    static constexpr int kBBytes = kHalf * kBK;   // 16 KB
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kBarOff = STAGES * kStageBytes;
    // full[S], empty[S], tmem_full[2], tmem_empty[2], tmem slot (16 B), the stream-K fixup
    // barrier and a word for the epilogue group
    static constexpr int kFixBarOff = kBarOff + (2 * STAGES + 4) * 8 + 16;
    static constexpr int kSchOff = (kFixBarOff + 16 + 15) & ~15;
    // channel scales [4 warps][2][256], then each epilogue warp's 4 KB store staging buffer
    static constexpr int kOutOff = kSchOff + 4 * 2 * 256 * 4;
    static constexpr int kSmemBytes = kOutOff + 4 * 4096 + 1024;
    static constexpr int kTmemCols = 512;         // two 128 x 256 accumulators per CTA
    // stream-K: a CTA's partial of a split tile, 128 rows x 256 columns of accumulator words,
    // stored as [64 column quads][128 rows][4] so that the rows of a warp are consecutive
    static constexpr int kPartBytes = kHalf * 256 * 4;
    static constexpr int kPartHalf = kPartBytes / 2; // columns 0..127 or 128..255
    static constexpr int kMaxContrib = 3;            // contributors per split tile
    static_assert(kMaxContrib * kPartHalf <= STAGES * kStageBytes,
                  "the fixup stages contributor halves in the idle ring");
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

// Persistent 256 x 256 tiles on CTA pairs (cta_group::2). Two schedules:
//   tile-persistent (ws_flag == nullptr): pair p takes tiles p, p + P, ...;
//   stream-K (ws_flag != nullptr): the tiles x k-blocks units are split evenly over the P
//     pairs; a pair walks its range in segments (the part inside one tile). A tile split
//     between pairs is finished by its owner, the pair holding its k-block 0 (that segment is
//     the owner's last, so it completes last); the later pairs sharing the tile (at most
//     kMaxContrib; the host sizes shares so) store their int32 partial (binary32 for FP8)
//     halves in their CTA's workspace slot and raise the CTA's flag. The owner, whose ring is
//     idle by then, brings the contributors' column halves into it with bulk copies, adds
//     them to its accumulator chunk by chunk and finishes the tile; it lowers the flags, so
//     the workspace is ready for the next call.
template <int STAGES, bool SILU = false, bool F8 = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_prefill_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                             const __grid_constant__ CUtensorMap tmB,
                             const float *__restrict__ s_tok, const float *__restrict__ s_ch,
                             int M, int N, int K, uint16_t *__restrict__ y,
                             int32_t *__restrict__ acc_out, SiluOut so,
                             int32_t *__restrict__ ws_part, unsigned int *__restrict__ ws_flag,
                             int group_m, int prefetch_static, unsigned long long limit_ns)
{
    using Cfg = PairCfg<STAGES>;
    constexpr int TN = 256, TM = 256;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sA = sbase;
    const uint32_t sB = sbase + STAGES * Cfg::kABytes;
    const uint32_t bar_full = sbase + Cfg::kBarOff;     // used in the even CTA
    const uint32_t bar_empty = bar_full + 8 * STAGES;   // both CTAs
    const uint32_t bar_tfull = bar_empty + 8 * STAGES;  // both CTAs
    const uint32_t bar_tempty = bar_tfull + 16;         // used in the even CTA
    const uint32_t tslot = bar_tempty + 16;
    const uint32_t bar_fix = sbase + Cfg::kFixBarOff;
    uint32_t *tslot_ptr = reinterpret_cast<uint32_t *>(smem + Cfg::kBarOff + (2 * STAGES + 4) * 8);
    volatile uint32_t *sh_word = reinterpret_cast<volatile uint32_t *>(smem + Cfg::kFixBarOff + 8);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank(); // 0: leader (issues the MMAs), 1: peer
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;
    const int num_m = (M + TM - 1) / TM;
    const int num_n = (N + TN - 1) / TN;
    const int tiles = num_m * num_n;
    const int kblocks = (K + kBK - 1) / kBK;
    const bool sk = ws_flag != nullptr;
    const int64_t U = static_cast<int64_t>(tiles) * kblocks;
    const int64_t u_begin = sk ? (static_cast<int64_t>(pair) * U) / npairs : pair;
    const int64_t u_end = sk ? (static_cast<int64_t>(pair + 1) * U) / npairs : tiles;
    // The segments of this pair's work, in order: (tile, k-blocks [kb0, kb1)). cursor starts
    // at u_begin; every role walks the same sequence.
    auto next_seg = [&](int64_t &cursor, int &t, int &kb0, int &kb1) -> bool {
        if (cursor >= u_end)
            return false;
        if (sk) {
            const SkSegment sg = sk_segment(cursor, u_end, kblocks);
            t = static_cast<int>(sg.t);
            kb0 = sg.kb0;
            kb1 = sg.kb1;
            cursor += kb1 - kb0;
        } else {
            t = static_cast<int>(cursor);
            kb0 = 0;
            kb1 = kblocks;
            cursor += npairs;
        }
        return true;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_tfull + 8 * b, 1);
            mbar_init(bar_tempty + 8 * b, 8); // 4 epilogue warps in each CTA of the pair
        }
        mbar_init(bar_fix, 1);
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    // Both CTAs' barriers are initialized before either uses the other's, and both CTAs are
    // running before the pair allocates tensor memory together (allocating first, with the
    // pair launched early behind the previous kernel, intermittently never returned).
    cluster_sync();
    if (warp == 1) {
        tmem_alloc_pair(tslot, Cfg::kTmemCols);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t *>(tslot_ptr);

    if (warp == 0) {
        if (lane == 0) {
            const uint32_t full0 = map_peer_smem(bar_full, 0); // the leader's full barriers
            uint32_t npre = 0;
            if (prefetch_static) {
                int64_t cur = u_begin;
                int t, kb0, kb1;
                while (npre < STAGES && next_seg(cur, t, kb0, kb1)) {
                    int mb, nb;
                    tile_coords(t, num_m, num_n, group_m, mb, nb);
                    for (int kb = kb0; kb < kb1 && npre < STAGES; ++kb, ++npre) {
                        if (rank == 0)
                            mbar_expect_tx(bar_full + 8 * npre, 2 * Cfg::kStageBytes);
                        tma_load_2d_pair(sB + npre * Cfg::kBBytes, &tmB, full0 + 8 * npre,
                                         kb * kBK, nb * TN + rank * Cfg::kHalf);
                    }
                }
            }
            pdl_wait();
            uint32_t it = 0;
            bool ok = true;
            int64_t cur = u_begin;
            int t, kb0, kb1;
            while (ok && next_seg(cur, t, kb0, kb1)) {
                int mb, nb;
                tile_coords(t, num_m, num_n, group_m, mb, nb);
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const uint32_t s = it % STAGES;
                    if (it < npre) {
                        tma_load_2d_pair(sA + s * Cfg::kABytes, &tmA, full0 + 8 * s, kb * kBK,
                                         mb * TM + rank * Cfg::kHalf);
                        continue;
                    }
                    const uint32_t ph = (it / STAGES) & 1u;
                    if (!mbar_wait(bar_empty + 8 * s, ph ^ 1u, limit_ns)) {
                        ok = false;
                        break;
                    }
                    if (rank == 0)
                        mbar_expect_tx(bar_full + 8 * s, 2 * Cfg::kStageBytes);
                    tma_load_2d_pair(sA + s * Cfg::kABytes, &tmA, full0 + 8 * s, kb * kBK,
                                     mb * TM + rank * Cfg::kHalf);
                    tma_load_2d_pair(sB + s * Cfg::kBBytes, &tmB, full0 + 8 * s, kb * kBK,
                                     nb * TN + rank * Cfg::kHalf);
                }
            }
            // Producer tail (each CTA): the leader's multicast commits have released every
            // stage of this CTA's ring before it may exit (a stage wait that ran out leaves
            // it at once).
            if (ok)
                drain_ring(bar_empty, it, STAGES, limit_ns);
            pdl_launch_dependents(); // the pair's main loop is done in this CTA
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            constexpr uint32_t idesc = idesc_8bit<F8>(TM, TN);
            uint32_t it = 0, seg = 0;
            bool ok = true;
            int64_t cur = u_begin;
            int t, kb0, kb1;
            while (ok && next_seg(cur, t, kb0, kb1)) {
                const uint32_t buf = seg & 1u;
                const uint32_t aph = (seg >> 1) & 1u;
                ++seg;
                if (!mbar_wait(bar_tempty + 8 * buf, aph ^ 1u, limit_ns))
                    break;
                tc_fence_after();
                const uint32_t d = tmem_base + buf * TN;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
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
                        umma_8bit_pair<F8>(d, sw128_kmajor_desc(a0 + k * kUmmaK),
                                           sw128_kmajor_desc(b0 + k * kUmmaK), idesc,
                                           (kb > kb0 || k > 0) ? 1u : 0u);
                    umma_commit_pair(bar_empty + 8 * s, 0x3); // frees the stage in both CTAs
                }
                if (ok)
                    umma_commit_pair(bar_tfull + 8 * buf, 0x3);
            }
        }
    } else {
        // epilogue warps 2..5: this CTA's 128 accumulator rows of the 256-row tile
        pdl_wait();
        const int quarter = warp & 3;
        const int etid = threadIdx.x - 64;
        const int rl = quarter * 32 + lane; // row within this CTA's half of the tile
        const uint32_t tempty0 = map_peer_smem(bar_tempty, 0);
        const int row_in_tile = static_cast<int>(rank) * Cfg::kHalf + rl;
        float *sh_sch = reinterpret_cast<float *>(smem + Cfg::kSchOff) + (warp - 2) * 2 * TN;
        const int4 *ring = reinterpret_cast<const int4 *>(smem);
        uint4 *stage_w = reinterpret_cast<uint4 *>(smem + Cfg::kOutOff) + (warp - 2) * 256;
        int4 *my_slot = sk ? reinterpret_cast<int4 *>(ws_part) +
                                 static_cast<int64_t>(blockIdx.x) * (Cfg::kPartBytes / 16)
                           : nullptr;
        TileScales<TN> nxt;
        auto fetch = [&](int tile) {
            int mb, nb;
            tile_coords(tile, num_m, num_n, group_m, mb, nb);
            nxt.fetch(s_ch, s_tok, nb * TN, N, mb * TM + row_in_tile, M, lane);
        };
        int64_t peek = u_begin, cur = u_begin;
        int pt, pk0, pk1, t, kb0, kb1;
        if (next_seg(peek, pt, pk0, pk1))
            fetch(pt);
        uint32_t seg = 0;
        while (next_seg(cur, t, kb0, kb1)) {
            int mb, nb;
            tile_coords(t, num_m, num_n, group_m, mb, nb);
            const uint32_t buf = seg & 1u;
            const uint32_t aph = (seg >> 1) & 1u;
            ++seg;
            // this segment's scales to the warp's shared memory, the next segment's requested
            nxt.publish(sh_sch + buf * TN, lane);
            const float st = nxt.st;
            if (next_seg(peek, pt, pk0, pk1))
                fetch(pt);
            if (!mbar_wait(bar_tfull + 8 * buf, aph, limit_ns))
                break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + buf * TN + (static_cast<uint32_t>(quarter * 32) << 16);
            if (kb0 > 0) {
                // a later piece of a split tile: the partial to this CTA's slot, then its flag
#pragma unroll 1
                for (int c = 0; c < TN / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tbase + c * 32, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        __stcg(my_slot + (c * 8 + i) * Cfg::kHalf + rl,
                               make_int4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive_cluster(tempty0 + 8 * buf);
                named_bar_sync(1, 128);
                if (etid == 0) {
                    fence_acq_rel_gpu();
                    st_relaxed_gpu(ws_flag + blockIdx.x, 1u);
                }
                continue;
            }
            // The tile's first piece: whole, or owned with ncon later pieces to add.
            int ncon = 0;
            if (kb1 < kblocks) {
                ncon = static_cast<int>(
                    sk_owner_of(static_cast<int64_t>(t) * kblocks + kblocks - 1, U, npairs) - pair);
                if (etid == 0) {
                    bool all = true;
                    for (int j = 1; j <= ncon && all; ++j) {
                        const unsigned int *f = ws_flag + 2 * (pair + j) + rank;
                        if (ld_acquire_gpu(f) == 0u) {
                            const uint64_t t0 = globaltimer_ns();
                            while (ld_acquire_gpu(f) == 0u) {
                                if (globaltimer_ns() - t0 > limit_ns) {
                                    flag_timeout();
                                    all = false;
                                    break;
                                }
                            }
                        }
                    }
                    fence_proxy_async_global(); // the partials came from generic stores
                    *sh_word = all ? 1u : 0u;
                }
                named_bar_sync(1, 128);
                if (*sh_word == 0u)
                    ncon = -1; // a wait ran out: leave the tile unwritten
            }
            const int row = mb * TM + row_in_tile;
            const bool row_ok = row < M && ncon >= 0;
            const int wrow0 = mb * TM + static_cast<int>(rank) * Cfg::kHalf + quarter * 32;
            // nadd is uniform over the epilogue group (it guards a named barrier); a fixup wait
            // that runs out only keeps this thread from storing
            const int nadd = ncon > 0 ? ncon : 0;
            // adds the contributors' words of chunk c (staged in the ring for half h) to r
            auto add_parts = [&](uint32_t (&r)[32], int c, int h) {
                for (int j = 0; j < nadd; ++j) {
                    const int4 *src = ring + j * (Cfg::kPartHalf / 16) +
                                      (c * 8 - h * 32) * Cfg::kHalf + rl;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int4 v = src[i * Cfg::kHalf];
                        r[4 * i] = acc_add<F8>(r[4 * i], static_cast<uint32_t>(v.x));
                        r[4 * i + 1] = acc_add<F8>(r[4 * i + 1], static_cast<uint32_t>(v.y));
                        r[4 * i + 2] = acc_add<F8>(r[4 * i + 2], static_cast<uint32_t>(v.z));
                        r[4 * i + 3] = acc_add<F8>(r[4 * i + 3], static_cast<uint32_t>(v.w));
                    }
                }
            };
            for (int h = 0; h < 2; ++h) {
                bool ok_h = ncon >= 0;
                if (nadd > 0) {
                    // the contributors' column half h into the (idle) ring
                    if (etid == 0) {
                        fence_proxy_async_smem(); // earlier reads of the ring, before the copies
                        mbar_expect_tx(bar_fix, static_cast<uint32_t>(ncon) * Cfg::kPartHalf);
                        for (int j = 0; j < ncon; ++j)
                            bulk_load_g2s(sbase + j * Cfg::kPartHalf,
                                          ws_part + (static_cast<int64_t>(2 * (pair + 1 + j) + rank) *
                                                         Cfg::kPartBytes + h * Cfg::kPartHalf) / 4,
                                          Cfg::kPartHalf, bar_fix);
                    }
                    if (!mbar_wait(bar_fix, static_cast<uint32_t>(h), limit_ns))
                        ok_h = false;
                }
                // the warp's 32 rows go out together (staged stores): which of them are rows
                // of the output, and whether every lane's values are good
                const bool ok_w = __all_sync(0xffffffffu, ok_h) && ncon >= 0;
                const int rows_valid = ok_w ? min(32, M - wrow0) : 0;
                if constexpr (SILU) {
#pragma unroll 1
                    for (int p = 2 * h; p < 2 * h + 2; ++p) {
                        const int cg = (p >> 1) * 4 + (p & 1);
                        const int ch0 = nb * (TN / 2) + (p >> 1) * 64 + (p & 1) * 32;
                        uint32_t rg[32], ru[32];
                        tmem_ld_32x32b_x32(tbase + cg * 32, rg);
                        tmem_ld_32x32b_x32(tbase + (cg + 2) * 32, ru);
                        tmem_ld_wait();
                        if (nadd > 0) {
                            add_parts(rg, cg, h);
                            add_parts(ru, cg + 2, h);
                        }
                        uint4 v[8];
                        silu_row_chunk_regs<F8>(rg, ru, st, sh_sch + buf * TN + cg * 32,
                                                sh_sch + buf * TN + (cg + 2) * 32, v);
                        warp_store_rows(stage_w, v, lane,
                                        reinterpret_cast<char *>(so.a + static_cast<int64_t>(wrow0) * so.I + ch0),
                                        static_cast<int64_t>(so.I) * 4, rows_valid,
                                        min(128, (so.I - ch0) * 4));
                    }
                } else {
                    // the half's four chunks requested together: one wait for their latency
                    uint32_t r[4][32];
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc)
                        tmem_ld_32x32b_x32(tbase + (4 * h + cc) * 32, r[cc]);
                    tmem_ld_wait();
#pragma unroll
                    for (int c2 = 0; c2 < 2; ++c2) {
                        uint4 v[8];
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc) {
                            const int c = 4 * h + 2 * c2 + cc;
                            if (nadd > 0)
                                add_parts(r[2 * c2 + cc], c, h);
                            dequant_chunk_bf16<F8>(r[2 * c2 + cc], st, sh_sch + buf * TN + c * 32,
                                                   v + 4 * cc);
                            if (acc_out && row_ok && ok_h)
                                store_acc_chunk(r[2 * c2 + cc], row, nb * TN + c * 32, N, acc_out);
                        }
                        const int n0 = nb * TN + (2 * h + c2) * 64;
                        warp_store_rows(stage_w, v, lane,
                                        reinterpret_cast<char *>(y + static_cast<int64_t>(wrow0) * N + n0),
                                        static_cast<int64_t>(N) * 2, rows_valid, min(128, (N - n0) * 2));
                    }
                }
                if (nadd > 0)
                    named_bar_sync(1, 128); // every thread is done with this half in the ring
            }
            if (ncon > 0 && etid == 0) // the contributors' flags down for the next call
                for (int j = 1; j <= ncon; ++j)
                    st_relaxed_gpu(ws_flag + 2 * (pair + j) + rank, 0u);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_cluster(tempty0 + 8 * buf); // release the leader's accumulator
        }
    }
    __syncwarp();
    if (warp == 1)
        tmem_relinquish_pair(); // after the work, as the allocator's permit protocol expects
    // every MMA, commit and remote arrive of the pair is done before either CTA frees
    // its tensor memory or leaves
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (warp == 1)
        tmem_dealloc_pair(tmem_base, Cfg::kTmemCols);
}

// ---------------------------------------------------------------- decode (swap-AB)
//
// Work units are (channel block t, k-block kb) pairs in block-major order, U = NB * KB of
// them; a CTA owns a contiguous unit range and walks it in segments (the part of its range
// inside one channel block). Two schedules:
//
// CLUSTER (few channel blocks): grid (S, NB) with thread-block clusters of S CTAs along K;
//   CTA r of block t takes k-blocks [r KB / S, (r+1) KB / S). The S partial accumulators meet
//   in shared memory: each CTA writes its partial tile [token][128 channels] to its own (now
//   idle) stage buffers; CTA r owns tokens [r M / S, (r+1) M / S) and every other CTA adds
//   its rows for them into r's tile with one asynchronous bulk reduction (counted in bytes on
//   r's barrier); r then dequantizes and stores its rows. No global workspace.
//
// stream-K (many channel blocks): G persistent CTAs (one per SM) take equal contiguous
//   ranges [g U / G, (g+1) U / G), so every SM streams the same weight bytes. A block split
//   between CTAs has one owner, the segment holding k-block 0 (its CTA's last segment, so it
//   finishes last); the other segments (first segments of later CTAs) store their int32
//   partials in their CTA's workspace slot and raise the CTA's flag; the owner waits for the
//   flags of the later CTAs sharing its block (as soon as its own first segment is done, so
//   the partial sums are fetched while its MMAs still run), adds their partials, dequantizes,
//   stores and
//   lowers the flags so the workspace is ready for the next call.

// Token tiles per launch of the swap-AB kernel: M <= kDecodeMaxTiles * NT. Each channel block
// is computed once per token tile (tile tt holds tokens tt NT .. tt NT + NT - 1); a block's
// consecutive units walk its token tiles first, so the weight rows re-read for the second
// tile come from L2.
constexpr int kDecodeMaxTiles = 4;

template <int NT, int STAGES, int KPS, bool CLUSTER> struct DecodeCfg {
    static constexpr int kWBytes = kBM * kBK;  // one k-block of 128 weight rows
    static constexpr int kXBytes = NT * kBK;   // one k-block of NT token rows
    static constexpr int kStageBytes = KPS * (kWBytes + kXBytes);
    // stream-K stages its bf16 output tile [NT][128] for coalesced stores
    static constexpr int kYBytes = CLUSTER ? 0 : NT * kBM * 2;
    static constexpr int kYOff = STAGES * kStageBytes;
    static constexpr int kStokOff = kYOff + kYBytes; // fp32 token scales [tiles * NT]
    static constexpr int kBarOff = kStokOff + kDecodeMaxTiles * NT * 4;
    // full[S], empty[S], tmem_full[2], tmem_empty[2], tmem slot, flag word, then the
    // cluster reduction barrier
    static constexpr int kRedBarOff = kBarOff + (2 * STAGES + 4) * 8 + 32;
    static constexpr int kSmemBytes = kRedBarOff + 8 + 1024;
    static constexpr int kTmemCols = 2 * NT < 32 ? 32 : 2 * NT;
    static_assert(kXBytes % 1024 == 0, "token tile must keep stages 1024-byte aligned");
    static_assert(kTmemCols <= 512, "two accumulators must fit TMEM");
    static_assert(!CLUSTER || NT * kBM * 4 <= STAGES * kStageBytes,
                  "the cluster partial tile reuses the stage buffers");
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};


// The SiLU*up form of the final step of a block (see SiluOut): the block's 128 weight rows
// are gate rows 0..63 and up rows 64..127 of output channels [64 t, 64 t + 64); v8 = (token,
// group of 8 channels) vectors, 8 per token. gate_up(m, j0, g, u) gives the bf16-rounded gate
// and up values of channels j0 .. j0 + 7 of token m; tokens m0 .. m0 + mt - 1.
template <typename GateUp>
__device__ __forceinline__ void silu_block_rows(int m0, int mt, int t, int etid, const SiluOut &so,
                                                GateUp gate_up)
{
    // every lane of a warp runs the same trips (the group max is a shuffle over the 8 lanes
    // that hold one token's 64 channels)
    for (int base = 0; base < mt * 8; base += 128) {
        const int v = base + etid;
        const bool act = v < mt * 8;
        const int m = m0 + (v >> 3), j0 = (v & 7) * 8;
        float mx = 0.0f;
        if (act) {
            float g[8], u[8], a[8];
            gate_up(m, j0, g, u);
            silu_mul8(g, u, a);
            float *dst = so.a + static_cast<int64_t>(m) * so.I + static_cast<int64_t>(t) * 64 + j0;
            reinterpret_cast<float4 *>(dst)[0] = make_float4(a[0], a[1], a[2], a[3]);
            reinterpret_cast<float4 *>(dst)[1] = make_float4(a[4], a[5], a[6], a[7]);
#pragma unroll
            for (int i = 0; i < 8; ++i)
                mx = fmaxf(mx, fabsf(a[i]));
        }
        if (so.amax != nullptr) {
#pragma unroll
            for (int o = 1; o < 8; o <<= 1)
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            if (act && (v & 7) == 0)
                so.amax[static_cast<int64_t>(m) * (so.I / 64) + t] = mx;
        }
    }
}

template <int NT, int STAGES, int KPS, bool CLUSTER, bool SILU = false, bool F8 = false,
          int RNV = 0>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_decode_kernel(const __grid_constant__ CUtensorMap tmW,
                       const __grid_constant__ CUtensorMap tmX, const float *__restrict__ s_tok,
                       const float *__restrict__ s_ch, int M, int N, int K,
                       uint16_t *__restrict__ y, int32_t *__restrict__ acc_out,
                       int32_t *__restrict__ ws_part, unsigned int *__restrict__ ws_flag,
                       SiluOut so, RowNormOut rn, int prefetch_static, unsigned long long limit_ns)
{
    static_assert(!(SILU && F8 && CLUSTER), "the fused SiLU epilogue of the FP8 cluster split-K is not built");
    // RNV > 0: the residual RMSNorm tail, rows of up to 8 * 128 * RNV values (INT8 cluster
    // split-K with the plain epilogue only)
    static_assert(RNV == 0 || (CLUSTER && !SILU && !F8), "the RMSNorm tail is built for the INT8 cluster split-K");
    using Cfg = DecodeCfg<NT, STAGES, KPS, CLUSTER>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sW = sbase;                               // [STAGES][KPS][128 x 128 B]
    const uint32_t sX = sbase + STAGES * KPS * Cfg::kWBytes; // [STAGES][KPS][NT x 128 B]
    uint16_t *ysm = reinterpret_cast<uint16_t *>(smem + Cfg::kYOff);
    float *sh_stok = reinterpret_cast<float *>(smem + Cfg::kStokOff);
    const uint32_t bar_full = sbase + Cfg::kBarOff;
    const uint32_t bar_empty = bar_full + 8 * STAGES;
    const uint32_t bar_tfull = bar_empty + 8 * STAGES;
    const uint32_t bar_tempty = bar_tfull + 16;
    const uint32_t tslot = bar_tempty + 16;
    uint32_t *tslot_ptr = reinterpret_cast<uint32_t *>(smem + Cfg::kBarOff + (2 * STAGES + 4) * 8);
    volatile uint32_t *sh_word = tslot_ptr + 4;
    const uint32_t bar_red = sbase + Cfg::kRedBarOff;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int KB = (K + kBK - 1) / kBK;
    const int TT = (M + NT - 1) / NT;                  // token tiles
    const int64_t NB = ((N + kBM - 1) / kBM) * TT;     // blocks: (channel block, token tile)
    const int64_t U = NB * KB;
    const int64_t G = gridDim.x;
    const int64_t g = blockIdx.x;
    int64_t u_begin, u_end;
    if constexpr (CLUSTER) {
        const int64_t t = blockIdx.y;
        u_begin = t * KB + (g * KB) / G;
        u_end = t * KB + ((g + 1) * KB) / G;
    } else {
        u_begin = (g * U) / G;
        u_end = ((g + 1) * U) / G;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_tfull + 8 * b, 1);
            mbar_init(bar_tempty + 8 * b, 4);
        }
        if constexpr (CLUSTER)
            mbar_init(bar_red, 1);
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmW);
        tma_prefetch_desc(&tmX);
    }
    if (warp == 1) {
        tmem_alloc(tslot, Cfg::kTmemCols);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t *>(tslot_ptr);
    // Cluster split-K: an owner thread dequantizes 4 channels, the same 4 for every row it
    // handles; their scales are read when the epilogue starts, not after the reduction.
    float4 cl_sc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first(); // weights are streamed once
            // With prefetch_static the weight tiles of the first ring of stages are requested
            // before waiting for the previous kernel (the caller guarantees no kernel still
            // in flight writes the weights); token tiles always come after the wait.
            uint32_t npre = 0;
            if (prefetch_static) {
                for (int64_t u = u_begin; u < u_end && npre < STAGES;) {
                    const SkSegment sg = sk_segment(u, u_end, KB);
                    for (int kb = sg.kb0; kb < sg.kb1 && npre < STAGES; kb += KPS, ++npre) {
                        const int nk = min(KPS, sg.kb1 - kb);
                        mbar_expect_tx(bar_full + 8 * npre, nk * (Cfg::kWBytes + Cfg::kXBytes));
                        for (int j = 0; j < nk; ++j)
                            tma_load_2d_hint(sW + (npre * KPS + j) * Cfg::kWBytes, &tmW,
                                             bar_full + 8 * npre, (kb + j) * kBK,
                                             static_cast<int32_t>((sg.t / TT) * kBM), pol_w);
                    }
                    u += sg.kb1 - sg.kb0;
                }
            }
            pdl_wait();
            uint32_t it = 0;
            bool ok = true;
            for (int64_t u = u_begin; u < u_end && ok;) {
                const SkSegment sg = sk_segment(u, u_end, KB);
                for (int kb = sg.kb0; kb < sg.kb1; kb += KPS, ++it) {
                    const int nk = min(KPS, sg.kb1 - kb);
                    const uint32_t s = it % STAGES;
                    const int32_t xrow = static_cast<int32_t>((sg.t % TT) * NT);
                    if (it < npre) { // weights already requested; add the token tiles
                        for (int j = 0; j < nk; ++j)
                            tma_load_2d(sX + (s * KPS + j) * Cfg::kXBytes, &tmX, bar_full + 8 * s,
                                        (kb + j) * kBK, xrow);
                        continue;
                    }
                    const uint32_t ph = (it / STAGES) & 1u;
                    if (!mbar_wait(bar_empty + 8 * s, ph ^ 1u, limit_ns)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(bar_full + 8 * s, nk * (Cfg::kWBytes + Cfg::kXBytes));
                    for (int j = 0; j < nk; ++j) {
                        tma_load_2d_hint(sW + (s * KPS + j) * Cfg::kWBytes, &tmW, bar_full + 8 * s,
                                         (kb + j) * kBK, static_cast<int32_t>((sg.t / TT) * kBM),
                                         pol_w);
                        tma_load_2d(sX + (s * KPS + j) * Cfg::kXBytes, &tmX, bar_full + 8 * s,
                                    (kb + j) * kBK, xrow);
                    }
                }
                u += sg.kb1 - sg.kb0;
            }
            // Producer tail: every stage released by the MMA warp before the CTA may exit.
            if (ok)
                drain_ring(bar_empty, it, STAGES, limit_ns);
            // every stage consumed: the next kernel in the stream may launch now
            pdl_launch_dependents();
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_8bit<F8>(kBM, NT);
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
                            umma_8bit<F8>(d, sw128_kmajor_desc(w0 + k * kUmmaK),
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
        // Epilogue warps: warp w reads TMEM lanes 32*(w%4)..+31 = channels of the block.
        pdl_wait(); // s_tok and the workspace may still be in use by the previous kernel
        const int quarter = warp & 3;
        const int etid = threadIdx.x - 64; // 0..127
        const int r = quarter * 32 + lane; // channel within the block
        for (int i = etid; i < M; i += 128)
            sh_stok[i] = __ldg(s_tok + i);
        if constexpr (CLUSTER) {
            const int n = static_cast<int>((blockIdx.y / TT) * kBM) + (etid % (kBM / 4)) * 4;
            if (n < N)
                cl_sc = __ldg(reinterpret_cast<const float4 *>(s_ch + n));
        }
        named_bar_sync(1, 128);
        // tokens of block b's tile held in the accumulator (tile b % TT)
        auto tile_tokens = [&](int64_t b) {
            const int rest = M - static_cast<int>(b % TT) * NT;
            return rest < NT ? rest : NT;
        };
        const int Mp = ((M < NT ? M : NT) + 3) & ~3; // tokens per partial row in the workspace
        // an owner's contributor sums, per token of its channel (small token tiles only)
        constexpr int kPre = (!CLUSTER && NT <= 64) ? NT : 0;
        uint32_t pre[kPre > 0 ? kPre : 1];
        // This CTA owns a block shared with later CTAs iff its range ends inside a block it
        // starts; the later CTAs' shares of that block are their first segments.
        int64_t own_t = -1, own_last = g;
        if constexpr (!CLUSTER) {
            const int64_t tl = (u_end - 1) / KB;
            if (u_end > u_begin && tl * KB >= u_begin && u_end < (tl + 1) * KB) {
                own_t = tl;
                own_last = sk_owner_of(tl * KB + KB - 1, U, G);
            }
        }
        // Waits for the contributors' flags and, for small token tiles, adds their partial
        // sums into pre[]. Done as soon as this CTA's first segment is finished (the
        // contributors' first segments finish at about the same time), so that the loads
        // overlap the MMAs of this CTA's remaining segments.
        auto fetch_contributions = [&]() -> bool {
            if (etid == 0) {
                bool all = true;
                for (int64_t c = g + 1; c <= own_last && all; ++c) {
                    if (ld_acquire_gpu(ws_flag + c) == 0u) {
                        const uint64_t t0 = globaltimer_ns();
                        while (ld_acquire_gpu(ws_flag + c) == 0u) {
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
            const bool all_ok = *sh_word != 0u;
            if constexpr (kPre > 0) {
                const int mt = tile_tokens(own_t);
#pragma unroll
                for (int j = 0; j < kPre; ++j)
                    pre[j] = 0u; // +0 in both accumulator types
                for (int64_t c = g + 1; c <= own_last; ++c) {
                    const int4 *src = reinterpret_cast<const int4 *>(ws_part + (c * kBM + r) * Mp);
#pragma unroll
                    for (int q = 0; q < kPre / 4; ++q) {
                        if (4 * q < mt) {
                            const int4 v = __ldcg(src + q);
                            pre[4 * q] = acc_add<F8>(pre[4 * q], v.x);
                            pre[4 * q + 1] = acc_add<F8>(pre[4 * q + 1], v.y);
                            pre[4 * q + 2] = acc_add<F8>(pre[4 * q + 2], v.z);
                            pre[4 * q + 3] = acc_add<F8>(pre[4 * q + 3], v.w);
                        }
                    }
                }
            }
            return all_ok;
        };
        bool fetched = false;
        uint32_t seg = 0;
        bool ok = true;
        for (int64_t u = u_begin; u < u_end && ok; ++seg) {
            const SkSegment sg = sk_segment(u, u_end, KB);
            u += sg.kb1 - sg.kb0;
            const uint32_t buf = seg & 1u;
            const uint32_t aph = (seg >> 1) & 1u;
            // a segment is a whole block, the owned start of a split block, or a contribution
            const bool owner = !CLUSTER && sg.t == own_t && sg.kb0 == 0;
            const bool contrib = !CLUSTER && sg.kb0 > 0;
            const int64_t tch = sg.t / TT;                 // channel block
            const int mbase = static_cast<int>(sg.t % TT) * NT; // first token of the tile
            const int mt = tile_tokens(sg.t);
            const int n = static_cast<int>(tch * kBM) + r;
            const bool n_ok = n < N;
            const float sc = n_ok ? __ldg(s_ch + n) : 0.0f;
            if (own_t >= 0 && !fetched && (seg >= 1 || owner)) {
                fetched = true;
                if (!fetch_contributions())
                    ok = false;
            }
            // contributors to an owned block: CTAs g+1 .. g_last
            const int64_t g_last = owner ? own_last : g;
            if (!mbar_wait(bar_tfull + 8 * buf, aph, limit_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if constexpr (CLUSTER)
                fence_proxy_async_smem(); // the partial tile reuses TMA-written smem
            const uint32_t tbase = tmem_base + buf * NT + (static_cast<uint32_t>(quarter * 32) << 16);
            // 16 tokens of this thread's channel
            auto chunk = [&](const int c0) {
                uint32_t a[16];
                tmem_ld_32x32b_x16(tbase + c0, a);
                tmem_ld_wait();
                if constexpr (CLUSTER) {
                    // partial tile P[m][128] int32 in this CTA's stage buffers
                    int32_t *P = reinterpret_cast<int32_t *>(smem);
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (c0 + j < mt)
                            P[(c0 + j) * kBM + r] = static_cast<int32_t>(a[j]);
                    return;
                }
                if (contrib) {
                    // this CTA's slot: [128 channels][Mp tokens] int32, 16-byte vectors
                    int4 *dst = reinterpret_cast<int4 *>(ws_part + (g * kBM + r) * Mp + c0);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        if (c0 + 4 * q < mt)
                            __stcg(dst + q, make_int4(a[4 * q], a[4 * q + 1], a[4 * q + 2], a[4 * q + 3]));
                    return;
                }
                if (owner) {
                    if constexpr (kPre > 0) {
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            a[j] = acc_add<F8>(a[j], pre[c0 + j]);
                    } else {
#pragma unroll 2
                        for (int64_t c = g + 1; c <= g_last; ++c) {
                            const int4 *src =
                                reinterpret_cast<const int4 *>(ws_part + (c * kBM + r) * Mp + c0);
                            int4 v[4];
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                v[q] = (c0 + 4 * q < mt) ? __ldcg(src + q) : make_int4(0, 0, 0, 0);
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                a[4 * q] = acc_add<F8>(a[4 * q], v[q].x);
                                a[4 * q + 1] = acc_add<F8>(a[4 * q + 1], v[q].y);
                                a[4 * q + 2] = acc_add<F8>(a[4 * q + 2], v[q].z);
                                a[4 * q + 3] = acc_add<F8>(a[4 * q + 3], v[q].w);
                            }
                        }
                    }
                }
                // dequantize into the staged output tile [m][128] bf16 (two tokens per
                // conversion instruction)
#pragma unroll
                for (int j = 0; j < 16; j += 2) {
                    const int m = c0 + j;
                    if (m < mt) {
                        const uint32_t pr = pack_bf16x2(
                            dequant_acc<F8>(a[j], sh_stok[mbase + m], sc),
                            dequant_acc<F8>(a[j + 1], sh_stok[mbase + m + 1], sc));
                        ysm[m * kBM + r] = static_cast<uint16_t>(pr & 0xFFFFu);
                        if (m + 1 < mt)
                            ysm[(m + 1) * kBM + r] = static_cast<uint16_t>(pr >> 16);
                        if (acc_out && n_ok) {
                            acc_out[static_cast<int64_t>(mbase + m) * N + n] =
                                static_cast<int32_t>(a[j]);
                            if (m + 1 < mt)
                                acc_out[static_cast<int64_t>(mbase + m + 1) * N + n] =
                                    static_cast<int32_t>(a[j + 1]);
                        }
                    }
                }
            };
            if constexpr (kPre > 0) {
#pragma unroll
                for (int c0 = 0; c0 < NT; c0 += 16)
                    if (c0 < mt)
                        chunk(c0);
            } else {
#pragma unroll 1
                for (int c0 = 0; c0 < mt; c0 += 16)
                    chunk(c0);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar_tempty + 8 * buf);
            if constexpr (!CLUSTER) {
                if (contrib) {
                    // publish the partial: every thread's stores, a CTA barrier, then one
                    // release of the flag
                    named_bar_sync(1, 128);
                    if (etid == 0) {
                        fence_acq_rel_gpu();
                        st_relaxed_gpu(ws_flag + g, 1u);
                    }
                } else {
                    // whole or owned block: copy the staged tile out, 16 bytes per thread
                    named_bar_sync(1, 128);
                    if constexpr (SILU) {
                        silu_block_rows(mbase, mt, static_cast<int>(tch), etid, so,
                                        [&](int m, int j0, float (&g)[8], float (&u)[8]) {
                                            const uint16_t *row = ysm + (m - mbase) * kBM;
                                            unpack8(*reinterpret_cast<const uint4 *>(row + j0), g);
                                            unpack8(*reinterpret_cast<const uint4 *>(row + 64 + j0), u);
                                        });
                    } else {
                        const int nvalid = min(kBM, N - static_cast<int>(tch * kBM));
                        for (int v = etid; v < mt * 16; v += 128) {
                            const int m = v >> 4, cv = v & 15;
                            if (cv * 8 < nvalid)
                                *reinterpret_cast<uint4 *>(y + static_cast<int64_t>(mbase + m) * N +
                                                           tch * kBM + cv * 8) =
                                    *reinterpret_cast<const uint4 *>(ysm + m * kBM + cv * 8);
                        }
                    }
                    named_bar_sync(1, 128);
                    if (owner && etid == 0) // ready for the next call
                        for (int64_t c = g + 1; c <= g_last; ++c)
                            st_relaxed_gpu(ws_flag + c, 0u);
                }
            }
        }
    }
    __syncwarp();
    if constexpr (CLUSTER && F8) {
        // Split-K sum in distributed shared memory, binary32 partials (the bulk reduction
        // into peer shared memory has integer forms only): after the cluster barrier, CTA q
        // reads the rows of its tokens [q mt / S, (q+1) mt / S) from every CTA's tile, in
        // rank order (so the sum does not depend on which CTA owns the rows), adds them,
        // dequantizes and stores.
        const uint32_t S = gridDim.x;
        const uint32_t rank = cluster_ctarank();
        const int64_t blk = blockIdx.y;
        const int tch = static_cast<int>(blk / TT);             // channel block
        const int mbase = static_cast<int>(blk % TT) * NT;      // first token of the tile
        const uint32_t mt = static_cast<uint32_t>(M - mbase < NT ? M - mbase : NT);
        const uint32_t m0 = (rank * mt) / S, m1 = ((rank + 1) * mt) / S;
        cluster_sync(); // every CTA's partial tile complete and visible to the cluster
        if (warp >= 2) {
            const int etid = threadIdx.x - 64;
            const int nv = static_cast<int>(m1 - m0) * (kBM / 4);
            for (int v = etid; v < nv; v += 128) {
                const int ml = static_cast<int>(m0) + v / (kBM / 4); // token within the tile
                const int m = mbase + ml;
                const int c = (v % (kBM / 4)) * 4;
                const int n = tch * kBM + c;
                if (n < N) { // N % 8 == 0: the 4 channels are all valid or all past N
                    const uint32_t off = sbase + static_cast<uint32_t>(ml * kBM + c) * 4u;
                    uint4 s4 = ld_dsmem_v4(map_peer_smem(off, 0));
                    for (uint32_t q = 1; q < S; ++q) {
                        const uint4 p4 = ld_dsmem_v4(map_peer_smem(off, q));
                        s4.x = acc_add<true>(s4.x, p4.x);
                        s4.y = acc_add<true>(s4.y, p4.y);
                        s4.z = acc_add<true>(s4.z, p4.z);
                        s4.w = acc_add<true>(s4.w, p4.w);
                    }
                    const float4 c4 = cl_sc; // the scales of channels n .. n + 3
                    const float st = sh_stok[m];
                    uint2 o;
                    o.x = bf16_bits(dequant_acc<true>(s4.x, st, c4.x)) |
                          (bf16_bits(dequant_acc<true>(s4.y, st, c4.y)) << 16);
                    o.y = bf16_bits(dequant_acc<true>(s4.z, st, c4.z)) |
                          (bf16_bits(dequant_acc<true>(s4.w, st, c4.w)) << 16);
                    const int64_t goff = static_cast<int64_t>(m) * N + n;
                    *reinterpret_cast<uint2 *>(y + goff) = o;
                    if (acc_out)
                        *reinterpret_cast<uint4 *>(acc_out + goff) = s4;
                }
            }
        }
        // nobody leaves, or reuses its tile, while a peer may still read it
        cluster_sync();
    } else if constexpr (CLUSTER) {
        // Split-K sum in distributed shared memory. CTA q of the cluster owns the tokens
        // [q mt / S, (q+1) mt / S) of the block; every other CTA adds its partial rows for
        // those tokens into q's tile with one bulk reduction, counted in bytes on q's
        // barrier; q then dequantizes its rows.
        const uint32_t S = gridDim.x;
        const uint32_t rank = cluster_ctarank();
        const int64_t blk = blockIdx.y;
        const int tch = static_cast<int>(blk / TT);             // channel block
        const int mbase = static_cast<int>(blk % TT) * NT;      // first token of the tile
        const uint32_t mt = static_cast<uint32_t>(M - mbase < NT ? M - mbase : NT);
        const uint32_t m0 = (rank * mt) / S, m1 = ((rank + 1) * mt) / S;
        constexpr uint32_t kRowBytes = kBM * 4;
        if (threadIdx.x == 64)
            mbar_expect_tx(bar_red, (m1 - m0) * kRowBytes * (S - 1));
        fence_proxy_async_smem(); // this thread's partial-tile writes, before the bulk reads
        cluster_sync();           // every tile complete, every reduction barrier armed
        if (threadIdx.x == 64) {
            for (uint32_t q = 0; q < S; ++q) {
                const uint32_t a0 = (q * mt) / S, a1 = ((q + 1) * mt) / S;
                if (q != rank && a1 > a0)
                    bulk_reduce_add_s32_peer(map_peer_smem(sbase + a0 * kRowBytes, q),
                                             sbase + a0 * kRowBytes, (a1 - a0) * kRowBytes,
                                             map_peer_smem(bar_red, q));
            }
        }
        if constexpr (SILU) {
            // a warp takes part as a whole (the group maxima are warp shuffles)
            if (warp >= 2 && __all_sync(0xffffffffu, mbar_wait(bar_red, 0, limit_ns))) {
                const int etid = threadIdx.x - 64;
                const int32_t *P = reinterpret_cast<const int32_t *>(smem);
                // this CTA's tokens only: rows m0 .. m1 - 1 of the summed tile
                silu_block_rows(mbase + static_cast<int>(m0), static_cast<int>(m1 - m0), tch,
                                etid, so, [&](int m, int j0, float (&g)[8], float (&u)[8]) {
                                    const float st = sh_stok[m];
                                    const int32_t *row = P + (m - mbase) * kBM;
#pragma unroll
                                    for (int i = 0; i < 8; ++i) {
                                        const int ng = tch * kBM + j0 + i, nu = ng + 64;
                                        g[i] = bf16_round(dequant_f32(row[j0 + i], st, __ldg(s_ch + ng)));
                                        u[i] = bf16_round(dequant_f32(row[64 + j0 + i], st, __ldg(s_ch + nu)));
                                    }
                                });
            }
        } else if (warp >= 2 && mbar_wait(bar_red, 0, limit_ns)) {
            const int etid = threadIdx.x - 64;
            const int32_t *P = reinterpret_cast<const int32_t *>(smem);
            // 4 channels per thread per row: 16-byte tile reads, 8-byte output stores
            const int nv = static_cast<int>(m1 - m0) * (kBM / 4);
            for (int v = etid; v < nv; v += 128) {
                const int ml = static_cast<int>(m0) + v / (kBM / 4); // token within the tile
                const int m = mbase + ml;
                const int c = (v % (kBM / 4)) * 4;
                const int n = tch * kBM + c;
                if (n < N) { // N % 8 == 0: the 4 channels are all valid or all past N
                    const int4 s4 = *reinterpret_cast<const int4 *>(P + ml * kBM + c);
                    const float4 c4 = cl_sc; // the scales of channels n .. n + 3
                    const float st = sh_stok[m];
                    uint2 o;
                    o.x = bf16_bits(dequant_f32(s4.x, st, c4.x)) |
                          (bf16_bits(dequant_f32(s4.y, st, c4.y)) << 16);
                    o.y = bf16_bits(dequant_f32(s4.z, st, c4.z)) |
                          (bf16_bits(dequant_f32(s4.w, st, c4.w)) << 16);
                    const int64_t off = static_cast<int64_t>(m) * N + n;
                    *reinterpret_cast<uint2 *>(y + off) = o;
                    if (acc_out)
                        *reinterpret_cast<int4 *>(acc_out + off) = s4;
                }
            }
        }
        // nobody leaves, or reuses its tile, while a peer's reduction may still read it
        cluster_sync();
    }
    if (warp == 1)
        tmem_relinquish(); // after the work, as the allocator's permit protocol expects
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::kTmemCols);
    }
    if constexpr (RNV > 0) {
        // The residual RMSNorm of the output rows, by the last CTAs to finish. Every CTA takes
        // a ticket once its output stores are done (the barrier above orders them before
        // thread 0's release); the CTAs holding the last R tickets (R = min(M, 64, grid))
        // wait until every ticket is taken, then run rows slot, slot + R, ... reading y back
        // through L2. The others exit at once. The last row CTA to finish zeroes both
        // counters for the next call.
        const unsigned int total = gridDim.x * gridDim.y;
        const unsigned int R = min(min(static_cast<unsigned int>(M), 64u), total);
        volatile uint32_t *sh_ok = tslot_ptr + 5;
        if (threadIdx.x == 0) {
            fence_acq_rel_gpu();
            *sh_word = atomicAdd(rn.bar, 1u);
        }
        __syncthreads();
        const unsigned int ticket = *sh_word;
        if (ticket + R >= total && warp >= 2) {
            const int etid = threadIdx.x - 64;
            const int slot = static_cast<int>(ticket - (total - R));
            // the first row's residual and gamma' do not depend on y: requested before the wait
            RmsRow<RNV> row;
            rms_row_load_side<RNV>(rn.res + static_cast<int64_t>(slot) * N, rn.gamma, N, etid, row);
            if (etid == 0) {
                bool all = true;
                if (ld_acquire_gpu(rn.bar) < total) {
                    const uint64_t t0 = globaltimer_ns();
                    while (ld_acquire_gpu(rn.bar) < total) {
                        if (globaltimer_ns() - t0 > limit_ns) {
                            flag_timeout();
                            all = false;
                            break;
                        }
                    }
                }
                *sh_ok = all ? 1u : 0u;
            }
            named_bar_sync(1, 128);
            // reductions' scratch: the (idle) stage ring
            double *shd = reinterpret_cast<double *>(smem);
            float *shf = reinterpret_cast<float *>(smem + 64);
            if (*sh_ok != 0u) {
                for (int m = slot; m < M; m += static_cast<int>(R)) {
                    const int64_t off = static_cast<int64_t>(m) * N;
                    if (m != slot)
                        rms_row_load_side<RNV>(rn.res + off, rn.gamma, N, etid, row);
                    rms_row_load_x<RNV>(y + off, true, N, etid, row);
                    rms_row_finish<RNV>(row, true, rn.h + off, rn.eps, N, rn.q + off, rn.s + m,
                                        etid, shd, shf);
                }
            }
            named_bar_sync(1, 128);
            if (etid == 0 && atom_add_acq_rel_gpu(rn.bar + 1, 1u) == R - 1) {
                // every ticket is taken and every row CTA is past its wait
                rn.bar[0] = 0u;
                rn.bar[1] = 0u;
            }
        }
    }
}

} // namespace w8a8
