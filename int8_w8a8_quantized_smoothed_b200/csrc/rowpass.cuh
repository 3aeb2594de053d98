// Row passes run by the 128 threads of a GEMM kernel's epilogue group (warps 2..5, named
// barrier 2) inside a persistent launch: the fused decoder block's row phases and the
// residual RMSNorm tail of the decode GEMM. The per-element arithmetic is that of the
// stand-alone row kernels (rowquant.cuh); only the binary64 order of the RMSNorm sums
// differs, which the method leaves free.
#pragma once

#include "ptx.cuh"
#include "rowquant.cuh"

namespace w8a8 {

__device__ __forceinline__ unsigned int atom_add_acq_rel_gpu(unsigned int *p, unsigned int v)
{
    unsigned int old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// Sum / max over the 128 threads of the epilogue group (named barrier 2), using sh[0..3].
__device__ __forceinline__ double group_sum(double v, double *sh, int etid)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((etid & 31) == 0)
        sh[etid >> 5] = v;
    named_bar_sync(2, 128);
    const double r = (sh[0] + sh[1]) + (sh[2] + sh[3]);
    named_bar_sync(2, 128);
    return r;
}

__device__ __forceinline__ float group_max(float v, float *sh, int etid)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if ((etid & 31) == 0)
        sh[etid >> 5] = v;
    named_bar_sync(2, 128);
    const float r = fmaxf(fmaxf(sh[0], sh[1]), fmaxf(sh[2], sh[3]));
    named_bar_sync(2, 128);
    return r;
}

// Codes of the eight values of one vector given the row's s and r = RN(1/s), or by the exact
// quotient when the product path is unavailable (the same decisions as quantize_and_store).
__device__ __forceinline__ uint2 quant8_int8(const float (&y)[8], float s, float r, bool by_product,
                                             float amax)
{
    uint2 out = make_uint2(0u, 0u);
    if (by_product) {
        uint32_t b[8];
        quant_bits8(y, s, r, b);
        out.x = pack_low_bytes(b[0], b[1], b[2], b[3]);
        out.y = pack_low_bytes(b[4], b[5], b[6], b[7]);
    } else if (amax > 0.0f) {
        out.x = pack_low_bytes(quant_bits(y[0], s), quant_bits(y[1], s), quant_bits(y[2], s),
                               quant_bits(y[3], s));
        out.y = pack_low_bytes(quant_bits(y[4], s), quant_bits(y[5], s), quant_bits(y[6], s),
                               quant_bits(y[7], s));
    }
    return out;
}

__device__ __forceinline__ void load8_gamma(const float *p, float (&v)[8])
{
    const float4 lo = __ldg(reinterpret_cast<const float4 *>(p));
    const float4 hi = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    v[0] = lo.x; v[1] = lo.y; v[2] = lo.z; v[3] = lo.w;
    v[4] = hi.x; v[5] = hi.y; v[6] = hi.z; v[7] = hi.w;
}

// Smoothed RMSNorm + quant of one row of K <= 8 * 128 * NV values by the 128-thread group,
// the row held in registers: with a residual the row is h = bf16(x + res), also written to
// h_out. Arithmetic as rmsnorm_quant_kernel. The loads come in two parts so that a caller
// can issue the residual and gamma' (which do not depend on x) before it waits for x.
template <int NV> struct RmsRow {
    uint4 raw[NV]; // x
    uint4 rr[NV];  // residual (zero when there is none)
    float gm[NV][8]; // gamma'
};

// The residual (res may be null) and gamma' of this thread's vectors c * 128 + etid.
template <int NV>
__device__ __forceinline__ void rms_row_load_side(const uint16_t *res, const float *gamma, int K,
                                                  int etid, RmsRow<NV> &r)
{
    const int nvec = K >> 3;
#pragma unroll
    for (int c = 0; c < NV; ++c) {
        const int v = c * 128 + etid;
        r.rr[c] = make_uint4(0u, 0u, 0u, 0u);
        if (v < nvec) {
            if (res)
                r.rr[c] = ldg_nc_v4(reinterpret_cast<const uint4 *>(res) + v);
            load8_gamma(gamma + 8 * v, r.gm[c]);
        }
    }
}

// x of this thread's vectors; xin_coherent: x was written in this launch (read through L2).
template <int NV>
__device__ __forceinline__ void rms_row_load_x(const uint16_t *xin, bool xin_coherent, int K,
                                               int etid, RmsRow<NV> &r)
{
    const int nvec = K >> 3;
#pragma unroll
    for (int c = 0; c < NV; ++c) {
        const int v = c * 128 + etid;
        r.raw[c] = make_uint4(0u, 0u, 0u, 0u);
        if (v < nvec)
            r.raw[c] = xin_coherent ? __ldcg(reinterpret_cast<const uint4 *>(xin) + v)
                                    : ldg_nc_v4(reinterpret_cast<const uint4 *>(xin) + v);
    }
}

template <int NV>
__device__ __forceinline__ void rms_row_finish(const RmsRow<NV> &row, bool has_res,
                                               uint16_t *h_out, float eps, int K, int8_t *qrow,
                                               float *s_out, int etid, double *shd, float *shf)
{
    const int nvec = K >> 3;
    const uint4 (&raw)[NV] = row.raw;
    const uint4 (&rr)[NV] = row.rr;
    const float (&gm)[NV][8] = row.gm;
    float f[NV][8];
    double ss = 0.0;
#pragma unroll
    for (int c = 0; c < NV; ++c) {
        const int v = c * 128 + etid;
        unpack8(raw[c], f[c]);
        if (has_res) {
            float r8[8];
            unpack8(rr[c], r8);
            uint4 hb;
            hb.x = pack_bf16x2(__fadd_rn(f[c][0], r8[0]), __fadd_rn(f[c][1], r8[1]));
            hb.y = pack_bf16x2(__fadd_rn(f[c][2], r8[2]), __fadd_rn(f[c][3], r8[3]));
            hb.z = pack_bf16x2(__fadd_rn(f[c][4], r8[4]), __fadd_rn(f[c][5], r8[5]));
            hb.w = pack_bf16x2(__fadd_rn(f[c][6], r8[6]), __fadd_rn(f[c][7], r8[7]));
            if (v < nvec)
                reinterpret_cast<uint4 *>(h_out)[v] = hb;
            unpack8(hb, f[c]);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) // each square of a bf16 value is exact in binary32
            ss = __dadd_rn(ss, static_cast<double>(__fmul_rn(f[c][i], f[c][i])));
    }
    const double sum = group_sum(ss, shd, etid);
    const double mean = (K & (K - 1)) == 0 ? __dmul_rn(sum, 1.0 / static_cast<double>(K))
                                           : __ddiv_rn(sum, static_cast<double>(K));
    const float ms = __double2float_rn(mean);
    const float rstd = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
    float amax = 0.0f;
#pragma unroll
    for (int c = 0; c < NV; ++c) {
        const int v = c * 128 + etid;
        if (v < nvec) {
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                const float2 p = mul2(mul2(make_float2(f[c][i], f[c][i + 1]), splat2(rstd)),
                                      make_float2(gm[c][i], gm[c][i + 1]));
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

template <int NV>
__device__ __forceinline__ void row_rmsnorm(const uint16_t *xin, bool xin_coherent,
                                            const uint16_t *res, uint16_t *h_out,
                                            const float *gamma, float eps, int K, int8_t *qrow,
                                            float *s_out, int etid, double *shd, float *shf)
{
    RmsRow<NV> r;
    rms_row_load_x<NV>(xin, xin_coherent, K, etid, r);
    rms_row_load_side<NV>(res, gamma, K, etid, r);
    rms_row_finish<NV>(r, res != nullptr, h_out, eps, K, qrow, s_out, etid, shd, shf);
}

} // namespace w8a8
