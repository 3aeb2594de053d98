// Per-token quantization kernels (HBM-bound): quantize_rows, smoothed RMSNorm + quant and
// SiLU(gate)*up + quant. One CTA per row; each thread keeps NCH vectors of 8 values in
// registers, so the row is read from HBM once and written once. Loads and stores are
// 16-byte (bf16 x 8) / 8-byte (int8 x 8) and coalesced: vector v = c*blockDim + tid.
#pragma once

#include "ptx.cuh"

namespace w8a8 {

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ double warp_sum(double v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Block-wide max of non-negative floats; `sh` holds >= 33 floats. Exact (max is
// order-free). All threads receive the result.
__device__ __forceinline__ float block_max(float v, float *sh)
{
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    const int nw = (blockDim.x + 31) >> 5;
    v = warp_max(v);
    if (l == 0)
        sh[w] = v;
    __syncthreads();
    if (w == 0) {
        float t = (l < nw) ? sh[l] : 0.0f;
        t = warp_max(t);
        if (l == 0)
            sh[32] = t;
    }
    __syncthreads();
    return sh[32];
}

__device__ __forceinline__ double block_sum(double v, double *sh)
{
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    const int nw = (blockDim.x + 31) >> 5;
    v = warp_sum(v);
    if (l == 0)
        sh[w] = v;
    __syncthreads();
    if (w == 0) {
        double t = (l < nw) ? sh[l] : 0.0;
        t = warp_sum(t);
        if (l == 0)
            sh[32] = t;
    }
    __syncthreads();
    return sh[32];
}

// Adding 1.5 * 2^23 to a binary32 v with |v| < 2^22 leaves v rounded to an integer
// (round half to even, like rint) in the low bits of the sum: integer rounding on the FMA
// pipe instead of a float-to-int conversion. For |v| <= 127 the sum's low byte is the int8.
constexpr float kRoundMagic = 12582912.0f;
constexpr int kRoundMagicBits = 0x4B400000;

// Bits of RN(clamp(RN(y / s), -127, 127) + 1.5 * 2^23): the low byte is
// clamp(round_half_even(y / s), -127, 127) as int8 (rounding and clamping commute here).
__device__ __forceinline__ uint32_t quant_bits(float y, float s)
{
    const float t = fminf(fmaxf(__fdiv_rn(y, s), -127.0f), 127.0f);
    return __float_as_uint(__fadd_rn(t, kRoundMagic));
}

// Four codes from the low bytes of four quant_bits results.
__device__ __forceinline__ uint32_t pack_low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// ---- packed binary32 pairs (sm_100 f32x2): each lane is an IEEE RN operation

__device__ __forceinline__ unsigned long long f2_bits(float2 v)
{
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(v.x), "f"(v.y));
    return r;
}

__device__ __forceinline__ float2 bits_f2(unsigned long long r)
{
    float2 v;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
    return v;
}

__device__ __forceinline__ float2 mul2(float2 a, float2 b)
{
    unsigned long long r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)));
    return bits_f2(r);
}

__device__ __forceinline__ float2 add2(float2 a, float2 b)
{
    unsigned long long r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)));
    return bits_f2(r);
}

__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c)
{
    unsigned long long r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)),
        "l"(f2_bits(c)));
    return bits_f2(r);
}

__device__ __forceinline__ float2 splat2(float v)
{
    return make_float2(v, v);
}

// Quantizes the row held in registers (v[c][0..7] for vector c*blockDim + tid) given its
// absmax, writes q and the scale.
template <int NCH>
__device__ __forceinline__ void quantize_and_store(const float (&v)[NCH][8], float amax,
                                                   int nvec, int8_t *__restrict__ qrow,
                                                   float *__restrict__ s_out)
{
    const float s = __fdiv_rn(amax, 127.0f);
    if (threadIdx.x == 0)
        *s_out = s;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        const int vi = c * blockDim.x + threadIdx.x;
        if (vi < nvec) {
            uint2 out = make_uint2(0u, 0u);
            if (amax > 0.0f) {
                out.x = pack_low_bytes(quant_bits(v[c][0], s), quant_bits(v[c][1], s),
                                       quant_bits(v[c][2], s), quant_bits(v[c][3], s));
                out.y = pack_low_bytes(quant_bits(v[c][4], s), quant_bits(v[c][5], s),
                                       quant_bits(v[c][6], s), quant_bits(v[c][7], s));
            }
            reinterpret_cast<uint2 *>(qrow)[vi] = out;
        }
    }
}

__device__ __forceinline__ void unpack8(const uint4 u, float (&f)[8])
{
    f[0] = bf16_lo(u.x);
    f[1] = bf16_hi(u.x);
    f[2] = bf16_lo(u.y);
    f[3] = bf16_hi(u.y);
    f[4] = bf16_lo(u.z);
    f[5] = bf16_hi(u.z);
    f[6] = bf16_lo(u.w);
    f[7] = bf16_hi(u.w);
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// ----------------------------------------------------------------- quantize_rows

template <int NCH>
__global__ void __launch_bounds__(1024) quantize_rows_kernel(const uint16_t *__restrict__ x,
                                                             const float *__restrict__ sinv,
                                                             int K, int8_t *__restrict__ q,
                                                             float *__restrict__ s_tok)
{
    __shared__ float sh[33];
    if (threadIdx.x == 0)
        pdl_launch_dependents();
    pdl_wait(); // every input may come from the previous kernel
    const int64_t row = blockIdx.x;
    const int nvec = K >> 3;
    const uint4 *xr = reinterpret_cast<const uint4 *>(x + row * K);
    float v[NCH][8];
    float amax = 0.0f;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        const int vi = c * blockDim.x + threadIdx.x;
        if (vi < nvec) {
            unpack8(ldg_nc_v4(xr + vi), v[c]);
            if (sinv) {
                const float4 a = __ldg(reinterpret_cast<const float4 *>(sinv) + 2 * vi);
                const float4 b = __ldg(reinterpret_cast<const float4 *>(sinv) + 2 * vi + 1);
                const float2 p0 = mul2(make_float2(v[c][0], v[c][1]), make_float2(a.x, a.y));
                const float2 p1 = mul2(make_float2(v[c][2], v[c][3]), make_float2(a.z, a.w));
                const float2 p2 = mul2(make_float2(v[c][4], v[c][5]), make_float2(b.x, b.y));
                const float2 p3 = mul2(make_float2(v[c][6], v[c][7]), make_float2(b.z, b.w));
                v[c][0] = p0.x; v[c][1] = p0.y; v[c][2] = p1.x; v[c][3] = p1.y;
                v[c][4] = p2.x; v[c][5] = p2.y; v[c][6] = p3.x; v[c][7] = p3.y;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i)
                amax = fmaxf(amax, fabsf(v[c][i]));
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                v[c][i] = 0.0f;
        }
    }
    amax = block_max(amax, sh);
    quantize_and_store<NCH>(v, amax, nvec, q + row * K, s_tok + row);
}

// ----------------------------------------------------------------- smoothed RMSNorm + quant

template <int NCH, bool RES>
__global__ void __launch_bounds__(1024) rmsnorm_quant_kernel(
    const uint16_t *__restrict__ x, const uint16_t *__restrict__ res, uint16_t *__restrict__ h_out,
    const float *__restrict__ gamma, float eps, int K, int8_t *__restrict__ q,
    float *__restrict__ s_tok)
{
    __shared__ double shd[33];
    __shared__ float shf[33];
    if (threadIdx.x == 0)
        pdl_launch_dependents();
    pdl_wait(); // every input may come from the previous kernel
    const int64_t row = blockIdx.x;
    const int nvec = K >> 3;
    const uint4 *xr = reinterpret_cast<const uint4 *>(x + row * K);
    float v[NCH][8];
    double ss = 0.0;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        const int vi = c * blockDim.x + threadIdx.x;
        if (vi < nvec) {
            unpack8(ldg_nc_v4(xr + vi), v[c]);
            if (RES) {
                float r[8];
                unpack8(ldg_nc_v4(reinterpret_cast<const uint4 *>(res + row * K) + vi), r);
                uint4 hb;
                hb.x = pack_bf16x2(__fadd_rn(v[c][0], r[0]), __fadd_rn(v[c][1], r[1]));
                hb.y = pack_bf16x2(__fadd_rn(v[c][2], r[2]), __fadd_rn(v[c][3], r[3]));
                hb.z = pack_bf16x2(__fadd_rn(v[c][4], r[4]), __fadd_rn(v[c][5], r[5]));
                hb.w = pack_bf16x2(__fadd_rn(v[c][6], r[6]), __fadd_rn(v[c][7], r[7]));
                reinterpret_cast<uint4 *>(h_out + row * K)[vi] = hb;
                unpack8(hb, v[c]);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) // each square of a bf16 value is exact in binary32
                ss = __dadd_rn(ss, static_cast<double>(__fmul_rn(v[c][i], v[c][i])));
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                v[c][i] = 0.0f;
        }
    }
    const double sum = block_sum(ss, shd);
    const float ms = __double2float_rn(__ddiv_rn(sum, static_cast<double>(K)));
    const float rstd = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
    float amax = 0.0f;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        const int vi = c * blockDim.x + threadIdx.x;
        if (vi < nvec) {
            const float4 a = __ldg(reinterpret_cast<const float4 *>(gamma) + 2 * vi);
            const float4 b = __ldg(reinterpret_cast<const float4 *>(gamma) + 2 * vi + 1);
            const float g[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 8; i += 2) { // (h * rstd) * gamma', two lanes at a time
                const float2 p = mul2(mul2(make_float2(v[c][i], v[c][i + 1]), splat2(rstd)),
                                      make_float2(g[i], g[i + 1]));
                v[c][i] = p.x;
                v[c][i + 1] = p.y;
                amax = fmaxf(amax, fmaxf(fabsf(p.x), fabsf(p.y)));
            }
        }
    }
    amax = block_max(amax, shf);
    quantize_and_store<NCH>(v, amax, nvec, q + row * K, s_tok + row);
}

// ----------------------------------------------------------------- SiLU(gate)*up + quant

// Binary32 exp fixed by the library's contract (header w8a8.h), two lanes at a time:
// Cody-Waite reduction with a 16-bit head of ln 2, degree-7 Taylor polynomial by Horner in
// fused multiply-adds, exact scaling by two powers of two; every step is the scalar
// definition's IEEE operation, lane by lane.
__device__ __forceinline__ float2 w8a8_exp2(float2 x)
{
    const float kInvLn2 = 1.44269502162933349609375f;           // RN(1 / ln 2)
    const float kLn2Hi = 0.693145751953125f;                    // ln 2, 16 significant bits
    const float kLn2Lo = 1.428606765330187045037746429443359375e-06f; // RN(ln 2 - kLn2Hi)
    // k = rint(x / ln 2) (|x / ln 2| < 2^22 in range: magic-constant rounding is rint)
    const float2 km = add2(mul2(x, splat2(kInvLn2)), splat2(kRoundMagic));
    const float2 kf = add2(km, splat2(-kRoundMagic));
    float2 r = fma2(kf, splat2(-kLn2Hi), x);
    r = fma2(kf, splat2(-kLn2Lo), r);
    float2 p = splat2(1.0f / 5040.0f);
    p = fma2(p, r, splat2(1.0f / 720.0f));
    p = fma2(p, r, splat2(1.0f / 120.0f));
    p = fma2(p, r, splat2(1.0f / 24.0f));
    p = fma2(p, r, splat2(1.0f / 6.0f));
    p = fma2(p, r, splat2(0.5f));
    p = fma2(p, r, splat2(1.0f));
    p = fma2(p, r, splat2(1.0f));
    const int ka = __float_as_int(km.x) - kRoundMagicBits;
    const int kb = __float_as_int(km.y) - kRoundMagicBits;
    const int ka1 = ka / 2, kb1 = kb / 2; // truncation toward zero
    const float2 s1 = make_float2(__int_as_float((ka1 + 127) << 23), __int_as_float((kb1 + 127) << 23));
    const float2 s2 = make_float2(__int_as_float((ka - ka1 + 127) << 23),
                                  __int_as_float((kb - kb1 + 127) << 23));
    float2 e = mul2(mul2(p, s1), s2);
    // outside the reduction's range: NaN stays NaN, x > 89 gives +inf, x < -104 gives +0
    const float inf = __int_as_float(0x7f800000);
    e.x = (x.x != x.x) ? x.x : (x.x > 89.0f ? inf : (x.x < -104.0f ? 0.0f : e.x));
    e.y = (x.y != x.y) ? x.y : (x.y > 89.0f ? inf : (x.y < -104.0f ? 0.0f : e.y));
    return e;
}

// a = silu(g) * u = (g / (1 + exp(-g))) * u for two lanes; the division stays IEEE scalar.
__device__ __forceinline__ float2 silu_mul2(float2 g, float2 u)
{
    const float2 d = add2(splat2(1.0f), w8a8_exp2(make_float2(-g.x, -g.y)));
    return mul2(make_float2(__fdiv_rn(g.x, d.x), __fdiv_rn(g.y, d.y)), u);
}

template <int NCH>
__global__ void __launch_bounds__(1024) silu_mul_quant_kernel(const uint16_t *__restrict__ gu,
                                                              int I, int8_t *__restrict__ q,
                                                              float *__restrict__ s_tok)
{
    __shared__ float sh[33];
    if (threadIdx.x == 0)
        pdl_launch_dependents();
    pdl_wait(); // every input may come from the previous kernel
    const int64_t row = blockIdx.x;
    const int nvec = I >> 3;
    const uint4 *gr = reinterpret_cast<const uint4 *>(gu + row * 2 * static_cast<int64_t>(I));
    const uint4 *ur = gr + nvec;
    float v[NCH][8];
    float amax = 0.0f;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        const int vi = c * blockDim.x + threadIdx.x;
        if (vi < nvec) {
            float g[8], u[8];
            unpack8(ldg_nc_v4(gr + vi), g);
            unpack8(ldg_nc_v4(ur + vi), u);
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                const float2 a2 = silu_mul2(make_float2(g[i], g[i + 1]), make_float2(u[i], u[i + 1]));
                v[c][i] = a2.x;
                v[c][i + 1] = a2.y;
                amax = fmaxf(amax, fmaxf(fabsf(a2.x), fabsf(a2.y)));
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                v[c][i] = 0.0f;
        }
    }
    amax = block_max(amax, sh);
    quantize_and_store<NCH>(v, amax, nvec, q + row * I, s_tok + row);
}

} // namespace w8a8
