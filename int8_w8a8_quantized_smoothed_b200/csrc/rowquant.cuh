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

// q = clamp(round_half_even(y / s), -127, 127) with IEEE division; s == 0 gives 0.
__device__ __forceinline__ int quant1(float y, float s)
{
    const int v = __float2int_rn(__fdiv_rn(y, s));
    return max(-127, min(127, v));
}

__device__ __forceinline__ uint32_t pack_i8x4(int a, int b, int c, int d)
{
    return (static_cast<uint32_t>(a) & 0xFFu) | ((static_cast<uint32_t>(b) & 0xFFu) << 8) |
           ((static_cast<uint32_t>(c) & 0xFFu) << 16) | ((static_cast<uint32_t>(d) & 0xFFu) << 24);
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
                out.x = pack_i8x4(quant1(v[c][0], s), quant1(v[c][1], s), quant1(v[c][2], s),
                                  quant1(v[c][3], s));
                out.y = pack_i8x4(quant1(v[c][4], s), quant1(v[c][5], s), quant1(v[c][6], s),
                                  quant1(v[c][7], s));
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
                v[c][0] = __fmul_rn(v[c][0], a.x);
                v[c][1] = __fmul_rn(v[c][1], a.y);
                v[c][2] = __fmul_rn(v[c][2], a.z);
                v[c][3] = __fmul_rn(v[c][3], a.w);
                v[c][4] = __fmul_rn(v[c][4], b.x);
                v[c][5] = __fmul_rn(v[c][5], b.y);
                v[c][6] = __fmul_rn(v[c][6], b.z);
                v[c][7] = __fmul_rn(v[c][7], b.w);
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
            for (int i = 0; i < 8; ++i) {
                v[c][i] = __fmul_rn(__fmul_rn(v[c][i], rstd), g[i]);
                amax = fmaxf(amax, fabsf(v[c][i]));
            }
        }
    }
    amax = block_max(amax, shf);
    quantize_and_store<NCH>(v, amax, nvec, q + row * K, s_tok + row);
}

// ----------------------------------------------------------------- SiLU(gate)*up + quant

// Binary32 exp fixed by the library's contract (header w8a8.h): Cody-Waite reduction with
// a 16-bit head of ln 2, degree-7 Taylor polynomial by Horner in fused multiply-adds,
// exact scaling by two powers of two.
__device__ __forceinline__ float w8a8_exp(float x)
{
    if (x != x)
        return x;
    if (x > 89.0f)
        return __int_as_float(0x7f800000);
    if (x < -104.0f)
        return 0.0f;
    const float kInvLn2 = 1.44269502162933349609375f;           // RN(1 / ln 2)
    const float kLn2Hi = 0.693145751953125f;                    // ln 2, 16 significant bits
    const float kLn2Lo = 1.428606765330187045037746429443359375e-06f; // RN(ln 2 - kLn2Hi)
    const float kf = rintf(__fmul_rn(x, kInvLn2));
    const int k = static_cast<int>(kf);
    float r = __fmaf_rn(-kf, kLn2Hi, x);
    r = __fmaf_rn(-kf, kLn2Lo, r);
    float p = 1.0f / 5040.0f;
    p = __fmaf_rn(p, r, 1.0f / 720.0f);
    p = __fmaf_rn(p, r, 1.0f / 120.0f);
    p = __fmaf_rn(p, r, 1.0f / 24.0f);
    p = __fmaf_rn(p, r, 1.0f / 6.0f);
    p = __fmaf_rn(p, r, 0.5f);
    p = __fmaf_rn(p, r, 1.0f);
    p = __fmaf_rn(p, r, 1.0f);
    const int k1 = k / 2;
    const int k2 = k - k1;
    return __fmul_rn(__fmul_rn(p, __int_as_float((k1 + 127) << 23)),
                     __int_as_float((k2 + 127) << 23));
}

__device__ __forceinline__ float silu_f32(float g)
{
    return __fdiv_rn(g, __fadd_rn(1.0f, w8a8_exp(-g)));
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
            for (int i = 0; i < 8; ++i) {
                v[c][i] = __fmul_rn(silu_f32(g[i]), u[i]);
                amax = fmaxf(amax, fabsf(v[c][i]));
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
