// Per-token quantization kernels (HBM-bound): quantize_rows, smoothed RMSNorm + quant and
// SiLU(gate)*up + quant. A CTA handles one row at a time and keeps it in registers (NCH
// vectors of 8 values per thread), so the row is read from HBM once and written once. The
// grid is persistent (at most as many CTAs as are resident on the device, looping over
// rows). Loads and stores are 16-byte (bf16 x 8) / 8-byte (int8 x 8) and coalesced: vector
// v = c*blockDim + tid.
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

// Block-wide reductions with one barrier: each warp reduces its values and publishes the
// result in sh[warp]; after the barrier every warp reduces all the warps' results itself
// (in the same fixed order, so every thread gets the same value). A buffer may be written
// again only after a later barrier that every thread reaches after reading it.

// Max of non-negative floats (exact: max is order-free); sh holds >= 32 floats.
__device__ __forceinline__ float block_max(float v, float *sh)
{
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    const int nw = (blockDim.x + 31) >> 5;
    v = warp_max(v);
    if (l == 0)
        sh[w] = v;
    __syncthreads();
    return warp_max(l < nw ? sh[l] : 0.0f);
}

// Sum in binary64 (any order: the caller accepts either neighbour where it matters); sh
// holds >= 32 doubles.
__device__ __forceinline__ double block_sum(double v, double *sh)
{
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    const int nw = (blockDim.x + 31) >> 5;
    v = warp_sum(v);
    if (l == 0)
        sh[w] = v;
    __syncthreads();
    return warp_sum(l < nw ? sh[l] : 0.0);
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

// Codes of eight values given the row's scale s and r = RN(1 / s) (s >= 2^-100), as the
// bits whose low bytes are the int8 codes (see quant_bits). t = RN(y r) is within 2^-15 of
// RN(y / s) (both within 127 * 2^-23 + 2^-18 of y / s), so when t is more than 2^-14 away
// from every half-integer, rint(t) = rint(RN(y / s)) and |rint(t)| <= 127 needs no clamp.
// When any of the eight is that close (probability about 2^-10 per vector), the exact
// quotient decides all eight (one branch per vector keeps the common path branch-free).
// SAT: values may lie beyond +-127 s (a fixed scale); t is clamped to [-127, 127] first,
// which commutes with the rounding because the bounds are integers.
template <bool SAT = false>
__device__ __forceinline__ void quant_bits8(const float (&y)[8], float s, float r, uint32_t (&b)[8])
{
    constexpr float kNearHalf = 0.5f - 6.103515625e-05f; // 0.5 - 2^-14
    bool near = false;
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        float2 t = mul2(make_float2(y[i], y[i + 1]), splat2(r));
        if constexpr (SAT)
            t = make_float2(fminf(fmaxf(t.x, -127.0f), 127.0f), fminf(fmaxf(t.y, -127.0f), 127.0f));
        const float2 m = add2(t, splat2(kRoundMagic));     // rint(t) + 1.5 * 2^23
        const float2 n = add2(m, splat2(-kRoundMagic));    // rint(t)
        const float2 d = add2(t, make_float2(-n.x, -n.y)); // t - rint(t), exact
        near |= !(fabsf(d.x) < kNearHalf) | !(fabsf(d.y) < kNearHalf);
        b[i] = __float_as_uint(m.x);
        b[i + 1] = __float_as_uint(m.y);
    }
    if (near) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            b[i] = quant_bits(y[i], s);
    }
}

// ---- FP8 (OCP E4M3) codes
//
// E4M3: sign, 4 exponent bits (bias 7), 3 fraction bits, no infinities; largest finite 448.
// A value's code is RN-even of it to E4M3 with saturation to +-448 (cvt.rn.satfinite), and
// the per-token scale is s = amax / 448, so code = e4m3(RN(y / s)).

// Codes of two binary32 values, lo in the low byte of the result.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

constexpr float kBracketLo = 0x1.ffffep-1f; // 1 - 2^-20
constexpr float kBracketHi = 0x1.00001p+0f; // 1 + 2^-20

// Codes of eight values (two 32-bit words, value i in byte i) given s, rl = RN(r (1 - 2^-20))
// and rh = RN(r (1 + 2^-20)) with r = RN(1 / s), s >= 2^-100. Each of RN(y rl), RN(y rh)
// carries at most three binary32 roundings (relative 3 * 2^-24 together) on top of the
// +-2^-20 offset, so they bracket RN(y / s) strictly in magnitude, and rounding to E4M3 is
// monotone: when both ends give the same code, so does the exact quotient. Otherwise (an
// E4M3 rounding midpoint within about 2^-20 relative of y / s: probability about 2^-12 per
// vector) the IEEE quotients decide all eight. Results in the binary32 subnormal range
// (|y / s| < 2^-126) are all far below the smallest E4M3 step, so every form gives +-0 with
// the sign of y.
__device__ __forceinline__ uint2 quant_e4m3_8(const float (&y)[8], float s, float rl, float rh)
{
    uint32_t lo[4], hi[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 a = mul2(make_float2(y[2 * i], y[2 * i + 1]), splat2(rl));
        const float2 b = mul2(make_float2(y[2 * i], y[2 * i + 1]), splat2(rh));
        lo[i] = e4m3x2(a.x, a.y);
        hi[i] = e4m3x2(b.x, b.y);
    }
    uint2 out = make_uint2(lo[0] | (lo[1] << 16), lo[2] | (lo[3] << 16));
    const uint2 chk = make_uint2(hi[0] | (hi[1] << 16), hi[2] | (hi[3] << 16));
    if (out.x != chk.x || out.y != chk.y) {
        uint32_t e[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            e[i] = e4m3x2(__fdiv_rn(y[2 * i], s), __fdiv_rn(y[2 * i + 1], s));
        out = make_uint2(e[0] | (e[1] << 16), e[2] | (e[3] << 16));
    }
    return out;
}

// Codes by the IEEE quotient alone (tiny scales, whose reciprocal may not be finite).
__device__ __forceinline__ uint2 quant_e4m3_8_exact(const float (&y)[8], float s)
{
    uint32_t e[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        e[i] = e4m3x2(__fdiv_rn(y[2 * i], s), __fdiv_rn(y[2 * i + 1], s));
    return make_uint2(e[0] | (e[1] << 16), e[2] | (e[3] << 16));
}

// Quantizes the part of a row held in registers (v[c][0..7] for vector v0 + c*blockDim + tid,
// vectors below v1) given the row's absmax, writes its codes; the CTA's thread 0 writes the
// scale when s_out is given. F8: E4M3 codes with s = amax / 448, else int8 with s = amax / 127.
template <int NCH, bool F8 = false>
__device__ __forceinline__ void quantize_and_store(const float (&v)[NCH][8], float amax, int v0,
                                                   int v1, int8_t *__restrict__ qrow,
                                                   float *__restrict__ s_out)
{
    const float s = __fdiv_rn(amax, F8 ? 448.0f : 127.0f);
    if (s_out && threadIdx.x == 0)
        *s_out = s;
    // the product path needs a finite reciprocal; tiny scales take the exact quotient
    const bool by_product = s >= 7.888609052210118e-31f; // 2^-100
    const float r = by_product ? __frcp_rn(s) : 0.0f;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        const int vi = v0 + c * blockDim.x + threadIdx.x;
        if (vi < v1) {
            uint2 out = make_uint2(0u, 0u); // an all-zero row: s = 0, every code +0
            if constexpr (F8) {
                if (by_product)
                    out = quant_e4m3_8(v[c], s, __fmul_rn(r, kBracketLo), __fmul_rn(r, kBracketHi));
                else if (amax > 0.0f)
                    out = quant_e4m3_8_exact(v[c], s);
            } else if (by_product) {
                uint32_t b[8];
                quant_bits8(v[c], s, r, b);
                out.x = pack_low_bytes(b[0], b[1], b[2], b[3]);
                out.y = pack_low_bytes(b[4], b[5], b[6], b[7]);
            } else if (amax > 0.0f) {
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

// Raw 16-byte vectors of one row for this thread (zero past the row's end).
template <int NCH>
__device__ __forceinline__ void load_row(const uint4 *__restrict__ xr, int nvec, uint4 (&raw)[NCH])
{
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        const int vi = c * blockDim.x + threadIdx.x;
        raw[c] = vi < nvec ? ldg_nc_v4(xr + vi) : make_uint4(0u, 0u, 0u, 0u);
    }
}

// ----------------------------------------------------------------- quantize_rows
//
// Rows of up to 4096 values run with at most 256 threads (NCH <= 2); those kernels are
// compiled for several resident CTAs per SM (at most 40 registers for quantize_rows and
// SiLU, 85 for RMSNorm, which keeps gamma' in registers and loads the next row while it
// reduces the current one), since with so little work per thread the arithmetic and the
// reductions' latency, not HBM, set their pace.

template <int NCH, bool F8 = false>
__global__ void __launch_bounds__(NCH <= 2 ? 256 : 1024, NCH <= 2 ? 6 : 1) quantize_rows_kernel(const uint16_t *__restrict__ x,
                                                             const float *__restrict__ sinv,
                                                             int K, int M,
                                                             int8_t *__restrict__ q,
                                                             float *__restrict__ s_tok)
{
    __shared__ float sh[2][32]; // by row parity: one barrier per row
    if (threadIdx.x == 0)
        pdl_launch_dependents();
    pdl_wait(); // every input may come from the previous kernel
    const int nvec = K >> 3;
    int64_t row = blockIdx.x;
    for (uint32_t it = 0; row < M; row += gridDim.x, ++it) {
        uint4 raw[NCH];
        load_row<NCH>(reinterpret_cast<const uint4 *>(x + row * K), nvec, raw);
        float v[NCH][8];
#pragma unroll
        for (int c = 0; c < NCH; ++c)
            unpack8(raw[c], v[c]);
        float amax = 0.0f;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const int vi = c * blockDim.x + threadIdx.x;
            if (vi < nvec) {
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
            }
        }
        amax = block_max(amax, sh[it & 1u]);
        quantize_and_store<NCH, F8>(v, amax, 0, nvec, q + row * K, s_tok + row);
    }
}

// ----------------------------------------------------------------- static per-tensor scale
//
// One scale S for every token, fixed offline by min-max calibration: no reduction, so the
// kernel is a grid-stride pass over the 8-value vectors of all rows (HBM-bound). Values
// beyond the calibrated range saturate at +-127.

__global__ void __launch_bounds__(256) quantize_rows_static_kernel(
    const uint16_t *__restrict__ x, const float *__restrict__ sinv, float S, int K,
    int64_t nvec_total, int M, int8_t *__restrict__ q, float *__restrict__ s_tok)
{
    constexpr int kU = 4; // vectors per thread per pass, all loads issued before any use
    if (threadIdx.x == 0)
        pdl_launch_dependents();
    pdl_wait(); // every input may come from the previous kernel
    const int nvec = K >> 3;
    const bool by_product = S >= 7.888609052210118e-31f; // 2^-100: finite reciprocal
    const float r = by_product ? __frcp_rn(S) : 0.0f;
    const uint4 *xv = reinterpret_cast<const uint4 *>(x);
    // each CTA walks one contiguous range of vectors (DRAM locality), kU * blockDim.x
    // vectors per pass, consecutive threads on consecutive vectors
    const int64_t per_cta = (nvec_total + gridDim.x - 1) / gridDim.x;
    const int64_t begin = static_cast<int64_t>(blockIdx.x) * per_cta;
    const int64_t end = begin + per_cta < nvec_total ? begin + per_cta : nvec_total;
    const int step = static_cast<int>(blockDim.x) % nvec; // column advance per vector step
    int c0 = static_cast<int>((begin + threadIdx.x) % nvec);
    for (int64_t v0 = begin + threadIdx.x; v0 < end; v0 += kU * blockDim.x) {
        uint4 raw[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int64_t v = v0 + u * static_cast<int64_t>(blockDim.x);
            raw[u] = v < end ? ldg_nc_v4(xv + v) : make_uint4(0u, 0u, 0u, 0u);
        }
        int c = c0;
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int64_t v = v0 + u * static_cast<int64_t>(blockDim.x);
            if (v >= end)
                break;
            float y[8];
            unpack8(raw[u], y);
            if (sinv) {
                const float4 a = __ldg(reinterpret_cast<const float4 *>(sinv) + 2 * c);
                const float4 b = __ldg(reinterpret_cast<const float4 *>(sinv) + 2 * c + 1);
                const float w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
                for (int i = 0; i < 8; i += 2) {
                    const float2 p = mul2(make_float2(y[i], y[i + 1]), make_float2(w[i], w[i + 1]));
                    y[i] = p.x;
                    y[i + 1] = p.y;
                }
            }
            uint32_t bits[8];
            if (by_product) {
                quant_bits8<true>(y, S, r, bits);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    bits[i] = quant_bits(y[i], S);
            }
            reinterpret_cast<uint2 *>(q)[v] =
                make_uint2(pack_low_bytes(bits[0], bits[1], bits[2], bits[3]),
                           pack_low_bytes(bits[4], bits[5], bits[6], bits[7]));
            c += step;
            if (c >= nvec)
                c -= nvec;
        }
        c0 = c; // after kU steps (or the end)
    }
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    if (s_tok)
        for (int64_t m = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; m < M;
             m += stride)
            s_tok[m] = S;
}

// ----------------------------------------------------------------- smoothed RMSNorm + quant

template <int NCH, bool RES, bool F8 = false>
__global__ void __launch_bounds__(NCH <= 2 ? 256 : 1024, NCH <= 2 ? 3 : 1) rmsnorm_quant_kernel(
    const uint16_t *__restrict__ x, const uint16_t *__restrict__ res, uint16_t *__restrict__ h_out,
    const float *__restrict__ gamma, float eps, int K, int M, int8_t *__restrict__ q,
    float *__restrict__ s_tok, bool gamma_early)
{
    // the sum's and the max's buffers alternate, so each is rewritten only after the other's
    // barrier: two barriers per row
    __shared__ double shd[32];
    __shared__ float shf[32];
    if (threadIdx.x == 0)
        pdl_launch_dependents();
    const int nvec = K >> 3;
    // gamma' of this thread's vectors, the same for every row: for short rows read once and
    // kept in registers, for long rows re-read per row. gamma_early (overlap mode 2: no
    // kernel still in flight writes gamma') reads it, or brings it into L2, before the
    // dependency wait; otherwise it is read together with the first row, so its latency
    // overlaps the row's.
    constexpr bool kKeepGamma = NCH <= 2;
    float gk[kKeepGamma ? NCH : 1][8];
    auto read_gamma = [&]() {
        if constexpr (kKeepGamma) {
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                const int vi = c * blockDim.x + threadIdx.x;
                const float4 a = vi < nvec ? __ldg(reinterpret_cast<const float4 *>(gamma) + 2 * vi)
                                           : make_float4(0.f, 0.f, 0.f, 0.f);
                const float4 b = vi < nvec
                                     ? __ldg(reinterpret_cast<const float4 *>(gamma) + 2 * vi + 1)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
                gk[c][0] = a.x; gk[c][1] = a.y; gk[c][2] = a.z; gk[c][3] = a.w;
                gk[c][4] = b.x; gk[c][5] = b.y; gk[c][6] = b.z; gk[c][7] = b.w;
            }
        }
    };
    if (gamma_early) {
        if constexpr (kKeepGamma) {
            read_gamma();
        } else {
            // one 128-byte line (32 values) per 4 vectors of gamma'
            for (int l = threadIdx.x; l < (nvec + 3) / 4; l += blockDim.x)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(gamma + 32 * l));
        }
    }
    pdl_wait(); // every other input may come from the previous kernel
    if (!gamma_early)
        read_gamma();
    int64_t row = blockIdx.x;
    // short rows: the next row's loads are issued before this row's reductions, so each CTA
    // keeps a row in flight while it works on another
    constexpr bool kPre = NCH <= 2;
    uint4 nx[kPre ? NCH : 1], nr[kPre && RES ? NCH : 1];
    if constexpr (kPre) {
        if (row < M) {
            load_row<NCH>(reinterpret_cast<const uint4 *>(x + row * K), nvec, nx);
            if constexpr (RES)
                load_row<NCH>(reinterpret_cast<const uint4 *>(res + row * K), nvec, nr);
        }
    }
    for (; row < M; row += gridDim.x) {
        uint4 rx[NCH], rr[RES ? NCH : 1];
        if constexpr (kPre) {
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                rx[c] = nx[c];
                if constexpr (RES)
                    rr[c] = nr[c];
            }
            const int64_t next = row + gridDim.x;
            if (next < M) {
                load_row<NCH>(reinterpret_cast<const uint4 *>(x + next * K), nvec, nx);
                if constexpr (RES)
                    load_row<NCH>(reinterpret_cast<const uint4 *>(res + next * K), nvec, nr);
            }
        } else {
            load_row<NCH>(reinterpret_cast<const uint4 *>(x + row * K), nvec, rx);
            if constexpr (RES)
                load_row<NCH>(reinterpret_cast<const uint4 *>(res + row * K), nvec, rr);
        }
        float v[NCH][8];
        double ss = 0.0;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            unpack8(rx[c], v[c]);
            if constexpr (RES) {
                const int vi = c * blockDim.x + threadIdx.x;
                float r[8];
                unpack8(rr[c], r);
                uint4 hb;
                hb.x = pack_bf16x2(__fadd_rn(v[c][0], r[0]), __fadd_rn(v[c][1], r[1]));
                hb.y = pack_bf16x2(__fadd_rn(v[c][2], r[2]), __fadd_rn(v[c][3], r[3]));
                hb.z = pack_bf16x2(__fadd_rn(v[c][4], r[4]), __fadd_rn(v[c][5], r[5]));
                hb.w = pack_bf16x2(__fadd_rn(v[c][6], r[6]), __fadd_rn(v[c][7], r[7]));
                if (vi < nvec)
                    reinterpret_cast<uint4 *>(h_out + row * K)[vi] = hb;
                unpack8(hb, v[c]);
            }
        }
#pragma unroll
        for (int c = 0; c < NCH; ++c)
#pragma unroll
            for (int i = 0; i < 8; ++i) // each square of a bf16 value is exact in binary32
                ss = __dadd_rn(ss, static_cast<double>(__fmul_rn(v[c][i], v[c][i])));
        const double sum = block_sum(ss, shd);
        // sum / K: a power-of-two K divides exactly by scaling
        const double mean = (K & (K - 1)) == 0 ? __dmul_rn(sum, 1.0 / static_cast<double>(K))
                                               : __ddiv_rn(sum, static_cast<double>(K));
        const float ms = __double2float_rn(mean);
        const float rstd = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
        float amax = 0.0f;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const int vi = c * blockDim.x + threadIdx.x;
            if (vi < nvec) {
                float g[8];
                if constexpr (kKeepGamma) {
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        g[i] = gk[c][i];
                } else {
                    const float4 a = __ldg(reinterpret_cast<const float4 *>(gamma) + 2 * vi);
                    const float4 b = __ldg(reinterpret_cast<const float4 *>(gamma) + 2 * vi + 1);
                    g[0] = a.x; g[1] = a.y; g[2] = a.z; g[3] = a.w;
                    g[4] = b.x; g[5] = b.y; g[6] = b.z; g[7] = b.w;
                }
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
        quantize_and_store<NCH, F8>(v, amax, 0, nvec, q + row * K, s_tok + row);
    }
}

// ----------------------------------------------------------------- SiLU(gate)*up + quant

// Binary32 exp fixed by the library's contract (header w8a8.h), two lanes at a time:
// Cody-Waite reduction with a 16-bit head of ln 2, degree-7 Taylor polynomial by Horner in
// fused multiply-adds, exact scaling by two powers of two; every step is the scalar
// definition's IEEE operation, lane by lane. exp_poly2 returns the polynomial p and k.
__device__ __forceinline__ float2 exp_poly2(float2 x, int &ka, int &kb)
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
    ka = __float_as_int(km.x) - kRoundMagicBits;
    kb = __float_as_int(km.y) - kRoundMagicBits;
    return p;
}

// p * 2^k1 * 2^k2 (k1 = k / 2 truncated, k2 = k - k1), and the range rules: NaN stays NaN,
// x > 89 gives +inf, x < -104 gives +0.
__device__ __forceinline__ float exp_scale_full(float p, int k, float x)
{
    const int k1 = k / 2; // truncation toward zero
    const float e = __fmul_rn(__fmul_rn(p, __int_as_float((k1 + 127) << 23)),
                              __int_as_float((k - k1 + 127) << 23));
    const float inf = __int_as_float(0x7f800000);
    return (x != x) ? x : (x > 89.0f ? inf : (x < -104.0f ? 0.0f : e));
}

// a = silu(g) * u = (g / (1 + exp(-g))) * u for the eight values of one vector; the
// divisions stay IEEE scalar. When every |g| <= 80 (one test per vector), |k| <= 115 and
// p in [0.7, 1.5) make every partial product of the two power-of-two scalings a normal
// number, so both are exact and equal adding k to p's exponent.
__device__ __forceinline__ void silu_mul8(const float (&g)[8], const float (&u)[8], float (&a)[8])
{
    float e[8];
    int k[8];
    bool in_range = true;
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        const float2 p = exp_poly2(make_float2(-g[i], -g[i + 1]), k[i], k[i + 1]);
        e[i] = p.x;
        e[i + 1] = p.y;
        in_range &= (fabsf(g[i]) <= 80.0f) & (fabsf(g[i + 1]) <= 80.0f);
    }
    if (in_range) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            e[i] = __uint_as_float(__float_as_uint(e[i]) + (static_cast<uint32_t>(k[i]) << 23));
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            e[i] = exp_scale_full(e[i], k[i], -g[i]);
    }
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        const float2 d = add2(splat2(1.0f), make_float2(e[i], e[i + 1]));
        const float2 q = make_float2(__fdiv_rn(g[i], d.x), __fdiv_rn(g[i + 1], d.y));
        const float2 r = mul2(q, make_float2(u[i], u[i + 1]));
        a[i] = r.x;
        a[i + 1] = r.y;
    }
}

template <int NCH, bool F8 = false>
__global__ void __launch_bounds__(NCH <= 2 ? 256 : 1024, NCH <= 2 ? 6 : 1) silu_mul_quant_kernel(const uint16_t *__restrict__ gu,
                                                              int I, int M,
                                                              int8_t *__restrict__ q,
                                                              float *__restrict__ s_tok)
{
    __shared__ float sh[2][32]; // by row parity: one barrier per row
    if (threadIdx.x == 0)
        pdl_launch_dependents();
    pdl_wait(); // every input may come from the previous kernel
    const int nvec = I >> 3;
    int64_t row = blockIdx.x;
    for (uint32_t it = 0; row < M; row += gridDim.x, ++it) {
        uint4 cg[NCH], cu[NCH];
        const uint4 *gr = reinterpret_cast<const uint4 *>(gu + row * 2 * static_cast<int64_t>(I));
        load_row<NCH>(gr, nvec, cg);
        load_row<NCH>(gr + nvec, nvec, cu);
        float v[NCH][8];
        float amax = 0.0f;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const int vi = c * blockDim.x + threadIdx.x;
            if (vi < nvec) {
                float g[8], u[8];
                unpack8(cg[c], g);
                unpack8(cu[c], u);
                silu_mul8(g, u, v[c]);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    amax = fmaxf(amax, fabsf(v[c][i]));
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    v[c][i] = 0.0f;
            }
        }
        amax = block_max(amax, sh[it & 1u]);
        quantize_and_store<NCH, F8>(v, amax, 0, nvec, q + row * I, s_tok + row);
    }
}

// ----------------------------------------------------------------- quantization of fp32 rows
//
// Second half of the fused SiLU*up path: a (binary32 [M, I], written by the GEMM epilogue)
// is quantized per token with s = max_j |a[m, j]| / 127, exactly as the SiLU*up row kernel
// quantizes the same values.

template <int NCH, bool F8 = false>
__global__ void __launch_bounds__(NCH <= 2 ? 256 : 1024, NCH <= 2 ? 6 : 1) quantize_f32_rows_kernel(
    const float *__restrict__ a, int I, int M, int8_t *__restrict__ q, float *__restrict__ s_tok)
{
    __shared__ float sh[2][32]; // by row parity: one barrier per row
    if (threadIdx.x == 0)
        pdl_launch_dependents();
    pdl_wait(); // a comes from the previous kernel
    const int nvec = I >> 3;
    int64_t row = blockIdx.x;
    for (uint32_t it = 0; row < M; row += gridDim.x, ++it) {
        const float4 *ar = reinterpret_cast<const float4 *>(a + row * I);
        float v[NCH][8];
        float amax = 0.0f;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const int vi = c * blockDim.x + threadIdx.x;
            if (vi < nvec) {
                const float4 lo = __ldcs(ar + 2 * vi);
                const float4 hi = __ldcs(ar + 2 * vi + 1);
                v[c][0] = lo.x; v[c][1] = lo.y; v[c][2] = lo.z; v[c][3] = lo.w;
                v[c][4] = hi.x; v[c][5] = hi.y; v[c][6] = hi.z; v[c][7] = hi.w;
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    v[c][i] = 0.0f;
            }
        }
#pragma unroll
        for (int c = 0; c < NCH; ++c)
#pragma unroll
            for (int i = 0; i < 8; ++i)
                amax = fmaxf(amax, fabsf(v[c][i]));
        amax = block_max(amax, sh[it & 1u]);
        quantize_and_store<NCH, F8>(v, amax, 0, nvec, q + row * I, s_tok + row);
    }
}

// The same quantization of a when the SiLU*up epilogue has already taken the max |a| of
// every (token, group of 64 channels) (SiluOut::amax): a token's scale is the max of its I / 64
// partial maxima divided by 127 (448 for E4M3). The max is exact and order-free, so the scale,
// and with it every code, is bit-identical to a pass over the whole row. With the row's range
// known, a row no longer has to sit in one CTA: CTA (x, m) codes the x-th slice of
// 8 * blockDim values of row m, so a pass over few tokens still spreads over many SMs; the
// CTAs of slice 0 write the scales.
template <bool F8 = false>
__global__ void __launch_bounds__(256) quantize_f32_parts_kernel(
    const float *__restrict__ a, const float *__restrict__ amax_part, int I, int M,
    int8_t *__restrict__ q, float *__restrict__ s_tok)
{
    __shared__ float sh[32];
    if (threadIdx.x == 0)
        pdl_launch_dependents();
    pdl_wait(); // a and the maxima come from the previous kernel
    const int64_t m = blockIdx.y;
    const int groups = I >> 6;
    const int nvec = I >> 3;
    const int v0 = blockIdx.x * blockDim.x;
    const int vi = v0 + threadIdx.x;
    // this thread's 8 values, requested before the reduction so that the two overlap
    float v[1][8];
    if (vi < nvec) {
        const float4 *ar = reinterpret_cast<const float4 *>(a + m * I);
        const float4 lo = __ldcs(ar + 2 * vi);
        const float4 hi = __ldcs(ar + 2 * vi + 1);
        v[0][0] = lo.x; v[0][1] = lo.y; v[0][2] = lo.z; v[0][3] = lo.w;
        v[0][4] = hi.x; v[0][5] = hi.y; v[0][6] = hi.z; v[0][7] = hi.w;
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            v[0][i] = 0.0f;
    }
    float mx = 0.0f;
    for (int j = threadIdx.x; j < groups; j += blockDim.x)
        mx = fmaxf(mx, __ldcg(amax_part + m * groups + j));
    mx = block_max(mx, sh);
    quantize_and_store<1, F8>(v, mx, v0, nvec, q + m * I, blockIdx.x == 0 ? s_tok + m : nullptr);
}

} // namespace w8a8
