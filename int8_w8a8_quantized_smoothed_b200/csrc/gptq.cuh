// GPTQ weight quantization on the GPU, in binary64 (offline preparation of the int8 weights).
//
// For each output channel (row of W [N, K]) the columns are quantized in order; after each
// rounding the error is spread over the columns not yet quantized through U, the upper
// Cholesky factor of the inverse Hessian (H^-1 = U^T U, H = (2/T) X^T X of the calibration
// inputs, dampened). Pipeline, all on the device:
//   hessian      H = (2/T) X^T X                         64 x 64 tiles of the lower half
//   diag         dead channels (H_jj = 0 -> 1), H_jj += damp * mean(H_jj)
//   UL Cholesky  H = V V^T with V upper, by 64-column blocks from the last to the first
//                (diagonal block, panel solve, trailing update of the blocks above-left)
//   inverse      U = V^-1 (upper): diagonal blocks inverted, then the off-diagonal blocks
//                right-looking from the bottom block row (every finished block row adds its
//                contributions to all pending blocks at once)
//   quantize     64-column blocks in order: four lanes per row (one thread per row when
//                the rows exceed one wave) run the block's columns sequentially
//                (quantize, error, compensate inside the block); the lazy
//                batch form applies the errors later, in two levels: each block's errors
//                go at once to the rest of its group of four blocks, and a group's 256
//                columns of errors go to every column after the group in one tiled pass
//                (the same sums as the column-by-column form, in another order)
// U = V^-1 is the Cholesky factor GPTQ needs: H = V V^T gives H^-1 = V^-T V^-1 = U^T U.
// The dense steps run on tiles staged in shared memory by asynchronous copies, each thread
// owning a register micro-tile of the result (4 x 4 in the Hessian, 8 x 4 in the trailing
// and lazy-batch updates) accumulated with fused multiply-adds.
#pragma once

#include <stdint.h>

namespace w8a8 {
namespace gptq {

constexpr int kT = 64;    // tile / column-block size
constexpr int kLd = 65;   // padded shared-memory row (doubles)
constexpr int kThreads = 256;
// dynamic shared memory of the two-tile kernels
constexpr int kTwoTileBytes = 2 * kT * kLd * 8;

extern __shared__ __align__(16) double gptq_smem[];

// The trailing-update tile kernels run 128 threads, each owning an 8 x 4 micro-tile of the
// 64 x 64 result (rows ty + 8a, columns tx + 16b): twelve shared-memory loads per 32 FMAs.
constexpr int kTileThreads = 128;

// acc[a][b] += sum_k A[ty + 8a][k] * B[k][tx + 16b], or B[tx + 16b][k] when BT
template <bool BT>
__device__ __forceinline__ void mm84(const double *A, const double *B, double (&acc)[8][4])
{
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll 4
    for (int k = 0; k < kT; ++k) {
        double a[8], b[4];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            a[i] = A[(ty + 8 * i) * kLd + k];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            b[i] = BT ? B[(tx + 16 * i) * kLd + k] : B[k * kLd + tx + 16 * i];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j)
                acc[i][j] = fma(a[i], b[j], acc[i][j]);
    }
}

__device__ __forceinline__ void zero_acc84(double (&acc)[8][4])
{
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            acc[i][j] = 0.0;
}

// the 64 x 64 block (r0, c0) of a row-major matrix into L2 (four 128-byte lines per row)
__device__ __forceinline__ void prefetch_tile_l2(const double *g, int64_t ld, int64_t r0,
                                                 int64_t c0)
{
    for (int l = threadIdx.x; l < kT * 4; l += blockDim.x)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(g + (r0 + (l >> 2)) * ld + c0 + (l & 3) * 16));
}

// asynchronous global -> shared copies (complete after cp_async_wait_all)
__device__ __forceinline__ void cp_async8(double *smem, const double *gmem)
{
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(a), "l"(gmem) : "memory");
}

__device__ __forceinline__ void cp_async16(double *smem, const double *gmem)
{
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(a), "l"(gmem) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all()
{
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// 64 x 64 block (r0, c0) of a row-major matrix with leading dimension ld -> smem [64][kLd],
// issued as asynchronous copies: the caller waits (cp_async_wait_all) and synchronizes.
template <int NT = kThreads>
__device__ __forceinline__ void load_tile(double *sm, const double *g, int64_t ld, int64_t r0,
                                          int64_t c0)
{
#pragma unroll 4
    for (int e = threadIdx.x; e < kT * kT; e += NT) {
        const int r = e >> 6, c = e & 63;
        cp_async8(sm + r * kLd + c, g + (r0 + r) * ld + c0 + c);
    }
}

__device__ __forceinline__ void zero_acc(double (&acc)[4][4])
{
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            acc[i][j] = 0.0;
}

// ------------------------------------------------------------------ Hessian

// One CTA per 64 x 64 tile (ti >= tj) of H = (2/T) X^T X, X binary32 [T, K] (K % 64 == 0);
// the tile and its mirror are written.
__global__ void __launch_bounds__(kThreads) hessian_kernel(const float *__restrict__ x, int64_t T,
                                                          int64_t K, double *__restrict__ H)
{
    __shared__ double sa[16][kT + 1], sb[16][kT + 1];
    // blockIdx.x -> (ti, tj), ti >= tj, row-major over the lower triangle of tiles
    int64_t b = blockIdx.x, ti = 0;
    while (b > ti) {
        b -= ti + 1;
        ++ti;
    }
    const int64_t tj = b;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    double acc[4][4];
    zero_acc(acc);
    for (int64_t t0 = 0; t0 < T; t0 += 16) {
        for (int e = threadIdx.x; e < 16 * kT; e += kThreads) {
            const int r = e >> 6, c = e & 63;
            const bool ok = t0 + r < T;
            sa[r][c] = ok ? static_cast<double>(x[(t0 + r) * K + ti * kT + c]) : 0.0;
            sb[r][c] = ok ? static_cast<double>(x[(t0 + r) * K + tj * kT + c]) : 0.0;
        }
        __syncthreads();
#pragma unroll 4
        for (int t = 0; t < 16; ++t) {
            double a[4], bb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[i] = sa[t][ty + 16 * i];
                bb[i] = sb[t][tx + 16 * i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    acc[i][j] = fma(a[i], bb[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t r = ti * kT + ty + 16 * i, c = tj * kT + tx + 16 * j;
            const double h = 2.0 * acc[i][j] / static_cast<double>(T);
            H[r * K + c] = h;
            H[c * K + r] = h;
        }
}

// Dead channels and dampening (one CTA): H_jj = 0 -> 1 and dead[j] = 1; then
// H_jj += damp * mean_j H_jj.
__global__ void __launch_bounds__(1024) diag_kernel(double *__restrict__ H, int64_t K,
                                                   double damp, uint8_t *__restrict__ dead)
{
    __shared__ double red[32];
    double sum = 0.0;
    for (int64_t j = threadIdx.x; j < K; j += blockDim.x) {
        double h = H[j * K + j];
        const bool d = h == 0.0;
        dead[j] = d ? 1 : 0;
        if (d) {
            h = 1.0;
            H[j * K + j] = h;
        }
        sum += h;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if ((threadIdx.x & 31) == 0)
        red[threadIdx.x >> 5] = sum;
    __syncthreads();
    if (threadIdx.x < 32) {
        double v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            v += __shfl_xor_sync(0xffffffffu, v, o);
        if (threadIdx.x == 0)
            red[0] = v;
    }
    __syncthreads();
    const double add = damp * (red[0] / static_cast<double>(K));
    for (int64_t j = threadIdx.x; j < K; j += blockDim.x)
        H[j * K + j] += add;
}

// ------------------------------------------------------------------ UL Cholesky H = V V^T

// Diagonal block kb: D = V_kk V_kk^T, V_kk upper, right-looking from the last column; the
// block's upper triangle is overwritten with V_kk. A non-positive pivot (H not positive
// definite) is replaced by the smallest normal double and reported through *bad.
// One barrier per column: every thread forms the pivot and its reciprocal itself, the scaled
// column V[i][j] = D[i][j] / V[j][j] (i < j) goes to the unused lower triangle (d[j][i]) and
// the pivot to dg[j], so nothing read in a step is written in it.
__global__ void __launch_bounds__(kThreads) chol_diag_kernel(double *__restrict__ A, int64_t K,
                                                            int kb, int *__restrict__ bad)
{
    __shared__ double d[kT * kLd];
    __shared__ double dg[kT];
    const int64_t o = static_cast<int64_t>(kb) * kT;
    load_tile(d, A, K, o, o);
    cp_async_wait_all();
    __syncthreads();
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    for (int j = kT - 1; j >= 0; --j) {
        double p = d[j * kLd + j];
        const bool ok = p > 0.0;
        if (!ok)
            p = 2.2250738585072014e-308;
        const double vjj = sqrt(p);
        const double rinv = 1.0 / vjj;
        if (threadIdx.x == 0) {
            if (!ok)
                atomicExch(bad, 1);
            dg[j] = vjj;
        }
        if (threadIdx.x < j)
            d[j * kLd + threadIdx.x] = d[threadIdx.x * kLd + j] * rinv;
        // D[i][i'] -= V[i][j] V[i'][j] for i <= i' < j (upper triangle of the rest); thread
        // (ty, tx) owns rows ty + 16a and columns tx + 16b
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const int i = ty + 16 * a;
            if (i < j) {
                const double vi = d[i * kLd + j] * rinv;
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const int i2 = tx + 16 * b;
                    if (i <= i2 && i2 < j)
                        d[i * kLd + i2] -= vi * (d[i2 * kLd + j] * rinv);
                }
            }
        }
        __syncthreads();
    }
    for (int e = threadIdx.x; e < kT * kT; e += kThreads) {
        const int r = e >> 6, c = e & 63;
        if (r <= c)
            A[(o + r) * K + o + c] = r == c ? dg[r] : d[c * kLd + r];
    }
}

// Panel of block column kb: V[ib][kb] = A[ib][kb] V_kk^-T for every ib < kb (one CTA each):
// X V_kk^T = A solved from the last column: x_j = a_j / V[j][j], then a_k -= x_j V[k][j]
// for k < j. The rows are independent: one thread per row holds its 64 values in registers
// (loops unrolled, constant register indices) and reads V's column j as a shared-memory
// broadcast, so the column loop needs no barrier; a compiler barrier per column keeps the
// next column's loads of V from being hoisted (register pressure).
__global__ void __launch_bounds__(kT) chol_panel_kernel(double *__restrict__ A, int64_t K, int kb)
{
    __shared__ __align__(16) double v[kT * kT]; // V_kk, unpadded
    __shared__ double vinv[kT];                 // 1 / V[j][j]
    const int64_t oc = static_cast<int64_t>(kb) * kT, orow = static_cast<int64_t>(blockIdx.x) * kT;
    for (int e = threadIdx.x; e < kT * (kT / 2); e += kT) {
        const int r = e >> 5, c = (e & 31) * 2;
        cp_async16(v + r * kT + c, A + (oc + r) * K + oc + c);
    }
    cp_async_wait_all();
    __syncthreads();
    vinv[threadIdx.x] = 1.0 / v[threadIdx.x * kT + threadIdx.x];
    __syncthreads();
    double a[kT];
    double2 *row = reinterpret_cast<double2 *>(A + (orow + threadIdx.x) * K + oc);
#pragma unroll
    for (int i = 0; i < kT / 2; ++i) {
        const double2 t = row[i];
        a[2 * i] = t.x;
        a[2 * i + 1] = t.y;
    }
#pragma unroll
    for (int j = kT - 1; j >= 0; --j) {
        const double x = a[j] * vinv[j];
        a[j] = x;
#pragma unroll
        for (int k = 0; k < kT; ++k)
            if (k < j)
                a[k] -= x * v[k * kT + j];
        asm volatile("" ::: "memory");
    }
#pragma unroll
    for (int i = 0; i < kT / 2; ++i)
        row[i] = make_double2(a[2 * i], a[2 * i + 1]);
}

// Trailing update after block column kb: A[ib][jb] -= V[ib][kb] V[jb][kb]^T for
// ib <= jb < kb (the upper triangle of the remaining blocks); one CTA per pair.
__global__ void __launch_bounds__(kTileThreads) chol_update_kernel(double *__restrict__ A,
                                                                  int64_t K, int kb)
{
    double *p1 = gptq_smem, *p2 = gptq_smem + kT * kLd;
    int64_t b = blockIdx.x, jb = 0;
    while (b > jb) { // pairs (ib <= jb), enumerated jb-major
        b -= jb + 1;
        ++jb;
    }
    const int64_t ib = b;
    const int64_t oc = static_cast<int64_t>(kb) * kT;
    prefetch_tile_l2(A, K, ib * kT, jb * kT);
    load_tile<kTileThreads>(p1, A, K, ib * kT, oc);
    load_tile<kTileThreads>(p2, A, K, jb * kT, oc);
    cp_async_wait_all();
    __syncthreads();
    double acc[8][4];
    zero_acc84(acc);
    mm84<true>(p1, p2, acc);
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t r = ib * kT + ty + 8 * i, c = jb * kT + tx + 16 * j;
            A[r * K + c] -= acc[i][j];
        }
}

// ------------------------------------------------------------------ U = V^-1 (upper)

// Diagonal blocks (one CTA each): U_kk = V_kk^-1 by back substitution, one column per
// thread: U[c][c] = 1 / V[c][c], U[i][c] = -(sum_{k=i+1..c} V[i][k] U[k][c]) / V[i][i].
// The block's lower triangle is written as zeros.
__global__ void __launch_bounds__(kT) trtri_diag_kernel(const double *__restrict__ V,
                                                       double *__restrict__ U, int64_t K)
{
    double *v = gptq_smem, *u = gptq_smem + kT * kLd;
    const int64_t o = static_cast<int64_t>(blockIdx.x) * kT;
    for (int e = threadIdx.x; e < kT * kT; e += blockDim.x) {
        const int r = e >> 6, c = e & 63;
        v[r * kLd + c] = r <= c ? V[(o + r) * K + o + c] : 0.0;
        u[r * kLd + c] = 0.0;
    }
    __syncthreads();
    const int c = threadIdx.x;
    u[c * kLd + c] = 1.0 / v[c * kLd + c];
    for (int i = c - 1; i >= 0; --i) {
        double s = 0.0;
        for (int k = i + 1; k <= c; ++k)
            s = fma(v[i * kLd + k], u[k * kLd + c], s);
        u[i * kLd + c] = -s / v[i * kLd + i];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < kT * kT; e += blockDim.x) {
        const int r = e >> 6, cc = e & 63;
        U[(o + r) * K + o + cc] = u[r * kLd + cc];
    }
}

// Off-diagonal blocks, right-looking from the bottom block row: U[i][j] (i < j) is
// -U_ii T[i][j] with T[i][j] = sum_{k=i+1..j} V[i][k] U[k][j]. The off-diagonal blocks of U hold
// the running sums T (zero to begin with); once block row k is final (trtri_final_kernel),
// trtri_update_kernel adds V[i][k] U[k][j] into T[i][j] for every i < k <= j, one product per
// CTA, so each T[i][j] receives its terms in the fixed order k = j, j-1, .., i+1.
__global__ void __launch_bounds__(kTileThreads) trtri_update_kernel(const double *__restrict__ V,
                                                                   double *__restrict__ U,
                                                                   int64_t K, int k)
{
    double *sa = gptq_smem, *sb = gptq_smem + kT * kLd;
    const int64_t nb = K / kT;
    const int64_t i = blockIdx.x % k, j = k + blockIdx.x / k; // i < k <= j < nb
    if (j >= nb)
        return;
    prefetch_tile_l2(U, K, i * kT, j * kT);
    load_tile<kTileThreads>(sa, V, K, i * kT, k * kT);
    load_tile<kTileThreads>(sb, U, K, k * kT, j * kT);
    cp_async_wait_all();
    __syncthreads();
    double acc[8][4];
    zero_acc84(acc);
    mm84<false>(sa, sb, acc);
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b)
            U[(i * kT + ty + 8 * a) * K + j * kT + tx + 16 * b] += acc[a][b];
}

// Block row k final: U[k][j] = -U_kk T[k][j] for every j > k (one CTA per j).
__global__ void __launch_bounds__(kTileThreads) trtri_final_kernel(double *__restrict__ U,
                                                                  int64_t K, int k)
{
    double *sa = gptq_smem, *sb = gptq_smem + kT * kLd;
    const int64_t j = k + 1 + blockIdx.x;
    load_tile<kTileThreads>(sa, U, K, static_cast<int64_t>(k) * kT, static_cast<int64_t>(k) * kT);
    load_tile<kTileThreads>(sb, U, K, static_cast<int64_t>(k) * kT, j * kT);
    cp_async_wait_all();
    __syncthreads();
    double acc[8][4];
    zero_acc84(acc);
    mm84<false>(sa, sb, acc);
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b)
            U[(static_cast<int64_t>(k) * kT + ty + 8 * a) * K + j * kT + tx + 16 * b] = -acc[a][b];
}

// Lower off-diagonal blocks of U are zero (U is returned whole to callers that ask for it).
__global__ void __launch_bounds__(kThreads) zero_lower_kernel(double *__restrict__ U, int64_t K)
{
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; e < K * K;
         e += static_cast<int64_t>(gridDim.x) * kThreads) {
        const int64_t r = e / K, c = e % K;
        if (r / kT > c / kT)
            U[e] = 0.0;
    }
}

// ------------------------------------------------------------------ quantize and compensate

// Working copy of the smoothed weight, binary64: W'[n][j] = bf16(w[n][j]) * s_j (binary32
// product, as the RTN path computes it), 0 for dead channels; s_ch[n] = max_j |W'[n][j]| / 127
// over the weight as given (binary32). One warp per row.
__global__ void __launch_bounds__(kThreads) prep_kernel(const uint16_t *__restrict__ w,
                                                       const float *__restrict__ smooth,
                                                       const uint8_t *__restrict__ dead,
                                                       int64_t N, int64_t K,
                                                       double *__restrict__ wd,
                                                       float *__restrict__ s_ch)
{
    const int lane = threadIdx.x & 31;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
    for (int64_t n = static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5);
         n < N; n += warps) {
        float amax = 0.0f;
        for (int64_t j = lane; j < K; j += 32) {
            float f = __uint_as_float(static_cast<uint32_t>(w[n * K + j]) << 16);
            if (smooth)
                f = __fmul_rn(f, smooth[j]);
            amax = fmaxf(amax, fabsf(f));
            wd[n * K + j] = dead[j] ? 0.0 : static_cast<double>(f);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (lane == 0)
            s_ch[n] = __fdiv_rn(amax, 127.0f);
    }
}

// Column block jb (columns j0 .. j0 + 63), four lanes per weight row: lane l of a quad holds
// columns 4i + l (i = 0..15) in registers. For each column j = 4i + o in order the quad's
// lane o rounds w_j / s and forms the error e = (w_j - q s) / U[j][j]; a quad shuffle hands e
// to the other three, and each lane subtracts e U[j][k] from its columns k > j (U's rows
// are read from shared memory, four distinct words per warp access). Every lane forms the
// code and error of its own column i and lane o's are kept, so the loop has no branch; the
// loops are unrolled, so register indices and o are compile-time constants, and a compiler
// barrier per column keeps the next column's loads of U from being hoisted. A zero scale has
// a zero reciprocal, so its codes are 0. Errors go to err[n * err_ld + t] (t = 0..63),
// codes to wq. The whole warp walks its 8 rows together (shuffles need every lane); a row
// past N repeats row N - 1 and stores nothing.
constexpr int kQuantThreads = 128;

__global__ void __launch_bounds__(kQuantThreads) quant_block_kernel(
    double *__restrict__ wd, const double *__restrict__ U, const float *__restrict__ s_ch,
    int64_t N, int64_t K, int jb, int8_t *__restrict__ wq, double *__restrict__ err,
    int64_t err_ld)
{
    __shared__ __align__(16) double u[kT * kT]; // the diagonal block of U, unpadded
    __shared__ double uinv[kT];                 // 1 / U[j][j]
    const int64_t j0 = static_cast<int64_t>(jb) * kT;
    for (int e = threadIdx.x; e < kT * (kT / 2); e += blockDim.x) {
        const int r = e >> 5, c = (e & 31) * 2;
        cp_async16(u + r * kT + c, U + (j0 + r) * K + j0 + c);
    }
    cp_async_wait_all();
    __syncthreads();
    for (int t = threadIdx.x; t < kT; t += blockDim.x)
        uinv[t] = 1.0 / u[t * kT + t];
    __syncthreads();
    const int l = threadIdx.x & 3, lane = threadIdx.x & 31;
    const int qbase = lane & ~3;
    double ui[kT / 4]; // 1 / U[c][c] of this lane's columns
#pragma unroll
    for (int i = 0; i < kT / 4; ++i)
        ui[i] = uinv[4 * i + l];
    const int64_t warp = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x / 32);
    for (int64_t n0 = warp * 8; n0 < N; n0 += warps * 8) {
        const int64_t n = n0 + (lane >> 2);
        const int64_t nr = n < N ? n : N - 1;
        double w[kT / 4];
#pragma unroll
        for (int i = 0; i < kT / 4; ++i)
            w[i] = wd[nr * K + j0 + 4 * i + l];
        const double s = static_cast<double>(s_ch[nr]);
        const double sinv = s > 0.0 ? 1.0 / s : 0.0;
        uint32_t qp[kT / 16];
#pragma unroll
        for (int i = 0; i < kT / 16; ++i)
            qp[i] = 0u;
#pragma unroll
        for (int j = 0; j < kT; ++j) {
            const int i = j >> 2, o = j & 3;
            const double qc = fmin(fmax(rint(w[i] * sinv), -127.0), 127.0);
            const double ec = (w[i] - qc * s) * ui[i];
            const double e = __shfl_sync(0xffffffffu, ec, qbase | o);
            if (l == o)
                qp[i >> 2] |= (static_cast<uint32_t>(static_cast<int>(qc)) & 0xffu)
                              << (8 * (i & 3));
#pragma unroll
            for (int ii = 0; ii < kT / 4; ++ii)
                if (ii > i || (ii == i && l > o))
                    w[ii] -= e * u[j * kT + 4 * ii + l];
            if (l == o)
                w[i] = e;
            asm volatile("" ::: "memory");
        }
        if (n < N) {
#pragma unroll
            for (int i = 0; i < kT / 4; ++i) {
                err[n * err_ld + 4 * i + l] = w[i];
                wq[n * K + j0 + 4 * i + l] = static_cast<int8_t>((qp[i >> 2] >> (8 * (i & 3))) & 0xffu);
            }
        }
    }
}

// Column block jb for many rows (one wave of the four-lane form does not hold them): one
// thread per weight row with the row's 64 block columns in registers: for each column j in order it rounds w_j / s, forms the error
// e = (w_j - q s) / U[j][j] and subtracts e U[j][k] from its columns k > j (U's rows are
// shared-memory broadcasts: every thread of a warp reads the same word). The loops are
// unrolled, so every register index is a compile-time constant; nothing crosses lanes, so the
// only serial chain is one row's own column steps. A zero scale has a zero reciprocal, so its
// codes are 0. Each error replaces its dead column value, so the row's 64 errors go to
// err[n * err_ld + t] (t = 0..63) as vector stores, and its 64 codes to wq as four 16-byte
// stores.
__global__ void __launch_bounds__(128) quant_block_rows_kernel(double *__restrict__ wd,
                                                         const double *__restrict__ U,
                                                         const float *__restrict__ s_ch,
                                                         int64_t N, int64_t K, int jb,
                                                         int8_t *__restrict__ wq,
                                                         double *__restrict__ err,
                                                         int64_t err_ld)
{
    __shared__ __align__(16) double u[kT * kT]; // the diagonal block of U, unpadded
    __shared__ double uinv[kT];                 // 1 / U[j][j]
    const int64_t j0 = static_cast<int64_t>(jb) * kT;
    for (int e = threadIdx.x; e < kT * (kT / 2); e += blockDim.x) {
        const int r = e >> 5, c = (e & 31) * 2;
        cp_async16(u + r * kT + c, U + (j0 + r) * K + j0 + c);
    }
    cp_async_wait_all();
    __syncthreads();
    for (int t = threadIdx.x; t < kT; t += blockDim.x)
        uinv[t] = 1.0 / u[t * kT + t];
    __syncthreads();
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t n = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; n < N;
         n += stride) {
        double w[kT];
        const double2 *src = reinterpret_cast<const double2 *>(wd + n * K + j0);
#pragma unroll
        for (int i = 0; i < kT / 2; ++i) {
            const double2 v = src[i];
            w[2 * i] = v.x;
            w[2 * i + 1] = v.y;
        }
        const double s = static_cast<double>(s_ch[n]);
        const double sinv = s > 0.0 ? 1.0 / s : 0.0;
        uint32_t qp[kT / 4];
#pragma unroll
        for (int i = 0; i < kT / 4; ++i)
            qp[i] = 0u;
#pragma unroll
        for (int j = 0; j < kT; ++j) {
            const double q = fmin(fmax(rint(w[j] * sinv), -127.0), 127.0);
            const double e = (w[j] - q * s) * uinv[j];
            qp[j >> 2] |= (static_cast<uint32_t>(static_cast<int>(q)) & 0xffu) << (8 * (j & 3));
#pragma unroll
            for (int k = 0; k < kT; ++k)
                if (k > j)
                    w[k] -= e * u[j * kT + k];
            w[j] = e;
            // keeps the next step's loads of U out of this one (register pressure)
            asm volatile("" ::: "memory");
        }
        double2 *eo = reinterpret_cast<double2 *>(err + n * err_ld);
#pragma unroll
        for (int i = 0; i < kT / 2; ++i)
            eo[i] = make_double2(w[2 * i], w[2 * i + 1]);
        uint4 *qo = reinterpret_cast<uint4 *>(wq + n * K + j0);
#pragma unroll
        for (int i = 0; i < kT / 16; ++i)
            qo[i] = make_uint4(qp[4 * i], qp[4 * i + 1], qp[4 * i + 2], qp[4 * i + 3]);
    }
}

// Update tiles: 128 rows x 64 columns; the depth is staged 32 at a time (err [128][32] and
// U [32][64], rows padded to 16-byte multiples), two stages in flight; dynamic shared memory.
constexpr int kRT = 128;
constexpr int kDC = 32;
constexpr int kLdE = kDC + 2;
constexpr int kLdU = kT + 2;
constexpr int kStage = kRT * kLdE + kDC * kLdU; // doubles
constexpr int kUpdateBytes = 2 * kStage * 8;

// Lazy batch update: W'[n][c] -= sum_t err[n][t] U[j0 + t][c] for t < 64 * chunks and the
// columns c = c_first + 64 * blockIdx.x + (0..63). One CTA per 128 x 64 tile of W' (a tile
// past row N reads row N - 1 and writes nothing there); each thread owns an 8 x 4
// micro-tile (rows ty + 16a, columns tx + 16b). The depth runs in 32-deep stages copied to
// shared memory with 16-byte asynchronous copies, the next stage's copies in flight while
// the current one is multiplied; the tile of W' is prefetched into L2 at the start.
// err rows, U rows and c_first are multiples of 16 bytes apart (64-column blocks, binary64).
__global__ void __launch_bounds__(kThreads) update_kernel(double *__restrict__ wd,
                                                         const double *__restrict__ U,
                                                         const double *__restrict__ err,
                                                         int64_t err_ld, int64_t N, int64_t K,
                                                         int64_t j0, int chunks,
                                                         int64_t c_first)
{
    const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kRT;
    const int64_t c0 = c_first + static_cast<int64_t>(blockIdx.x) * kT;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    // the W' tile: 128 rows of four 128-byte lines
    for (int l = threadIdx.x; l < kRT * 4; l += kThreads) {
        const int64_t r = r0 + (l >> 2);
        if (r < N)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(wd + r * K + c0 + (l & 3) * 16));
    }
    auto stage = [&](int buf, int cc) {
        double *se = gptq_smem + buf * kStage, *su = se + kRT * kLdE;
#pragma unroll
        for (int e = threadIdx.x; e < kRT * (kDC / 2); e += kThreads) {
            const int r = e >> 4, c = (e & 15) * 2;
            const int64_t n = r0 + r < N ? r0 + r : N - 1;
            cp_async16(se + r * kLdE + c, err + n * err_ld + cc * kDC + c);
        }
#pragma unroll
        for (int e = threadIdx.x; e < kDC * (kT / 2); e += kThreads) {
            const int r = e >> 5, c = (e & 31) * 2;
            cp_async16(su + r * kLdU + c,
                       U + (j0 + static_cast<int64_t>(cc) * kDC + r) * K + c0 + c);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    double acc[8][4];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b)
            acc[a][b] = 0.0;
    const int stages = chunks * (kT / kDC);
    stage(0, 0);
    for (int cc = 0; cc < stages; ++cc) {
        if (cc + 1 < stages) {
            stage((cc + 1) & 1, cc + 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        const double *se = gptq_smem + (cc & 1) * kStage, *su = se + kRT * kLdE;
#pragma unroll 4
        for (int k = 0; k < kDC; ++k) {
            double a[8], b[4];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                a[i] = se[(ty + 16 * i) * kLdE + k];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                b[i] = su[k * kLdU + tx + 16 * i];
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    acc[i][j] = fma(a[i], b[j], acc[i][j]);
        }
        __syncthreads(); // the buffer is refilled two stages on
    }
#pragma unroll
    for (int a = 0; a < 8; ++a) {
        const int64_t r = r0 + ty + 16 * a;
        if (r < N) {
#pragma unroll
            for (int b = 0; b < 4; ++b)
                wd[r * K + c0 + tx + 16 * b] -= acc[a][b];
        }
    }
}

} // namespace gptq
} // namespace w8a8
