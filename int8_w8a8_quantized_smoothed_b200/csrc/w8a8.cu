// C ABI of the W8A8 SmoothQuant linear path (declared in include/w8a8.h): argument
// validation, kernel selection, TMA descriptor encoding and launches. Every compute step
// runs in the kernels of rowquant.cuh and gemm.cuh; there is no host fallback.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <map>
#include <mutex>
#include <set>
#include <tuple>
#include <utility>

#include "block.cuh"
#include "gemm.cuh"
#include "gptq.cuh"
#include "probe.cuh"
#include "rowquant.cuh"
#include "w8a8.h"

namespace {

using namespace w8a8;

constexpr unsigned long long kWaitLimitNs = 2000000000ull; // 2 s per bounded wait
constexpr int kMaxDevices = 64;

struct DeviceInfo {
    int ok = -1; // -1 unknown, 0 unsupported, 1 sm_100
    int num_sms = 0;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
std::set<std::pair<const void *, int>> g_smem_set;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool aligned16(const void *p)
{
    return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

// Current device if it is an sm_100 part; fills its SM count.
int current_device(int *dev, int *num_sms)
{
    int d = -1;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) {
        cudaGetLastError();
        return W8A8_ERR_NO_DEVICE;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceInfo &info = g_dev[d];
    if (info.ok < 0) {
        int major = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, d) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, d) != cudaSuccess) {
            cudaGetLastError();
            return W8A8_ERR_NO_DEVICE;
        }
        info.ok = (major == 10) ? 1 : 0;
        info.num_sms = sms;
    }
    if (info.ok != 1)
        return W8A8_ERR_NO_DEVICE;
    if (!g_encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000,
                                             cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr) {
            cudaGetLastError();
            return W8A8_ERR_CUDA;
        }
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    *dev = d;
    *num_sms = info.num_sms;
    return W8A8_OK;
}

// Once per kernel and device: raise the dynamic shared-memory limit, and ask for the
// largest shared-memory carveout for every kernel of the library, so consecutive launches
// of row kernels and GEMMs never reconfigure the L1/shared split between them.
int ensure_smem(const void *kernel, int dev, int bytes)
{
    std::lock_guard<std::mutex> lk(g_mu);
    auto key = std::make_pair(kernel, dev);
    if (g_smem_set.count(key))
        return W8A8_OK;
    if ((bytes > 0 && cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           bytes) != cudaSuccess) ||
        cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess) {
        cudaGetLastError();
        return W8A8_ERR_CUDA;
    }
    g_smem_set.insert(key);
    return W8A8_OK;
}

// Overlap mode (w8a8_set_overlap): 0 plain stream order, 1 programmatic dependent launch,
// 2 dependent launch + weight prefetch before the dependency wait.
std::atomic<int> g_overlap{1};

// Launches `kernel`, with programmatic stream serialization when the overlap mode asks for
// it (the kernels call griddepcontrol.wait before touching dependent data either way).
template <typename... KArgs, typename... Args>
int launch_kernel_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t st, unsigned cluster_x, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    unsigned n = 0;
    if (g_overlap.load(std::memory_order_relaxed) >= 1) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    if (cluster_x > 0) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster_x;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    if (cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) != cudaSuccess) {
        cudaGetLastError();
        return W8A8_ERR_CUDA;
    }
    return W8A8_OK;
}

template <typename... KArgs, typename... Args>
int launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                  Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    if (g_overlap.load(std::memory_order_relaxed) >= 1) {
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    if (cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) != cudaSuccess) {
        cudaGetLastError();
        return W8A8_ERR_CUDA;
    }
    return W8A8_OK;
}

// 2-D int8 [rows, K] K-contiguous tensor, box = 128 bytes of K x box_rows, 128B swizzle,
// out-of-range elements read as zero.
int encode_kmajor_i8(CUtensorMap *map, const void *base, int64_t rows, int64_t K, int box_rows)
{
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? W8A8_OK : W8A8_ERR_CUDA;
}

// ------------------------------------------------------------------ row kernels

struct RowLaunch {
    int nch;
    int threads;
};

// One CTA per row; each thread holds nch vectors of 8 values (nch <= 4, <= 1024 threads).
RowLaunch row_launch(int64_t K)
{
    const int64_t nvec = K / 8;
    int nch = static_cast<int>((nvec + 255) / 256);
    nch = nch < 1 ? 1 : (nch > 4 ? 4 : nch);
    if (nch == 3)
        nch = 4;
    int64_t t = (nvec + nch - 1) / nch;
    t = ((t + 31) / 32) * 32;
    return RowLaunch{nch, static_cast<int>(t)};
}

int check_row_shape(int64_t M, int64_t K)
{
    if (M < 1 || K < 16)
        return W8A8_ERR_INVALID_ARG;
    if (K % 16 != 0 || K > 32768 || M > 0x7fffffffLL)
        return W8A8_ERR_UNSUPPORTED_SHAPE;
    return W8A8_OK;
}

// Persistent row grid: at most as many CTAs as are resident on the device at once (cached
// per kernel, block size and device), never more than there are rows.
unsigned row_grid(const void *kernel, int threads, int64_t M, int dev, int sms)
{
    static std::mutex mu;
    static std::map<std::tuple<const void *, int, int>, int> cache;
    int occ = 0;
    {
        std::lock_guard<std::mutex> lk(mu);
        auto key = std::make_tuple(kernel, threads, dev);
        auto it = cache.find(key);
        if (it != cache.end()) {
            occ = it->second;
        } else {
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, threads, 0) !=
                cudaSuccess) {
                cudaGetLastError();
                occ = 1;
            }
            occ = occ < 1 ? 1 : occ;
            cache[key] = occ;
        }
    }
    const int64_t g = static_cast<int64_t>(sms) * occ;
    return static_cast<unsigned>(M < g ? M : g);
}

template <int NCH, bool F8>
int launch_quantize_rows(const uint16_t *x, const float *sinv, int64_t M, int K, int8_t *q,
                         float *s, int threads, int dev, int sms, cudaStream_t st)
{
    const void *fn = reinterpret_cast<const void *>(&quantize_rows_kernel<NCH, F8>);
    if (int rc = ensure_smem(fn, dev, 0))
        return rc;
    return launch_kernel(quantize_rows_kernel<NCH, F8>, dim3(row_grid(fn, threads, M, dev, sms)),
                         dim3(threads), 0, st, x, sinv, K, static_cast<int>(M), q, s);
}

template <int NCH, bool RES, bool F8>
int launch_rmsnorm_t(const uint16_t *x, const uint16_t *r, uint16_t *h, const float *g, float eps,
                     int64_t M, int K, int8_t *q, float *s, int threads, int dev, int sms,
                     cudaStream_t st)
{
    const void *fn = reinterpret_cast<const void *>(&rmsnorm_quant_kernel<NCH, RES, F8>);
    if (int rc = ensure_smem(fn, dev, 0))
        return rc;
    const bool gamma_early = g_overlap.load(std::memory_order_relaxed) >= 2;
    return launch_kernel(rmsnorm_quant_kernel<NCH, RES, F8>, dim3(row_grid(fn, threads, M, dev, sms)),
                         dim3(threads), 0, st, x, r, h, g, eps, K, static_cast<int>(M), q, s,
                         gamma_early);
}

template <int NCH, bool F8>
int launch_rmsnorm(const uint16_t *x, const uint16_t *r, uint16_t *h, const float *g, float eps,
                   int64_t M, int K, int8_t *q, float *s, int threads, int dev, int sms,
                   cudaStream_t st)
{
    if (r)
        return launch_rmsnorm_t<NCH, true, F8>(x, r, h, g, eps, M, K, q, s, threads, dev, sms, st);
    return launch_rmsnorm_t<NCH, false, F8>(x, r, h, g, eps, M, K, q, s, threads, dev, sms, st);
}

template <int NCH, bool F8>
int launch_silu(const uint16_t *gu, int64_t M, int I, int8_t *q, float *s, int threads, int dev,
                int sms, cudaStream_t st)
{
    const void *fn = reinterpret_cast<const void *>(&silu_mul_quant_kernel<NCH, F8>);
    if (int rc = ensure_smem(fn, dev, 0))
        return rc;
    return launch_kernel(silu_mul_quant_kernel<NCH, F8>, dim3(row_grid(fn, threads, M, dev, sms)),
                         dim3(threads), 0, st, gu, I, static_cast<int>(M), q, s);
}

template <bool F8 = false>
int launch_quantize_f32_parts(const float *a, const float *parts, int64_t M, int I, int8_t *q,
                              float *s, int dev, cudaStream_t st)
{
    const void *fn = reinterpret_cast<const void *>(&quantize_f32_parts_kernel<F8>);
    if (int rc = ensure_smem(fn, dev, 0))
        return rc;
    const unsigned slices = static_cast<unsigned>((I / 8 + 255) / 256);
    return launch_kernel(quantize_f32_parts_kernel<F8>, dim3(slices, static_cast<unsigned>(M)),
                         dim3(256), 0, st, a, parts, I, static_cast<int>(M), q, s);
}

template <int NCH, bool F8 = false>
int launch_quantize_f32(const float *a, int64_t M, int I, int8_t *q, float *s, int threads,
                        int dev, int sms, cudaStream_t st)
{
    const void *fn = reinterpret_cast<const void *>(&quantize_f32_rows_kernel<NCH, F8>);
    if (int rc = ensure_smem(fn, dev, 0))
        return rc;
    return launch_kernel(quantize_f32_rows_kernel<NCH, F8>, dim3(row_grid(fn, threads, M, dev, sms)),
                         dim3(threads), 0, st, a, I, static_cast<int>(M), q, s);
}

// ------------------------------------------------------------------ GEMM planning

struct GemmPlan {
    int variant = 0;   // 1 prefill tiles, 2 decode stream-K, 3 decode cluster split-K
    int tile_n = 256;  // prefill tile width
    int nt = 16;       // decode token tile
    int ctas = 1;      // stream-K persistent grid, or cluster size
    int sk_pairs = 0;  // pair tile kernel: stream-K over this many CTA pairs (0: whole tiles)
    size_t ws_bytes = 0;
    size_t flag_off = 0;
    size_t part_off = 0;
};

// stream-K workspace: one flag word per CTA (at most kMaxCtas) in the first kFlagBytes
constexpr int kMaxCtas = 1024;
constexpr size_t kFlagBytes = kMaxCtas * 4;
// the pair tile kernel's partial slot per CTA (128 x 256 accumulator words)
constexpr size_t kPairPartBytes = 128 * 256 * 4;

int decode_nt(int64_t M)
{
    return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256;
}

// Bytes of the per-(token, 64-channel group) maxima the fused SiLU*up call keeps in its
// workspace after the GEMM's own part (small-M plans only), and where they start: never
// inside the flag words, which every later stream-K call on the same workspace must find zero
// (the maxima are written before they are read in every call, so they need no clearing).
size_t silu_parts_off(const GemmPlan &p)
{
    const size_t base = p.ws_bytes > kFlagBytes ? p.ws_bytes : kFlagBytes;
    return (base + 255) & ~static_cast<size_t>(255);
}
size_t silu_parts_bytes(const GemmPlan &p, int64_t M, int64_t I)
{
    return p.variant == 1 ? 0 : static_cast<size_t>(M) * static_cast<size_t>(I / 64) * 4u;
}



int plan_gemm(int64_t M, int64_t N, int64_t K, int variant, int ctas, int tile_n, int num_sms,
              GemmPlan *p)
{
    if (variant < 0 || variant > 3 || ctas < 0 ||
        (tile_n != 0 && tile_n != 128 && tile_n != 256 && tile_n != 512))
        return W8A8_ERR_INVALID_ARG;
    const int64_t KB = (K + kBK - 1) / kBK;
    const int64_t NB = (N + kBM - 1) / kBM;
    if (variant == 0) {
        if (M > 64)
            variant = 1;
        else // few channel blocks: split K inside clusters; many: stream-K over all SMs
            variant = (2 * NB <= num_sms && KB >= 2) ? 3 : 2;
    }
    if ((variant == 2 || variant == 3) && M > kDecodeMaxTiles * 256)
        return W8A8_ERR_UNSUPPORTED_SHAPE;
    p->variant = variant;
    if (variant == 1) {
        if (tile_n == 0) {
            // Cost model: a tile is bound by its SMs' shared-memory traffic (TMA writes plus
            // tensor-core operand reads) for its MACs. Relative tile times: 128x128 on one SM
            // -> 2, 128x256 on one SM -> 3, 256x256 on a CTA pair -> 2 (each SM does 128x256
            // MACs with two thirds of the traffic). A launch takes ceil(tiles / concurrent
            // tiles) tile times.
            const int64_t cand[3][4] = {{128, 128, 2, 1}, {128, 256, 3, 1}, {256, 256, 2, 2}};
            int64_t best = -1, best_cost = 0;
            for (int i = 0; i < 3; ++i) {
                const int64_t tiles = ((M + cand[i][0] - 1) / cand[i][0]) *
                                      ((N + cand[i][1] - 1) / cand[i][1]);
                const int64_t slots = num_sms / cand[i][3];
                const int64_t cost = ((tiles + slots - 1) / slots) * cand[i][2];
                if (best < 0 || cost < best_cost) {
                    best = i;
                    best_cost = cost;
                }
            }
            tile_n = best == 0 ? 128 : best == 1 ? 256 : 512;
            // Stream-K over the pairs for few, long tiles: at most half the pairs would have a
            // whole tile, each of at least 64 k-blocks. Every pair then takes an equal share
            // of the tiles' k-blocks; a split tile's owner adds the later pieces at its end,
            // a fixed cost of a few microseconds that only tiles this long amortize
            // (measured: 512 x 4096 x 14336 38.3 -> 34.0 us; with K = 4096 stream-K was
            // slower than whole tiles at M = 512 and 2048).
            const int64_t P = num_sms / 2;
            const int64_t tp = ((M + 255) / 256) * ((N + 255) / 256);
            if (2 * tp <= P && KB >= 64) {
                tile_n = 512;
                ctas = static_cast<int>(P);
            }
        }
        p->tile_n = tile_n;
        p->ws_bytes = 0;
        if (tile_n == 512 && ctas > 0) {
            // at most kMaxContrib (3) later pieces per split tile: shares of >= KB / 3 units
            const int64_t tp = ((M + 255) / 256) * ((N + 255) / 256);
            int64_t P = ctas < num_sms / 2 ? ctas : num_sms / 2;
            if (P > 3 * tp)
                P = 3 * tp;
            p->sk_pairs = static_cast<int>(P < 1 ? 1 : P);
            p->flag_off = 0;
            p->part_off = kFlagBytes;
            p->ws_bytes = kFlagBytes + static_cast<size_t>(2 * p->sk_pairs) * kPairPartBytes;
        }
        return W8A8_OK;
    }
    p->nt = decode_nt(M);
    const int64_t TT = (M + p->nt - 1) / p->nt; // token tiles (M > 256: tiles of 256)
    if (variant == 3) {
        int64_t S = ctas > 0 ? ctas : num_sms / (NB * TT);
        S = S < 1 ? 1 : S;
        S = S > kMaxClusterSize ? kMaxClusterSize : S;
        S = S > KB ? KB : S;
        p->ctas = static_cast<int>(S);
        p->ws_bytes = 0;
        return W8A8_OK;
    }
    const int64_t U = NB * TT * KB;
    // every CTA must be resident at once (owners wait on later CTAs): at most one per SM
    int64_t G = (ctas == 0 || ctas > num_sms) ? num_sms : ctas;
    if (ctas == 0) {
        // Whole blocks per CTA when that keeps most SMs streaming: no block is split, so no
        // partial sums cross CTAs (e.g. 224 channel blocks as 2 per CTA on 112 SMs beats the
        // even split over 148 SMs at every decode size: the split-K tail costs more than the
        // 36 idle SMs' share of the weight stream).
        const int64_t blocks = NB * TT;
        const int64_t per = (blocks + num_sms - 1) / num_sms;
        if (per <= 2 && blocks % per == 0 && (blocks / per) * 10 >= static_cast<int64_t>(num_sms) * 7)
            G = blocks / per;
    }
    if (G > U)
        G = U;
    if (G > kMaxCtas)
        G = kMaxCtas;
    p->ctas = static_cast<int>(G);
    // a workspace is needed only if some CTA boundary falls inside a channel block
    bool split = false;
    for (int64_t g = 1; g < G && !split; ++g)
        split = ((g * U) / G) % KB != 0;
    if (split) {
        // flag words first, at a fixed place whatever the shape (they are the only part that
        // must be zero when a call starts); partial slots after them
        const int64_t Mp = ((M < p->nt ? M : p->nt) + 3) & ~static_cast<int64_t>(3);
        p->flag_off = 0;
        p->part_off = kFlagBytes;
        p->ws_bytes = kFlagBytes + static_cast<size_t>(G) * kBM * static_cast<size_t>(Mp) * 4u;
    } else {
        p->ws_bytes = 0;
    }
    return W8A8_OK;
}

int check_gemm_shape(int64_t M, int64_t N, int64_t K)
{
    if (M < 1 || N < 8 || K < 16)
        return W8A8_ERR_INVALID_ARG;
    if (N % 8 != 0 || K % 16 != 0 || K > 133144 || M > 0x7fffffffLL || N > 0x7fffffffLL)
        return W8A8_ERR_UNSUPPORTED_SHAPE;
    return W8A8_OK;
}

template <int BN, int STAGES, bool SILU, bool F8 = false>
int launch_prefill(const CUtensorMap &ta, const CUtensorMap &tb, const float *s_tok,
                   const float *s_ch, int64_t M, int64_t N, int64_t K, uint16_t *y, int32_t *acc,
                   const SiluOut &so, int dev, int num_sms, cudaStream_t st)
{
    using Cfg = PrefillCfg<BN, STAGES>;
    const void *fn = reinterpret_cast<const void *>(&gemm_prefill_kernel<BN, STAGES, SILU, F8>);
    int rc = ensure_smem(fn, dev, Cfg::kSmemBytes);
    if (rc)
        return rc;
    const int64_t tiles = ((M + kBM - 1) / kBM) * ((N + BN - 1) / BN);
    const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
    const int prefetch = g_overlap.load(std::memory_order_relaxed) >= 2 ? 1 : 0;
    return launch_kernel(gemm_prefill_kernel<BN, STAGES, SILU, F8>, dim3(grid), dim3(kGemmThreads),
                         Cfg::kSmemBytes, st, ta, tb, s_tok, s_ch, static_cast<int>(M),
                         static_cast<int>(N), static_cast<int>(K), y, acc, so, prefetch,
                         kWaitLimitNs);
}

// Resident pair clusters of the pair kernel on this device (cached per device).
int pair_clusters(const void *kernel, int smem, int dev, int num_sms)
{
    static std::mutex mu;
    static int cached[kMaxDevices] = {0};
    {
        std::lock_guard<std::mutex> lk(mu);
        if (cached[dev] > 0)
            return cached[dev];
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (num_sms / 2));
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n < 1)
        n = num_sms / 2;
    cudaGetLastError();
    std::lock_guard<std::mutex> lk(mu);
    cached[dev] = n;
    return n;
}

template <int STAGES, bool SILU, bool F8 = false>
int launch_prefill_pair(const CUtensorMap &ta, const CUtensorMap &tb, const float *s_tok,
                        const float *s_ch, int64_t M, int64_t N, int64_t K, uint16_t *y,
                        int32_t *acc, const SiluOut &so, const GemmPlan &p, void *ws, int dev,
                        int num_sms, cudaStream_t st)
{
    using Cfg = PairCfg<STAGES>;
    static_assert(Cfg::kPartBytes == kPairPartBytes, "pair partial slot");
    auto kernel = gemm_prefill_pair_kernel<STAGES, SILU, F8>;
    int rc = ensure_smem(reinterpret_cast<const void *>(kernel), dev, Cfg::kSmemBytes);
    if (rc)
        return rc;
    const int64_t tiles = ((M + 255) / 256) * ((N + 255) / 256);
    int64_t pairs = pair_clusters(reinterpret_cast<const void *>(kernel), Cfg::kSmemBytes, dev,
                                  num_sms);
    int32_t *ws_part = nullptr;
    unsigned int *ws_flag = nullptr;
    if (p.sk_pairs > 0) { // stream-K: every pair resident, each with a partial slot
        if (pairs > p.sk_pairs)
            pairs = p.sk_pairs;
        ws_part = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + p.part_off);
        ws_flag = reinterpret_cast<unsigned int *>(static_cast<char *>(ws) + p.flag_off);
    } else if (pairs > tiles) {
        pairs = tiles;
    }
    // Tile order: groups of row-tiles whose A row-panels (256 x K bytes each) total at most
    // 32 MiB, so that they stay in L2 while the group's column sweep passes (32 row-tiles at
    // K = 4096, 16 at 8192, 8 at 14336): B is read once per group, A about once.
    int64_t group_m = (32ll << 20) / (256 * K);
    group_m = group_m < 2 ? 2 : group_m > 32 ? 32 : group_m;
    const int prefetch = g_overlap.load(std::memory_order_relaxed) >= 2 ? 1 : 0;
    return launch_kernel_cluster(kernel, dim3(static_cast<unsigned>(2 * pairs)),
                                 dim3(kGemmThreads), Cfg::kSmemBytes, st, 2u, ta, tb, s_tok, s_ch,
                                 static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), y,
                                 acc, so, ws_part, ws_flag, static_cast<int>(group_m), prefetch,
                                 kWaitLimitNs);
}

// Largest cluster size <= want whose clusters can all be resident at once (one wave).
template <typename Kern>
int fit_cluster(Kern kernel, int want, int64_t clusters_needed, int smem, int dev)
{
    static std::mutex mu;
    static std::set<std::tuple<const void *, int, int, int>> ok_set, bad_set;
    for (int S = want; S > 1; --S) {
        const auto key = std::make_tuple(reinterpret_cast<const void *>(kernel), S, dev,
                                         static_cast<int>(clusters_needed));
        {
            std::lock_guard<std::mutex> lk(mu);
            if (ok_set.count(key))
                return S;
            if (bad_set.count(key))
                continue;
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(S, static_cast<unsigned>(clusters_needed));
        cfg.blockDim = dim3(kGemmThreads);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = S;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        const bool fits = cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) == cudaSuccess &&
                          n >= clusters_needed;
        cudaGetLastError();
        std::lock_guard<std::mutex> lk(mu);
        (fits ? ok_set : bad_set).insert(key);
        if (fits)
            return S;
    }
    return 1;
}

// RNV > 0: the cluster split-K with the residual RMSNorm tail (rn), rows of up to 1024 RNV
// values; only the INT8 plain-epilogue cluster plans take it.
template <int NT, int STAGES, int KPS, bool SILU, bool F8 = false, int RNV = 0>
int launch_decode(const CUtensorMap &tw, const CUtensorMap &tx, const float *s_tok,
                  const float *s_ch, int64_t M, int64_t N, int64_t K, const GemmPlan &p,
                  uint16_t *y, int32_t *acc, void *ws, const SiluOut &so, int dev, cudaStream_t st,
                  const RowNormOut &rn = RowNormOut{})
{
    const int prefetch = g_overlap.load(std::memory_order_relaxed) >= 2 ? 1 : 0;
    if constexpr (RNV > 0) {
        if (p.variant != 3)
            return W8A8_ERR_UNSUPPORTED_SHAPE;
    }
    if constexpr (SILU && F8) {
        if (p.variant == 3) // the FP8 cluster split-K has no SiLU epilogue: planned away
            return W8A8_ERR_UNSUPPORTED_SHAPE;
    } else if (p.variant == 3) {
        using Cfg = DecodeCfg<NT, STAGES, KPS, true>;
        auto kernel = gemm_decode_kernel<NT, STAGES, KPS, true, SILU, F8, RNV>;
        if (int rc = ensure_smem(reinterpret_cast<const void *>(kernel), dev, Cfg::kSmemBytes))
            return rc;
        const int64_t NB = ((N + kBM - 1) / kBM) * ((M + NT - 1) / NT); // x token tiles
        const int S = fit_cluster(kernel, p.ctas, NB, Cfg::kSmemBytes, dev);
        return launch_kernel_cluster(kernel, dim3(S, static_cast<unsigned>(NB)), dim3(kGemmThreads),
                                     Cfg::kSmemBytes, st, static_cast<unsigned>(S), tw, tx, s_tok,
                                     s_ch, static_cast<int>(M), static_cast<int>(N),
                                     static_cast<int>(K), y, acc, static_cast<int32_t *>(nullptr),
                                     static_cast<unsigned int *>(nullptr), so, rn, prefetch,
                                     kWaitLimitNs);
    }
    if constexpr (RNV == 0) {
        using Cfg = DecodeCfg<NT, STAGES, KPS, false>;
        auto kernel = gemm_decode_kernel<NT, STAGES, KPS, false, SILU, F8>;
        if (int rc = ensure_smem(reinterpret_cast<const void *>(kernel), dev, Cfg::kSmemBytes))
            return rc;
        int32_t *ws_part =
            p.ws_bytes ? reinterpret_cast<int32_t *>(static_cast<char *>(ws) + p.part_off) : nullptr;
        unsigned int *ws_flag =
            p.ws_bytes ? reinterpret_cast<unsigned int *>(static_cast<char *>(ws) + p.flag_off)
                       : nullptr;
        return launch_kernel(kernel, dim3(p.ctas), dim3(kGemmThreads), Cfg::kSmemBytes, st, tw, tx,
                             s_tok, s_ch, static_cast<int>(M), static_cast<int>(N),
                             static_cast<int>(K), y, acc, ws_part, ws_flag, so, RowNormOut{},
                             prefetch, kWaitLimitNs);
    }
    return W8A8_ERR_UNSUPPORTED_SHAPE;
}

// Decode launch by token tile: (stages, k-blocks per stage) keep ~200 KB of weight and
// token bytes in flight per SM.
template <bool SILU, bool F8 = false>
int launch_decode_nt(const CUtensorMap &tw, const CUtensorMap &tx, const float *s_tok,
                     const float *s_ch, int64_t M, int64_t N, int64_t K, const GemmPlan &p,
                     uint16_t *y, int32_t *acc, void *ws, const SiluOut &so, int dev,
                     cudaStream_t st)
{
    switch (p.nt) {
    case 16: return launch_decode<16, 3, 4, SILU, F8>(tw, tx, s_tok, s_ch, M, N, K, p, y, acc, ws, so, dev, st);
    case 32: return launch_decode<32, 5, 2, SILU, F8>(tw, tx, s_tok, s_ch, M, N, K, p, y, acc, ws, so, dev, st);
    case 64: return launch_decode<64, 4, 2, SILU, F8>(tw, tx, s_tok, s_ch, M, N, K, p, y, acc, ws, so, dev, st);
    case 128: return launch_decode<128, 5, 1, SILU, F8>(tw, tx, s_tok, s_ch, M, N, K, p, y, acc, ws, so, dev, st);
    default: return launch_decode<256, 3, 1, SILU, F8>(tw, tx, s_tok, s_ch, M, N, K, p, y, acc, ws, so, dev, st);
    }
}

// The INT8 cluster split-K GEMM with the residual RMSNorm tail: token tiles of at most 64,
// rows of at most 8192 values.
int launch_decode_rn(const CUtensorMap &tw, const CUtensorMap &tx, const float *s_tok,
                     const float *s_ch, int64_t M, int64_t N, int64_t K, const GemmPlan &p,
                     uint16_t *y, const RowNormOut &rn, int dev, cudaStream_t st)
{
    const SiluOut none{nullptr, 0};
    const bool wide = N > 4096;
    switch (p.nt) {
    case 16: return wide ? launch_decode<16, 3, 4, false, false, 8>(tw, tx, s_tok, s_ch, M, N, K, p, y, nullptr, nullptr, none, dev, st, rn)
                         : launch_decode<16, 3, 4, false, false, 4>(tw, tx, s_tok, s_ch, M, N, K, p, y, nullptr, nullptr, none, dev, st, rn);
    case 32: return wide ? launch_decode<32, 5, 2, false, false, 8>(tw, tx, s_tok, s_ch, M, N, K, p, y, nullptr, nullptr, none, dev, st, rn)
                         : launch_decode<32, 5, 2, false, false, 4>(tw, tx, s_tok, s_ch, M, N, K, p, y, nullptr, nullptr, none, dev, st, rn);
    case 64: return wide ? launch_decode<64, 4, 2, false, false, 8>(tw, tx, s_tok, s_ch, M, N, K, p, y, nullptr, nullptr, none, dev, st, rn)
                         : launch_decode<64, 4, 2, false, false, 4>(tw, tx, s_tok, s_ch, M, N, K, p, y, nullptr, nullptr, none, dev, st, rn);
    default: return W8A8_ERR_UNSUPPORTED_SHAPE;
    }
}

// The FP8 GEMM launch for a plan: plain dequant epilogue (so == nullptr) or the fused
// SiLU*up epilogue (tile kernels and stream-K; not the cluster split-K).
int gemm_run_fp8(const uint8_t *xq, const float *s_tok, const uint8_t *wq, const float *s_ch,
                 int64_t M, int64_t N, int64_t K, uint16_t *y, float *acc_out, void *workspace,
                 const GemmPlan &p, int dev, int sms, cudaStream_t st, const SiluOut *so = nullptr)
{
    const SiluOut none{nullptr, 0};
    int32_t *acc = reinterpret_cast<int32_t *>(acc_out); // raw binary32 words
    if (p.variant == 1) {
        const int bn = p.tile_n == 128 ? 128 : p.tile_n == 256 ? 256 : 128;
        CUtensorMap ta, tb;
        if (encode_kmajor_i8(&ta, xq, M, K, kBM) || encode_kmajor_i8(&tb, wq, N, K, bn))
            return W8A8_ERR_CUDA;
        if (so) {
            if (p.tile_n == 512)
                return launch_prefill_pair<6, true, true>(ta, tb, s_tok, s_ch, M, N, K, y, acc, *so, p, workspace, dev, sms, st);
            if (p.tile_n == 256)
                return launch_prefill<256, 4, true, true>(ta, tb, s_tok, s_ch, M, N, K, y, acc, *so, dev, sms, st);
            return launch_prefill<128, 6, true, true>(ta, tb, s_tok, s_ch, M, N, K, y, acc, *so, dev, sms, st);
        }
        if (p.tile_n == 512)
            return launch_prefill_pair<6, false, true>(ta, tb, s_tok, s_ch, M, N, K, y, acc, none, p, workspace, dev, sms, st);
        if (p.tile_n == 256)
            return launch_prefill<256, 4, false, true>(ta, tb, s_tok, s_ch, M, N, K, y, acc, none, dev, sms, st);
        return launch_prefill<128, 6, false, true>(ta, tb, s_tok, s_ch, M, N, K, y, acc, none, dev, sms, st);
    }
    CUtensorMap tw, tx;
    if (encode_kmajor_i8(&tw, wq, N, K, kBM) || encode_kmajor_i8(&tx, xq, M, K, p.nt))
        return W8A8_ERR_CUDA;
    if (so)
        return launch_decode_nt<true, true>(tw, tx, s_tok, s_ch, M, N, K, p, y, acc, workspace, *so, dev, st);
    return launch_decode_nt<false, true>(tw, tx, s_tok, s_ch, M, N, K, p, y, acc, workspace, none, dev, st);
}

// The GEMM launch for a plan: plain dequant epilogue (so == nullptr) or the fused SiLU*up
// epilogue.
int gemm_run(const int8_t *xq, const float *s_tok, const int8_t *wq, const float *s_ch,
             int64_t M, int64_t N, int64_t K, uint16_t *y, int32_t *acc_out, void *workspace,
             const GemmPlan &p, const SiluOut *so, int dev, int sms, cudaStream_t st)
{
    const SiluOut none{nullptr, 0};
    if (p.variant == 1) {
        // tile_n: 128 -> 128 x 128, 256 -> 128 x 256, 512 -> 256 x 256 by a CTA pair
        const int bn = p.tile_n == 128 ? 128 : p.tile_n == 256 ? 256 : 128;
        CUtensorMap ta, tb;
        if (encode_kmajor_i8(&ta, xq, M, K, kBM) || encode_kmajor_i8(&tb, wq, N, K, bn))
            return W8A8_ERR_CUDA;
        if (so) {
            if (p.tile_n == 512)
                return launch_prefill_pair<6, true>(ta, tb, s_tok, s_ch, M, N, K, y, acc_out, *so, p, workspace, dev, sms, st);
            if (p.tile_n == 256)
                return launch_prefill<256, 4, true>(ta, tb, s_tok, s_ch, M, N, K, y, acc_out, *so, dev, sms, st);
            return launch_prefill<128, 6, true>(ta, tb, s_tok, s_ch, M, N, K, y, acc_out, *so, dev, sms, st);
        }
        if (p.tile_n == 512)
            return launch_prefill_pair<6, false>(ta, tb, s_tok, s_ch, M, N, K, y, acc_out, none, p, workspace, dev, sms, st);
        if (p.tile_n == 256)
            return launch_prefill<256, 4, false>(ta, tb, s_tok, s_ch, M, N, K, y, acc_out, none, dev, sms, st);
        return launch_prefill<128, 6, false>(ta, tb, s_tok, s_ch, M, N, K, y, acc_out, none, dev, sms, st);
    }
    CUtensorMap tw, tx;
    if (encode_kmajor_i8(&tw, wq, N, K, kBM) || encode_kmajor_i8(&tx, xq, M, K, p.nt))
        return W8A8_ERR_CUDA;
    if (so)
        return launch_decode_nt<true>(tw, tx, s_tok, s_ch, M, N, K, p, y, acc_out, workspace, *so, dev, st);
    return launch_decode_nt<false>(tw, tx, s_tok, s_ch, M, N, K, p, y, acc_out, workspace, none, dev, st);
}


// ------------------------------------------------------------------ fused decoder block

// Workspace: the barrier counter and the SiLU maxima, then per GEMM phase a count word per
// 128-channel block and an int32 accumulation tile [128 channels x Mp tokens] per block.
size_t block_phase_bytes(int64_t M, int64_t N)
{
    const size_t Mp = static_cast<size_t>((M + 3) & ~3LL);
    const size_t NB = static_cast<size_t>((N + kBM - 1) / kBM);
    return (kFlagBytes + NB * kBM * Mp * 4u + 255) & ~static_cast<size_t>(255);
}

template <int NT, int STAGES, int KPS, int NV>
int launch_block(const BlockMaps &maps, const BlockArgs &args, int dev, int sms, cudaStream_t st)
{
    using Cfg = BlockCfg<NT, STAGES, KPS>;
    auto kernel = block_decode_kernel<NT, STAGES, KPS, NV>;
    if (int rc = ensure_smem(reinterpret_cast<const void *>(kernel), dev, Cfg::kSmemBytes))
        return rc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(sms));
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = Cfg::kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative; // every CTA resident: they wait on each other
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, maps, args);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return W8A8_ERR_CUDA;
    }
    return W8A8_OK;
}

// ------------------------------------------------------------------ GPTQ workspace

struct GptqLayout {
    size_t a_off, u_off, w_off, e_off, d_off, b_off, total;
};

size_t round256(size_t b)
{
    return (b + 255) & ~static_cast<size_t>(255);
}

// column blocks whose errors are batched into one update of the later columns
constexpr int kGptqGroup = 4;

// H/V [K,K] fp64, U [K,K] fp64, working weight [N,K] fp64, the errors of one group of column
// blocks [N, 64 * kGptqGroup] fp64, dead flags [K], the non-positive-pivot flag.
GptqLayout gptq_layout(int64_t N, int64_t K)
{
    GptqLayout L;
    const size_t kk = static_cast<size_t>(K) * static_cast<size_t>(K) * sizeof(double);
    L.a_off = 0;
    L.u_off = L.a_off + round256(kk);
    L.w_off = L.u_off + round256(kk);
    L.e_off = L.w_off + round256(static_cast<size_t>(N) * static_cast<size_t>(K) * sizeof(double));
    L.d_off = L.e_off + round256(static_cast<size_t>(N) * 64 * kGptqGroup * sizeof(double));
    L.b_off = L.d_off + round256(static_cast<size_t>(K));
    L.total = L.b_off + 256;
    return L;
}

// ------------------------------------------------------------------ row entry points
// (F8: E4M3 codes with scale amax / 448, else int8 codes with amax / 127)

template <bool F8>
int quantize_rows_impl(const uint16_t *x, const float *smooth_inv, int64_t M, int64_t K,
                       int8_t *q, float *s_tok, w8a8_stream_t stream)
{
    if (!x || !q || !s_tok)
        return W8A8_ERR_INVALID_ARG;
    int rc = check_row_shape(M, K);
    if (rc)
        return rc;
    if (!aligned16(x) || !aligned16(q) || (smooth_inv && !aligned16(smooth_inv)))
        return W8A8_ERR_ALIGNMENT;
    if (static_cast<const void *>(x) == static_cast<const void *>(q))
        return W8A8_ERR_INVALID_ARG;
    int dev, sms;
    if ((rc = current_device(&dev, &sms)))
        return rc;
    const RowLaunch L = row_launch(K);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    switch (L.nch) {
    case 1: return launch_quantize_rows<1, F8>(x, smooth_inv, M, (int)K, q, s_tok, L.threads, dev, sms, st);
    case 2: return launch_quantize_rows<2, F8>(x, smooth_inv, M, (int)K, q, s_tok, L.threads, dev, sms, st);
    default: return launch_quantize_rows<4, F8>(x, smooth_inv, M, (int)K, q, s_tok, L.threads, dev, sms, st);
    }
}

template <bool F8>
int rmsnorm_quant_impl(const uint16_t *x, const uint16_t *residual, uint16_t *h_out,
                       const float *gamma_smoothed, float eps, int64_t M, int64_t K, int8_t *q,
                       float *s_tok, w8a8_stream_t stream)
{
    if (!x || !gamma_smoothed || !q || !s_tok || ((residual == nullptr) != (h_out == nullptr)))
        return W8A8_ERR_INVALID_ARG;
    if (!(eps >= 0.0f))
        return W8A8_ERR_INVALID_ARG;
    int rc = check_row_shape(M, K);
    if (rc)
        return rc;
    if (!aligned16(x) || !aligned16(q) || !aligned16(gamma_smoothed) ||
        (residual && (!aligned16(residual) || !aligned16(h_out))))
        return W8A8_ERR_ALIGNMENT;
    if (h_out && static_cast<const void *>(h_out) == static_cast<const void *>(x))
        return W8A8_ERR_INVALID_ARG;
    int dev, sms;
    if ((rc = current_device(&dev, &sms)))
        return rc;
    const RowLaunch L = row_launch(K);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    switch (L.nch) {
    case 1: return launch_rmsnorm<1, F8>(x, residual, h_out, gamma_smoothed, eps, M, (int)K, q, s_tok, L.threads, dev, sms, st);
    case 2: return launch_rmsnorm<2, F8>(x, residual, h_out, gamma_smoothed, eps, M, (int)K, q, s_tok, L.threads, dev, sms, st);
    default: return launch_rmsnorm<4, F8>(x, residual, h_out, gamma_smoothed, eps, M, (int)K, q, s_tok, L.threads, dev, sms, st);
    }
}

template <bool F8>
int silu_mul_quant_impl(const uint16_t *gate_up, int64_t M, int64_t I, int8_t *q, float *s_tok,
                        w8a8_stream_t stream)
{
    if (!gate_up || !q || !s_tok)
        return W8A8_ERR_INVALID_ARG;
    int rc = check_row_shape(M, I);
    if (rc)
        return rc;
    if (!aligned16(gate_up) || !aligned16(q))
        return W8A8_ERR_ALIGNMENT;
    int dev, sms;
    if ((rc = current_device(&dev, &sms)))
        return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const RowLaunch L = row_launch(I);
    switch (L.nch) {
    case 1: return launch_silu<1, F8>(gate_up, M, (int)I, q, s_tok, L.threads, dev, sms, st);
    case 2: return launch_silu<2, F8>(gate_up, M, (int)I, q, s_tok, L.threads, dev, sms, st);
    default: return launch_silu<4, F8>(gate_up, M, (int)I, q, s_tok, L.threads, dev, sms, st);
    }
}

} // namespace

namespace {

template <int N>
int launch_probe(long long iters, int grid, int dev, cudaStream_t st)
{
    const int smem = 128 * 128 + N * 128 + 64 + 1024;
    const void *fn = reinterpret_cast<const void *>(&mma_i8_probe_kernel<N>);
    int rc = ensure_smem(fn, dev, smem);
    if (rc)
        return rc;
    return launch_kernel(mma_i8_probe_kernel<N>, dim3(grid), dim3(128), smem, st, iters,
                         kWaitLimitNs);
}

} // namespace

extern "C" {

int w8a8_version(void)
{
    return (1 << 16) | 0;
}

const char *w8a8_status_string(int status)
{
    switch (status) {
    case W8A8_OK:
        return "ok";
    case W8A8_ERR_INVALID_ARG:
        return "invalid argument";
    case W8A8_ERR_ALIGNMENT:
        return "pointer not 16-byte aligned";
    case W8A8_ERR_UNSUPPORTED_SHAPE:
        return "unsupported shape";
    case W8A8_ERR_WORKSPACE:
        return "workspace missing or too small";
    case W8A8_ERR_CUDA:
        return "CUDA error";
    case W8A8_ERR_TIMEOUT:
        return "device-side wait timed out";
    case W8A8_ERR_NO_DEVICE:
        return "no sm_100 device";
    case W8A8_ERR_NUMERIC:
        return "matrix not positive definite";
    default:
        return "unknown status";
    }
}


int w8a8_quantize_rows(const w8a8_bf16 *x, const float *smooth_inv, int64_t M, int64_t K,
                       int8_t *q, float *s_tok, w8a8_stream_t stream)
{
    return quantize_rows_impl<false>(x, smooth_inv, M, K, q, s_tok, stream);
}

int w8a8_quantize_rows_fp8(const w8a8_bf16 *x, const float *smooth_inv, int64_t M, int64_t K,
                           uint8_t *q, float *s_tok, w8a8_stream_t stream)
{
    return quantize_rows_impl<true>(x, smooth_inv, M, K, reinterpret_cast<int8_t *>(q), s_tok,
                                    stream);
}

int w8a8_quantize_rows_static(const w8a8_bf16 *x, const float *smooth_inv, float scale,
                              int64_t M, int64_t K, int8_t *q, float *s_tok,
                              w8a8_stream_t stream)
{
    if (!x || !q)
        return W8A8_ERR_INVALID_ARG;
    if (!(scale > 0.0f) || !(scale <= 3.4028234663852886e38f))
        return W8A8_ERR_INVALID_ARG;
    int rc = check_row_shape(M, K);
    if (rc)
        return rc;
    if (!aligned16(x) || !aligned16(q) || (smooth_inv && !aligned16(smooth_inv)))
        return W8A8_ERR_ALIGNMENT;
    if (static_cast<const void *>(x) == static_cast<const void *>(q))
        return W8A8_ERR_INVALID_ARG;
    int dev, sms;
    if ((rc = current_device(&dev, &sms)))
        return rc;
    const void *fn = reinterpret_cast<const void *>(&quantize_rows_static_kernel);
    if ((rc = ensure_smem(fn, dev, 0)))
        return rc;
    const int64_t nvec_total = M * (K / 8);
    const int64_t want = (nvec_total + 255) / 256;
    const unsigned grid = static_cast<unsigned>(std::min<int64_t>(want, static_cast<int64_t>(sms) * 8));
    return launch_kernel(quantize_rows_static_kernel, dim3(grid), dim3(256), 0,
                         reinterpret_cast<cudaStream_t>(stream), x, smooth_inv, scale,
                         static_cast<int>(K), nvec_total, static_cast<int>(M), q, s_tok);
}



int w8a8_smooth_rmsnorm_quant(const w8a8_bf16 *x, const w8a8_bf16 *residual, w8a8_bf16 *h_out,
                              const float *gamma_smoothed, float eps, int64_t M, int64_t K,
                              int8_t *q, float *s_tok, w8a8_stream_t stream)
{
    return rmsnorm_quant_impl<false>(x, residual, h_out, gamma_smoothed, eps, M, K, q, s_tok,
                                     stream);
}

int w8a8_smooth_rmsnorm_quant_fp8(const w8a8_bf16 *x, const w8a8_bf16 *residual,
                                  w8a8_bf16 *h_out, const float *gamma_smoothed, float eps,
                                  int64_t M, int64_t K, uint8_t *q, float *s_tok,
                                  w8a8_stream_t stream)
{
    return rmsnorm_quant_impl<true>(x, residual, h_out, gamma_smoothed, eps, M, K,
                                    reinterpret_cast<int8_t *>(q), s_tok, stream);
}

int w8a8_silu_mul_quant(const w8a8_bf16 *gate_up, int64_t M, int64_t I, int8_t *q, float *s_tok,
                        w8a8_stream_t stream)
{
    return silu_mul_quant_impl<false>(gate_up, M, I, q, s_tok, stream);
}

int w8a8_silu_mul_quant_fp8(const w8a8_bf16 *gate_up, int64_t M, int64_t I, uint8_t *q,
                            float *s_tok, w8a8_stream_t stream)
{
    return silu_mul_quant_impl<true>(gate_up, M, I, reinterpret_cast<int8_t *>(q), s_tok, stream);
}

size_t w8a8_gemm_silu_quant_workspace_size(int64_t M, int64_t I, int64_t K)
{
    if (I < 64 || I % 64 != 0 || check_row_shape(M, I) || check_gemm_shape(M, 2 * I, K))
        return 0;
    int dev, sms = 148;
    if (current_device(&dev, &sms))
        sms = 148;
    GemmPlan p;
    if (plan_gemm(M, 2 * I, K, 0, 0, 0, sms, &p))
        return 0;
    const size_t parts = silu_parts_bytes(p, M, I);
    return parts ? silu_parts_off(p) + parts : p.ws_bytes;
}

int w8a8_gemm_silu_quant(const int8_t *xq, const float *s_tok, const int8_t *wq_il,
                         const float *s_ch_il, int64_t M, int64_t I, int64_t K, float *a,
                         int8_t *q, float *s_out, void *workspace, size_t workspace_bytes,
                         w8a8_stream_t stream)
{
    if (!xq || !s_tok || !wq_il || !s_ch_il || !a || !q || !s_out)
        return W8A8_ERR_INVALID_ARG;
    if (I < 64 || I % 64 != 0)
        return W8A8_ERR_UNSUPPORTED_SHAPE;
    int rc = check_gemm_shape(M, 2 * I, K);
    if (rc || (rc = check_row_shape(M, I)))
        return rc;
    if (!aligned16(xq) || !aligned16(wq_il) || !aligned16(s_ch_il) || !aligned16(a) ||
        !aligned16(q) || (workspace && !aligned16(workspace)))
        return W8A8_ERR_ALIGNMENT;
    int dev, sms;
    if ((rc = current_device(&dev, &sms)))
        return rc;
    GemmPlan p;
    if ((rc = plan_gemm(M, 2 * I, K, 0, 0, 0, sms, &p)))
        return rc;
    const size_t parts = silu_parts_bytes(p, M, I);
    const size_t need = parts ? silu_parts_off(p) + parts : p.ws_bytes;
    if (need > 0 && (workspace == nullptr || workspace_bytes < need))
        return W8A8_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    float *amax = parts ? reinterpret_cast<float *>(static_cast<char *>(workspace) +
                                                    silu_parts_off(p))
                        : nullptr;
    const SiluOut so{a, static_cast<int>(I), amax};
    if ((rc = gemm_run(xq, s_tok, wq_il, s_ch_il, M, 2 * I, K, nullptr, nullptr, workspace, p,
                       &so, dev, sms, st)))
        return rc;
    if (amax) // small M: each token's range from the epilogue's group maxima
        return launch_quantize_f32_parts(a, amax, M, static_cast<int>(I), q, s_out, dev, st);
    const RowLaunch L = row_launch(I);
    switch (L.nch) {
    case 1: return launch_quantize_f32<1>(a, M, (int)I, q, s_out, L.threads, dev, sms, st);
    case 2: return launch_quantize_f32<2>(a, M, (int)I, q, s_out, L.threads, dev, sms, st);
    default: return launch_quantize_f32<4>(a, M, (int)I, q, s_out, L.threads, dev, sms, st);
    }
}

// ------------------------------------------------------------------ GEMM + residual RMSNorm

// The RMSNorm tail's two counter words: the last two flag words, which no stream-K plan
// reaches (its CTAs, at most one per SM, use the words 0 .. grid - 1).
constexpr size_t kRowBarWord = kMaxCtas - 2;

// Whether the one-launch form (the cluster split-K with the RMSNorm tail) applies.
bool gemm_rn_fused(const GemmPlan &p, int64_t N, int sms)
{
    return p.variant == 3 && p.nt <= 64 && N <= 8192 && sms <= static_cast<int>(kRowBarWord);
}

size_t w8a8_gemm_rmsnorm_quant_workspace_size(int64_t M, int64_t N, int64_t K)
{
    if (check_gemm_shape(M, N, K) || check_row_shape(M, N))
        return 0;
    int dev, sms = 148;
    if (current_device(&dev, &sms))
        sms = 148;
    GemmPlan p;
    if (plan_gemm(M, N, K, 0, 0, 0, sms, &p))
        return 0;
    return p.ws_bytes > kFlagBytes ? p.ws_bytes : kFlagBytes;
}

int w8a8_gemm_rmsnorm_quant_one_launch_ok(int64_t M, int64_t N, int64_t K)
{
    if (check_gemm_shape(M, N, K) || check_row_shape(M, N))
        return 0;
    int dev, sms = 148;
    if (current_device(&dev, &sms))
        sms = 148;
    GemmPlan p;
    if (plan_gemm(M, N, K, 0, 0, 0, sms, &p))
        return 0;
    return gemm_rn_fused(p, N, sms) ? 1 : 0;
}

int w8a8_gemm_rmsnorm_quant_ex(const int8_t *xq, const float *s_tok, const int8_t *wq,
                               const float *s_ch, int64_t M, int64_t N, int64_t K, w8a8_bf16 *y,
                               const w8a8_bf16 *residual, w8a8_bf16 *h_out,
                               const float *gamma_smoothed, float eps, int8_t *q, float *s_out,
                               void *workspace, size_t workspace_bytes, int one_launch,
                               w8a8_stream_t stream)
{
    if (one_launch != 0 && one_launch != 1)
        return W8A8_ERR_INVALID_ARG;
    if (!xq || !s_tok || !wq || !s_ch || !y || !residual || !h_out || !gamma_smoothed || !q ||
        !s_out || !(eps >= 0.0f))
        return W8A8_ERR_INVALID_ARG;
    int rc = check_gemm_shape(M, N, K);
    if (rc || (rc = check_row_shape(M, N)))
        return rc;
    if (!aligned16(xq) || !aligned16(wq) || !aligned16(s_ch) || !aligned16(y) ||
        !aligned16(residual) || !aligned16(h_out) || !aligned16(gamma_smoothed) ||
        !aligned16(q) || (workspace && !aligned16(workspace)))
        return W8A8_ERR_ALIGNMENT;
    // h_out may alias residual (in place); y is written by the GEMM and read by the row pass
    if (static_cast<const void *>(h_out) == static_cast<const void *>(y) ||
        static_cast<const void *>(residual) == static_cast<const void *>(y))
        return W8A8_ERR_INVALID_ARG;
    int dev, sms;
    if ((rc = current_device(&dev, &sms)))
        return rc;
    GemmPlan p;
    if ((rc = plan_gemm(M, N, K, 0, 0, 0, sms, &p)))
        return rc;
    const size_t need = p.ws_bytes > kFlagBytes ? p.ws_bytes : kFlagBytes;
    if (workspace == nullptr || workspace_bytes < need)
        return W8A8_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (one_launch) {
        if (!gemm_rn_fused(p, N, sms))
            return W8A8_ERR_UNSUPPORTED_SHAPE;
        CUtensorMap tw, tx;
        if (encode_kmajor_i8(&tw, wq, N, K, kBM) || encode_kmajor_i8(&tx, xq, M, K, p.nt))
            return W8A8_ERR_CUDA;
        RowNormOut rn;
        rn.res = residual;
        rn.h = h_out;
        rn.gamma = gamma_smoothed;
        rn.eps = eps;
        rn.q = q;
        rn.s = s_out;
        rn.bar = static_cast<unsigned int *>(workspace) + kRowBarWord;
        return launch_decode_rn(tw, tx, s_tok, s_ch, M, N, K, p, y, rn, dev, st);
    }
    if ((rc = gemm_run(xq, s_tok, wq, s_ch, M, N, K, y, nullptr, workspace, p, nullptr, dev, sms,
                       st)))
        return rc;
    return rmsnorm_quant_impl<false>(y, residual, h_out, gamma_smoothed, eps, M, N, q, s_out,
                                     stream);
}

int w8a8_gemm_rmsnorm_quant(const int8_t *xq, const float *s_tok, const int8_t *wq,
                            const float *s_ch, int64_t M, int64_t N, int64_t K, w8a8_bf16 *y,
                            const w8a8_bf16 *residual, w8a8_bf16 *h_out,
                            const float *gamma_smoothed, float eps, int8_t *q, float *s_out,
                            void *workspace, size_t workspace_bytes, w8a8_stream_t stream)
{
    return w8a8_gemm_rmsnorm_quant_ex(xq, s_tok, wq, s_ch, M, N, K, y, residual, h_out,
                                      gamma_smoothed, eps, q, s_out, workspace, workspace_bytes,
                                      0, stream);
}

// The FP8 fused gate|up plan: as the GEMM's own, with stream-K in place of the cluster
// split-K (which has no SiLU epilogue).
int plan_silu_fp8(int64_t M, int64_t I, int64_t K, int sms, GemmPlan *p)
{
    int rc = plan_gemm(M, 2 * I, K, 0, 0, 0, sms, p);
    if (rc == W8A8_OK && p->variant == 3)
        rc = plan_gemm(M, 2 * I, K, 2, 0, 0, sms, p);
    return rc;
}

size_t w8a8_gemm_silu_quant_fp8_workspace_size(int64_t M, int64_t I, int64_t K)
{
    if (I < 64 || I % 64 != 0 || check_gemm_shape(M, 2 * I, K))
        return 0;
    int dev, sms = 148;
    if (current_device(&dev, &sms))
        sms = 148;
    GemmPlan p;
    if (plan_silu_fp8(M, I, K, sms, &p))
        return 0;
    const size_t parts = silu_parts_bytes(p, M, I);
    return parts ? silu_parts_off(p) + parts : p.ws_bytes;
}

int w8a8_gemm_silu_quant_fp8(const uint8_t *xq, const float *s_tok, const uint8_t *wq_il,
                             const float *s_ch_il, int64_t M, int64_t I, int64_t K, float *a,
                             uint8_t *q, float *s_out, void *workspace, size_t workspace_bytes,
                             w8a8_stream_t stream)
{
    if (!xq || !s_tok || !wq_il || !s_ch_il || !a || !q || !s_out)
        return W8A8_ERR_INVALID_ARG;
    if (I < 64 || I % 64 != 0)
        return W8A8_ERR_UNSUPPORTED_SHAPE;
    int rc = check_gemm_shape(M, 2 * I, K);
    if (rc || (rc = check_row_shape(M, I)))
        return rc;
    if (!aligned16(xq) || !aligned16(wq_il) || !aligned16(s_ch_il) || !aligned16(a) ||
        !aligned16(q) || (workspace && !aligned16(workspace)))
        return W8A8_ERR_ALIGNMENT;
    int dev, sms;
    if ((rc = current_device(&dev, &sms)))
        return rc;
    GemmPlan p;
    if ((rc = plan_silu_fp8(M, I, K, sms, &p)))
        return rc;
    const size_t parts = silu_parts_bytes(p, M, I);
    const size_t need = parts ? silu_parts_off(p) + parts : p.ws_bytes;
    if (need > 0 && (workspace == nullptr || workspace_bytes < need))
        return W8A8_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    float *amax = parts ? reinterpret_cast<float *>(static_cast<char *>(workspace) +
                                                    silu_parts_off(p))
                        : nullptr;
    const SiluOut so{a, static_cast<int>(I), amax};
    if ((rc = gemm_run_fp8(xq, s_tok, wq_il, s_ch_il, M, 2 * I, K, nullptr, nullptr, workspace,
                           p, dev, sms, st, &so)))
        return rc;
    int8_t *qc = reinterpret_cast<int8_t *>(q);
    if (amax)
        return launch_quantize_f32_parts<true>(a, amax, M, static_cast<int>(I), qc, s_out, dev, st);
    const RowLaunch L = row_launch(I);
    switch (L.nch) {
    case 1: return launch_quantize_f32<1, true>(a, M, (int)I, qc, s_out, L.threads, dev, sms, st);
    case 2: return launch_quantize_f32<2, true>(a, M, (int)I, qc, s_out, L.threads, dev, sms, st);
    default: return launch_quantize_f32<4, true>(a, M, (int)I, qc, s_out, L.threads, dev, sms, st);
    }
}

size_t w8a8_gemm_workspace_size_ex(int64_t M, int64_t N, int64_t K, int variant, int ctas,
                                   int tile_n)
{
    if (check_gemm_shape(M, N, K))
        return 0;
    int dev, sms = 148;
    if (current_device(&dev, &sms))
        sms = 148;
    GemmPlan p;
    if (plan_gemm(M, N, K, variant, ctas, tile_n, sms, &p))
        return 0;
    return p.ws_bytes;
}

size_t w8a8_gemm_workspace_size(int64_t M, int64_t N, int64_t K)
{
    return w8a8_gemm_workspace_size_ex(M, N, K, 0, 0, 0);
}

int w8a8_gemm_dequant_ex(const int8_t *xq, const float *s_tok, const int8_t *wq,
                         const float *s_ch, int64_t M, int64_t N, int64_t K, w8a8_bf16 *y,
                         int32_t *acc_out, void *workspace, size_t workspace_bytes, int variant,
                         int ctas, int tile_n, w8a8_stream_t stream)
{
    if (!xq || !s_tok || !wq || !s_ch || !y)
        return W8A8_ERR_INVALID_ARG;
    int rc = check_gemm_shape(M, N, K);
    if (rc)
        return rc;
    if (!aligned16(xq) || !aligned16(wq) || !aligned16(s_ch) || !aligned16(y) ||
        (acc_out && !aligned16(acc_out)) || (workspace && !aligned16(workspace)))
        return W8A8_ERR_ALIGNMENT;
    int dev, sms;
    if ((rc = current_device(&dev, &sms)))
        return rc;
    GemmPlan p;
    if ((rc = plan_gemm(M, N, K, variant, ctas, tile_n, sms, &p)))
        return rc;
    if (p.ws_bytes > 0 && (workspace == nullptr || workspace_bytes < p.ws_bytes))
        return W8A8_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    return gemm_run(xq, s_tok, wq, s_ch, M, N, K, y, acc_out, workspace, p, nullptr, dev, sms,
                    st);
}

int w8a8_gemm_dequant(const int8_t *xq, const float *s_tok, const int8_t *wq, const float *s_ch,
                      int64_t M, int64_t N, int64_t K, w8a8_bf16 *y, int32_t *acc_out,
                      void *workspace, size_t workspace_bytes, w8a8_stream_t stream)
{
    return w8a8_gemm_dequant_ex(xq, s_tok, wq, s_ch, M, N, K, y, acc_out, workspace,
                                workspace_bytes, 0, 0, 0, stream);
}

size_t w8a8_gemm_fp8_workspace_size(int64_t M, int64_t N, int64_t K, int variant, int ctas,
                                    int tile_n)
{
    if (check_gemm_shape(M, N, K))
        return 0;
    int dev, sms = 148;
    if (current_device(&dev, &sms))
        sms = 148;
    GemmPlan p;
    if (plan_gemm(M, N, K, variant, ctas, tile_n, sms, &p))
        return 0;
    return p.ws_bytes;
}

int w8a8_gemm_dequant_fp8(const uint8_t *xq, const float *s_tok, const uint8_t *wq,
                          const float *s_ch, int64_t M, int64_t N, int64_t K, w8a8_bf16 *y,
                          float *acc_out, void *workspace, size_t workspace_bytes, int variant,
                          int ctas, int tile_n, w8a8_stream_t stream)
{
    if (!xq || !s_tok || !wq || !s_ch || !y)
        return W8A8_ERR_INVALID_ARG;
    int rc = check_gemm_shape(M, N, K);
    if (rc)
        return rc;
    if (!aligned16(xq) || !aligned16(wq) || !aligned16(s_ch) || !aligned16(y) ||
        (acc_out && !aligned16(acc_out)) || (workspace && !aligned16(workspace)))
        return W8A8_ERR_ALIGNMENT;
    int dev, sms;
    if ((rc = current_device(&dev, &sms)))
        return rc;
    GemmPlan p;
    if ((rc = plan_gemm(M, N, K, variant, ctas, tile_n, sms, &p)))
        return rc;
    if (p.ws_bytes > 0 && (workspace == nullptr || workspace_bytes < p.ws_bytes))
        return W8A8_ERR_WORKSPACE;
    return gemm_run_fp8(xq, s_tok, wq, s_ch, M, N, K, y, acc_out, workspace, p, dev, sms,
                        reinterpret_cast<cudaStream_t>(stream));
}

size_t w8a8_block_decode_workspace_size(int64_t M, int64_t H, int64_t I, int64_t QKV)
{
    if (M < 1 || M > 64 || H < 128 || H % 128 || I < 128 || I % 128 || QKV < 8 || QKV % 8)
        return 0;
    return 512 + block_phase_bytes(M, QKV) + 2 * block_phase_bytes(M, H) +
           block_phase_bytes(M, 2 * I);
}

int w8a8_block_decode(const w8a8_block_io *io, void *workspace, size_t workspace_bytes,
                      w8a8_stream_t stream)
{
    if (!io)
        return W8A8_ERR_INVALID_ARG;
    const w8a8_block_io &b = *io;
    const void *ptrs[] = {b.x, b.attn, b.gamma1, b.sinv_o, b.gamma2, b.qkv.wq, b.qkv.s_ch, b.o.wq,
                          b.o.s_ch, b.gate_up_il.wq, b.gate_up_il.s_ch, b.down.wq, b.down.s_ch,
                          b.qkv_out, b.o_out, b.h_out, b.y_out, b.a_out, b.q1, b.q2, b.q3, b.q4,
                          b.s1, b.s2, b.s3, b.s4};
    for (const void *p : ptrs)
        if (!p)
            return W8A8_ERR_INVALID_ARG;
    if (!(b.eps >= 0.0f))
        return W8A8_ERR_INVALID_ARG;
    if (b.M < 1 || b.M > 64 || b.H < 128 || b.H % 128 || b.I < 128 || b.I % 128 || b.QKV < 8 ||
        b.QKV % 8 || b.H > 8192 || b.I > 32768 || b.QKV > 0x7fffffffLL)
        return W8A8_ERR_UNSUPPORTED_SHAPE;
    for (const void *p : ptrs)
        if (!aligned16(p))
            return W8A8_ERR_ALIGNMENT;
    if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256 != 0)
        return workspace ? W8A8_ERR_ALIGNMENT : W8A8_ERR_WORKSPACE;
    int dev, sms;
    int rc = current_device(&dev, &sms);
    if (rc)
        return rc;
    if (sms > kMaxCtas || (2 * b.I + kBM - 1) / kBM > kMaxCtas || (b.QKV + kBM - 1) / kBM > kMaxCtas)
        return W8A8_ERR_UNSUPPORTED_SHAPE;
    const size_t need = 512 + block_phase_bytes(b.M, b.QKV) + 2 * block_phase_bytes(b.M, b.H) +
                        block_phase_bytes(b.M, 2 * b.I);
    if (workspace_bytes < need)
        return W8A8_ERR_WORKSPACE;
    const int M = static_cast<int>(b.M), H = static_cast<int>(b.H), I = static_cast<int>(b.I),
              Q = static_cast<int>(b.QKV);
    const int nt = M <= 16 ? 16 : M <= 32 ? 32 : 64;
    BlockMaps maps;
    const int8_t *wq[4] = {b.qkv.wq, b.o.wq, b.gate_up_il.wq, b.down.wq};
    const int8_t *xq[4] = {b.q1, b.q2, b.q3, b.q4};
    const int Ns[4] = {Q, H, 2 * I, H}, Ks[4] = {H, H, H, I};
    for (int p = 0; p < 4; ++p)
        if (encode_kmajor_i8(&maps.w[p], wq[p], Ns[p], Ks[p], kBM) ||
            encode_kmajor_i8(&maps.x[p], xq[p], M, Ks[p], nt))
            return W8A8_ERR_CUDA;
    BlockArgs a;
    a.M = M;
    a.H = H;
    a.I = I;
    a.eps = b.eps;
    a.x = b.x;
    a.attn = b.attn;
    a.g1 = b.gamma1;
    a.sinv_o = b.sinv_o;
    a.g2 = b.gamma2;
    int8_t *qs[4] = {b.q1, b.q2, b.q3, b.q4};
    float *ss[4] = {b.s1, b.s2, b.s3, b.s4};
    for (int p = 0; p < 4; ++p) {
        a.q[p] = qs[p];
        a.s[p] = ss[p];
    }
    a.h = b.h_out;
    a.a = b.a_out;
    const float *sch[4] = {b.qkv.s_ch, b.o.s_ch, b.gate_up_il.s_ch, b.down.s_ch};
    uint16_t *ys[4] = {b.qkv_out, b.o_out, nullptr, b.y_out};
    char *ws = static_cast<char *>(workspace);
    size_t off = 512;
    for (int p = 0; p < 4; ++p) {
        char *base = ws + off;
        a.g[p] = BlockGemm{sch[p], ys[p], Ns[p], Ks[p], reinterpret_cast<int32_t *>(base + kFlagBytes),
                           reinterpret_cast<unsigned int *>(base)};
        off += block_phase_bytes(b.M, Ns[p]);
    }
    a.bar = reinterpret_cast<unsigned long long *>(ws);
    a.amax_w = reinterpret_cast<unsigned int *>(ws + 256);
    a.limit_ns = kWaitLimitNs;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // two k-blocks per stage, as many stages as fit: the ring holds a CTA's whole share of the
    // small projections
    if (H <= 4096) {
        switch (nt) {
        case 16: return launch_block<16, 6, 2, 4>(maps, a, dev, sms, st);
        case 32: return launch_block<32, 5, 2, 4>(maps, a, dev, sms, st);
        default: return launch_block<64, 4, 2, 4>(maps, a, dev, sms, st);
        }
    }
    switch (nt) {
    case 16: return launch_block<16, 6, 2, 8>(maps, a, dev, sms, st);
    case 32: return launch_block<32, 5, 2, 8>(maps, a, dev, sms, st);
    default: return launch_block<64, 4, 2, 8>(maps, a, dev, sms, st);
    }
}

size_t w8a8_gptq_workspace_size(int64_t N, int64_t K)
{
    if (N < 1 || K < 64 || K % 64 != 0 || K > 32768)
        return 0;
    const GptqLayout L = gptq_layout(N, K);
    return L.total;
}

int w8a8_gptq_quantize(const w8a8_bf16 *w, const float *smooth, const float *x_cal, int64_t N,
                       int64_t K, int64_t T, double damp, int8_t *wq, float *s_ch,
                       double *u_out, void *workspace, size_t workspace_bytes,
                       w8a8_stream_t stream)
{
    namespace g = w8a8::gptq;
    if (!w || !x_cal || !wq || !s_ch || N < 1 || T < 1 || !(damp > 0.0) || !(damp < 1e300))
        return W8A8_ERR_INVALID_ARG;
    if (K < 64 || K % 64 != 0 || K > 32768 || N > 0x7fffffffLL || T > 0x7fffffffLL)
        return W8A8_ERR_UNSUPPORTED_SHAPE;
    const GptqLayout L = gptq_layout(N, K);
    if (!workspace || workspace_bytes < L.total)
        return W8A8_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0 ||
        reinterpret_cast<uintptr_t>(u_out) % 8 != 0 || reinterpret_cast<uintptr_t>(wq) % 16 != 0)
        return W8A8_ERR_ALIGNMENT;
    int dev, sms;
    int rc = current_device(&dev, &sms);
    if (rc)
        return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    char *base = static_cast<char *>(workspace);
    double *A = reinterpret_cast<double *>(base + L.a_off);   // H, then V in its upper part
    double *U = reinterpret_cast<double *>(base + L.u_off);
    double *wd = reinterpret_cast<double *>(base + L.w_off);
    double *err = reinterpret_cast<double *>(base + L.e_off);
    uint8_t *dead = reinterpret_cast<uint8_t *>(base + L.d_off);
    int *bad = reinterpret_cast<int *>(base + L.b_off);
    const int nb = static_cast<int>(K / g::kT);
    const int sm2 = g::kTwoTileBytes;
    for (const void *fn : {reinterpret_cast<const void *>(&g::chol_update_kernel),
                           reinterpret_cast<const void *>(&g::trtri_diag_kernel),
                           reinterpret_cast<const void *>(&g::trtri_update_kernel),
                           reinterpret_cast<const void *>(&g::trtri_final_kernel)})
        if ((rc = ensure_smem(fn, dev, sm2)))
            return rc;
    if ((rc = ensure_smem(reinterpret_cast<const void *>(&g::update_kernel), dev,
                          g::kUpdateBytes)))
        return rc;
    if (cudaMemsetAsync(bad, 0, sizeof(int), st) != cudaSuccess)
        return W8A8_ERR_CUDA;
    g::hessian_kernel<<<nb * (nb + 1) / 2, g::kThreads, 0, st>>>(x_cal, T, K, A);
    g::diag_kernel<<<1, 1024, 0, st>>>(A, K, damp, dead);
    for (int kb = nb - 1; kb >= 0; --kb) {
        g::chol_diag_kernel<<<1, g::kThreads, 0, st>>>(A, K, kb, bad);
        if (kb > 0) {
            g::chol_panel_kernel<<<kb, g::kT, 0, st>>>(A, K, kb);
            g::chol_update_kernel<<<kb * (kb + 1) / 2, g::kTileThreads, sm2, st>>>(A, K, kb);
        }
    }
    // U's off-diagonal blocks start as zero running sums
    if (cudaMemsetAsync(U, 0, static_cast<size_t>(K * K) * sizeof(double), st) != cudaSuccess)
        return W8A8_ERR_CUDA;
    g::trtri_diag_kernel<<<nb, g::kT, sm2, st>>>(A, U, K);
    for (int k = nb - 1; k >= 1; --k) {
        // block row k is final from here on (row nb-1 is its diagonal block only)
        if (k < nb - 1)
            g::trtri_final_kernel<<<nb - 1 - k, g::kTileThreads, sm2, st>>>(U, K, k);
        g::trtri_update_kernel<<<k * (nb - k), g::kTileThreads, sm2, st>>>(A, U, K, k);
    }
    if (nb > 1)
        g::trtri_final_kernel<<<nb - 1, g::kTileThreads, sm2, st>>>(U, K, 0);
    const unsigned rows_grid =
        static_cast<unsigned>(std::min<int64_t>((N + 7) / 8, static_cast<int64_t>(sms) * 8));
    g::prep_kernel<<<rows_grid, g::kThreads, 0, st>>>(w, smooth, dead, N, K, wd, s_ch);
    // groups of kGptqGroup column blocks: inside a group each block's errors reach the
    // group's later blocks at once; the group's errors then reach every later column in one
    // pass over the working weight
    const unsigned row_tiles = static_cast<unsigned>((N + g::kRT - 1) / g::kRT);
    // the quantize kernel: four lanes per row (32 rows per CTA) while one wave holds the
    // rows; beyond that one thread per row (CTAs of 32..128 threads)
    int quad_per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&quad_per_sm, g::quant_block_kernel,
                                                      g::kQuantThreads, 0) != cudaSuccess)
        return W8A8_ERR_CUDA;
    const int64_t quad_ctas = (N + g::kQuantThreads / 4 - 1) / (g::kQuantThreads / 4);
    const bool quad = quad_ctas <= static_cast<int64_t>(sms) * std::max(quad_per_sm, 1);
    const int row_threads = static_cast<int>(
        std::min<int64_t>(128, std::max<int64_t>(32, ((N + sms - 1) / sms + 31) / 32 * 32)));
    const unsigned quant_grid = static_cast<unsigned>(
        quad ? quad_ctas : (N + row_threads - 1) / row_threads);
    const int64_t eld = static_cast<int64_t>(g::kT) * kGptqGroup;
    const int ub = g::kUpdateBytes;
    for (int b0 = 0; b0 < nb; b0 += kGptqGroup) {
        const int b1 = std::min(nb, b0 + kGptqGroup);
        for (int jb = b0; jb < b1; ++jb) {
            double *ej = err + static_cast<int64_t>(jb - b0) * g::kT;
            if (quad)
                g::quant_block_kernel<<<quant_grid, g::kQuantThreads, 0, st>>>(wd, U, s_ch, N, K,
                                                                                jb, wq, ej, eld);
            else
                g::quant_block_rows_kernel<<<quant_grid, row_threads, 0, st>>>(wd, U, s_ch, N, K,
                                                                               jb, wq, ej, eld);
            if (jb + 1 < b1)
                g::update_kernel<<<dim3(b1 - 1 - jb, row_tiles), g::kThreads, ub, st>>>(
                    wd, U, ej, eld, N, K, static_cast<int64_t>(jb) * g::kT, 1,
                    static_cast<int64_t>(jb + 1) * g::kT);
        }
        if (b1 < nb)
            g::update_kernel<<<dim3(nb - b1, row_tiles), g::kThreads, ub, st>>>(
                wd, U, err, eld, N, K, static_cast<int64_t>(b0) * g::kT, b1 - b0,
                static_cast<int64_t>(b1) * g::kT);
    }
    if (u_out) {
        g::zero_lower_kernel<<<sms * 4, g::kThreads, 0, st>>>(U, K);
        if (cudaMemcpyAsync(u_out, U, static_cast<size_t>(K * K) * sizeof(double),
                            cudaMemcpyDeviceToDevice, st) != cudaSuccess)
            return W8A8_ERR_CUDA;
    }
    if (cudaGetLastError() != cudaSuccess)
        return W8A8_ERR_CUDA;
    int bad_h = 0;
    if (cudaMemcpyAsync(&bad_h, bad, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return W8A8_ERR_CUDA;
    return bad_h ? W8A8_ERR_NUMERIC : W8A8_OK;
}

int w8a8_probe_i8_mma(long long iters, int n, int ctas, w8a8_stream_t stream)
{
    if (iters < 1 || ctas < 0)
        return W8A8_ERR_INVALID_ARG;
    int dev, sms;
    int rc = current_device(&dev, &sms);
    if (rc)
        return rc;
    const int grid = ctas == 0 ? sms : ctas;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    switch (n) {
    case 16: return launch_probe<16>(iters, grid, dev, st);
    case 32: return launch_probe<32>(iters, grid, dev, st);
    case 64: return launch_probe<64>(iters, grid, dev, st);
    case 128: return launch_probe<128>(iters, grid, dev, st);
    case 256: return launch_probe<256>(iters, grid, dev, st);
    default: return W8A8_ERR_INVALID_ARG;
    }
}

int w8a8_probe_f64_fma(long long iters, int ctas, double *out, w8a8_stream_t stream)
{
    if (iters < 1 || ctas < 1 || !out)
        return W8A8_ERR_INVALID_ARG;
    int dev, sms;
    int rc = current_device(&dev, &sms);
    if (rc)
        return rc;
    fma_f64_probe_kernel<<<ctas, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(iters, out);
    return cudaGetLastError() == cudaSuccess ? W8A8_OK : W8A8_ERR_CUDA;
}

int w8a8_set_overlap(int mode)
{
    if (mode < 0 || mode > 2)
        return W8A8_ERR_INVALID_ARG;
    return g_overlap.exchange(mode);
}

int w8a8_get_overlap(void)
{
    return g_overlap.load();
}

int w8a8_selftest_wait_timeout(unsigned long long limit_ns, w8a8_stream_t stream)
{
    if (limit_ns < 1000ull || limit_ns > 2000000000ull)
        return W8A8_ERR_INVALID_ARG;
    int dev, sms;
    int rc = current_device(&dev, &sms);
    if (rc)
        return rc;
    wait_timeout_selftest_kernel<<<1, 64, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_ns);
    if (cudaGetLastError() != cudaSuccess)
        return W8A8_ERR_CUDA;
    return W8A8_OK;
}

int w8a8_last_device_status(w8a8_stream_t stream)
{
    int dev, sms;
    int rc = current_device(&dev, &sms);
    if (rc)
        return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // the read is ordered after this stream's work; the host copy target is pageable, so the
    // call returns once the stream has reached it
    unsigned int word = 0;
    if (cudaMemcpyFromSymbolAsync(&word, g_status_word, sizeof(word), 0,
                                  cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess) {
        cudaGetLastError();
        return W8A8_ERR_CUDA;
    }
    return (word & kStatusTimeout) ? W8A8_ERR_TIMEOUT : W8A8_OK;
}

int w8a8_device_status(int reset)
{
    int dev, sms;
    int rc = current_device(&dev, &sms);
    if (rc)
        return rc;
    if (cudaDeviceSynchronize() != cudaSuccess)
        return W8A8_ERR_CUDA;
    unsigned int word = 0;
    if (cudaMemcpyFromSymbol(&word, g_status_word, sizeof(word)) != cudaSuccess)
        return W8A8_ERR_CUDA;
    if (reset) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_status_word, &zero, sizeof(zero)) != cudaSuccess)
            return W8A8_ERR_CUDA;
    }
    return (word & kStatusTimeout) ? W8A8_ERR_TIMEOUT : W8A8_OK;
}

} // extern "C"

// ------------------------------------------------------------------ no-allocation GEMM

// Split-K scratch of w8a8_gemm_dequant_noalloc: flag words and partial sums live here instead
// of in a caller-provided workspace. Host code must not pass `g_noalloc_scratch` itself to a
// kernel (on the host it names a host-side shadow, not device memory); it passes the device
// address looked up by noalloc_scratch().
static __device__ __align__(256) unsigned char g_noalloc_scratch[W8A8_NOALLOC_SCRATCH_BYTES];

namespace {

void *g_noalloc_ptr[kMaxDevices];

// Device address of the scratch array on device `dev` (the current device), looked up once.
int noalloc_scratch(int dev, void **out)
{
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return W8A8_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return W8A8_OK;
}

} // namespace

extern "C" int w8a8_gemm_dequant_noalloc(const int8_t *xq, const float *s_tok, const int8_t *wq,
                                         const float *s_ch, int64_t M, int64_t N, int64_t K,
                                         w8a8_bf16 *y, w8a8_stream_t stream)
{
    if (!xq || !s_tok || !wq || !s_ch || !y)
        return W8A8_ERR_INVALID_ARG;
    int rc = check_gemm_shape(M, N, K);
    if (rc)
        return rc;
    if (M > 256)
        return W8A8_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(xq) || !aligned16(wq) || !aligned16(s_ch) || !aligned16(y))
        return W8A8_ERR_ALIGNMENT;
    int dev, sms;
    if ((rc = current_device(&dev, &sms)))
        return rc;
    // the decode kernels, chosen as w8a8_gemm_dequant chooses them for small M
    const int64_t NB = (N + kBM - 1) / kBM, KB = (K + kBK - 1) / kBK;
    GemmPlan p;
    if ((rc = plan_gemm(M, N, K, (2 * NB <= sms && KB >= 2) ? 3 : 2, 0, 0, sms, &p)))
        return rc;
    if (p.ws_bytes > W8A8_NOALLOC_SCRATCH_BYTES)
        return W8A8_ERR_WORKSPACE;
    void *scratch = nullptr;
    if (p.ws_bytes > 0) {
        if ((rc = noalloc_scratch(dev, &scratch)))
            return rc;
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // Only the flag words must be zero when the kernel starts (each contributor writes its
    // partial sums before raising its flag, and the owner lowers the flags it consumed);
    // clearing them on every call also drops flags left raised by a call whose wait ran out.
    if (p.ws_bytes > 0 &&
        cudaMemsetAsync(static_cast<char *>(scratch) + p.flag_off, 0, kFlagBytes, st) !=
            cudaSuccess) {
        cudaGetLastError();
        return W8A8_ERR_CUDA;
    }
    CUtensorMap tw, tx;
    if (encode_kmajor_i8(&tw, wq, N, K, kBM) || encode_kmajor_i8(&tx, xq, M, K, p.nt))
        return W8A8_ERR_CUDA;
    return launch_decode_nt<false>(tw, tx, s_tok, s_ch, M, N, K, p, y, nullptr, scratch,
                                   SiluOut{nullptr, 0}, dev, st);
}
