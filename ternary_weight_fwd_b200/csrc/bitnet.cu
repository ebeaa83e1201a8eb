// bitnet.cu -- C ABI of the BitLinear forward library (the only translation
// unit; the kernels live in the .cuh files included below).
//
// Host side: argument validation (before anything is launched), kernel
// selection by M, TMA descriptor encoding, and launches with programmatic
// dependent launch so consecutive kernels overlap their prologues.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <queue>
#include <utility>
#include <vector>

#include "bitnet.h"
#include "common.cuh"
#include "decode.cuh"
#include "decode_cluster.cuh"
#include "decode_tasks.cuh"
#include "pack_quant.cuh"
#include "prefill.cuh"

namespace bitnet {


namespace {

constexpr int kMaxDevices = 64;
constexpr int64_t kMaxDim = int64_t(1) << 24;
constexpr int64_t kMaxK = 65536;
constexpr int kDecodeMaxM = 64;
constexpr size_t kSmemLimit = 227 * 1024;

std::atomic<int> g_dispatch{BITNET_DISPATCH_AUTO};
std::atomic<uint64_t> g_launches{0};

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

int current_device()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    return dev;
}

int num_sms_for(int dev)
{
    static std::atomic<int> cache[kMaxDevices];
    if (dev < 0 || dev >= kMaxDevices) return 0;
    int v = cache[dev].load();
    if (v > 0) return v;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev].store(v);
    return v;
}

// Raise the dynamic shared-memory limit of a kernel once per device.
template <typename Kern>
cudaError_t ensure_smem(Kern *kern, size_t bytes, std::atomic<int> (&done)[kMaxDevices], int dev)
{
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (done[dev].load() >= (int)bytes) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemLimit);
    if (e == cudaSuccess) done[dev].store((int)kSmemLimit);
    return e;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

bitnet_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA; }

bitnet_status_t check_shape(int64_t M, int64_t N, int64_t K)
{
    if (M < 1 || N < 1 || K < 1) return BITNET_ERR_INVALID_ARG;
    if (K % 64 != 0 || K > kMaxK || M > kMaxDim || N > kMaxDim) return BITNET_ERR_UNSUPPORTED_SHAPE;
    return BITNET_OK;
}

// ---- workspace layout shared by linear / ffn -------------------------------
struct Workspace {
    int8_t *xq;
    float *s;
    int32_t *rs;
};

size_t ws_bytes_for(int64_t M, int64_t K)
{
    return align_up((size_t)M * (size_t)K, 256) + 2 * align_up((size_t)M * 4, 256);
}

Workspace carve(void *ws, int64_t M, int64_t K)
{
    char *p = static_cast<char *>(ws);
    Workspace w;
    w.xq = reinterpret_cast<int8_t *>(p);
    p += align_up((size_t)M * (size_t)K, 256);
    w.s = reinterpret_cast<float *>(p);
    p += align_up((size_t)M * 4, 256);
    w.rs = reinterpret_cast<int32_t *>(p);
    return w;
}

// ---- prefill: the partly filled last wave of tiles (see k_prefill) -------------
// A BitLinear whose last wave holds at most a quarter (half) of the grid runs each
// of its tiles as 4 (2) sub-tiles of 64 (128) output columns on separate CTAs.
int pf_tail_q(int64_t M, int64_t N, int nmat, int sms)
{
    if (nmat != 1) return 1;
    const int64_t tiles = cdiv(M, PF_BM) * cdiv(N, PF_BN);
    const int64_t grid = std::min<int64_t>(tiles, sms);
    if (grid <= 0) return 1;
    const int64_t full = tiles / grid * grid, rem = tiles - full;
    if (full == 0 || rem == 0) return 1;
    if (4 * rem <= grid) return 4;
    if (2 * rem <= grid) return 2;
    return 1;
}

// ---- TMA descriptors ---------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D uint8 tensor [rows][cols] (row pitch = cols bytes), box [box_rows][box_cols].
bool encode_u8_2d(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                  uint32_t box_cols, bool swizzle128)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D output tensor [rows][cols] of fp32 (128-byte swizzle) or bf16 (64-byte
// swizzle), box [box_rows][box_cols]: the box rows are exactly one swizzle span.
bool encode_2d_out(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                   uint32_t box_cols, bool bf16)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * (bf16 ? 2 : 4)};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
                    const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    bf16 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ---- decode configuration -----------------------------------------------------
struct DecodeCfg {
    bool ok;
    int grid, rg, w_stride, rp, ch;
    size_t smem;
};

// Row-split decode kernel (quantiser kernel first): one CTA per slice of rows.
DecodeCfg decode_config(int64_t N, int64_t K, int nmat, int sms)
{
    DecodeCfg c = {};
    c.w_stride = (int)(K / 4 + ((16 - (K / 4) % 128) + 128) % 128);
    int64_t grid = std::min<int64_t>(sms, cdiv(N, 16));
    for (;;) {
        const int64_t rmax = cdiv(N, grid);
        const int rg = (int)cdiv(rmax, 16);
        if (rg > DEC_RGM) {
            grid = cdiv(N, 16 * DEC_RGM);
            continue;
        }
        const int rp = rg * 16 + ((4 - (rg * 16) % 32) + 32) % 32;
        const size_t smem = DEC_HDR + (size_t)nmat * rg * 16 * c.w_stride + (size_t)nmat * 8 * rp * 4;
        if (smem > kSmemLimit) {
            if (rg == 1) return c; // K too large for the decode kernel
            grid = cdiv(N, 16 * (rg - 1));
            continue;
        }
        c.grid = (int)grid;
        c.rg = rg;
        c.rp = rp;
        c.smem = smem;
        break;
    }
    const int64_t steps = cdiv(K / 64, DEC_WARPS);
    c.ch = steps <= 4 ? 4 : (steps <= 8 ? 8 : 16);
    c.ok = true;
    return c;
}

template <int NMAT, int CH>
cudaError_t launch_decode_t(const DecodeArgs &a, const DecodeCfg &c, cudaStream_t stream, int dev)
{
    static std::atomic<int> done[kMaxDevices];
    auto kern = k_decode<NMAT, CH>;
    cudaError_t e = ensure_smem(kern, c.smem, done, dev);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3(c.grid), dim3(DEC_THREADS), c.smem, stream, a);
}

template <int NMAT>
cudaError_t launch_decode(const DecodeArgs &a, const DecodeCfg &c, cudaStream_t stream, int dev)
{
    switch (c.ch) {
    case 4: return launch_decode_t<NMAT, 4>(a, c, stream, dev);
    case 8: return launch_decode_t<NMAT, 8>(a, c, stream, dev);
    default: return launch_decode_t<NMAT, 16>(a, c, stream, dev);
    }
}

template <bool XF32, int WPR>
cudaError_t launch_quant_w(const void *x, int64_t M, int64_t K, int8_t *xq, float *s, int32_t *rs,
                           const float *amax_in, float *amax_zero, cudaStream_t stream)
{
    const int64_t nch = K / (XF32 ? 4 : 8);
    const int64_t per_lane = cdiv(nch, 32 * WPR); // chunks a lane holds
    const dim3 grid((unsigned)cdiv(M, 8 / WPR));
    if (per_lane <= 8)
        return launch_pdl(k_quant_rows_reg<XF32, WPR, 8>, grid, dim3(256), 0, stream, x, M, K, xq, s, rs, amax_in,
                          amax_zero);
    if (per_lane <= 12)
        return launch_pdl(k_quant_rows_reg<XF32, WPR, 12>, grid, dim3(256), 0, stream, x, M, K, xq, s, rs, amax_in,
                          amax_zero);
    return launch_pdl(k_quant_rows_reg<XF32, WPR, QR_NCH>, grid, dim3(256), 0, stream, x, M, K, xq, s, rs, amax_in,
                      amax_zero);
}

// Per-token quantiser: rows held in registers (one HBM read) when a row fits
// in 8 warps x 32 lanes x QR_NCH chunks, otherwise the two-pass kernel (one
// pass when the row maxima are given).  amax_in: optional given row maxima;
// amax_zero: optional [M] zeroed for the next kernel's atomicMax.
template <bool XF32>
cudaError_t launch_quant_t(const void *x, int64_t M, int64_t K, int8_t *xq, float *s, int32_t *rs,
                           const float *amax_in, float *amax_zero, cudaStream_t stream)
{
    const int64_t nch = K / (XF32 ? 4 : 8);
    const int64_t per_warp = 32 * QR_NCH;
    if (nch <= per_warp) return launch_quant_w<XF32, 1>(x, M, K, xq, s, rs, amax_in, amax_zero, stream);
    if (nch <= 2 * per_warp) return launch_quant_w<XF32, 2>(x, M, K, xq, s, rs, amax_in, amax_zero, stream);
    if (nch <= 4 * per_warp) return launch_quant_w<XF32, 4>(x, M, K, xq, s, rs, amax_in, amax_zero, stream);
    if (nch <= 8 * per_warp) return launch_quant_w<XF32, 8>(x, M, K, xq, s, rs, amax_in, amax_zero, stream);
    return launch_pdl(k_quant_rows<XF32>, dim3((unsigned)cdiv(M, 8)), dim3(256), 0, stream, x, M, K, xq, s, rs,
                      amax_in, amax_zero);
}

// RMS normalisation + quantiser: the row layout of launch_quant_t (1, 2, 4 or 8
// warps per row by the number of 16-byte chunks), rows of up to kNormMaxK.
template <bool XF32>
cudaError_t launch_norm_quant_t(const void *x, int64_t M, int64_t K, const float *g, float eps, int8_t *xq, float *s,
                                int32_t *rs, float *amax_zero, cudaStream_t stream)
{
    const int64_t nch = K / (XF32 ? 4 : 8);
    const int64_t per_warp = 32 * QR_NCH;
    if (nch <= per_warp)
        return launch_pdl(k_rmsnorm_quant_rows<XF32, 1>, dim3((unsigned)cdiv(M, 8)), dim3(256), 0, stream, x, M, K,
                          g, eps, xq, s, rs, amax_zero);
    if (nch <= 2 * per_warp)
        return launch_pdl(k_rmsnorm_quant_rows<XF32, 2>, dim3((unsigned)cdiv(M, 4)), dim3(256), 0, stream, x, M, K,
                          g, eps, xq, s, rs, amax_zero);
    if (nch <= 4 * per_warp)
        return launch_pdl(k_rmsnorm_quant_rows<XF32, 4>, dim3((unsigned)cdiv(M, 2)), dim3(256), 0, stream, x, M, K,
                          g, eps, xq, s, rs, amax_zero);
    return launch_pdl(k_rmsnorm_quant_rows<XF32, 8>, dim3((unsigned)M), dim3(256), 0, stream, x, M, K, g, eps, xq, s,
                      rs, amax_zero);
}

cudaError_t launch_norm_quant(const void *x, bool xf32, int64_t M, int64_t K, const float *g, float eps, int8_t *xq,
                              float *s, int32_t *rs, cudaStream_t stream, float *amax_zero = nullptr)
{
    return xf32 ? launch_norm_quant_t<true>(x, M, K, g, eps, xq, s, rs, amax_zero, stream)
                : launch_norm_quant_t<false>(x, M, K, g, eps, xq, s, rs, amax_zero, stream);
}

cudaError_t launch_quant(const void *x, bool xf32, int64_t M, int64_t K, int8_t *xq, float *s, int32_t *rs,
                         cudaStream_t stream, const float *amax_in = nullptr, float *amax_zero = nullptr)
{
    return xf32 ? launch_quant_t<true>(x, M, K, xq, s, rs, amax_in, amax_zero, stream)
                : launch_quant_t<false>(x, M, K, xq, s, rs, amax_in, amax_zero, stream);
}

// ---- cluster (K-split, fused quantiser) decode kernel -------------------------
struct DcCfg {
    bool ok;
    int nc;  // clusters launched
    int rgw; // row groups per warp
    size_t smem;
    DcArgs a;
};

// Shared-memory layout for `rpc` rows per cluster and cluster size C.
bool dc_layout(DcArgs &a, size_t &smem, int64_t K, int nmat, bool xf32, int C, int rpc, bool single_tile)
{
    const int KS = (int)(K / 64);
    a.C = C;
    a.ks = (int)cdiv(KS, C);
    if (a.ks > 16) return false; // at most 1024 k per CTA
    a.rpc = (int)align_up((size_t)rpc, 8);
    if (nmat * cdiv(a.rpc, 16) > 8 * DC_RGW_MAX) return false; // row groups per warp
    const uint32_t box_w = (uint32_t)a.ks * 16;
    a.w_mat_bytes = (uint32_t)align_up(align_up((size_t)a.rpc, 16) * box_w, 128);
    a.xs_row = (uint32_t)align_up((size_t)a.ks * 64 * (xf32 ? 4 : 2), 128);
    a.xs_off = (uint32_t)(DC_HDR + (size_t)nmat * a.w_mat_bytes);
    a.xq_stride = (uint32_t)(a.ks * 64 + ((64 - (a.ks * 64) % 128) + 128) % 128);
    a.xq_off = a.xs_off + 8 * a.xs_row;
    a.own_rows = (int)cdiv(a.rpc, C);
    a.orp = (int)align_up((size_t)a.own_rows, 4);
    if (a.orp % 8 == 0) a.orp += 4; // token rows of a block land 8 banks apart
    a.blk_bytes = (uint32_t)(nmat * 8 * a.orp * 4);
    const size_t part_bytes = (size_t)C * a.blk_bytes;
    const size_t after_xq = align_up((size_t)a.xq_off + 8 * (size_t)a.xq_stride, 128);
    if (single_tile && part_bytes <= (size_t)nmat * a.w_mat_bytes) {
        a.part_off = DC_HDR; // one token tile: the weights are dead once the contraction is done
        a.recv_off = (uint32_t)after_xq;
    } else {
        a.part_off = (uint32_t)after_xq;
        a.recv_off = (uint32_t)(after_xq + align_up(part_bytes, 128));
    }
    smem = (size_t)a.recv_off + part_bytes + 128;
    return smem <= kSmemLimit;
}

// Row groups per warp for a layout (template argument of the kernel).
int dc_rgw(const DcArgs &a, int nmat)
{
    const int64_t per_warp = cdiv(nmat * cdiv(a.rpc, 16), 8);
    return per_warp <= 4 ? (int)per_warp : per_warp <= 6 ? 6 : 8;
}

template <int NMAT, bool XF32, int RGW>
cudaError_t dc_kernel_setup(int dev, int C, size_t smem, int *max_clusters)
{
    static std::atomic<int> done[kMaxDevices];
    auto kern = k_decode_cluster<NMAT, XF32, RGW>;
    cudaError_t e = ensure_smem(kern, smem, done, dev);
    if (e != cudaSuccess || !max_clusters) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C * 64);
    cfg.blockDim = dim3(DC_THREADS);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaOccupancyMaxActiveClusters(max_clusters, kern, &cfg);
}

template <int NMAT, bool XF32>
cudaError_t dc_setup_rgw(int rgw, int dev, int C, size_t smem, int *max_clusters)
{
    switch (rgw) {
    case 1: return dc_kernel_setup<NMAT, XF32, 1>(dev, C, smem, max_clusters);
    case 2: return dc_kernel_setup<NMAT, XF32, 2>(dev, C, smem, max_clusters);
    case 3: return dc_kernel_setup<NMAT, XF32, 3>(dev, C, smem, max_clusters);
    case 4: return dc_kernel_setup<NMAT, XF32, 4>(dev, C, smem, max_clusters);
    case 6: return dc_kernel_setup<NMAT, XF32, 6>(dev, C, smem, max_clusters);
    default: return dc_kernel_setup<NMAT, XF32, 8>(dev, C, smem, max_clusters);
    }
}

cudaError_t dc_setup(int nmat, bool xf32, int rgw, int dev, int C, size_t smem, int *max_clusters)
{
    if (nmat == 1)
        return xf32 ? dc_setup_rgw<1, true>(rgw, dev, C, smem, max_clusters)
                    : dc_setup_rgw<1, false>(rgw, dev, C, smem, max_clusters);
    return xf32 ? dc_setup_rgw<2, true>(rgw, dev, C, smem, max_clusters)
                : dc_setup_rgw<2, false>(rgw, dev, C, smem, max_clusters);
}

// Cluster size C = 8 (K split 8 ways) when K has at least 8 k-steps of 64;
// rows per cluster sized so that one wave of resident clusters covers N.
DcCfg dc_config(int64_t N, int64_t K, int nmat, bool xf32, bool single_tile, int dev, int sms)
{
    struct Entry {
        int64_t N, K;
        int nmat, xf32, single, dev;
        DcCfg cfg;
    };
    static std::mutex mu;
    static Entry cache[64];
    static int ncache = 0;
    {
        std::lock_guard<std::mutex> lk(mu);
        for (int i = 0; i < ncache; ++i)
            if (cache[i].N == N && cache[i].K == K && cache[i].nmat == nmat && cache[i].xf32 == (int)xf32 &&
                cache[i].single == (int)single_tile && cache[i].dev == dev)
                return cache[i].cfg;
    }
    DcCfg c = {};
    const int KS = (int)(K / 64);
    const int C = std::min(8, KS);
    int nc = std::max(1, sms / C);
    size_t smem = 0;
    for (int iter = 0; iter < 4; ++iter) {
        int rpc = (int)align_up((size_t)cdiv(N, nc), 8);
        while (!dc_layout(c.a, smem, K, nmat, xf32, C, rpc, single_tile)) {
            if (rpc <= 8 || cdiv(K / 64, C) > 16) return c; // not supported: caller falls back
            rpc = (int)align_up((size_t)(rpc / 2), 8);
        }
        int resident = 0;
        c.rgw = dc_rgw(c.a, nmat);
        if (dc_setup(nmat, xf32, c.rgw, dev, C, smem, &resident) != cudaSuccess || resident < 1) return c;
        const int want = (int)cdiv(N, c.a.rpc);
        if (want <= resident || iter == 3) {
            c.nc = want;
            break;
        }
        nc = resident; // fewer clusters fit: give each more rows and re-check
    }
    c.smem = smem;
    c.ok = true;
    std::lock_guard<std::mutex> lk(mu);
    if (ncache < 64) cache[ncache++] = {N, K, nmat, (int)xf32, (int)single_tile, dev, c};
    return c;
}

template <int NMAT, bool XF32, int RGW>
cudaError_t dc_launch_t(const DcCfg &c, const DcArgs &a, cudaStream_t stream)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(c.nc * a.C));
    cfg.blockDim = dim3(DC_THREADS);
    cfg.dynamicSmemBytes = c.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = a.C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaLaunchKernelEx(&cfg, k_decode_cluster<NMAT, XF32, RGW>, a);
}

template <int NMAT, bool XF32>
cudaError_t dc_launch(const DcCfg &c, const DcArgs &a, cudaStream_t stream)
{
    switch (c.rgw) {
    case 1: return dc_launch_t<NMAT, XF32, 1>(c, a, stream);
    case 2: return dc_launch_t<NMAT, XF32, 2>(c, a, stream);
    case 3: return dc_launch_t<NMAT, XF32, 3>(c, a, stream);
    case 4: return dc_launch_t<NMAT, XF32, 4>(c, a, stream);
    case 6: return dc_launch_t<NMAT, XF32, 6>(c, a, stream);
    default: return dc_launch_t<NMAT, XF32, 8>(c, a, stream);
    }
}

// Input and output options of the BitLinear entry points (the plain entry
// points use the defaults): x_amax = given per-token maxima of x; y_bf16 =
// store y as bf16; y_amax = emit the per-token maxima of y.
struct IoOpts {
    const float *x_amax = nullptr;
    bool y_bf16 = false;
    float *y_amax = nullptr;
};

bitnet_status_t dc_forward(const DcCfg &c, const void *x, bool xf32, int64_t M, int64_t K, const uint8_t *w0,
                           const float *gamma0, const uint8_t *w1, const float *gamma1, int64_t N, void *y,
                           int8_t *x_q_out, float *s_out, int32_t *acc0, int32_t *acc1, cudaStream_t stream,
                           int nmat, const IoOpts &io)
{
    DcArgs a = c.a;
    a.x = x;
    a.x_amax = io.x_amax;
    a.gamma0 = gamma0;
    a.gamma1 = gamma1;
    a.y = y;
    a.y_bf16 = io.y_bf16 ? 1 : 0;
    a.y_amax = io.y_amax;
    a.acc0 = acc0;
    a.acc1 = acc1;
    a.xq_out = x_q_out;
    a.s_out = s_out;
    a.M = (int)M;
    a.N = (int)N;
    a.K = (int)K;
    a.w0 = w0;
    a.w1 = w1;
    cudaError_t e = cudaSuccess;
    // the maxima are folded in with atomicMax by every cluster: zero them first
    if (io.y_amax) e = launch_pdl(k_zero_f32, dim3(1), dim3(128), 0, stream, io.y_amax, (int)M);
    if (e != cudaSuccess) return cuda_status(e);
    if (nmat == 1)
        e = xf32 ? dc_launch<1, true>(c, a, stream) : dc_launch<1, false>(c, a, stream);
    else
        e = xf32 ? dc_launch<2, true>(c, a, stream) : dc_launch<2, false>(c, a, stream);
    return cuda_status(e);
}

// Shared body of the BitLinear entry points (nmat = 1: BitLinear, 2: gated
// FFN gate/up).  norm_g (optional): RMS-normalise x with weight norm_g and
// epsilon norm_eps before quantising it.  io: given maxima of x, bf16 output,
// emitted maxima of y.
bitnet_status_t forward(const void *x, bitnet_dtype_t x_dtype, int64_t M, int64_t K, const uint8_t *w0,
                        const float *gamma0, const uint8_t *w1, const float *gamma1, int64_t N, void *y,
                        int8_t *x_q_out, float *s_out, int32_t *acc0, int32_t *acc1, void *workspace,
                        size_t ws_bytes, cudaStream_t stream, int nmat, const float *norm_g = nullptr,
                        float norm_eps = 0.0f, const IoOpts &io = IoOpts())
{
    bitnet_status_t st = check_shape(M, N, K);
    if (st != BITNET_OK) return st;
    if (x_dtype != BITNET_DTYPE_BF16 && x_dtype != BITNET_DTYPE_F32) return BITNET_ERR_INVALID_ARG;
    if (!x || !w0 || !gamma0 || !y || (nmat == 2 && (!w1 || !gamma1))) return BITNET_ERR_INVALID_ARG;
    if (norm_g && (K > kNormMaxK || !(norm_eps >= 0.0f) || !std::isfinite(norm_eps)))
        return norm_g && K > kNormMaxK ? BITNET_ERR_UNSUPPORTED_SHAPE : BITNET_ERR_INVALID_ARG;
    // the maxima of the raw input are not those of its normalised form; the
    // given and the emitted maxima must not share memory (one is read while
    // the other is zeroed and folded)
    if (io.x_amax && norm_g) return BITNET_ERR_INVALID_ARG;
    if (io.x_amax && io.y_amax) {
        const uintptr_t a0 = reinterpret_cast<uintptr_t>(io.x_amax), b0 = reinterpret_cast<uintptr_t>(io.y_amax);
        const uintptr_t bytes = (uintptr_t)M * 4;
        if (a0 < b0 + bytes && b0 < a0 + bytes) return BITNET_ERR_INVALID_ARG;
    }
    const void *ptrs[] = {x, w0, gamma0, w1, gamma1, y, x_q_out, s_out, acc0, acc1, workspace, norm_g,
                          io.x_amax, io.y_amax};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return BITNET_ERR_MISALIGNED;
    if (!workspace || ws_bytes < ws_bytes_for(M, K)) return BITNET_ERR_WORKSPACE;
    const int dev = current_device();
    const int sms = num_sms_for(dev);
    if (sms <= 0) return BITNET_ERR_CUDA;
    const bool xf32 = x_dtype == BITNET_DTYPE_F32;
    const int dispatch = g_dispatch.load();
    Workspace ws = carve(workspace, M, K);
    int8_t *xq = x_q_out ? x_q_out : ws.xq;
    float *s = s_out ? s_out : ws.s;

    // the normalising quantiser runs as its own kernel ahead of the GEMM
    // and zeroes the emitted maxima for the contraction kernel's epilogue
    auto quantise = [&](int8_t *q, float *sc, int32_t *rs) {
        return norm_g ? launch_norm_quant(x, xf32, M, K, norm_g, norm_eps, q, sc, rs, stream, io.y_amax)
                      : launch_quant(x, xf32, M, K, q, sc, rs, stream, io.x_amax, io.y_amax);
    };
    if (M <= kDecodeMaxM && dispatch != BITNET_DISPATCH_PREFILL) {
        // cluster kernel with the quantiser fused in (automatic choice for decode)
        if (dispatch != BITNET_DISPATCH_DECODE && !norm_g) {
            const DcCfg c = dc_config(N, K, nmat, xf32, M <= 8, dev, sms);
            if (c.ok)
                return dc_forward(c, x, xf32, M, K, w0, gamma0, w1, gamma1, N, y, x_q_out, s_out, acc0, acc1,
                                  stream, nmat, io);
            if (dispatch == BITNET_DISPATCH_DECODE_FUSED) return BITNET_ERR_UNSUPPORTED_SHAPE;
        }
        if (norm_g && dispatch == BITNET_DISPATCH_DECODE_FUSED) return BITNET_ERR_UNSUPPORTED_SHAPE;
        // quantiser kernel, then the row-split decode kernel
        const DecodeCfg c = decode_config(N, K, nmat, sms);
        if (c.ok) {
            DecodeArgs a = {};
            a.xq = xq;
            a.s_in = s;
            a.rs_in = ws.rs;
            a.w0 = w0;
            a.w1 = w1;
            a.gamma0 = gamma0;
            a.gamma1 = gamma1;
            a.y = y;
            a.y_bf16 = io.y_bf16 ? 1 : 0;
            a.y_amax = io.y_amax;
            a.acc0 = acc0;
            a.acc1 = acc1;
            a.M = (int)M;
            a.N = (int)N;
            a.K = (int)K;
            a.grid = c.grid;
            a.rg = c.rg;
            a.w_stride = c.w_stride;
            a.rp = c.rp;
            cudaError_t e = quantise(xq, s, ws.rs);
            if (e == cudaSuccess)
                e = nmat == 1 ? launch_decode<1>(a, c, stream, dev) : launch_decode<2>(a, c, stream, dev);
            return cuda_status(e);
        }
        if (dispatch != BITNET_DISPATCH_AUTO) return BITNET_ERR_UNSUPPORTED_SHAPE;
    } else if (M > kDecodeMaxM && (dispatch == BITNET_DISPATCH_DECODE || dispatch == BITNET_DISPATCH_DECODE_FUSED)) {
        return BITNET_ERR_UNSUPPORTED_SHAPE;
    }

    // ---- prefill: quantiser kernel, then the tcgen05 GEMM ----
    PrefillArgs a = {};
    a.M = (int)M;
    a.N = (int)N;
    a.K = (int)K;
    a.num_m = (int)cdiv(M, PF_BM);
    a.num_n = (int)cdiv(N, nmat == 1 ? PF_BN : PF_BN / 2);
    a.num_k = (int)cdiv(K, PF_BK);
    a.num_tiles = a.num_m * a.num_n;
    a.gamma0 = gamma0;
    a.gamma1 = gamma1;
    a.s = s;
    a.y = y;
    a.y_bf16 = io.y_bf16 ? 1 : 0;
    a.y_amax = io.y_amax;
    a.acc0 = acc0;
    a.acc1 = acc1;
    a.vec_ok = (N % (io.y_bf16 ? 8 : 4)) == 0; // 16-byte rows
    CUtensorMap tmA, tmB0, tmB1, tmY;
    const uint32_t brows = nmat == 1 ? PF_BN : PF_BN / 2;
    if (!encode_u8_2d(&tmA, xq, (uint64_t)M, (uint64_t)K, PF_BM, PF_BK, true) ||
        !encode_u8_2d(&tmB0, w0, (uint64_t)N, (uint64_t)(K / 4), brows, PF_BK / 4, false))
        return BITNET_ERR_CUDA;
    if (nmat == 2) {
        if (!encode_u8_2d(&tmB1, w1, (uint64_t)N, (uint64_t)(K / 4), brows, PF_BK / 4, false))
            return BITNET_ERR_CUDA;
    } else {
        tmB1 = tmB0;
    }
    // the last, partly filled wave of a BitLinear as sub-tiles (tmB1: a box of their rows)
    const int grid = std::min(a.num_tiles, sms);
    a.tail_q = pf_tail_q(M, N, nmat, sms);
    a.full_units = a.num_tiles;
    a.num_units = a.num_tiles;
    if (a.tail_q > 1) {
        a.full_units = a.num_tiles / grid * grid;
        a.num_units = a.full_units + (a.num_tiles - a.full_units) * a.tail_q;
        if (!encode_u8_2d(&tmB1, w0, (uint64_t)N, (uint64_t)(K / 4), (uint32_t)(PF_BN / a.tail_q), PF_BK / 4, false))
            return BITNET_ERR_CUDA;
    }
    // output through TMA stores when rows are 16-byte multiples: 32 x 32 boxes,
    // 128-byte swizzle for fp32, 64-byte swizzle for bf16
    tmY = tmA;
    if (a.vec_ok && !encode_2d_out(&tmY, y, (uint64_t)M, (uint64_t)N, 32, 32, io.y_bf16)) return BITNET_ERR_CUDA;
    cudaError_t e = quantise(xq, s, nullptr);
    if (e != cudaSuccess) return BITNET_ERR_CUDA;
    if (nmat == 1) {
        static std::atomic<int> done[kMaxDevices];
        e = ensure_smem(k_prefill<false>, PF_SMEM, done, dev);
        if (e == cudaSuccess)
            e = launch_pdl(k_prefill<false>, dim3(grid), dim3(PF_THREADS), PF_SMEM, stream, tmA, tmB0, tmB1, tmY, a);
    } else {
        static std::atomic<int> done[kMaxDevices];
        e = ensure_smem(k_prefill<true>, PF_SMEM, done, dev);
        if (e == cudaSuccess)
            e = launch_pdl(k_prefill<true>, dim3(grid), dim3(PF_THREADS), PF_SMEM, stream, tmA, tmB0, tmB1, tmY, a);
    }
    return cuda_status(e);
}

// ---- decode sequences: one persistent launch for many ops -----------------
constexpr int64_t kSeqMaxK = 8192; // the exact sum of squares and the x_q fragment layout are sized for this

struct ByteRange {
    uintptr_t lo, hi;
};
inline bool overlaps(ByteRange a, ByteRange b) { return a.lo < b.hi && b.lo < a.hi; }
inline ByteRange range_of(const void *p, size_t bytes)
{
    const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
    return {lo, lo + bytes};
}

// Validation (host only, shared by plan, schedule, tasks and run); fills the
// byte ranges each op reads (x) and writes (y).  extra: one more range no op may
// write or read (the workspace), may be empty.
bitnet_status_t seq_validate(const bitnet_op_t *ops, int n, int64_t M, ByteRange extra, std::vector<ByteRange> &xr,
                             std::vector<ByteRange> &yr)
{
    if (!ops || n < 1 || n > BITNET_SEQ_MAX_OPS || M < 1) return BITNET_ERR_INVALID_ARG;
    if (M > BITNET_SEQ_MAX_M) return BITNET_ERR_UNSUPPORTED_SHAPE;
    xr.assign(n, ByteRange{0, 0});
    yr.assign(n, ByteRange{0, 0});
    std::vector<ByteRange> ro; // weights, gammas and norm weights (read-only for the launch)
    ro.reserve(5 * (size_t)n);
    for (int i = 0; i < n; ++i) {
        const bitnet_op_t &o = ops[i];
        if (o.kind != BITNET_OP_LINEAR && o.kind != BITNET_OP_FFN_GATE_UP) return BITNET_ERR_INVALID_ARG;
        if (o.x_dtype != BITNET_DTYPE_BF16 && o.x_dtype != BITNET_DTYPE_F32) return BITNET_ERR_INVALID_ARG;
        const bool ffn = o.kind == BITNET_OP_FFN_GATE_UP;
        if (!o.x || !o.w0 || !o.gamma0 || !o.y || (ffn && (!o.w1 || !o.gamma1))) return BITNET_ERR_INVALID_ARG;
        if (o.norm_g && !(o.norm_eps >= 0.0f && std::isfinite(o.norm_eps))) return BITNET_ERR_INVALID_ARG;
        const bitnet_status_t st = check_shape(M, o.N, o.K);
        if (st != BITNET_OK) return st;
        if (o.K > kSeqMaxK || o.N > 32767 * 64) return BITNET_ERR_UNSUPPORTED_SHAPE;
        const void *ptrs[] = {o.x, o.w0, o.gamma0, ffn ? o.w1 : nullptr, ffn ? o.gamma1 : nullptr, o.y, o.norm_g};
        for (const void *q : ptrs)
            if (q && !aligned16(q)) return BITNET_ERR_MISALIGNED;
        xr[i] = range_of(o.x, (size_t)M * (size_t)o.K * (o.x_dtype == BITNET_DTYPE_F32 ? 4 : 2));
        yr[i] = range_of(o.y, (size_t)M * (size_t)o.N * 4);
        if (overlaps(xr[i], yr[i])) return BITNET_ERR_INVALID_ARG;
        const size_t wbytes = (size_t)o.N * (size_t)(o.K / 4);
        ro.push_back(range_of(o.w0, wbytes));
        ro.push_back(range_of(o.gamma0, 4));
        if (ffn) {
            ro.push_back(range_of(o.w1, wbytes));
            ro.push_back(range_of(o.gamma1, 4));
        }
        if (o.norm_g) ro.push_back(range_of(o.norm_g, (size_t)o.K * 4));
    }
    for (int j = 0; j < n; ++j) {
        for (const ByteRange &w : ro)
            if (overlaps(yr[j], w)) return BITNET_ERR_INVALID_ARG;
        if (extra.hi > extra.lo && (overlaps(yr[j], extra) || overlaps(xr[j], extra))) return BITNET_ERR_INVALID_ARG;
    }
    if (extra.hi > extra.lo)
        for (const ByteRange &w : ro)
            if (overlaps(w, extra)) return BITNET_ERR_INVALID_ARG;
    return BITNET_OK;
}

// Op i must precede op j (i before j in the list): one writes what the other reads or writes.
inline bool hazard(const std::vector<ByteRange> &xr, const std::vector<ByteRange> &yr, int i, int j)
{
    return overlaps(yr[i], xr[j]) || overlaps(yr[i], yr[j]) || overlaps(xr[i], yr[j]);
}

// Hazard waits of the ops in list order (see bitnet_sequence_plan).
bitnet_status_t seq_plan(const bitnet_op_t *ops, int n, int64_t M, int32_t *wait_x, int32_t *wait_y,
                         ByteRange extra)
{
    std::vector<ByteRange> xr, yr;
    const bitnet_status_t st = seq_validate(ops, n, M, extra, xr, yr);
    if (st != BITNET_OK) return st;
    for (int j = 0; j < n; ++j) {
        int wx = -1, wy = -1;
        for (int i = 0; i < j; ++i) {
            if (overlaps(yr[i], xr[j])) wx = i;
            if (overlaps(yr[i], yr[j]) || overlaps(xr[i], yr[j])) wy = i;
        }
        if (wait_x) wait_x[j] = wx;
        if (wait_y) wait_y[j] = wy;
    }
    return BITNET_OK;
}

// Execution order (see bitnet_sequence_schedule): a topological order of the
// hazard graph, so every op reads and leaves exactly what it would in list
// order.  Greedy, in list order, except that an op reading the output of the
// op scheduled just before it is deferred while another op is ready.
bitnet_status_t seq_schedule(const bitnet_op_t *ops, int n, int64_t M, int32_t *order, ByteRange extra)
{
    std::vector<ByteRange> xr, yr;
    const bitnet_status_t st = seq_validate(ops, n, M, extra, xr, yr);
    if (st != BITNET_OK) return st;
    std::vector<int> pending(n, 0);              // unscheduled predecessors
    std::vector<unsigned char> hz((size_t)n * n); // hz[i * n + j]: i must precede j
    for (int j = 0; j < n; ++j)
        for (int i = 0; i < j; ++i)
            if (hazard(xr, yr, i, j)) {
                hz[(size_t)i * n + j] = 1;
                ++pending[j];
            }
    std::vector<unsigned char> done(n, 0);
    int last = -1;
    for (int k = 0; k < n; ++k) {
        int pick = -1, first = -1;
        for (int j = 0; j < n && pick < 0; ++j) {
            if (done[j] || pending[j] != 0) continue;
            if (first < 0) first = j;
            if (last < 0 || !overlaps(yr[last], xr[j])) pick = j;
        }
        if (pick < 0) pick = first;
        order[k] = pick;
        done[pick] = 1;
        last = pick;
        for (int j = pick + 1; j < n; ++j)
            if (hz[(size_t)pick * n + j]) --pending[j];
    }
    return BITNET_OK;
}

inline int seq_mp(int64_t M) { return M <= 8 ? 8 : M <= 16 ? 16 : M <= 32 ? 32 : 64; }
// Row groups per compute warp: two at one token tile (each activation fragment feeds two
// weight fragments, halving the activation loads from shared memory), else one.
// quantisation tasks of an op: one per token for M <= 8 (on all compute warps),
// else one per 8 tokens (a compute warp per token)
inline int seq_qtasks(int64_t M) { return (int)(M <= 8 ? M : (M + 7) / 8); }
inline int seq_rg(int64_t M) { return M <= 8 ? 2 : 1; }
inline int seq_rtasks(const bitnet_op_t &o, int64_t M)
{
    const int64_t rows_per_task = (o.kind == BITNET_OP_FFN_GATE_UP ? DT_ROWS / 2 : DT_ROWS) * seq_rg(M);
    return (int)cdiv(o.N, rows_per_task);
}

// Task groups of a sequence (ops in execution order): group 2j = the quant
// tasks of op j (one per token), group 2j + 1 = its row tasks.  Dependencies
// between groups (must complete first):
//   rows(j)  <- quant(j)                                  (always; implicit)
//   quant(j) <- rows(i),  i < j, y_i overlaps x_j         (read after write)
//   rows(j)  <- quant(i), i < j, x_i overlaps y_j         (write after read: quant(i) is x_i's only reader)
//   rows(j)  <- rows(i),  i < j, y_i overlaps y_j         (write after write)
// reduced to the edges not implied by others.  [0, 2n) is a topological order.
struct SeqGroups {
    std::vector<std::vector<int>> preds; // reduced predecessors of every group
};

bitnet_status_t seq_groups(const bitnet_op_t *ops, int n, int64_t M, ByteRange extra, SeqGroups &G)
{
    std::vector<ByteRange> xr, yr;
    const bitnet_status_t st = seq_validate(ops, n, M, extra, xr, yr);
    if (st != BITNET_OK) return st;
    const int ng = 2 * n, words = (ng + 63) / 64;
    std::vector<std::vector<int>> full(ng);
    for (int j = 0; j < n; ++j) {
        full[2 * j + 1].push_back(2 * j);
        for (int i = 0; i < j; ++i) {
            if (overlaps(yr[i], xr[j])) full[2 * j].push_back(2 * i + 1);
            if (overlaps(xr[i], yr[j])) full[2 * j + 1].push_back(2 * i);
            if (overlaps(yr[i], yr[j])) full[2 * j + 1].push_back(2 * i + 1);
        }
    }
    std::vector<uint64_t> anc((size_t)ng * words, 0ull); // ancestors of each group (bitset)
    G.preds.assign(ng, {});
    for (int v = 0; v < ng; ++v) {
        uint64_t *av = &anc[(size_t)v * words];
        for (int u : full[v]) {
            const uint64_t *au = &anc[(size_t)u * words];
            for (int w = 0; w < words; ++w) av[w] |= au[w];
        }
        for (int u : full[v]) { // u is implied if another predecessor already has it as an ancestor
            bool implied = false;
            for (int u2 : full[v])
                if (u2 != u && ((anc[(size_t)u2 * words + u / 64] >> (u % 64)) & 1ull)) implied = true;
            if (!implied) G.preds[v].push_back(u);
        }
        for (int u : full[v]) av[u / 64] |= 1ull << (u % 64);
    }
    return BITNET_OK;
}

// Order of the task groups in the launch's global task list.  A list-scheduling
// simulation on `ctas` CTAs: at the time the first CTA frees up, among the
// groups whose predecessors are placed and finished by then, take the one with
// the longest chain of work after it (its own duration plus the longest chain
// of its successors), ties in execution order; if none is ready, the one whose
// predecessors finish first.  Its tasks go to the CTAs that free up first.
// Durations are estimates (a quant task 1.5 us for one token, 3 us for 8; a row
// task its packed weights at ~28 GB/s per SM, the rate a CTA sustains in a full
// step; a dependent group is ready kSeqHandOver after its predecessors finish:
// completion fence, counter, the consumer's poll and copies).  Chains such as gate/up -> down
// therefore start early and short independent work is left for the end, where
// it fills the CTAs instead of a few long tasks running on a mostly idle GPU.
// CTAs claim tasks in this order; every dependency points to an earlier group.
constexpr double kSeqHandOver = 3.0; // us

std::vector<int> seq_group_order(const bitnet_op_t *ops, int n, int64_t M, const SeqGroups &G, int ctas)
{
    const int ng = 2 * n;
    const int nc = std::max(1, ctas);
    std::vector<double> finish(ng, 0.0), dur(ng, 0.0), chain(ng, 0.0);
    std::vector<int> count(ng, 0), left(ng, 0), order;
    for (int j = 0; j < n; ++j) {
        count[2 * j] = seq_qtasks(M);
        dur[2 * j] = M <= 8 ? 1.5 : 3.0;
        count[2 * j + 1] = seq_rtasks(ops[j], M);
        dur[2 * j + 1] = (double)(DT_ROWS * seq_rg(M)) * (double)(ops[j].K / 4) / 28e3;
    }
    std::vector<std::vector<int>> succ(ng);
    for (int v = 0; v < ng; ++v) {
        left[v] = (int)G.preds[v].size();
        for (int u : G.preds[v]) succ[u].push_back(v);
    }
    // successors are later groups (dependencies point to earlier ops, or from an op's
    // rows to its own quant tasks), so one backward pass computes every chain
    for (int v = ng - 1; v >= 0; --v) {
        double after = 0.0;
        for (int w : succ[v]) after = std::max(after, chain[w]);
        chain[v] = dur[v] * (double)((count[v] + nc - 1) / nc) + after;
    }
    std::priority_queue<double, std::vector<double>, std::greater<double>> free_at;
    for (int c = 0; c < nc; ++c) free_at.push(0.0);
    std::vector<char> placed(ng, 0);
    for (int k = 0; k < ng; ++k) {
        const double now = free_at.top();
        int pick = -1, first = -1;
        double best_chain = -1.0, first_ready = 0.0, pick_ready = 0.0;
        for (int v = 0; v < ng; ++v) {
            if (placed[v] || left[v] != 0) continue;
            double ready = 0.0;
            for (int u : G.preds[v]) ready = std::max(ready, finish[u] + kSeqHandOver);
            if (first < 0 || ready < first_ready) {
                first = v;
                first_ready = ready;
            }
            if (ready <= now && chain[v] > best_chain) {
                pick = v;
                best_chain = chain[v];
                pick_ready = ready;
            }
        }
        if (pick < 0) {
            pick = first;
            pick_ready = first_ready;
        }
        placed[pick] = 1;
        order.push_back(pick);
        double fin = pick_ready;
        for (int t = 0; t < count[pick]; ++t) {
            const double f = free_at.top();
            free_at.pop();
            const double end = std::max(f, pick_ready) + dur[pick];
            free_at.push(end);
            fin = std::max(fin, end);
        }
        finish[pick] = fin;
        for (int v : succ[pick]) --left[v];
    }
    return order;
}

// Workspace: counters (per op: quant tasks done, row tasks done), the ops'
// weight tensor maps [n][2] x 128 bytes, then per op x_q [K/64][Mp][64],
// s [Mp], row sums [Mp].
inline size_t seq_counter_bytes(int n) { return align_up(4 * (size_t)(DT_CNT_OPS + 2 * n), 256); }
inline size_t seq_map_bytes(int n) { return align_up((size_t)n * 2 * sizeof(CUtensorMap) + 128, 256); } // + alignment
inline size_t seq_op_ws_bytes(int64_t K, int Mp) { return align_up((size_t)K * Mp, 256) + 512; }

std::atomic<int> g_seq_stall{-1};                        // tests: op (list index) whose rows never become ready
std::atomic<unsigned long long> g_wait_limit_set{kDefaultWaitLimitNs};

// Build the launch program for ops in execution order (user_index: list index
// of each).  ws: workspace (counters zero before the first launch).  stall:
// list index of the test stall's op, or -2 to read the test setting.
bitnet_status_t seq_build(DtProgram &p, const bitnet_op_t *ops, const int32_t *user_index, int n, int64_t M, int ctas,
                          void *ws, size_t ws_bytes, ByteRange extra, std::vector<int> *order_out = nullptr,
                          int stall = -2)
{
    SeqGroups G;
    bitnet_status_t st = seq_groups(ops, n, M, extra, G);
    if (st != BITNET_OK) return st;
    const int Mp = seq_mp(M);
    size_t need = seq_counter_bytes(n) + seq_map_bytes(n);
    for (int j = 0; j < n; ++j) need += seq_op_ws_bytes(ops[j].K, Mp);
    if (ws && ws_bytes < need) return BITNET_ERR_WORKSPACE;
    p.n_ops = n;
    p.M = (int)M;
    p.Mp = Mp;
    p.counters = static_cast<unsigned *>(ws);
    char *base = static_cast<char *>(ws);
    // tensor maps want 128-byte alignment; the workspace is only required to be 16-byte aligned
    p.wmaps = base ? reinterpret_cast<CUtensorMap *>(align_up(reinterpret_cast<uintptr_t>(base) + seq_counter_bytes(n),
                                                              (uintptr_t)128))
                   : nullptr;
    size_t off = seq_counter_bytes(n) + seq_map_bytes(n);
    if (stall == -2) stall = g_seq_stall.load();
    for (int j = 0; j < n; ++j) {
        const bitnet_op_t &o = ops[j];
        DtOp &d = p.ops[j];
        d = DtOp{};
        d.x = o.x;
        d.w0 = o.w0;
        d.w1 = o.kind == BITNET_OP_FFN_GATE_UP ? o.w1 : nullptr;
        d.gamma0 = o.gamma0;
        d.gamma1 = o.kind == BITNET_OP_FFN_GATE_UP ? o.gamma1 : nullptr;
        d.norm_g = o.norm_g;
        d.norm_eps = o.norm_eps;
        d.y = o.y;
        d.K = (int)o.K;
        d.N = (int)o.N;
        d.nmat = o.kind == BITNET_OP_FFN_GATE_UP ? 2 : 1;
        d.xf32 = o.x_dtype == BITNET_DTYPE_F32;
        d.rtasks = seq_rtasks(o, M);
        d.stall = (stall >= 0 && user_index && user_index[j] == stall) ? 1 : 0;
        if (base) {
            d.xq = reinterpret_cast<int8_t *>(base + off);
            d.s = reinterpret_cast<float *>(base + off + align_up((size_t)o.K * Mp, 256));
            d.rs = reinterpret_cast<int32_t *>(base + off + align_up((size_t)o.K * Mp, 256) + 256);
        }
        off += seq_op_ws_bytes(o.K, Mp);
        const std::vector<int> &qp = G.preds[2 * j], &rp = G.preds[2 * j + 1];
        int nd = 0;
        for (int u : qp) { // quant(j) waits only on row groups
            if (nd >= DT_MAX_DEPS) return BITNET_ERR_UNSUPPORTED_SHAPE;
            d.deps[nd++] = (uint16_t)(u / 2);
        }
        d.nq = nd;
        for (int u : rp) {
            if (u == 2 * j) continue; // the op's own quant tasks: always waited for
            if (nd >= DT_MAX_DEPS) return BITNET_ERR_UNSUPPORTED_SHAPE;
            d.deps[nd++] = (uint16_t)((u / 2) | ((u % 2 == 0) ? DT_DEP_QUANT : 0));
        }
        d.nr = nd - d.nq;
    }
    const std::vector<int> order = seq_group_order(ops, n, M, G, ctas);
    int t = 0, ns = 0;
    for (int v : order) {
        const int j = v / 2;
        const bool quant = v % 2 == 0;
        const int cnt = quant ? seq_qtasks(M) : p.ops[j].rtasks;
        if (ns >= DT_MAX_SEGS) return BITNET_ERR_UNSUPPORTED_SHAPE;
        p.segs[ns].start = t;
        p.segs[ns].op = (uint16_t)j;
        p.segs[ns].first = (uint16_t)(quant ? 0x8000u : 0u);
        ++ns;
        t += cnt;
    }
    p.n_segs = ns;
    p.n_tasks = t;
    p.slot_bytes = seq_rg(M) * DT_WBYTES + DT_KC * Mp;
    p.n_slots = (int)std::min<size_t>(DT_MAX_SLOTS, (kSmemLimit - 1024 - DT_HDR) / (size_t)p.slot_bytes);
    if (order_out) *order_out = order;
    return BITNET_OK;
}

static_assert(sizeof(DtProgram) <= 32000, "kernel parameter space");
static_assert(DT_MAX_OPS >= BITNET_SEQ_MAX_OPS && 2 * DT_MAX_OPS <= DT_MAX_SEGS, "sequence limits");
static_assert(DT_MAX_M >= BITNET_SEQ_MAX_M, "sequence token limit");

template <int TT, int RG>
cudaError_t seq_launch_t(const DtProgram &p, int ctas, cudaStream_t stream, int dev)
{
    static std::atomic<int> smem_done[kMaxDevices];
    cudaError_t e = ensure_smem(k_decode_tasks<TT, RG>, kSmemLimit, smem_done, dev);
    if (e != cudaSuccess) return e;
    const size_t smem = 1024 + DT_HDR + (size_t)p.n_slots * p.slot_bytes; // + alignment to 1024 bytes
    // the weights' tensor maps (after everything before it on the stream: a previous
    // sequence on this workspace may still read the old ones), then the sequence as its
    // programmatic dependent: everything but the weight producer starts while the maps
    // are written
    g_launches.fetch_add(1, std::memory_order_relaxed);
    k_decode_maps<<<p.n_ops, 32, 0, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_pdl(k_decode_tasks<TT, RG>, dim3(ctas), dim3(DT_THREADS), smem, stream, p);
}

cudaError_t seq_launch(const DtProgram &p, int ctas, cudaStream_t stream, int dev)
{
    switch (p.Mp) { // row groups per warp as seq_rg
    case 8: return seq_launch_t<1, 2>(p, ctas, stream, dev);
    case 16: return seq_launch_t<2, 1>(p, ctas, stream, dev);
    case 32: return seq_launch_t<4, 1>(p, ctas, stream, dev);
    default: return seq_launch_t<8, 1>(p, ctas, stream, dev);
    }
}

// Plans of recent sequence calls.  A decode loop calls with the same op list
// every step; planning a 120-op layer stack takes on the order of a
// millisecond of host time, the launch itself microseconds.
struct SeqCacheEntry {
    bool used = false;
    uint64_t stamp = 0;
    int n = 0, dev = -1, stall = -1;
    int64_t M = 0;
    const void *ws = nullptr;
    size_t ws_bytes = 0;
    bitnet_op_t ops[BITNET_SEQ_MAX_OPS];
    DtProgram prog;
};
constexpr int kSeqCacheEntries = 8;
SeqCacheEntry g_seq_cache[kSeqCacheEntries];
std::mutex g_seq_cache_mu;
uint64_t g_seq_cache_clock = 0;

bool same_op(const bitnet_op_t &a, const bitnet_op_t &b)
{
    return a.kind == b.kind && a.x_dtype == b.x_dtype && a.x == b.x && a.K == b.K && a.N == b.N && a.w0 == b.w0 &&
           a.gamma0 == b.gamma0 && a.w1 == b.w1 && a.gamma1 == b.gamma1 && a.y == b.y && a.norm_g == b.norm_g &&
           (a.norm_g == nullptr || a.norm_eps == b.norm_eps);
}

bool seq_cache_match(const SeqCacheEntry &e, const bitnet_op_t *ops, int n, int64_t M, int dev, int stall,
                     const void *ws, size_t ws_bytes)
{
    if (!e.used || e.n != n || e.M != M || e.dev != dev || e.stall != stall || e.ws != ws || e.ws_bytes != ws_bytes)
        return false;
    for (int i = 0; i < n; ++i)
        if (!same_op(e.ops[i], ops[i])) return false;
    return true;
}

int seq_ctas(int dev) { return num_sms_for(dev); } // one CTA per SM (227 KB of shared memory each)

// One launch of at most BITNET_SEQ_MAX_OPS ops.  whole: the byte range no op may
// touch (the caller's whole workspace), or null for this part's own; base: the
// list index of ops[0] in the caller's list (the test stall names a list index).
bitnet_status_t decode_sequence(const bitnet_op_t *ops, int n, int64_t M, void *workspace, size_t ws_bytes,
                                cudaStream_t stream, const ByteRange *whole = nullptr, int base = 0)
{
    if (workspace && !aligned16(workspace)) return BITNET_ERR_MISALIGNED;
    const int stall_set = g_seq_stall.load();
    const int stall = stall_set >= base && stall_set < base + n ? stall_set - base : -1;
    const int dev = current_device();
    if (ops && n >= 1 && n <= BITNET_SEQ_MAX_OPS && workspace && dev >= 0) {
        static DtProgram hit_proto;
        DtProgram p = hit_proto;
        bool hit = false;
        {
            std::lock_guard<std::mutex> lk(g_seq_cache_mu);
            for (SeqCacheEntry &e : g_seq_cache)
                if (seq_cache_match(e, ops, n, M, dev, stall, workspace, ws_bytes)) {
                    p = e.prog;
                    e.stamp = ++g_seq_cache_clock;
                    hit = true;
                    break;
                }
        }
        if (hit) return cuda_status(seq_launch(p, seq_ctas(dev), stream, dev));
    }
    const ByteRange wsr = whole ? *whole : workspace ? range_of(workspace, ws_bytes) : ByteRange{0, 0};
    int32_t order[BITNET_SEQ_MAX_OPS];
    bitnet_status_t st = seq_schedule(ops, n, M, order, wsr);
    if (st != BITNET_OK) return st;
    if (!workspace) return BITNET_ERR_WORKSPACE;
    if (dev < 0) return BITNET_ERR_CUDA;
    const int ctas = seq_ctas(dev);
    if (ctas < 1) return BITNET_ERR_CUDA;
    bitnet_op_t sched[BITNET_SEQ_MAX_OPS];
    for (int k = 0; k < n; ++k) sched[k] = ops[order[k]];
    static DtProgram prog_proto; // zero-initialised template; each call fills a copy
    DtProgram p = prog_proto;
    st = seq_build(p, sched, order, n, M, ctas, workspace, ws_bytes, wsr, nullptr, stall);
    if (st != BITNET_OK) return st;
    if (p.n_slots < 2) return BITNET_ERR_UNSUPPORTED_SHAPE;
    // the template of the weight maps (any op's first matrix: address, extent and pitch are replaced per op)
    if (!encode_u8_2d(&p.wtmpl, sched[0].w0, (uint64_t)sched[0].N, (uint64_t)(sched[0].K / 4), DT_BOX_ROWS,
                      DT_KC / 4, true))
        return BITNET_ERR_CUDA;
    {
        // remember the plan under the caller's op list (least recently used entry replaced)
        std::lock_guard<std::mutex> lk(g_seq_cache_mu);
        SeqCacheEntry *slot = &g_seq_cache[0];
        for (SeqCacheEntry &e : g_seq_cache) {
            if (!e.used) {
                slot = &e;
                break;
            }
            if (e.stamp < slot->stamp) slot = &e;
        }
        slot->used = true;
        slot->stamp = ++g_seq_cache_clock;
        slot->n = n;
        slot->M = M;
        slot->dev = dev;
        slot->stall = stall;
        slot->ws = workspace;
        slot->ws_bytes = ws_bytes;
        for (int i = 0; i < n; ++i) slot->ops[i] = ops[i];
        slot->prog = p;
    }
    return cuda_status(seq_launch(p, ctas, stream, dev));
}

// ---- fixed scratch for bitnet_linear_noalloc -------------------------------
// Callers of that entry point cannot allocate, so its scratch is a static
// device array (every GPU that loads the library holds it until exit).  Host
// code must not use the symbol as a pointer: it is a host-side stand-in, and
// the device address is looked up once per device and context below.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device (looked up on the
// first call per device and context, with that device current); nullptr on
// failure.  The context is part of the key: if the primary context is torn
// down and created again (cudaDeviceReset), the module is loaded again and
// the array may live at another address.
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

CUcontext current_context()
{
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    });
    CUcontext c = nullptr;
    if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
    return c;
}

void *noalloc_scratch(int dev)
{
    struct Entry {
        CUcontext ctx = nullptr;
        void *ptr = nullptr;
    };
    static Entry cache[kMaxDevices];
    static std::mutex mu;
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    const CUcontext ctx = current_context();
    if (!ctx) return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if (cache[dev].ptr && cache[dev].ctx == ctx) return cache[dev].ptr;
    void *q = nullptr;
    if (cudaGetSymbolAddress(&q, g_noalloc_scratch) != cudaSuccess || q == nullptr) return nullptr;
    cache[dev].ctx = ctx;
    cache[dev].ptr = q;
    return q;
}

} // namespace
} // namespace bitnet

using namespace bitnet;

extern "C" {

const char *bitnet_status_string(bitnet_status_t status)
{
    switch (status) {
    case BITNET_OK: return "BITNET_OK";
    case BITNET_ERR_INVALID_ARG: return "BITNET_ERR_INVALID_ARG";
    case BITNET_ERR_UNSUPPORTED_SHAPE: return "BITNET_ERR_UNSUPPORTED_SHAPE";
    case BITNET_ERR_MISALIGNED: return "BITNET_ERR_MISALIGNED";
    case BITNET_ERR_CUDA: return "BITNET_ERR_CUDA";
    case BITNET_ERR_TIMEOUT: return "BITNET_ERR_TIMEOUT";
    case BITNET_ERR_WORKSPACE: return "BITNET_ERR_WORKSPACE";
    }
    return "BITNET_ERR_UNKNOWN";
}

int bitnet_version(void) { return 100; }

size_t bitnet_pack_workspace_size(int64_t N, int64_t K)
{
    (void)K;
    return N > 0 ? (size_t)N * sizeof(double) : 0;
}

bitnet_status_t bitnet_pack_weights(const float *w, int64_t N, int64_t K, float eps, uint8_t *w_packed,
                                    float *gamma, void *workspace, size_t ws_bytes, cudaStream_t stream)
{
    if (!w || !w_packed || !gamma) return BITNET_ERR_INVALID_ARG;
    bitnet_status_t st = check_shape(1, N, K);
    if (st != BITNET_OK) return st;
    if (!(eps >= 0.0f) || !std::isfinite(eps)) return BITNET_ERR_INVALID_ARG;
    if (!aligned16(w) || !aligned16(w_packed) || !aligned16(gamma) || (workspace && !aligned16(workspace)))
        return BITNET_ERR_MISALIGNED;
    if (!workspace || ws_bytes < bitnet_pack_workspace_size(N, K)) return BITNET_ERR_WORKSPACE;
    double *rowsum = static_cast<double *>(workspace);
    g_launches.fetch_add(3, std::memory_order_relaxed);
    k_pack_rowsum<<<(unsigned)cdiv(N, 128), 128, 0, stream>>>(w, N, K, rowsum);
    k_pack_gamma<<<1, 1, 0, stream>>>(rowsum, N, K, gamma);
    const int64_t nwords = N * K / 16;
    k_pack_codes<<<(unsigned)cdiv(nwords, 256), 256, 0, stream>>>(w, nwords, eps, gamma,
                                                                   reinterpret_cast<uint32_t *>(w_packed));
    return cuda_status(cudaGetLastError());
}

bitnet_status_t bitnet_quant_act(const void *x, bitnet_dtype_t x_dtype, int64_t M, int64_t K, int8_t *x_q, float *s,
                                 int32_t *rowsum, cudaStream_t stream)
{
    bitnet_status_t st = check_shape(M, 1, K);
    if (st != BITNET_OK) return st;
    if (x_dtype != BITNET_DTYPE_BF16 && x_dtype != BITNET_DTYPE_F32) return BITNET_ERR_INVALID_ARG;
    if (!x || !x_q || !s) return BITNET_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(x_q) || !aligned16(s) || (rowsum && !aligned16(rowsum)))
        return BITNET_ERR_MISALIGNED;
    return cuda_status(launch_quant(x, x_dtype == BITNET_DTYPE_F32, M, K, x_q, s, rowsum, stream));
}

size_t bitnet_workspace_size(int64_t M, int64_t N, int64_t K)
{
    (void)N;
    if (M < 1 || K < 1) return 0;
    return ws_bytes_for(M, K);
}

bitnet_status_t bitnet_linear(const void *x, bitnet_dtype_t x_dtype, int64_t M, int64_t K, const uint8_t *w_packed,
                              const float *gamma, int64_t N, float *y, int8_t *x_q_out, float *s_out,
                              int32_t *acc_out, void *workspace, size_t ws_bytes, cudaStream_t stream)
{
    return forward(x, x_dtype, M, K, w_packed, gamma, nullptr, nullptr, N, y, x_q_out, s_out, acc_out, nullptr,
                   workspace, ws_bytes, stream, 1);
}

bitnet_status_t bitnet_linear_noalloc(const void *x, bitnet_dtype_t x_dtype, int64_t M, int64_t K,
                                      const uint8_t *w_packed, const float *gamma, int64_t N, float *y,
                                      cudaStream_t stream)
{
    bitnet_status_t st = check_shape(M, N, K);
    if (st != BITNET_OK) return st;
    if (ws_bytes_for(M, K) > kNoAllocScratchBytes) return BITNET_ERR_WORKSPACE;
    if (!x || !w_packed || !gamma || !y) return BITNET_ERR_INVALID_ARG;
    void *scratch = noalloc_scratch(current_device());
    if (!scratch) return BITNET_ERR_CUDA;
    return forward(x, x_dtype, M, K, w_packed, gamma, nullptr, nullptr, N, y, nullptr, nullptr, nullptr, nullptr,
                   scratch, kNoAllocScratchBytes, stream, 1);
}

bitnet_status_t bitnet_ffn_gate_up(const void *x, bitnet_dtype_t x_dtype, int64_t M, int64_t K,
                                   const uint8_t *wg_packed, const float *gamma_g, const uint8_t *wu_packed,
                                   const float *gamma_u, int64_t N, float *h, int32_t *acc_g_out,
                                   int32_t *acc_u_out, void *workspace, size_t ws_bytes, cudaStream_t stream)
{
    return forward(x, x_dtype, M, K, wg_packed, gamma_g, wu_packed, gamma_u, N, h, nullptr, nullptr, acc_g_out,
                   acc_u_out, workspace, ws_bytes, stream, 2);
}

// Workspace of one launch of n ops (all sized for K_max).
size_t seq_part_ws_bytes(int n, int64_t M, int64_t K_max)
{
    return seq_counter_bytes(n) + seq_map_bytes(n) + (size_t)n * seq_op_ws_bytes(align_up((size_t)K_max, 64), seq_mp(M));
}

size_t bitnet_sequence_workspace_size(int32_t n_ops, int64_t M, int64_t K_max)
{
    if (n_ops < 1 || n_ops > BITNET_SEQ_MAX_OPS_TOTAL || M < 1 || M > BITNET_SEQ_MAX_M || K_max < 64 ||
        K_max > kSeqMaxK)
        return 0;
    size_t total = 0;
    for (int c0 = 0; c0 < n_ops; c0 += BITNET_SEQ_MAX_OPS)
        total += seq_part_ws_bytes(std::min(BITNET_SEQ_MAX_OPS, n_ops - c0), M, K_max);
    return total;
}

bitnet_status_t bitnet_sequence_plan(const bitnet_op_t *ops, int32_t n_ops, int64_t M, int32_t *wait_x,
                                     int32_t *wait_y)
{
    return seq_plan(ops, n_ops, M, wait_x, wait_y, ByteRange{0, 0});
}

bitnet_status_t bitnet_decode_sequence(const bitnet_op_t *ops, int32_t n_ops, int64_t M, void *workspace,
                                       size_t ws_bytes, cudaStream_t stream)
{
    if (n_ops <= BITNET_SEQ_MAX_OPS) return decode_sequence(ops, n_ops, M, workspace, ws_bytes, stream);
    // a longer list: consecutive launches of BITNET_SEQ_MAX_OPS ops, each on its own part of the
    // workspace (sized for the largest K of the list), all validated before the first launch
    if (!ops || n_ops > BITNET_SEQ_MAX_OPS_TOTAL || M < 1 || M > BITNET_SEQ_MAX_M) return BITNET_ERR_INVALID_ARG;
    if (!workspace) return BITNET_ERR_WORKSPACE;
    if (!aligned16(workspace)) return BITNET_ERR_MISALIGNED;
    int64_t K_max = 64;
    for (int i = 0; i < n_ops; ++i) K_max = std::max(K_max, ops[i].K);
    if (K_max > kSeqMaxK) return BITNET_ERR_UNSUPPORTED_SHAPE;
    const ByteRange whole = range_of(workspace, ws_bytes);
    size_t need = 0;
    for (int c0 = 0; c0 < n_ops; c0 += BITNET_SEQ_MAX_OPS) {
        const int nc = std::min(BITNET_SEQ_MAX_OPS, n_ops - c0);
        int32_t order[BITNET_SEQ_MAX_OPS];
        const bitnet_status_t st = seq_schedule(ops + c0, nc, M, order, whole);
        if (st != BITNET_OK) return st;
        need += seq_part_ws_bytes(nc, M, K_max);
    }
    if (need > ws_bytes) return BITNET_ERR_WORKSPACE;
    size_t off = 0;
    for (int c0 = 0; c0 < n_ops; c0 += BITNET_SEQ_MAX_OPS) {
        const int nc = std::min(BITNET_SEQ_MAX_OPS, n_ops - c0);
        const size_t part = seq_part_ws_bytes(nc, M, K_max);
        const bitnet_status_t st =
            decode_sequence(ops + c0, nc, M, static_cast<unsigned char *>(workspace) + off, part, stream, &whole, c0);
        if (st != BITNET_OK) return st;
        off += part;
    }
    return BITNET_OK;
}

bitnet_status_t bitnet_sequence_schedule(const bitnet_op_t *ops, int32_t n_ops, int64_t M, int32_t *order)
{
    if (!order) return BITNET_ERR_INVALID_ARG;
    return seq_schedule(ops, n_ops, M, order, ByteRange{0, 0});
}

bitnet_status_t bitnet_sequence_tasks(const bitnet_op_t *ops, int32_t n_ops, int64_t M, int32_t ctas,
                                      int32_t *group_op, int32_t *group_kind, int32_t *group_tasks,
                                      int32_t *dep_count, int32_t *deps)
{
    if (!group_op || !group_kind || !group_tasks || !dep_count || !deps || ctas < 1) return BITNET_ERR_INVALID_ARG;
    int32_t order[BITNET_SEQ_MAX_OPS];
    bitnet_status_t st = seq_schedule(ops, n_ops, M, order, ByteRange{0, 0});
    if (st != BITNET_OK) return st;
    bitnet_op_t sched[BITNET_SEQ_MAX_OPS];
    for (int k = 0; k < n_ops; ++k) sched[k] = ops[order[k]];
    static DtProgram proto;
    DtProgram p = proto;
    std::vector<int> gorder;
    st = seq_build(p, sched, order, n_ops, M, ctas, nullptr, 0, ByteRange{0, 0}, &gorder);
    if (st != BITNET_OK) return st;
    SeqGroups G;
    st = seq_groups(sched, n_ops, M, ByteRange{0, 0}, G);
    if (st != BITNET_OK) return st;
    // position of each group in the task order, to report dependencies by position
    std::vector<int> pos(2 * n_ops, 0);
    for (int k = 0; k < 2 * n_ops; ++k) pos[gorder[k]] = k;
    for (int k = 0; k < 2 * n_ops; ++k) {
        const int v = gorder[k], j = v / 2;
        group_op[k] = order[j];
        group_kind[k] = v % 2;
        group_tasks[k] = v % 2 ? p.ops[j].rtasks : (int32_t)seq_qtasks(M);
        dep_count[k] = (int32_t)G.preds[v].size();
        for (int d = 0; d < DT_MAX_DEPS + 1; ++d)
            deps[k * (DT_MAX_DEPS + 1) + d] = d < (int)G.preds[v].size() ? pos[G.preds[v][d]] : -1;
    }
    return BITNET_OK;
}

uint64_t bitnet_set_wait_limit_ns(uint64_t ns)
{
    if (ns == 0) ns = kDefaultWaitLimitNs;
    const unsigned long long v = ns;
    if (cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v)) != cudaSuccess) return 0;
    return g_wait_limit_set.exchange(v);
}

int bitnet_set_sequence_test_stall(int op)
{
    if (op < -1 || op >= BITNET_SEQ_MAX_OPS_TOTAL) return -2;
    return g_seq_stall.exchange(op);
}

bitnet_status_t bitnet_rmsnorm_quant(const void *x, bitnet_dtype_t x_dtype, int64_t M, int64_t K, const float *g,
                                     float eps, int8_t *x_q, float *s, int32_t *rowsum, cudaStream_t stream)
{
    bitnet_status_t st = check_shape(M, 1, K);
    if (st != BITNET_OK) return st;
    if (x_dtype != BITNET_DTYPE_BF16 && x_dtype != BITNET_DTYPE_F32) return BITNET_ERR_INVALID_ARG;
    if (!x || !g || !x_q || !s || !(eps >= 0.0f) || !std::isfinite(eps)) return BITNET_ERR_INVALID_ARG;
    if (K > kNormMaxK) return BITNET_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x) || !aligned16(g) || !aligned16(x_q) || !aligned16(s) || (rowsum && !aligned16(rowsum)))
        return BITNET_ERR_MISALIGNED;
    return cuda_status(launch_norm_quant(x, x_dtype == BITNET_DTYPE_F32, M, K, g, eps, x_q, s, rowsum, stream));
}

bitnet_status_t bitnet_linear_norm(const void *x, bitnet_dtype_t x_dtype, int64_t M, int64_t K, const float *g,
                                   float eps, const uint8_t *w_packed, const float *gamma, int64_t N, float *y,
                                   int8_t *x_q_out, float *s_out, int32_t *acc_out, void *workspace, size_t ws_bytes,
                                   cudaStream_t stream)
{
    if (!g) return BITNET_ERR_INVALID_ARG;
    return forward(x, x_dtype, M, K, w_packed, gamma, nullptr, nullptr, N, y, x_q_out, s_out, acc_out, nullptr,
                   workspace, ws_bytes, stream, 1, g, eps);
}

bitnet_status_t bitnet_ffn_gate_up_norm(const void *x, bitnet_dtype_t x_dtype, int64_t M, int64_t K, const float *g,
                                        float eps, const uint8_t *wg_packed, const float *gamma_g,
                                        const uint8_t *wu_packed, const float *gamma_u, int64_t N, float *h,
                                        int32_t *acc_g_out, int32_t *acc_u_out, void *workspace, size_t ws_bytes,
                                        cudaStream_t stream)
{
    if (!g) return BITNET_ERR_INVALID_ARG;
    return forward(x, x_dtype, M, K, wg_packed, gamma_g, wu_packed, gamma_u, N, h, nullptr, nullptr, acc_g_out,
                   acc_u_out, workspace, ws_bytes, stream, 2, g, eps);
}

bitnet_status_t bitnet_linear_ex(const void *x, bitnet_dtype_t x_dtype, const float *x_amax, const float *norm_g,
                                 float norm_eps, int64_t M, int64_t K, const uint8_t *w_packed, const float *gamma,
                                 int64_t N, void *y, bitnet_dtype_t y_dtype, float *y_amax, void *workspace,
                                 size_t ws_bytes, cudaStream_t stream)
{
    if (y_dtype != BITNET_DTYPE_BF16 && y_dtype != BITNET_DTYPE_F32) return BITNET_ERR_INVALID_ARG;
    IoOpts io;
    io.x_amax = x_amax;
    io.y_bf16 = y_dtype == BITNET_DTYPE_BF16;
    io.y_amax = y_amax;
    return forward(x, x_dtype, M, K, w_packed, gamma, nullptr, nullptr, N, y, nullptr, nullptr, nullptr, nullptr,
                   workspace, ws_bytes, stream, 1, norm_g, norm_eps, io);
}

bitnet_status_t bitnet_ffn_gate_up_ex(const void *x, bitnet_dtype_t x_dtype, const float *x_amax,
                                      const float *norm_g, float norm_eps, int64_t M, int64_t K,
                                      const uint8_t *wg_packed, const float *gamma_g, const uint8_t *wu_packed,
                                      const float *gamma_u, int64_t N, void *h, bitnet_dtype_t h_dtype,
                                      float *h_amax, void *workspace, size_t ws_bytes, cudaStream_t stream)
{
    if (h_dtype != BITNET_DTYPE_BF16 && h_dtype != BITNET_DTYPE_F32) return BITNET_ERR_INVALID_ARG;
    IoOpts io;
    io.x_amax = x_amax;
    io.y_bf16 = h_dtype == BITNET_DTYPE_BF16;
    io.y_amax = h_amax;
    return forward(x, x_dtype, M, K, wg_packed, gamma_g, wu_packed, gamma_u, N, h, nullptr, nullptr, nullptr,
                   nullptr, workspace, ws_bytes, stream, 2, norm_g, norm_eps, io);
}

bitnet_status_t bitnet_device_status(int clear, bitnet_status_t *status_out, cudaStream_t stream)
{
    if (!status_out) return BITNET_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return BITNET_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return BITNET_ERR_CUDA;
    *status_out = static_cast<bitnet_status_t>(v);
    if (clear) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return BITNET_ERR_CUDA;
    }
    return BITNET_OK;
}

int bitnet_num_sms(void) { return num_sms_for(current_device()); }

uint64_t bitnet_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int bitnet_set_dispatch(int dispatch)
{
    if (dispatch < BITNET_DISPATCH_AUTO || dispatch > BITNET_DISPATCH_PREFILL) return -1;
    return g_dispatch.exchange(dispatch);
}

} // extern "C"
