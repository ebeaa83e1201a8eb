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
#include <utility>
#include <vector>

#include "bitnet.h"
#include "common.cuh"
#include "decode.cuh"
#include "decode_cluster.cuh"
#include "decode_seq.cuh"
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
    if (nch <= per_warp)
        return launch_pdl(k_quant_rows_reg<XF32, 1>, dim3((unsigned)cdiv(M, 8)), dim3(256), 0, stream, x, M, K, xq,
                          s, rs, amax_in, amax_zero);
    if (nch <= 2 * per_warp)
        return launch_pdl(k_quant_rows_reg<XF32, 2>, dim3((unsigned)cdiv(M, 4)), dim3(256), 0, stream, x, M, K, xq,
                          s, rs, amax_in, amax_zero);
    if (nch <= 4 * per_warp)
        return launch_pdl(k_quant_rows_reg<XF32, 4>, dim3((unsigned)cdiv(M, 2)), dim3(256), 0, stream, x, M, K, xq,
                          s, rs, amax_in, amax_zero);
    if (nch <= 8 * per_warp)
        return launch_pdl(k_quant_rows_reg<XF32, 8>, dim3((unsigned)M), dim3(256), 0, stream, x, M, K, xq, s, rs,
                          amax_in, amax_zero);
    return launch_pdl(k_quant_rows<XF32>, dim3((unsigned)cdiv(M, 8)), dim3(256), 0, stream, x, M, K, xq, s, rs,
                      amax_in, amax_zero);
}

// RMS normalisation + quantiser: rows of up to 4096 elements on 128 threads (two rows
// per CTA), longer rows (up to 8192) on 256.
constexpr int64_t kNormMaxK = 256 * RQ_MAX_PER_THREAD;

template <bool XF32>
cudaError_t launch_norm_quant_t(const void *x, int64_t M, int64_t K, const float *g, float eps, int8_t *xq, float *s,
                                int32_t *rs, float *amax_zero, cudaStream_t stream)
{
    if (K <= 128 * RQ_MAX_PER_THREAD)
        return launch_pdl(k_rmsnorm_quant_rows<XF32, 128>, dim3((unsigned)cdiv(M, 2)), dim3(256), 0, stream, x, M, K,
                          g, eps, xq, s, rs, amax_zero);
    return launch_pdl(k_rmsnorm_quant_rows<XF32, 256>, dim3((unsigned)M), dim3(256), 0, stream, x, M, K, g, eps, xq, s,
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
    // output through TMA stores when rows are 16-byte multiples: 32 x 32 boxes,
    // 128-byte swizzle for fp32, 64-byte swizzle for bf16
    tmY = tmA;
    if (a.vec_ok && !encode_2d_out(&tmY, y, (uint64_t)M, (uint64_t)N, 32, 32, io.y_bf16)) return BITNET_ERR_CUDA;
    cudaError_t e = quantise(xq, s, nullptr);
    if (e != cudaSuccess) return BITNET_ERR_CUDA;
    const int grid = std::min(a.num_tiles, sms);
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
std::atomic<int> g_seq_cluster{4};
constexpr int64_t kSeqMaxK = 64 * DS_MAX_KS * 4; // 8192: at most 32 k-steps per CTA with the smallest cluster (4)

struct ByteRange {
    uintptr_t lo, hi;
};
inline bool overlaps(ByteRange a, ByteRange b) { return a.lo < b.hi && b.lo < a.hi; }
inline ByteRange range_of(const void *p, size_t bytes)
{
    const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
    return {lo, lo + bytes};
}

// Validation (host only, shared by plan, schedule and run); fills the byte
// ranges each op reads (x) and writes (y).  extra: one more range no op may
// write or read (the workspace), may be empty.
bitnet_status_t seq_validate(const bitnet_op_t *ops, int n, int64_t M, ByteRange extra, std::vector<ByteRange> &xr,
                             std::vector<ByteRange> &yr)
{
    if (!ops || n < 1 || n > BITNET_SEQ_MAX_OPS || M < 1) return BITNET_ERR_INVALID_ARG;
    if (M > BITNET_SEQ_MAX_M) return BITNET_ERR_UNSUPPORTED_SHAPE;
    xr.assign(n, ByteRange{0, 0});
    yr.assign(n, ByteRange{0, 0});
    std::vector<ByteRange> ro; // weights and gammas (read-only for the launch)
    ro.reserve(4 * (size_t)n);
    for (int i = 0; i < n; ++i) {
        const bitnet_op_t &o = ops[i];
        if (o.kind != BITNET_OP_LINEAR && o.kind != BITNET_OP_FFN_GATE_UP) return BITNET_ERR_INVALID_ARG;
        if (o.x_dtype != BITNET_DTYPE_BF16 && o.x_dtype != BITNET_DTYPE_F32) return BITNET_ERR_INVALID_ARG;
        const bool ffn = o.kind == BITNET_OP_FFN_GATE_UP;
        if (!o.x || !o.w0 || !o.gamma0 || !o.y || (ffn && (!o.w1 || !o.gamma1))) return BITNET_ERR_INVALID_ARG;
        const bitnet_status_t st = check_shape(M, o.N, o.K);
        if (st != BITNET_OK) return st;
        if (o.K > kSeqMaxK) return BITNET_ERR_UNSUPPORTED_SHAPE;
        const void *ptrs[] = {o.x, o.w0, o.gamma0, ffn ? o.w1 : nullptr, ffn ? o.gamma1 : nullptr, o.y};
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
// op scheduled just before it is deferred while another op is ready: a
// consumer then waits less for its producer to finish on every CTA.
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

// Clusters of C CTAs (one CTA per SM) that are resident at once on `dev`.
int seq_clusters(int dev, int C)
{
    static std::atomic<int> cache[kMaxDevices][9];
    static std::atomic<int> smem_done[kMaxDevices];
    if (dev < 0 || dev >= kMaxDevices || C < 1 || C > 8) return 0;
    int v = cache[dev][C].load();
    if (v > 0) return v;
    if (ensure_smem(k_decode_seq, kSmemLimit, smem_done, dev) != cudaSuccess) return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C * 64);
    cfg.blockDim = dim3(DS_THREADS);
    cfg.dynamicSmemBytes = kSmemLimit;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&v, k_decode_seq, &cfg) != cudaSuccess || v < 1) return 0;
    cache[dev][C].store(v);
    return v;
}

// Partitions of the grid: user op i runs on clusters [cl0[of[i]], cl0[of[i]] +
// ncl[of[i]]) as slices[i] consecutive ops over slices of its output rows.
struct SeqParts {
    int n = 1;
    int cl0[DS_MAX_PARTS] = {0}, ncl[DS_MAX_PARTS] = {0};
    std::vector<int> of;     // partition of each user op
    std::vector<int> slices; // row slices of each user op
    int ring_share = 1;      // an op's weights may fill 1 / ring_share of the ring
};

// Rows per cluster of `rows` output rows spread over ncl clusters.
inline int seq_rpc(int64_t rows, int ncl) { return (int)align_up((size_t)cdiv(rows, ncl), 16); }

// Fewest row slices of an op (nmat matrices, N rows) for which every warp holds
// at most DS_RGW row groups on ncl clusters.
int seq_min_slices(int64_t N, int nmat, int ncl)
{
    int s = 1;
    while ((int64_t)nmat * (seq_rpc(cdiv(N, s), ncl) / 16) > 8 * DS_RGW) ++s;
    return s;
}

// Per-op layout and the launch-wide shared-memory map for G clusters of C CTAs.
// The user ops (in execution order, waits wx / wy between them) are cut into
// parts.slices[i] consecutive ops over slices of their output rows.  A slice
// waits for the last slice of the op its user op waits for; later slices of an
// op need no wait of their own (the first one's wait held on every CTA of the
// partition), and with one token tile they reuse the first slice's quantised x.
// too_big (optional, n entries): set to 1 for every user op one of whose
// slices does not fit the ring, else 0.
bitnet_status_t seq_build(DsProgram &p, const bitnet_op_t *ops, int n, int64_t M, int C, int G, const SeqParts &parts,
                          const int32_t *wx, const int32_t *wy, std::vector<char> *too_big = nullptr)
{
    if (too_big) too_big->assign(n, 0);
    int total = 0;
    for (int i = 0; i < n; ++i) total += parts.slices[i];
    if (total > DS_MAX_OPS) return BITNET_ERR_UNSUPPORTED_SHAPE;
    std::vector<int> last_of(n), user_of(total);
    int ks_max = 1;
    uint32_t blk_max = 0;
    int idx = 0;
    for (int i = 0; i < n; ++i) {
        const bitnet_op_t &o = ops[i];
        const int part = parts.of[i];
        const int ncl = parts.ncl[part];
        const int nmat = o.kind == BITNET_OP_FFN_GATE_UP ? 2 : 1;
        const int KS = (int)(o.K / 64);
        const int ks = (int)cdiv(KS, C);
        if (ks > DS_MAX_KS) return BITNET_ERR_UNSUPPORTED_SHAPE;
        const int ns = parts.slices[i];
        const size_t row_bytes = (size_t)(o.K / 4);
        for (int t = 0; t < ns; ++t, ++idx) {
            const int64_t r0 = o.N * t / ns, r1 = o.N * (t + 1) / ns;
            DsOp &d = p.ops[idx];
            d = DsOp{};
            user_of[idx] = i;
            d.cl0 = (int16_t)parts.cl0[part];
            d.ncl = (int16_t)ncl;
            d.ks = (int16_t)ks;
            const int rpc = seq_rpc(r1 - r0, ncl);
            if ((int64_t)nmat * (rpc / 16) > 8 * DS_RGW) return BITNET_ERR_UNSUPPORTED_SHAPE;
            d.rpc = (int16_t)rpc;
            const int own = rpc / C;
            int orp = (int)align_up((size_t)own, 4);
            if (orp % 8 == 0) orp += 4; // token rows of a block land 8 banks apart
            d.own_rows = (int16_t)own;
            d.orp = (int16_t)orp;
            d.box_w = (int16_t)(16 * (ks | 1)); // odd number of 16-byte chunks: conflict-free fragment loads
            d.x = o.x;
            d.w0 = o.w0 + (size_t)r0 * row_bytes;
            d.w1 = nmat == 2 ? o.w1 + (size_t)r0 * row_bytes : nullptr;
            d.gamma0 = o.gamma0;
            d.gamma1 = nmat == 2 ? o.gamma1 : nullptr;
            d.y = o.y + r0;
            d.K = (int)o.K;
            d.N = (int)(r1 - r0);
            d.ldy = (int)o.N;
            d.nmat = (uint8_t)nmat;
            d.xf32 = o.x_dtype == BITNET_DTYPE_F32;
            d.reuse = (t > 0 && M <= 8) ? 1 : 0;
            d.wait_x = (wx[i] >= 0 && !d.reuse) ? last_of[wx[i]] : -1;
            d.wait_y = (t == 0 && wy[i] >= 0) ? last_of[wy[i]] : -1;
            blk_max = std::max(blk_max, (uint32_t)(nmat * 8 * orp * 4));
        }
        last_of[i] = idx - 1;
        ks_max = std::max(ks_max, ks);
    }
    p.n_ops = total;
    p.M = (int)M;
    p.C = C;
    p.n_ctas = G * C;
    // partitions: each runs its ops in program order, linked through DsOp::nxt
    p.n_parts = parts.n;
    for (int q = 0; q < parts.n; ++q) {
        p.part_cl0[q] = parts.cl0[q];
        p.part_ncl[q] = parts.ncl[q];
        p.part_first[q] = -1;
    }
    {
        int last[DS_MAX_PARTS];
        for (int q = 0; q < DS_MAX_PARTS; ++q) last[q] = -1;
        for (int j = 0; j < total; ++j) {
            const int i = user_of[j];
            const int q = parts.of[i];
            p.ops[j].nxt = -1;
            if (last[q] < 0)
                p.part_first[q] = j;
            else
                p.ops[last[q]].nxt = j;
            last[q] = j;
            // every op an op waits for runs in its partition
            if ((wx[i] >= 0 && parts.of[wx[i]] != q) || (wy[i] >= 0 && parts.of[wy[i]] != q))
                return BITNET_ERR_INVALID_ARG;
        }
        for (int q = 0; q < parts.n; ++q)
            if (p.part_first[q] < 0) return BITNET_ERR_INVALID_ARG;
    }
    // x staging: ops whose x no op of the launch writes alternate between buffers 0 and 1 (the
    // next one is fetched while the current one runs); ops reading an earlier op's output are
    // marked buffer 2 and read their x in place from L2 once their wait is over (no staging);
    // ops reusing the previous op's x load nothing.  Rows as long as the largest K slice in
    // the buffer.
    uint32_t pitch[3] = {16, 16, 16};
    int alt[DS_MAX_PARTS] = {0};
    for (int j = 0; j < total; ++j) {
        DsOp &d = p.ops[j];
        if (d.reuse) continue;
        const int q = parts.of[user_of[j]];
        if (d.wait_x >= 0) {
            d.xbuf = 2;
        } else {
            d.xbuf = (uint8_t)alt[q];
            alt[q] ^= 1;
        }
        if (d.xbuf != 2) pitch[d.xbuf] = std::max(pitch[d.xbuf], (uint32_t)(d.ks * 64 * (d.xf32 ? 4 : 2)));
    }
    size_t off = DS_HDR;
    for (int b = 0; b < 3; ++b) {
        p.xs_off[b] = (uint32_t)off;
        p.xs_pitch[b] = pitch[b];
        off = align_up(off + 8 * (size_t)pitch[b], 128);
    }
    uint32_t xs = (uint32_t)ks_max * 64;
    xs += (uint32_t)(((64 - (int)(xs % 128)) + 128) % 128); // == 64 mod 128
    p.xq_stride = xs;
    p.xq_off = (uint32_t)off;
    p.part_off = (uint32_t)align_up(p.xq_off + 8 * (size_t)xs, 128);
    const size_t part_bytes = align_up((size_t)C * blk_max, 128);
    p.recv_off = (uint32_t)(p.part_off + part_bytes);
    p.ring_off = (uint32_t)(p.recv_off + part_bytes);
    const size_t usable = kSmemLimit - 128; // the kernel aligns its base to 128 bytes
    if (p.ring_off + 4096 > usable) return BITNET_ERR_UNSUPPORTED_SHAPE;
    p.ring_bytes = (uint32_t)((usable - p.ring_off) & ~size_t(127));
    bool fits = true;
    for (int j = 0; j < total; ++j)
        if ((size_t)ds_piece_bytes(p.ops[j]) * p.ops[j].nmat * parts.ring_share > p.ring_bytes) {
            fits = false;
            if (too_big) (*too_big)[user_of[j]] = 1;
        }
    return fits ? BITNET_OK : BITNET_ERR_UNSUPPORTED_SHAPE;
}

// Partition count for decode sequences: 0 = chosen by the cost estimate below.
std::atomic<int> g_seq_parts{0};
// Share of the weight ring one op may fill (1 = all of it).  Half the ring
// lets the next op's weights stream in while an op computes, but the extra row
// slices cost more than the wait (measured on the 30-layer decode step: 4
// partitions fit 256 ops at share 1, only 2 at share 2).
std::atomic<int> g_seq_ring_share{1};

// Estimated duration (µs) of the busiest partition of a built program, from
// per-phase timestamps of the 30-layer decode step on B200: per op ~2 µs of
// partial-sum exchange, epilogue and hand-over, ~2 µs more for x, the absmax
// exchange and quantisation unless the op reuses the previous op's, the
// contraction at ~0.055 µs per mma.sync per warp, and a producer's completion
// latency when an op reads the output of the op just before it; or the weight
// stream at ~45 GB/s per SM if that takes longer.
double seq_estimate(const DsProgram &p)
{
    double t_ops[DS_MAX_PARTS] = {0.0}, bytes[DS_MAX_PARTS] = {0.0};
    for (int q = 0; q < p.n_parts; ++q) {
        int prev = -1;
        for (int j = p.part_first[q]; j >= 0; j = p.ops[j].nxt) {
            const DsOp &d = p.ops[j];
            const double mma_per_warp = (double)d.nmat * (d.rpc / 16) * d.ks * 2.0 / 8.0;
            double t = 2.0 + mma_per_warp * 0.055;
            if (!d.reuse) t += 2.0;
            if (d.wait_x >= 0 && d.wait_x == prev) t += 2.3;
            t_ops[q] += t;
            bytes[q] += (double)d.nmat * d.N * (d.K / 4);
            prev = j;
        }
    }
    double worst = 0.0;
    for (int q = 0; q < p.n_parts; ++q) {
        const double stream_us = bytes[q] / (p.part_ncl[q] * p.C * 45e3);
        worst = std::max(worst, std::max(t_ops[q], stream_us));
    }
    return worst;
}

// Independent groups of ops run side by side: the connected components of the
// hazard graph never wait for each other.  For each partition count P (up to
// DS_MAX_PARTS, or the count set by bitnet_set_sequence_partitions) the
// components are dealt to P partitions by weight bytes (largest first, to the
// lightest partition), each partition gets clusters in proportion to its
// bytes, its ops are re-scheduled among themselves, and each op is cut into
// the fewest row slices whose weight pieces fit a CTA's ring.  The program with
// the smallest estimated duration is kept.  ops / wx / wy are rewritten in the
// chosen execution order.
// What the planner chose, per op of the returned execution order.
struct SeqLayout {
    std::vector<int> perm;    // index of the op in the list the planner was given
    std::vector<int> part_of; // partition
    std::vector<int> slices;  // row slices
};

bitnet_status_t seq_partitioned_build(DsProgram &p, bitnet_op_t *ops, int n, int64_t M, int C, int G, int32_t *wx,
                                      int32_t *wy, ByteRange extra, SeqLayout *layout = nullptr)
{
    std::vector<ByteRange> xr, yr;
    if (seq_validate(ops, n, M, extra, xr, yr) != BITNET_OK) return BITNET_ERR_INVALID_ARG;
    // components over the hazards (union-find)
    std::vector<int> root(n);
    for (int i = 0; i < n; ++i) root[i] = i;
    auto find = [&](int i) {
        while (root[i] != i) i = root[i] = root[root[i]];
        return i;
    };
    for (int j = 0; j < n; ++j)
        for (int i = 0; i < j; ++i)
            if (hazard(xr, yr, i, j)) root[find(i)] = find(j);
    std::vector<double> cbytes(n, 0.0);
    double total = 0.0;
    for (int i = 0; i < n; ++i) {
        const double b = (ops[i].kind == BITNET_OP_FFN_GATE_UP ? 2.0 : 1.0) * (double)ops[i].N * (double)(ops[i].K / 4);
        cbytes[find(i)] += b;
        total += b;
    }
    std::vector<int> comps;
    for (int i = 0; i < n; ++i)
        if (find(i) == i) comps.push_back(i);
    std::sort(comps.begin(), comps.end(), [&](int a, int b) { return cbytes[a] > cbytes[b] || (cbytes[a] == cbytes[b] && a < b); });

    const int forced = g_seq_parts.load();
    const int p_max = std::min({DS_MAX_PARTS, G, (int)comps.size()});
    double best_t = 0.0;
    bool have = false;
    static DsProgram cand_proto;
    DsProgram cand = cand_proto;
    std::vector<bitnet_op_t> best_ops;
    std::vector<int32_t> best_wx, best_wy;
    SeqLayout best_layout;
    for (int P = 1; P <= p_max; ++P) {
        if (forced > 0 && P != std::min(forced, p_max)) continue;
        // components to partitions: largest first, each to the lightest partition
        std::vector<double> pbytes(P, 0.0);
        std::vector<int> part_of_root(n, 0);
        for (int c : comps) {
            int q = 0;
            for (int k = 1; k < P; ++k)
                if (pbytes[k] < pbytes[q]) q = k;
            part_of_root[c] = q;
            pbytes[q] += cbytes[c];
        }
        // clusters in proportion to bytes, at least one each
        SeqParts parts;
        parts.n = P;
        int used = 0;
        for (int q = 0; q < P; ++q) {
            parts.ncl[q] = std::max(1, (int)(G * pbytes[q] / total));
            used += parts.ncl[q];
        }
        while (used > G) { // only when many partitions are tiny
            int q = 0;
            for (int k = 1; k < P; ++k)
                if (parts.ncl[k] > parts.ncl[q]) q = k;
            --parts.ncl[q];
            --used;
        }
        while (used < G) {
            int q = 0;
            for (int k = 1; k < P; ++k)
                if (pbytes[k] / parts.ncl[k] > pbytes[q] / parts.ncl[q]) q = k;
            ++parts.ncl[q];
            ++used;
        }
        for (int q = 1; q < P; ++q) parts.cl0[q] = parts.cl0[q - 1] + parts.ncl[q - 1];
        // execution order: partition by partition, each re-scheduled among its own ops
        std::vector<bitnet_op_t> ord;
        std::vector<int> perm;
        ord.reserve(n);
        for (int q = 0; q < P; ++q) {
            std::vector<bitnet_op_t> sub;
            std::vector<int> sub_idx;
            for (int i = 0; i < n; ++i)
                if (part_of_root[find(i)] == q) {
                    sub.push_back(ops[i]);
                    sub_idx.push_back(i);
                }
            if (sub.empty()) continue;
            std::vector<int32_t> o(sub.size());
            if (seq_schedule(sub.data(), (int)sub.size(), M, o.data(), extra) != BITNET_OK) return BITNET_ERR_INVALID_ARG;
            for (int32_t k : o) {
                ord.push_back(sub[k]);
                perm.push_back(sub_idx[k]);
            }
        }
        std::vector<int32_t> cwx(n), cwy(n);
        if (seq_plan(ord.data(), n, M, cwx.data(), cwy.data(), extra) != BITNET_OK) return BITNET_ERR_INVALID_ARG;
        // partition of each op in the new order
        parts.of.assign(n, 0);
        {
            int pos = 0;
            for (int q = 0; q < P; ++q)
                for (int i = 0; i < n; ++i)
                    if (part_of_root[find(i)] == q) parts.of[pos++] = q;
        }
        parts.ring_share = g_seq_ring_share.load();
        parts.slices.resize(n);
        for (int i = 0; i < n; ++i)
            parts.slices[i] = seq_min_slices(ord[i].N, ord[i].kind == BITNET_OP_FFN_GATE_UP ? 2 : 1,
                                             parts.ncl[parts.of[i]]);
        // cut ops whose pieces do not fit the ring finer until they do: each pass adds one slice
        // to every op that does not fit (the ring grows as slices shrink, through smaller
        // partial-sum blocks, so an op is cut no finer than the ring of its pass requires)
        bitnet_status_t st = BITNET_ERR_UNSUPPORTED_SHAPE;
        std::vector<char> big;
        for (int pass = 0; pass < 4 * DS_MAX_OPS; ++pass) {
            st = seq_build(cand, ord.data(), n, M, C, G, parts, cwx.data(), cwy.data(), &big);
            if (st == BITNET_OK) break;
            bool grew = false;
            for (int i = 0; i < n; ++i)
                if (big[i] && parts.slices[i] < ord[i].N) {
                    ++parts.slices[i];
                    grew = true;
                }
            if (!grew) break;
        }
        if (st != BITNET_OK) {
            if (st == BITNET_ERR_INVALID_ARG) return st;
            continue;
        }
        const double t = seq_estimate(cand);
        if (!have || t < best_t) {
            have = true;
            best_t = t;
            p = cand;
            best_ops = ord;
            best_wx = cwx;
            best_wy = cwy;
            best_layout.perm = perm;
            best_layout.part_of = parts.of;
            best_layout.slices = parts.slices;
        }
    }
    if (!have) return BITNET_ERR_UNSUPPORTED_SHAPE;
    for (int i = 0; i < n; ++i) {
        ops[i] = best_ops[i];
        wx[i] = best_wx[i];
        wy[i] = best_wy[i];
    }
    if (layout) *layout = best_layout;
    return BITNET_OK;
}

constexpr size_t kSeqWorkspaceBytes = 2048;
static_assert(4 * (DS_MAX_OPS + 1) <= (int)kSeqWorkspaceBytes, "sequence counters");
static_assert(DS_MAX_OPS >= BITNET_SEQ_MAX_OPS, "sequence op limit: every op fits unsliced");
static_assert(sizeof(DsProgram) <= 32000, "kernel parameter space");

// Plans of recent sequence calls.  A decode loop calls with the same op list
// every step; planning it (schedule, partitions, row slices) takes about 2 ms
// of host time for a 120-op layer stack, the launch itself microseconds.
struct SeqCacheEntry {
    bool used = false;
    uint64_t stamp = 0;
    int n = 0, dev = -1, C = 0, parts = 0, share = 0;
    int64_t M = 0;
    const void *ws = nullptr;
    bitnet_op_t ops[BITNET_SEQ_MAX_OPS];
    DsProgram prog;
};
constexpr int kSeqCacheEntries = 8;
SeqCacheEntry g_seq_cache[kSeqCacheEntries];
std::mutex g_seq_cache_mu;
uint64_t g_seq_cache_clock = 0;

bool same_op(const bitnet_op_t &a, const bitnet_op_t &b)
{
    return a.kind == b.kind && a.x_dtype == b.x_dtype && a.x == b.x && a.K == b.K && a.N == b.N && a.w0 == b.w0 &&
           a.gamma0 == b.gamma0 && a.w1 == b.w1 && a.gamma1 == b.gamma1 && a.y == b.y;
}

bool seq_cache_match(const SeqCacheEntry &e, const bitnet_op_t *ops, int n, int64_t M, int dev, int C, int parts,
                     int share, const void *ws)
{
    if (!e.used || e.n != n || e.M != M || e.dev != dev || e.C != C || e.parts != parts || e.share != share ||
        e.ws != ws)
        return false;
    for (int i = 0; i < n; ++i)
        if (!same_op(e.ops[i], ops[i])) return false;
    return true;
}

cudaError_t seq_launch(const DsProgram &p, cudaStream_t stream)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.n_ctas);
    cfg.blockDim = dim3(DS_THREADS);
    cfg.dynamicSmemBytes = kSmemLimit;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = p.C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaLaunchKernelEx(&cfg, k_decode_seq, p);
}

bitnet_status_t decode_sequence(const bitnet_op_t *ops, int n, int64_t M, void *workspace, size_t ws_bytes,
                                cudaStream_t stream)
{
    if (workspace && !aligned16(workspace)) return BITNET_ERR_MISALIGNED;
    const int parts_set = g_seq_parts.load(), share_set = g_seq_ring_share.load();
    // the plan of an op list seen before (validated then) on this device, workspace and settings
    if (ops && n >= 1 && n <= BITNET_SEQ_MAX_OPS && workspace && ws_bytes >= kSeqWorkspaceBytes) {
        int dev = -1;
        if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0) {
            const int C = g_seq_cluster.load();
            static DsProgram hit_proto;
            DsProgram p = hit_proto;
            bool hit = false;
            {
                std::lock_guard<std::mutex> lk(g_seq_cache_mu);
                for (SeqCacheEntry &e : g_seq_cache)
                    if (seq_cache_match(e, ops, n, M, dev, C, parts_set, share_set, workspace)) {
                        p = e.prog;
                        e.stamp = ++g_seq_cache_clock;
                        hit = true;
                        break;
                    }
            }
            if (hit) return cuda_status(seq_launch(p, stream));
        }
    }
    int32_t wx[BITNET_SEQ_MAX_OPS], wy[BITNET_SEQ_MAX_OPS], order[BITNET_SEQ_MAX_OPS];
    const bitnet_op_t *user_ops = ops;
    const ByteRange wsr = workspace ? range_of(workspace, kSeqWorkspaceBytes) : ByteRange{0, 0};
    bitnet_status_t st = seq_schedule(ops, n, M, order, wsr);
    if (st != BITNET_OK) return st;
    bitnet_op_t sched[BITNET_SEQ_MAX_OPS];
    for (int k = 0; k < n; ++k) sched[k] = ops[order[k]];
    ops = sched;
    st = seq_plan(ops, n, M, wx, wy, wsr);
    if (st != BITNET_OK) return st;
    if (!workspace || ws_bytes < kSeqWorkspaceBytes) return BITNET_ERR_WORKSPACE;
    const int dev = current_device();
    const int C = g_seq_cluster.load();
    const int G = seq_clusters(dev, C);
    if (G < 1) return BITNET_ERR_CUDA;
    static DsProgram prog_proto; // zero-initialised template; each call fills a copy
    DsProgram p = prog_proto;
    st = seq_partitioned_build(p, sched, n, M, C, G, wx, wy, wsr);
    if (st != BITNET_OK) return st;
    p.counters = static_cast<unsigned *>(workspace);
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
        slot->C = C;
        slot->parts = parts_set;
        slot->share = share_set;
        slot->ws = workspace;
        for (int i = 0; i < n; ++i) slot->ops[i] = user_ops[i];
        slot->prog = p;
    }
    return cuda_status(seq_launch(p, stream));
}

// ---- fixed scratch for bitnet_linear_noalloc -------------------------------
// Callers of that entry point cannot allocate, so its scratch is a static
// device array (every GPU that loads the library holds it until exit).  Host
// code must not use the symbol as a pointer: it is a host-side stand-in, and
// the device address is looked up once per device below.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device (looked up on the
// first call per device, with that device current); nullptr on failure.
void *noalloc_scratch(int dev)
{
    static std::atomic<void *> cache[kMaxDevices];
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    void *p = cache[dev].load();
    if (p) return p;
    void *q = nullptr;
    if (cudaGetSymbolAddress(&q, g_noalloc_scratch) != cudaSuccess || q == nullptr) return nullptr;
    cache[dev].store(q);
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

size_t bitnet_sequence_workspace_size(void) { return kSeqWorkspaceBytes; }

bitnet_status_t bitnet_sequence_plan(const bitnet_op_t *ops, int32_t n_ops, int64_t M, int32_t *wait_x,
                                     int32_t *wait_y)
{
    return seq_plan(ops, n_ops, M, wait_x, wait_y, ByteRange{0, 0});
}

bitnet_status_t bitnet_decode_sequence(const bitnet_op_t *ops, int32_t n_ops, int64_t M, void *workspace,
                                       size_t ws_bytes, cudaStream_t stream)
{
    return decode_sequence(ops, n_ops, M, workspace, ws_bytes, stream);
}

bitnet_status_t bitnet_sequence_schedule(const bitnet_op_t *ops, int32_t n_ops, int64_t M, int32_t *order)
{
    if (!order) return BITNET_ERR_INVALID_ARG;
    return seq_schedule(ops, n_ops, M, order, ByteRange{0, 0});
}

bitnet_status_t bitnet_sequence_layout(const bitnet_op_t *ops, int32_t n_ops, int64_t M, int32_t cluster_size,
                                       int32_t clusters, int32_t *order, int32_t *part_of, int32_t *slices,
                                       int32_t *n_parts, int32_t *part_clusters)
{
    if (!ops || n_ops < 1 || n_ops > BITNET_SEQ_MAX_OPS || !order || !part_of || !slices || !n_parts || !part_clusters)
        return BITNET_ERR_INVALID_ARG;
    if ((cluster_size != 4 && cluster_size != 8) || clusters < 1) return BITNET_ERR_INVALID_ARG;
    int32_t wx[BITNET_SEQ_MAX_OPS], wy[BITNET_SEQ_MAX_OPS], ord0[BITNET_SEQ_MAX_OPS];
    bitnet_status_t st = seq_schedule(ops, n_ops, M, ord0, ByteRange{0, 0});
    if (st != BITNET_OK) return st;
    bitnet_op_t sched[BITNET_SEQ_MAX_OPS];
    for (int k = 0; k < n_ops; ++k) sched[k] = ops[ord0[k]];
    st = seq_plan(sched, n_ops, M, wx, wy, ByteRange{0, 0});
    if (st != BITNET_OK) return st;
    static DsProgram proto;
    DsProgram p = proto;
    SeqLayout lay;
    st = seq_partitioned_build(p, sched, n_ops, M, cluster_size, clusters, wx, wy, ByteRange{0, 0}, &lay);
    if (st != BITNET_OK) return st;
    for (int k = 0; k < n_ops; ++k) {
        order[k] = ord0[lay.perm[k]];
        part_of[k] = lay.part_of[k];
        slices[k] = lay.slices[k];
    }
    *n_parts = p.n_parts;
    for (int q = 0; q < p.n_parts; ++q) part_clusters[q] = p.part_ncl[q];
    return BITNET_OK;
}

int bitnet_set_sequence_cluster(int cluster_size)
{
    if (cluster_size != 4 && cluster_size != 8) return -1;
    return g_seq_cluster.exchange(cluster_size);
}

int bitnet_set_sequence_partitions(int partitions)
{
    if (partitions < 0 || partitions > DS_MAX_PARTS) return -1;
    return g_seq_parts.exchange(partitions);
}

int bitnet_set_sequence_ring_share(int share)
{
    if (share < 1 || share > 4) return -1;
    return g_seq_ring_share.exchange(share);
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
