// pack_quant.cuh -- offline weight ternarisation/packing and the standalone
// per-token activation quantiser.
//
// BitNet model page, section "Model details", item "Quantization": ternary
// weights by absmean quantisation, 8-bit activations by per-token absmax
// quantisation; section "Model variants": the deployable weights are packed.
#pragma once

#include "common.cuh"
#include "exact_sumsq.cuh"

namespace bitnet {

// ---------------------------------------------------------------------------
// gamma = mean|W| in fp64, fixed order: each row left to right (one thread per
// row), then the row sums top to bottom (one thread).  The order is part of
// the contract: it makes gamma bit-reproducible against a sequential CPU sum.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) k_pack_rowsum(const float *__restrict__ w, int64_t N, int64_t K,
                                                     double *__restrict__ rowsum)
{
    const int64_t n = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N) return;
    const float4 *row = reinterpret_cast<const float4 *>(w + n * K);
    double acc = 0.0;
    const int64_t nv = K / 4;
    for (int64_t i = 0; i < nv; ++i) {
        const float4 v = __ldg(row + i);
        acc = __dadd_rn(acc, fabs((double)v.x));
        acc = __dadd_rn(acc, fabs((double)v.y));
        acc = __dadd_rn(acc, fabs((double)v.z));
        acc = __dadd_rn(acc, fabs((double)v.w));
    }
    rowsum[n] = acc;
}

__global__ void k_pack_gamma(const double *__restrict__ rowsum, int64_t N, int64_t K, float *__restrict__ gamma)
{
    if (blockIdx.x != 0 || threadIdx.x != 0) return;
    double total = 0.0;
    for (int64_t n = 0; n < N; ++n) total = __dadd_rn(total, rowsum[n]);
    gamma[0] = __double2float_rn(__ddiv_rn(total, (double)(N * K)));
}

// code = clamp(rne(w / d), -1, 1) + 1 with d = gamma + eps (IEEE fp32).
BITNET_DEVINL uint32_t ternary_code(float w, float d)
{
    float q = rintf(__fdiv_rn(w, d));
    q = fminf(fmaxf(q, -1.0f), 1.0f);
    return (uint32_t)((int)q + 1);
}

// One thread per 32-bit word = 16 consecutive weights of a row: weight
// 16g + 4j + b goes to byte b, bits 2j..2j+1.
__global__ void __launch_bounds__(256) k_pack_codes(const float *__restrict__ w, int64_t nwords, float eps,
                                                    const float *__restrict__ gamma, uint32_t *__restrict__ out)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nwords) return;
    const float d = __fadd_rn(gamma[0], eps);
    const float4 *src = reinterpret_cast<const float4 *>(w) + i * 4;
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float4 v = __ldg(src + j);
        word |= ternary_code(v.x, d) << (2 * j);
        word |= ternary_code(v.y, d) << (8 + 2 * j);
        word |= ternary_code(v.z, d) << (16 + 2 * j);
        word |= ternary_code(v.w, d) << (24 + 2 * j);
    }
    out[i] = word;
}

// ---------------------------------------------------------------------------
// Per-token absmax quantiser, one warp per row, natural [M][K] int8 output.
// s = 127 / max(max|x|, 1e-5); x_q = clamp(rne(x * s), -128, 127).
// ---------------------------------------------------------------------------
template <bool XF32>
BITNET_DEVINL float chunk_absmax(const uint4 v)
{
    if constexpr (XF32) {
        return fmaxf(fmaxf(fabsf(__uint_as_float(v.x)), fabsf(__uint_as_float(v.y))),
                     fmaxf(fabsf(__uint_as_float(v.z)), fabsf(__uint_as_float(v.w))));
    } else {
        // |bf16| bit patterns order like their values; compare in fp32
        const uint32_t m = 0x7fff7fffu;
        const uint32_t a = v.x & m, b = v.y & m, c = v.z & m, d = v.w & m;
        const float f0 = fmaxf(bf16_bits_lo(a), bf16_bits_hi(a));
        const float f1 = fmaxf(bf16_bits_lo(b), bf16_bits_hi(b));
        const float f2 = fmaxf(bf16_bits_lo(c), bf16_bits_hi(c));
        const float f3 = fmaxf(bf16_bits_lo(d), bf16_bits_hi(d));
        return fmaxf(fmaxf(f0, f1), fmaxf(f2, f3));
    }
}

// Quantise one 16-byte chunk (8 bf16 or 4 fp32 values); returns the packed
// int8 bytes in q.x (.y for bf16) and adds their sum to rs.
template <bool XF32>
BITNET_DEVINL uint2 chunk_quant(const uint4 v, float sc, int &rs)
{
    uint2 q;
    if constexpr (XF32) {
        const int a = quant_one(__uint_as_float(v.x), sc), b = quant_one(__uint_as_float(v.y), sc);
        const int c = quant_one(__uint_as_float(v.z), sc), d = quant_one(__uint_as_float(v.w), sc);
        rs += a + b + c + d;
        q.x = pack4_s8(a, b, c, d);
        q.y = 0;
    } else {
        const int a0 = quant_one(bf16_bits_lo(v.x), sc), a1 = quant_one(bf16_bits_hi(v.x), sc);
        const int b0 = quant_one(bf16_bits_lo(v.y), sc), b1 = quant_one(bf16_bits_hi(v.y), sc);
        const int c0 = quant_one(bf16_bits_lo(v.z), sc), c1 = quant_one(bf16_bits_hi(v.z), sc);
        const int d0 = quant_one(bf16_bits_lo(v.w), sc), d1 = quant_one(bf16_bits_hi(v.w), sc);
        rs += a0 + a1 + b0 + b1 + c0 + c1 + d0 + d1;
        q.x = pack4_s8(a0, a1, b0, b1);
        q.y = pack4_s8(c0, c1, d0, d1);
    }
    return q;
}

template <bool XF32>
__global__ void __launch_bounds__(256) k_quant_rows(const void *__restrict__ x, int64_t M, int64_t K,
                                                    int8_t *__restrict__ x_q, float *__restrict__ s,
                                                    int32_t *__restrict__ rowsum, const float *__restrict__ amax_in,
                                                    float *__restrict__ amax_zero)
{
    pdl_launch_dependents();
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t m = (int64_t)blockIdx.x * 8 + warp;
    if (m >= M) return;
    constexpr int EPC = XF32 ? 4 : 8; // elements per 16-byte chunk
    const int64_t nch = K / EPC;
    const uint4 *row = reinterpret_cast<const uint4 *>(static_cast<const char *>(x) + m * K * (XF32 ? 4 : 2));
    float amax = 0.0f;
    int64_t c = lane;
    if (amax_in) {
        amax = amax_in[m]; // the row maximum is given: one pass over x
    } else {
        for (; c + 96 < nch; c += 128) {
            const uint4 v0 = __ldg(row + c), v1 = __ldg(row + c + 32), v2 = __ldg(row + c + 64),
                        v3 = __ldg(row + c + 96);
            amax = fmaxf(amax, fmaxf(fmaxf(chunk_absmax<XF32>(v0), chunk_absmax<XF32>(v1)),
                                     fmaxf(chunk_absmax<XF32>(v2), chunk_absmax<XF32>(v3))));
        }
        for (; c < nch; c += 32) amax = fmaxf(amax, chunk_absmax<XF32>(__ldg(row + c)));
        amax = warp_max(amax);
    }
    const float sc = quant_scale(amax);
    int rs = 0;
    int8_t *qrow = x_q + m * K;
    for (c = lane; c < nch; c += 32) {
        const uint2 q = chunk_quant<XF32>(__ldg(row + c), sc, rs);
        if constexpr (XF32)
            reinterpret_cast<uint32_t *>(qrow)[c] = q.x;
        else
            reinterpret_cast<uint2 *>(qrow)[c] = q;
    }
    rs = warp_sum(rs);
    if (lane == 0) {
        s[m] = sc;
        if (rowsum) rowsum[m] = rs;
        if (amax_zero) amax_zero[m] = 0.0f;
    }
}

// One-read variant: each row is held in registers between the absmax and the
// quantise step, so x is read from HBM exactly once (the two-pass kernel above
// re-reads rows that no longer sit in cache once the input exceeds L2).  WPR
// warps share a row (8 / WPR rows per 256-thread CTA); every lane holds up to
// NCH <= QR_NCH 16-byte chunks of it (the fewest that hold the row: fewer
// registers, more rows in flight per SM).  Same arithmetic as k_quant_rows.
constexpr int QR_NCH = 16;

template <bool XF32, int WPR, int NCH>
__global__ void __launch_bounds__(256, NCH <= 12 ? 3 : 2) k_quant_rows_reg(const void *__restrict__ x, int64_t M, int64_t K,
                                                        int8_t *__restrict__ x_q, float *__restrict__ s,
                                                        int32_t *__restrict__ rowsum,
                                                        const float *__restrict__ amax_in,
                                                        float *__restrict__ amax_zero)
{
    __shared__ float red_max[8];
    __shared__ int red_sum[8];
    pdl_launch_dependents();
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int RPC = 8 / WPR; // rows per CTA
    const int wr = warp % WPR;   // this warp's part of the row
    const int64_t m = (int64_t)blockIdx.x * RPC + warp / WPR;
    const bool live = m < M;
    constexpr int EPC = XF32 ? 4 : 8; // elements per 16-byte chunk
    const int nch = (int)(K / EPC);
    const int c0 = wr * 32 + lane;
    const uint4 *row = reinterpret_cast<const uint4 *>(static_cast<const char *>(x) + (live ? m : 0) * K * (XF32 ? 4 : 2));
    uint4 v[NCH];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
        const int c = c0 + i * 32 * WPR;
        if (live && c < nch) {
            v[i] = __ldg(row + c);
            amax = fmaxf(amax, chunk_absmax<XF32>(v[i]));
        }
    }
    if (amax_in) {
        amax = live ? amax_in[m] : 0.0f; // the row maximum is given: no reduction
    } else {
        amax = warp_max(amax);
        if (WPR > 1) {
            if (lane == 0) red_max[warp] = amax;
            __syncthreads();
            const int w0 = warp - wr;
#pragma unroll
            for (int i = 0; i < WPR; ++i) amax = fmaxf(amax, red_max[w0 + i]);
        }
    }
    const float sc = quant_scale(amax);
    int rs = 0;
    int8_t *qrow = x_q + (live ? m : 0) * K;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
        const int c = c0 + i * 32 * WPR;
        if (live && c < nch) {
            const uint2 q = chunk_quant<XF32>(v[i], sc, rs);
            if constexpr (XF32)
                reinterpret_cast<uint32_t *>(qrow)[c] = q.x;
            else
                reinterpret_cast<uint2 *>(qrow)[c] = q;
        }
    }
    rs = warp_sum(rs);
    if (WPR > 1) {
        if (lane == 0) red_sum[warp] = rs;
        __syncthreads();
        rs = 0;
        const int w0 = warp - wr;
#pragma unroll
        for (int i = 0; i < WPR; ++i) rs += red_sum[w0 + i];
    }
    if (live && wr == 0 && lane == 0) {
        s[m] = sc;
        if (rowsum) rowsum[m] = rs;
        if (amax_zero) amax_zero[m] = 0.0f;
    }
}

// amax[0 .. n) <- 0 ahead of a kernel that folds row maxima into it with
// atomicMax (after the previous kernel, which may still read or write it).
__global__ void __launch_bounds__(128) k_zero_f32(float *__restrict__ amax, int n)
{
    pdl_launch_dependents();
    pdl_wait();
    for (int i = threadIdx.x; i < n; i += blockDim.x) amax[i] = 0.0f;
}

// ---------------------------------------------------------------------------
// RMS normalisation (subln) fused in front of the per-token absmax quantiser:
// y = (x * r) * g with r = 1 / sqrt(mean(x^2) + eps), then the quantiser on y.
// BitNet model page, "Model details" / "Architecture" (subln normalisation, no
// bias) and BitNetConfig (rms_norm_eps).  Same row layout as k_quant_rows_reg
// (WPR warps per row, 16-byte chunks in registers), so x is read from HBM once
// and x_q written in 8- or 4-byte pieces.  The sum of squares is the exact sum
// rounded once to binary64 (exact_sumsq.cuh: 128-bit integer partials anchored
// at the exponent of the row maximum, or a long accumulator for rows of very
// wide range), so no summation order enters the result; r is computed in
// binary64 (correctly rounded division and square root) and rounded once to
// binary32.  y is recomputed for the quantise step rather than kept.
// ---------------------------------------------------------------------------
constexpr int64_t kNormMaxK = 8192; // the 128-bit window and the long accumulator are sized for 8192 terms

// The EPC values of a 16-byte chunk as fp32.
template <bool XF32>
BITNET_DEVINL void chunk_values(const uint4 v, float (&f)[XF32 ? 4 : 8])
{
    if constexpr (XF32) {
        f[0] = __uint_as_float(v.x), f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z), f[3] = __uint_as_float(v.w);
    } else {
        f[0] = bf16_bits_lo(v.x), f[1] = bf16_bits_hi(v.x), f[2] = bf16_bits_lo(v.y), f[3] = bf16_bits_hi(v.y);
        f[4] = bf16_bits_lo(v.z), f[5] = bf16_bits_hi(v.z), f[6] = bf16_bits_lo(v.w), f[7] = bf16_bits_hi(v.w);
    }
}

// y = (x * r) * g for the EPC values of chunk c.
template <bool XF32>
BITNET_DEVINL void chunk_norm(const uint4 v, int c, float r, const float *__restrict__ g, float (&y)[XF32 ? 4 : 8])
{
    constexpr int EPC = XF32 ? 4 : 8;
    float gg[EPC];
    const float4 g0 = __ldg(reinterpret_cast<const float4 *>(g) + (EPC / 4) * c);
    gg[0] = g0.x, gg[1] = g0.y, gg[2] = g0.z, gg[3] = g0.w;
    if constexpr (!XF32) {
        const float4 g1 = __ldg(reinterpret_cast<const float4 *>(g) + 2 * c + 1);
        gg[4] = g1.x, gg[5] = g1.y, gg[6] = g1.z, gg[7] = g1.w;
    }
    chunk_values<XF32>(v, y);
#pragma unroll
    for (int j = 0; j < EPC; ++j) y[j] = __fmul_rn(__fmul_rn(y[j], r), gg[j]);
}

template <bool XF32, int WPR>
__global__ void __launch_bounds__(256) k_rmsnorm_quant_rows(const void *__restrict__ x, int64_t M, int64_t K,
                                                            const float *__restrict__ g, float eps,
                                                            int8_t *__restrict__ x_q, float *__restrict__ s,
                                                            int32_t *__restrict__ rowsum, float *__restrict__ amax_zero)
{
    constexpr int RPC = 8 / WPR;       // rows per CTA
    constexpr int EPC = XF32 ? 4 : 8;  // elements per 16-byte chunk
    __shared__ float red_x[8], red_y[8];
    __shared__ uint64_t red_lo[8], red_hi[8];
    __shared__ int red_fit[8], red_sum[8];
    __shared__ unsigned long long dig[RPC][SS_LONG_DIGITS];
    pdl_launch_dependents();
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wr = warp % WPR, lr = warp / WPR, w0 = warp - wr;
    const int64_t m = (int64_t)blockIdx.x * RPC + lr;
    const bool live = m < M;
    const int nch = (int)(K / EPC);
    const int c0 = wr * 32 + lane;
    const uint4 *row = reinterpret_cast<const uint4 *>(static_cast<const char *>(x) + (live ? m : 0) * K * (XF32 ? 4 : 2));
    uint4 v[QR_NCH];
    float xmax = 0.0f;
#pragma unroll
    for (int i = 0; i < QR_NCH; ++i) {
        const int c = c0 + i * 32 * WPR;
        if (live && c < nch) {
            v[i] = __ldg(row + c);
            xmax = fmaxf(xmax, chunk_absmax<XF32>(v[i]));
        }
    }
    // the exponent of the row maximum anchors the 128-bit window
    xmax = warp_max(xmax);
    if constexpr (WPR > 1) {
        if (lane == 0) red_x[warp] = xmax;
        __syncthreads();
#pragma unroll
        for (int i = 0; i < WPR; ++i) xmax = fmaxf(xmax, red_x[w0 + i]);
    }
    const uint32_t E = ss_exponent(xmax);
    SsWindow acc;
    if (E != 0) {
#pragma unroll
        for (int i = 0; i < QR_NCH; ++i) {
            const int c = c0 + i * 32 * WPR;
            if (live && c < nch) {
                float f[EPC];
                chunk_values<XF32>(v[i], f);
#pragma unroll
                for (int j = 0; j < EPC; ++j) ss_window_add(acc, f[j], E);
            }
        }
    }
    ss_warp_sum(acc.lo, acc.hi);
    bool row_slow = !__all_sync(0xffffffffu, acc.fits);
    uint64_t lo = acc.lo, hi = acc.hi;
    if constexpr (WPR > 1) {
        if (lane == 0) {
            red_lo[warp] = lo;
            red_hi[warp] = hi;
            red_fit[warp] = row_slow ? 0 : 1;
        }
        // a row with a value too far below its maximum takes the long accumulator
        const int any_slow = __syncthreads_or(row_slow ? 1 : 0);
        lo = hi = 0;
        row_slow = false;
#pragma unroll
        for (int i = 0; i < WPR; ++i) {
            ss_add128(lo, hi, red_lo[w0 + i], red_hi[w0 + i]);
            row_slow = row_slow || red_fit[w0 + i] == 0;
        }
        if (any_slow) { // uniform over the CTA
            if (wr == 0 && lane < SS_LONG_DIGITS) dig[lr][lane] = 0ull;
            __syncthreads();
            if (row_slow) {
#pragma unroll
                for (int i = 0; i < QR_NCH; ++i) {
                    const int c = c0 + i * 32 * WPR;
                    if (live && c < nch) {
                        float f[EPC];
                        chunk_values<XF32>(v[i], f);
#pragma unroll
                        for (int j = 0; j < EPC; ++j) ss_long_add(dig[lr], f[j]);
                    }
                }
            }
            __syncthreads();
        }
    } else if (row_slow) { // uniform over the warp, which holds the whole row
        if (lane < SS_LONG_DIGITS) dig[lr][lane] = 0ull;
        __syncwarp();
#pragma unroll
        for (int i = 0; i < QR_NCH; ++i) {
            const int c = c0 + i * 32;
            if (live && c < nch) {
                float f[EPC];
                chunk_values<XF32>(v[i], f);
#pragma unroll
                for (int j = 0; j < EPC; ++j) ss_long_add(dig[lr], f[j]);
            }
        }
        __syncwarp();
    }
    // every lane evaluates r (the same binary64 operations, no broadcast needed)
    const double ss = row_slow ? ss_long_round(dig[lr]) : (E ? ss_window_round(lo, hi, E) : 0.0);
    const double mean = __ddiv_rn(ss, (double)K);
    const float r = __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(mean, (double)eps))));
    float ymax = 0.0f;
#pragma unroll
    for (int i = 0; i < QR_NCH; ++i) {
        const int c = c0 + i * 32 * WPR;
        if (live && c < nch) {
            float y[EPC];
            chunk_norm<XF32>(v[i], c, r, g, y);
#pragma unroll
            for (int j = 0; j < EPC; ++j) ymax = fmaxf(ymax, fabsf(y[j]));
        }
    }
    ymax = warp_max(ymax);
    if constexpr (WPR > 1) {
        if (lane == 0) red_y[warp] = ymax;
        __syncthreads();
#pragma unroll
        for (int i = 0; i < WPR; ++i) ymax = fmaxf(ymax, red_y[w0 + i]);
    }
    const float sc = quant_scale(ymax);
    int rs = 0;
    int8_t *qrow = x_q + (live ? m : 0) * K;
#pragma unroll
    for (int i = 0; i < QR_NCH; ++i) {
        const int c = c0 + i * 32 * WPR;
        if (live && c < nch) {
            float y[EPC];
            chunk_norm<XF32>(v[i], c, r, g, y);
            int q[EPC];
#pragma unroll
            for (int j = 0; j < EPC; ++j) {
                q[j] = quant_one(y[j], sc);
                rs += q[j];
            }
            if constexpr (XF32)
                reinterpret_cast<uint32_t *>(qrow)[c] = pack4_s8(q[0], q[1], q[2], q[3]);
            else
                reinterpret_cast<uint2 *>(qrow)[c] = make_uint2(pack4_s8(q[0], q[1], q[2], q[3]),
                                                                pack4_s8(q[4], q[5], q[6], q[7]));
        }
    }
    rs = warp_sum(rs);
    if constexpr (WPR > 1) {
        if (lane == 0) red_sum[warp] = rs;
        __syncthreads();
        rs = 0;
#pragma unroll
        for (int i = 0; i < WPR; ++i) rs += red_sum[w0 + i];
    }
    if (live && wr == 0 && lane == 0) {
        s[m] = sc;
        if (rowsum) rowsum[m] = rs;
        if (amax_zero) amax_zero[m] = 0.0f;
    }
}

} // namespace bitnet
