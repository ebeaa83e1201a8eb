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
// QR_NCH 16-byte chunks of it.  Same arithmetic as k_quant_rows.
constexpr int QR_NCH = 16;

template <bool XF32, int WPR>
__global__ void __launch_bounds__(256) k_quant_rows_reg(const void *__restrict__ x, int64_t M, int64_t K,
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
    uint4 v[QR_NCH];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < QR_NCH; ++i) {
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
    for (int i = 0; i < QR_NCH; ++i) {
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
// bias) and BitNetConfig (rms_norm_eps).  Each row is held in registers by
// 128 or 256 threads, so x is read once.  The sum of squares is the exact sum
// rounded once to binary64 (exact_sumsq.cuh: 128-bit integer partials, or a
// long accumulator for rows of very wide range), so no summation order enters
// the result; r is computed in binary64 (correctly rounded division and square
// root) and rounded once to binary32.
// ---------------------------------------------------------------------------
constexpr int RQ_MAX_PER_THREAD = 32; // elements a thread holds in registers

// TPR threads per row (128 or 256), 256 / TPR rows per CTA.
template <bool XF32, int TPR>
__global__ void __launch_bounds__(256) k_rmsnorm_quant_rows(const void *__restrict__ x, int64_t M, int64_t K,
                                                            const float *__restrict__ g, float eps,
                                                            int8_t *__restrict__ x_q, float *__restrict__ s,
                                                            int32_t *__restrict__ rowsum, float *__restrict__ amax_zero)
{
    constexpr int RPC = 256 / TPR;         // rows per CTA
    constexpr int WPR = TPR / 32;          // warps per row
    __shared__ uint64_t red_lo[RPC][WPR], red_hi[RPC][WPR];
    __shared__ unsigned long long dig[RPC][SS_LONG_DIGITS];
    __shared__ uint32_t red_e[RPC][WPR];
    __shared__ int red_fit[RPC][WPR];
    __shared__ float red_max[RPC][WPR];
    __shared__ int red_sum[RPC][WPR];
    __shared__ float bcast[RPC][2];
    pdl_launch_dependents();
    pdl_wait();
    const int lr = threadIdx.x / TPR;      // row of this CTA
    const int t = threadIdx.x % TPR;       // thread within the row
    const int wr = t >> 5, lane = t & 31;  // warp within the row
    const int64_t m = (int64_t)blockIdx.x * RPC + lr;
    const bool live = m < M;
    float v[RQ_MAX_PER_THREAD];
    const int n = live ? (int)((K + TPR - 1 - t) / TPR) : 0; // elements k = t + TPR * e, e < n
    if constexpr (XF32) {
        const float *row = static_cast<const float *>(x) + (live ? m : 0) * K;
#pragma unroll
        for (int e = 0; e < RQ_MAX_PER_THREAD; ++e)
            if (e < n) v[e] = __ldg(row + t + (int64_t)e * TPR);
    } else {
        const unsigned short *row = static_cast<const unsigned short *>(x) + (live ? m : 0) * K;
#pragma unroll
        for (int e = 0; e < RQ_MAX_PER_THREAD; ++e)
            if (e < n) v[e] = __uint_as_float((uint32_t)__ldg(row + t + (int64_t)e * TPR) << 16);
    }
    // largest exponent of the row (anchors the 128-bit window)
    uint32_t emax = 0;
#pragma unroll
    for (int e = 0; e < RQ_MAX_PER_THREAD; ++e)
        if (e < n) emax = max(emax, ss_exponent(v[e]));
    emax = __reduce_max_sync(0xffffffffu, emax);
    if (lane == 0) red_e[lr][wr] = emax;
    if (t < SS_LONG_DIGITS) dig[lr][t] = 0ull;
    __syncthreads();
    uint32_t E = 0;
#pragma unroll
    for (int w = 0; w < WPR; ++w) E = max(E, red_e[lr][w]);
    SsWindow acc;
    if (E != 0) {
#pragma unroll
        for (int e = 0; e < RQ_MAX_PER_THREAD; ++e)
            if (e < n) ss_window_add(acc, v[e], E);
    }
    ss_warp_sum(acc.lo, acc.hi);
    const bool fits = __all_sync(0xffffffffu, acc.fits);
    if (lane == 0) {
        red_lo[lr][wr] = acc.lo;
        red_hi[lr][wr] = acc.hi;
        red_fit[lr][wr] = fits ? 1 : 0;
    }
    __syncthreads();
    // a row with a value too far below its largest takes the long accumulator
    bool row_slow = false, any_slow = false;
#pragma unroll
    for (int q = 0; q < RPC; ++q) {
        bool f = true;
#pragma unroll
        for (int w = 0; w < WPR; ++w) f = f && red_fit[q][w] != 0;
        if (q == lr) row_slow = !f;
        any_slow = any_slow || !f;
    }
    if (any_slow) { // uniform over the CTA
        if (row_slow) {
#pragma unroll
            for (int e = 0; e < RQ_MAX_PER_THREAD; ++e)
                if (e < n) ss_long_add(dig[lr], v[e]);
        }
        __syncthreads();
    }
    if (t == 0) {
        double ss;
        if (row_slow) {
            ss = ss_long_round(dig[lr]);
        } else {
            uint64_t lo = 0, hi = 0;
            for (int w = 0; w < WPR; ++w) ss_add128(lo, hi, red_lo[lr][w], red_hi[lr][w]);
            ss = E ? ss_window_round(lo, hi, E) : 0.0;
        }
        const double mean = __ddiv_rn(ss, (double)K);
        bcast[lr][0] = __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(mean, (double)eps))));
    }
    __syncthreads();
    const float r = bcast[lr][0];
    float mx = 0.0f;
#pragma unroll
    for (int e = 0; e < RQ_MAX_PER_THREAD; ++e)
        if (e < n) {
            v[e] = __fmul_rn(__fmul_rn(v[e], r), __ldg(g + t + e * TPR));
            mx = fmaxf(mx, fabsf(v[e]));
        }
    mx = warp_max(mx);
    if (lane == 0) red_max[lr][wr] = mx;
    __syncthreads();
    if (t == 0) {
        float am = 0.0f;
        for (int w = 0; w < WPR; ++w) am = fmaxf(am, red_max[lr][w]);
        bcast[lr][1] = quant_scale(am);
    }
    __syncthreads();
    const float sc = bcast[lr][1];
    int rs = 0;
    int8_t *qrow = x_q + (live ? m : 0) * K;
#pragma unroll
    for (int e = 0; e < RQ_MAX_PER_THREAD; ++e)
        if (e < n) {
            const int q = quant_one(v[e], sc);
            qrow[t + e * TPR] = (int8_t)q;
            rs += q;
        }
    rs = warp_sum(rs);
    if (lane == 0) red_sum[lr][wr] = rs;
    __syncthreads();
    if (t == 0 && live) {
        int tot = 0;
        for (int w = 0; w < WPR; ++w) tot += red_sum[lr][w];
        s[m] = sc;
        if (rowsum) rowsum[m] = tot;
        if (amax_zero) amax_zero[m] = 0.0f;
    }
}

} // namespace bitnet
