// exact_sumsq.cuh -- sum of squares of a row, exact, rounded once to binary64.
//
// The RMS normalisation in front of a BitLinear (BitNet model page, "Model
// details" / "Architecture": subln normalisation; BitNetConfig: rms_norm_eps)
// needs mean(x^2).  Its value here is the exact sum of the squares rounded once
// to the nearest binary64, ties to even: one well-defined number whatever the
// order in which threads add, so a different grid or block shape cannot move a
// quantised code.
//
// A nonzero finite binary32 value is v = +-mant * 2^(e - 150) with mant < 2^24
// an integer and e >= 1 the biased exponent field (1 for subnormals, which have
// no hidden bit), so v^2 = mant^2 * 2^(2e - 300) exactly.
//
// Fast path: with E the largest exponent of the row, every term with
// e >= E - 33 is the integer mant^2 << (2(e - E) + 67) in units of
// 2^(2E - 367); each is below 2^115, so up to 8192 of them add up exactly in
// 128 bits.  Integer addition is exact and order-free: threads, warps and the
// block combine partial sums in any order.
// Slow path (a row with a nonzero value more than 33 binades below its
// largest): every term goes into a long accumulator of 32-bit digits in shared
// memory (units of 2^-298), added with 64-bit atomics, carries resolved once.
#pragma once

#include "common.cuh"

namespace bitnet {

constexpr int SS_WINDOW_SPREAD = 33; // largest e_max - e a fast-path term may have
constexpr int SS_LONG_DIGITS = 20;   // 640 bits: terms < 2^554 in units of 2^-298, 8192 of them < 2^567

// Biased exponent of |v| for the sum of squares: 0 for zero, 1 for subnormals.
BITNET_DEVINL uint32_t ss_exponent(float v)
{
    const uint32_t b = __float_as_uint(v) & 0x7fffffffu;
    if (b == 0) return 0;
    const uint32_t f = b >> 23;
    return f ? f : 1u;
}

// mant^2 and e of a nonzero |v| (bits b = |v| as binary32).
BITNET_DEVINL uint64_t ss_mant2(uint32_t b, int &e)
{
    const uint32_t f = b >> 23;
    const uint64_t mant = (b & 0x7fffffu) | (f ? 0x800000u : 0u);
    e = f ? (int)f : 1;
    return mant * mant;
}

// 128-bit partial sum of the fast path (units of 2^(2E - 367)).
struct SsWindow {
    uint64_t lo = 0, hi = 0;
    bool fits = true; // false once a term lies below the window
};

BITNET_DEVINL void ss_add128(uint64_t &lo, uint64_t &hi, uint64_t alo, uint64_t ahi)
{
    lo += alo;
    hi += ahi + (lo < alo ? 1ull : 0ull);
}

// a += v^2 for a row whose largest exponent is E >= 1.
BITNET_DEVINL void ss_window_add(SsWindow &a, float v, uint32_t E)
{
    const uint32_t b = __float_as_uint(v) & 0x7fffffffu;
    if (b == 0) return;
    int e;
    const uint64_t m2 = ss_mant2(b, e);
    const int sh = 2 * (e - (int)E) + 2 * SS_WINDOW_SPREAD + 1; // 0 .. 67 inside the window
    if (sh < 0) {
        a.fits = false;
        return;
    }
    uint64_t tlo, thi;
    if (sh >= 64) {
        tlo = 0;
        thi = m2 << (sh - 64);
    } else {
        tlo = m2 << sh;
        thi = sh ? (m2 >> (64 - sh)) : 0;
    }
    ss_add128(a.lo, a.hi, tlo, thi);
}

// Sum of the 128-bit partials of a warp (every lane gets the total).
BITNET_DEVINL void ss_warp_sum(uint64_t &lo, uint64_t &hi)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t olo = __shfl_xor_sync(0xffffffffu, lo, o);
        const uint64_t ohi = __shfl_xor_sync(0xffffffffu, hi, o);
        ss_add128(lo, hi, olo, ohi);
    }
}

// (hi:lo) * 2^p2 rounded to the nearest binary64, ties to even.  The caller
// keeps the result inside the normal range (p2 >= -1000, (hi:lo) * 2^p2 <
// 2^1000).
BITNET_DEVINL double ss_round128(uint64_t lo, uint64_t hi, int p2)
{
    if ((lo | hi) == 0) return 0.0;
    const int top = hi ? 127 - __clzll((long long)hi) : 63 - __clzll((long long)lo);
    uint64_t mant;
    int sh = 0;
    if (top <= 52) {
        mant = lo; // hi == 0
    } else {
        sh = top - 52; // 1 .. 75
        mant = sh >= 64 ? (hi >> (sh - 64)) : ((lo >> sh) | (hi << (64 - sh)));
        const int r = sh - 1; // position of the rounding bit
        const uint64_t round = r >= 64 ? (hi >> (r - 64)) & 1ull : (lo >> r) & 1ull;
        const bool sticky = r >= 64 ? (lo != 0 || (hi & ((1ull << (r - 64)) - 1ull)) != 0)
                                    : (lo & ((1ull << r) - 1ull)) != 0;
        if (round && (sticky || (mant & 1ull))) ++mant; // mant <= 2^53: exact in binary64
    }
    const double scale = __longlong_as_double((long long)(1023 + p2 + sh) << 52);
    return __dmul_rn(__ull2double_rn(mant), scale);
}

// Fast-path result of a row: the exact sum (hi:lo) in units of 2^(2E - 367).
BITNET_DEVINL double ss_window_round(uint64_t lo, uint64_t hi, uint32_t E)
{
    return ss_round128(lo, hi, 2 * (int)E - 300 - (2 * SS_WINDOW_SPREAD + 1));
}

// Slow path: dig[d] collects (carry-save) digit d of the long integer
// sum of mant^2 * 2^(2e - 2); the value is that integer * 2^-298.
BITNET_DEVINL void ss_long_add(unsigned long long *dig, float v)
{
    const uint32_t b = __float_as_uint(v) & 0x7fffffffu;
    if (b == 0) return;
    int e;
    const uint64_t m2 = ss_mant2(b, e);
    const int o = 2 * e - 2, d = o >> 5, s = o & 31;
    const uint64_t lo = m2 << s, hi = s ? m2 >> (64 - s) : 0ull;
    atomicAdd(&dig[d], (unsigned long long)(lo & 0xffffffffull));
    atomicAdd(&dig[d + 1], (unsigned long long)(lo >> 32));
    if (hi) atomicAdd(&dig[d + 2], (unsigned long long)hi);
}

// Slow-path result: resolve the carries, take the top 128 bits (lower nonzero
// digits folded into the lowest bit, which lies below the rounding bit) and
// round once.
__device__ __noinline__ double ss_long_round(const unsigned long long *dig)
{
    uint32_t w[SS_LONG_DIGITS];
    unsigned long long c = 0;
    int top = -1;
    for (int i = 0; i < SS_LONG_DIGITS; ++i) {
        const unsigned long long t = dig[i] + c;
        w[i] = (uint32_t)t;
        c = t >> 32;
        if (w[i]) top = i;
    }
    if (top < 0) return 0.0;
    const int base = top >= 3 ? top - 3 : 0;
    uint32_t sticky = 0;
    for (int i = 0; i < base; ++i) sticky |= w[i];
    auto digit = [&](int i) -> uint64_t { return i < SS_LONG_DIGITS ? (uint64_t)w[i] : 0ull; };
    const uint64_t lo = digit(base) | (digit(base + 1) << 32) | (sticky ? 1ull : 0ull);
    const uint64_t hi = digit(base + 2) | (digit(base + 3) << 32);
    return ss_round128(lo, hi, 32 * base - 298);
}

} // namespace bitnet
