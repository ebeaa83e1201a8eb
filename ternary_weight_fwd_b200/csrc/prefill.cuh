// prefill.cuh -- large-M (prefill) BitLinear on the 5th-generation tensor
// cores: tcgen05.mma kind::i8, the ternary weights as the A operand in tensor
// memory, int32 accumulators in tensor memory.
//
// BitNet model page, "Model details" / "Quantization" (W1.58A8) and
// "Architecture" (BitLinear without bias, ReLU^2 in the FFN).
//
// The product is formed transposed, D[n, t] = sum_k W_q[n, k] * x_q[t, k]:
// 128 weight rows sit on the 128 TMEM lanes (MMA M), 192 tokens on the MMA N
// dimension.  Unpacked weights go from registers into tensor memory
// (tcgen05.st) and never through shared memory, and each unpacked stage serves
// 192 tokens.  Shared memory carries only the TMA copies of x_q and of the
// packed codes, and the tensor cores' reads of x_q.
//
// One persistent CTA per SM, warp-specialised, 448 threads:
//   warps 0-3   epilogue, warp w on TMEM lanes 32w..32w+31: gamma/s[t] of a
//               unit's tokens into shared memory while its MMAs run; then
//               tcgen05.ld 32 tokens of its rows at a time, dequantise
//               (acc * gamma/s[t]), write the chunk transposed into a staging
//               buffer (token rows) and send it with one TMA store; FFN: lanes
//               16-31 hold the up rows of the gate rows in lanes 0-15 and hand
//               their values over by warp shuffle
//   warps 4-11  unpackers, warp w on lanes 32(w%4)..: the 2-bit codes of one
//               64-k half of a stage -> signed int8 -> tcgen05.st
//   warp 12     producer: TMA (no multicast) of x_q (64-token boxes, 128-byte
//               swizzle) and of the packed weight rows
//   warp 13     TMEM owner + MMA issuer (one elected thread)
// Stage: 128 weight rows x 192 tokens x 128 k.  6 shared-memory stages, 4
// tensor-memory weight stages.  Accumulators: a ring of four 96-column slots
// of 96 tokens; a tile takes two consecutive slots, so the MMAs of tile i + 1
// write the slots of tile i - 1 while the epilogue reads those of tile i.
// FFN tiles: lanes 32q..32q+15 hold gate rows n0+16q..n0+16q+15 and lanes
// 32q+16..32q+31 the up rows with the same indices.
// Work units: whole tiles for the full waves; a partly filled last wave runs
// each of its tiles as Q = 2, 3 or 6 units of 192 / Q tokens (a multiple of
// the 32-token output chunk) on separate CTAs.
// Units own disjoint outputs: nothing is combined across CTAs.
#pragma once

#include "common.cuh"

namespace bitnet {

constexpr int PF_WM = 128;                     // weight rows per tile: MMA M, TMEM lanes
constexpr int PF_TN = 192;                     // tokens per tile
constexpr int PF_HN = 96;                      // tokens per accumulator slot (one MMA's N)
constexpr int PF_BK = 128;                     // k per stage
constexpr int PF_STAGES = 6;
constexpr int PF_XBOX = 64;                    // token rows per x_q TMA box
constexpr int PF_X_BYTES = PF_TN * PF_BK;      // 24 KiB of x_q
constexpr int PF_WP_BYTES = PF_WM * PF_BK / 4; // 4 KiB of packed codes
constexpr int PF_STAGE_BYTES = PF_X_BYTES + PF_WP_BYTES;
constexpr int PF_A_STAGES = 4;
constexpr uint32_t PF_A_COLS = PF_BK / 4;      // TMEM columns of one unpacked stage
constexpr int PF_D_SLOTS = 4;
constexpr uint32_t PF_A_COL0 = PF_D_SLOTS * PF_HN;
constexpr uint32_t PF_TMEM_COLS = 512;
constexpr int PF_OBUF = 32 * 32 * 4;           // one output staging buffer: 32 tokens x 32 fp32
constexpr int PF_OUT_BYTES = 4 * 2 * PF_OBUF;  // per epilogue warp, double-buffered
constexpr int PF_R_BYTES = 4 * 2 * PF_TN * 4;  // per epilogue warp: gamma0/s and gamma1/s of a unit's tokens
constexpr int PF_HDR = 1024;
constexpr int PF_SMEM = PF_HDR + PF_STAGES * PF_STAGE_BYTES + PF_OUT_BYTES + PF_R_BYTES + 1024; // + alignment slack
constexpr int PF_THREADS = 448;
constexpr int PF_EPI_WARPS = 4;
constexpr int PF_UNPACK_WARP0 = 4;
constexpr int PF_UNPACK_WARPS = 8;
constexpr int PF_TMA_WARP = 12;
constexpr int PF_MMA_WARP = 13;
static_assert(PF_A_COL0 + PF_A_STAGES * PF_A_COLS == PF_TMEM_COLS, "tensor-memory columns");
static_assert(PF_STAGE_BYTES % 1024 == 0, "stages keep the 1024-byte alignment of the 128-byte swizzle");
static_assert(PF_THREADS == 32 * (PF_MMA_WARP + 1), "warp roles");
static_assert(PF_TN == 2 * PF_HN && PF_HN % 32 == 0 && (PF_HN * PF_BK) % 1024 == 0, "token slots");
static_assert(PF_TN % PF_XBOX == 0, "x_q boxes");

// kind::i8 instruction descriptor: D = s32, A = s8, B = s8, both K-major,
// M = 128, N = n (a multiple of 16, <= 256).
BITNET_DEVINL uint32_t pf_idesc(int n)
{
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(PF_WM >> 4) << 24);
}

struct PrefillArgs {
    int M, N, K;
    int num_t, num_w, num_k, num_tiles; // token tiles, weight tiles (FFN: 64 gate + 64 up rows)
    const float *gamma0, *gamma1;
    const float *s;       // [M] per-token scales
    void *y;              // [M][N] fp32, or bf16 when y_bf16
    float *y_amax;        // optional [M]: max |y| per row, folded in with atomicMax (zeroed beforehand)
    int32_t *acc0, *acc1; // optional [M][N]
    int y_bf16;           // store y as bf16 (nearest even of the fp32 value)
    int tma_out;          // rows of y are 16-byte multiples: staged chunks, TMA stores
    int full_units;       // whole tiles (units [0, full_units))
    int tail_q;           // units per remaining tile (1: none; 2, 3 or 6)
    int num_units;        // full_units + (num_tiles - full_units) * tail_q
};

// Unit u: tokens [t0, t0 + ntok) (ntok a multiple of 16; 0: nothing to do) of
// weight tile wt.  Token tiles vary fastest, so CTAs that run at the same time
// share weight tiles.
struct PfUnit {
    int t0, ntok, wt;
};

BITNET_DEVINL PfUnit pf_unit(const PrefillArgs &a, int u)
{
    int tile, q = 0, qn = 1;
    if (u < a.full_units) {
        tile = u;
    } else {
        const int v = u - a.full_units;
        tile = a.full_units + v / a.tail_q;
        q = v % a.tail_q;
        qn = a.tail_q;
    }
    PfUnit r;
    const int span = PF_TN / qn;
    r.wt = tile / a.num_t;
    r.t0 = (tile % a.num_t) * PF_TN + q * span;
    const int left = a.M - r.t0;
    r.ntok = left <= 0 ? 0 : min(span, (left + 15) & ~15);
    return r;
}

// codes {0,1,2} (one per byte) -> int8 {-1,0,1}: per byte (c | 0x80) - 1 cannot
// borrow across bytes, xor 0x80 restores the sign.
BITNET_DEVINL uint32_t codes_to_s8(uint32_t c)
{
    return ((c | 0x80808080u) - 0x01010101u) ^ 0x80808080u;
}

// 16 packed bytes: words g = 4h .. 4h+3 of a stage row, word g holding k = 16g
// .. 16g+15 with k = 16g + 4j + b in byte b, bits 2j.  Output word 4(g - 4h) + j
// holds k = 16g + 4j + 0..3 in bytes 0..3, i.e. TMEM column 4g + j of the stage.
BITNET_DEVINL void pf_unpack16(const uint4 p, uint32_t (&o)[16])
{
    constexpr uint32_t M3 = 0x03030303u;
    const uint32_t wv[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
    for (int w = 0; w < 4; ++w)
#pragma unroll
        for (int j = 0; j < 4; ++j) o[4 * w + j] = codes_to_s8((wv[w] >> (2 * j)) & M3);
}

// A bounded wait whose outcome is the same on every lane of the warp.
BITNET_DEVINL bool mbar_wait_warp(uint64_t *bar, uint32_t parity)
{
    return __all_sync(0xffffffffu, mbar_wait(bar, parity)) != 0;
}

// Stores one lane's 32 outputs y[tb + j][n] (j < 32, tokens below M only)
// straight to global memory (rows of y that are not 16-byte multiples).
BITNET_DEVINL void pf_emit_direct(const PrefillArgs &a, const float (&o)[32], int tb, int n, bool nok, bool obf)
{
    const int jn = min(32, a.M - tb);
    if (obf) {
        uint16_t *y = static_cast<uint16_t *>(a.y) + (size_t)tb * a.N + n;
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (nok && j < jn) y[(size_t)j * a.N] = (uint16_t)bf16_rn_bits(o[j]);
    } else {
        float *y = static_cast<float *>(a.y) + (size_t)tb * a.N + n;
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (nok && j < jn) y[(size_t)j * a.N] = o[j];
    }
}

// Folds the magnitudes of the chunk's outputs (lanes with nok) into the per-token maxima.
BITNET_DEVINL void pf_token_max(const PrefillArgs &a, const float (&o)[32], int tb, bool nok, bool obf)
{
    const int lane = threadIdx.x & 31;
    const int jn = min(32, a.M - tb);
    uint32_t mine = 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const uint32_t m = __reduce_max_sync(0xffffffffu, nok ? out_mag_bits(o[j], obf) : 0u);
        if (lane == j) mine = m;
    }
    if (lane < jn && mine != 0u) atomicMax(reinterpret_cast<unsigned *>(a.y_amax) + tb + lane, mine);
}

// The int32 sums of one lane's 32 tokens (acc may be null: nothing stored).
BITNET_DEVINL void pf_store_acc(int32_t *acc, const PrefillArgs &a, const uint32_t (&v)[32], int tb, int n, bool nok)
{
    if (!acc || !nok) return;
    const int jn = min(32, a.M - tb);
    int32_t *p = acc + (size_t)tb * a.N + n;
#pragma unroll
    for (int j = 0; j < 32; ++j)
        if (j < jn) p[(size_t)j * a.N] = (int32_t)v[j];
}

template <bool FFN>
__global__ void __launch_bounds__(PF_THREADS, 1)
    k_prefill(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW0,
              const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmY, const PrefillArgs a)
{
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *fullx = reinterpret_cast<uint64_t *>(smem); // x_q of a stage landed
    uint64_t *fullw = fullx + PF_STAGES;                  // packed codes of a stage landed
    uint64_t *empty = fullw + PF_STAGES;                  // the stage's MMAs are done
    uint64_t *afull = empty + PF_STAGES;                  // unpacked weights in TMEM
    uint64_t *aempty = afull + PF_A_STAGES;
    uint64_t *dfull = aempty + PF_A_STAGES;               // accumulator slot complete
    uint64_t *dempty = dfull + PF_D_SLOTS;                // accumulator slot read out
    uint64_t *mma_done = dempty + PF_D_SLOTS;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    unsigned char *stages = smem + PF_HDR;
    unsigned char *obufs = stages + PF_STAGES * PF_STAGE_BYTES;
    float *rbuf = reinterpret_cast<float *>(obufs + PF_OUT_BYTES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < PF_STAGES; ++s) {
            mbar_init(&fullx[s], 1);
            mbar_init(&fullw[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < PF_A_STAGES; ++s) {
            mbar_init(&afull[s], PF_UNPACK_WARPS); // one arrival per unpack warp
            mbar_init(&aempty[s], 1);
        }
        for (int d = 0; d < PF_D_SLOTS; ++d) {
            mbar_init(&dfull[d], 1);
            mbar_init(&dempty[d], PF_EPI_WARPS); // one arrival per epilogue warp
        }
        mbar_init(mma_done, 1);
        fence_mbarrier_init();
    }
    if (warp == PF_TMA_WARP && lane == 0) {
        prefetch_tensormap(&tmX);
        prefetch_tensormap(&tmW0);
        if (FFN) prefetch_tensormap(&tmW1);
        if (a.tma_out) prefetch_tensormap(&tmY);
    }
    if (warp == PF_MMA_WARP) {
        tmem_alloc(tmem_slot, PF_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_launch_dependents();

    if (warp == PF_TMA_WARP) {
        // ---------------- producer ----------------
        if (lane == 0) {
            pdl_wait();
            int st = 0;
            uint32_t ph = 0;
            uint32_t issued = 0, last_par = 0; // per stage bit flags
            bool ok = true;
            for (int unit = blockIdx.x; unit < a.num_units && ok; unit += gridDim.x) {
                const PfUnit un = pf_unit(a, unit);
                if (un.ntok <= 0) continue;
                const int nbox = (un.ntok + PF_XBOX - 1) / PF_XBOX;
                for (int kb = 0; kb < a.num_k; ++kb) {
                    if (!mbar_wait(&empty[st], ph ^ 1)) {
                        ok = false;
                        break;
                    }
                    unsigned char *xs = stages + st * PF_STAGE_BYTES;
                    unsigned char *wp = xs + PF_X_BYTES;
                    mbar_arrive_expect_tx(&fullw[st], PF_WP_BYTES);
                    if constexpr (FFN) {
                        // rows 32q..32q+15 gate, 32q+16..32q+31 up (16-row boxes)
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            tma_load_2d(wp + i * (PF_WP_BYTES / 8), (i & 1) ? &tmW1 : &tmW0, kb * (PF_BK / 4),
                                        un.wt * (PF_WM / 2) + (i >> 1) * 16, &fullw[st]);
                    } else {
                        tma_load_2d(wp, &tmW0, kb * (PF_BK / 4), un.wt * PF_WM, &fullw[st]);
                    }
                    mbar_arrive_expect_tx(&fullx[st], nbox * PF_XBOX * PF_BK);
                    for (int b = 0; b < nbox; ++b)
                        tma_load_2d(xs + b * PF_XBOX * PF_BK, &tmX, kb * PF_BK, un.t0 + b * PF_XBOX, &fullx[st]);
                    issued |= 1u << st;
                    last_par = (last_par & ~(1u << st)) | (ph << st);
                    if (++st == PF_STAGES) {
                        st = 0;
                        ph ^= 1;
                    }
                }
            }
            // let every copy this CTA issued land before the CTA can exit
            for (int s = 0; s < PF_STAGES; ++s)
                if (issued & (1u << s)) {
                    mbar_wait_drain(&fullw[s], (last_par >> s) & 1);
                    mbar_wait_drain(&fullx[s], (last_par >> s) & 1);
                }
        }
    } else if (warp == PF_MMA_WARP) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            int st = 0, as = 0;
            uint32_t ph = 0, aph = 0, pos = 0;
            bool ok = true;
            for (int unit = blockIdx.x; unit < a.num_units && ok; unit += gridDim.x) {
                const PfUnit un = pf_unit(a, unit);
                if (un.ntok <= 0) continue;
                const uint32_t p0 = pos, p1 = pos + 1;
                pos += 2;
                const uint32_t sl0 = p0 % PF_D_SLOTS, sl1 = p1 % PF_D_SLOTS;
                if (!mbar_wait(&dempty[sl0], ((p0 / PF_D_SLOTS) & 1) ^ 1) ||
                    !mbar_wait(&dempty[sl1], ((p1 / PF_D_SLOTS) & 1) ^ 1))
                    break;
                tc_fence_after();
                const int n0 = min(un.ntok, PF_HN), n1 = un.ntok - PF_HN;
                const uint32_t id0 = pf_idesc(n0), id1 = n1 > 0 ? pf_idesc(n1) : 0u;
                const uint32_t d0 = tmem_base + sl0 * PF_HN, d1 = tmem_base + sl1 * PF_HN;
                for (int kb = 0; kb < a.num_k; ++kb) {
                    if (!mbar_wait(&fullx[st], ph) || !mbar_wait(&afull[as], aph)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const unsigned char *xs = stages + st * PF_STAGE_BYTES;
                    const uint64_t b0 = umma_desc_k_sw128(xs), b1 = umma_desc_k_sw128(xs + PF_HN * PF_BK);
                    const uint32_t at = tmem_base + PF_A_COL0 + as * PF_A_COLS;
#pragma unroll
                    for (int j = 0; j < PF_BK / 32; ++j) {
                        umma_i8_ts(d0, at + 8 * j, b0 + 2 * j, id0, (kb | j) != 0);
                        if (n1 > 0) umma_i8_ts(d1, at + 8 * j, b1 + 2 * j, id1, (kb | j) != 0);
                    }
                    umma_commit(&empty[st]);
                    umma_commit(&aempty[as]);
                    if (++st == PF_STAGES) {
                        st = 0;
                        ph ^= 1;
                    }
                    if (++as == PF_A_STAGES) {
                        as = 0;
                        aph ^= 1;
                    }
                }
                if (!ok) break;
                umma_commit(&dfull[sl0]);
                umma_commit(&dfull[sl1]);
            }
            // every MMA issued must finish before TMEM / shared memory is released
            umma_commit(mma_done);
            mbar_wait_drain(mma_done, 0);
        }
        __syncwarp();
    } else if (warp >= PF_UNPACK_WARP0) {
        // ---------------- unpackers ----------------
        const int q = warp & 3, hk = (warp - PF_UNPACK_WARP0) >> 2;
        const uint32_t tl = tmem_base + ((uint32_t)(32 * q) << 16) + PF_A_COL0 + 16 * hk;
        const int src = (32 * q + lane) * (PF_BK / 4) + 16 * hk;
        int st = 0, as = 0;
        uint32_t ph = 0, aph = 0;
        bool ok = true;
        for (int unit = blockIdx.x; unit < a.num_units && ok; unit += gridDim.x) {
            const PfUnit un = pf_unit(a, unit);
            if (un.ntok <= 0) continue;
            for (int kb = 0; kb < a.num_k; ++kb) {
                if (!mbar_wait_warp(&fullw[st], ph) || !mbar_wait_warp(&aempty[as], aph ^ 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint4 p = *reinterpret_cast<const uint4 *>(stages + st * PF_STAGE_BYTES + PF_X_BYTES + src);
                uint32_t o[16];
                pf_unpack16(p, o);
                tmem_st16(tl + as * PF_A_COLS, o);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&afull[as]);
                if (++st == PF_STAGES) {
                    st = 0;
                    ph ^= 1;
                }
                if (++as == PF_A_STAGES) {
                    as = 0;
                    aph ^= 1;
                }
            }
        }
    } else {
        // ---------------- epilogue (warps 0-3: TMEM lanes 32w..32w+31) ----------------
        pdl_wait();
        const bool obf = a.y_bf16 != 0;
        // FFN: lanes 0-15 gate rows, 16-31 the up rows of the same n
        const bool upl = FFN && lane >= 16;
        const float g0 = a.gamma0[0];
        const float g1 = FFN ? a.gamma1[0] : 0.0f;
        float *rw = rbuf + warp * 2 * PF_TN; // gamma0/s, then gamma1/s
        const float *rl = rw + (upl ? PF_TN : 0);
        const uint32_t tq = tmem_base + ((uint32_t)(32 * warp) << 16);
        unsigned char *wbuf = obufs + warp * 2 * PF_OBUF;
        constexpr int OW = FFN ? 16 : 32; // output columns of a warp's chunk
        int nbuf = 0;
        uint32_t pos = 0; // accumulator-slot positions
        bool ok = true;
        for (int unit = blockIdx.x; unit < a.num_units && ok; unit += gridDim.x) {
            const PfUnit un = pf_unit(a, unit);
            if (un.ntok <= 0) continue;
            const int nw = FFN ? un.wt * (PF_WM / 2) + 16 * warp : un.wt * PF_WM + 32 * warp; // first n of the warp
            const int n = nw + (FFN ? (lane & 15) : lane);
            const bool nok = n < a.N && (!FFN || lane < 16); // this lane stores
            {
                // gamma / s of the unit's tokens, while its MMAs run (all loads first)
                float sv[PF_TN / 32];
#pragma unroll
                for (int i = 0; i < PF_TN / 32; ++i) {
                    const int t = un.t0 + 32 * i + lane;
                    sv[i] = 32 * i < un.ntok && t < a.M ? a.s[t] : 1.0f;
                }
#pragma unroll
                for (int i = 0; i < PF_TN / 32; ++i) {
                    rw[32 * i + lane] = __fdiv_rn(g0, sv[i]);
                    if (FFN) rw[PF_TN + 32 * i + lane] = __fdiv_rn(g1, sv[i]);
                }
                __syncwarp();
            }
            for (int h = 0; h < 2 && ok; ++h) {
                const uint32_t p = pos++, sl = p % PF_D_SLOTS;
                if (!mbar_wait_warp(&dfull[sl], (p / PF_D_SLOTS) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int nh = min(PF_HN, un.ntok - h * PF_HN); // <= 0: slot unused
#pragma unroll 1
                for (int c = 0; c < nh; c += 32) {
                    const int tb = un.t0 + h * PF_HN + c; // first token of the chunk
                    const float *rc = rl + h * PF_HN + c;
                    uint32_t v[32];
                    tmem_ld32(tq + sl * PF_HN + c, v);
                    tmem_wait_ld(v);
                    float o[32];
                    if constexpr (!FFN) {
                        if (a.acc0) pf_store_acc(a.acc0, a, v, tb, n, nok);
#pragma unroll
                        for (int j = 0; j < 32; ++j) o[j] = __fmul_rn((float)(int)v[j], rc[j]);
                    } else {
                        if (a.acc0 || a.acc1) pf_store_acc(upl ? a.acc1 : a.acc0, a, v, tb, n, n < a.N);
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const float d = __fmul_rn((float)(int)v[j], rc[j]); // gate (lanes < 16) or up
                            const float u = __shfl_down_sync(0xffffffffu, d, 16);
                            const float gp = d > 0.0f ? d : 0.0f;
                            o[j] = __fmul_rn(__fmul_rn(gp, gp), u);
                        }
                    }
                    if (a.tma_out) {
                        unsigned char *buf = wbuf + nbuf * PF_OBUF;
                        if (lane == 0) bulk_wait_group_read<1>(); // the store that used this buffer has read it
                        __syncwarp();
                        if (!FFN || lane < 16) {
                            if (obf) {
                                uint16_t *b = reinterpret_cast<uint16_t *>(buf);
#pragma unroll
                                for (int j = 0; j < 32; ++j) b[j * OW + (lane & (OW - 1))] = (uint16_t)bf16_rn_bits(o[j]);
                            } else {
                                float *b = reinterpret_cast<float *>(buf);
#pragma unroll
                                for (int j = 0; j < 32; ++j) b[j * OW + (lane & (OW - 1))] = o[j];
                            }
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0 && nw < a.N) {
                            tma_store_2d(&tmY, nw, tb, buf); // rows / columns outside y are not written
                            bulk_commit_group();
                        }
                        nbuf ^= 1;
                    } else {
                        pf_emit_direct(a, o, tb, n, nok, obf);
                    }
                    if (a.y_amax) pf_token_max(a, o, tb, nok, obf);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&dempty[sl]);
            }
        }
        if (a.tma_out && lane == 0) bulk_wait_group_all();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == PF_MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem_base, PF_TMEM_COLS);
    }
}

} // namespace bitnet
