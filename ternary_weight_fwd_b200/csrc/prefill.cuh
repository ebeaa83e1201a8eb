// prefill.cuh -- large-M (prefill) BitLinear on the 5th-generation tensor
// cores: tcgen05.mma kind::i8 with int32 accumulators in tensor memory.
//
// BitNet model page, "Model details" / "Quantization" (W1.58A8) and
// "Architecture" (BitLinear without bias, ReLU^2 in the FFN).
//
// One persistent CTA per SM, warp-specialised, 448 threads:
//   warps 0-3  epilogue: tcgen05.ld the int32 tile, dequantise (acc * gamma/s),
//              optional ReLU^2 gate; 32 x 32 chunks are staged in swizzled
//              shared memory (fp32: 128-byte swizzle; bf16 outputs, rounded to
//              nearest even: 64-byte swizzle) and written by TMA stores; the
//              optional per-token maxima of the stored values are folded in
//              with one integer atomicMax per row and tile
//   warp 4     producer: TMA (no multicast) of the int8 activation tile
//              (128 tokens x 128 k, 128-byte swizzle) and of the packed
//              ternary tile (256 rows x 32 bytes)
//   warp 5     TMEM owner + MMA issuer (one elected thread)
//   warps 6-13 unpackers: packed 2-bit codes -> signed int8 {-1,0,1} written
//              straight into the UMMA K-major 128-byte-swizzled layout
// Tile: 128 tokens x 256 output columns x 128 k per stage, 3-stage ring.
// Accumulators double-buffered in TMEM (2 x 256 columns) so the epilogue of
// tile i overlaps the main loop of tile i+1.
// Work units (BitLinear): the first full waves of tiles (a multiple of the
// grid) are whole tiles; each tile of a last, partly filled wave runs as Q
// sub-tiles of 256 / Q output columns (Q = 2 or 4, an N = 128 or 64 MMA) on Q
// CTAs, so the last wave takes 1 / Q of a tile's time.  Sub-tiles own disjoint
// outputs: nothing is combined across CTAs.
// For the gate/up FFN the 256 B-rows of a tile are 128 gate rows followed by
// the same 128 up rows, so one N=256 MMA yields both halves of h's tile.
#pragma once

#include "common.cuh"

namespace bitnet {

constexpr int PF_BM = 128;                  // tokens per tile (MMA M)
constexpr int PF_BN = 256;                  // B rows per tile (MMA N)
constexpr int PF_BK = 128;                  // k (int8 bytes) per stage
constexpr int PF_STAGES = 3;
constexpr int PF_A_BYTES = PF_BM * PF_BK;   // 16 KiB
constexpr int PF_BU_BYTES = PF_BN * PF_BK;  // 32 KiB unpacked int8
constexpr int PF_BP_BYTES = PF_BN * PF_BK / 4; // 8 KiB packed codes
constexpr int PF_STAGE_BYTES = PF_A_BYTES + PF_BU_BYTES + PF_BP_BYTES;
constexpr int PF_HDR = 1024;
constexpr int PF_EPI_BUF = 32 * 128;              // one warp's 32 rows x 32 fp32 columns
constexpr int PF_EPI_BYTES = 4 * 2 * PF_EPI_BUF;  // 4 epilogue warps, double-buffered
constexpr int PF_SMEM = PF_HDR + PF_STAGES * PF_STAGE_BYTES + PF_EPI_BYTES + 1024; // + alignment slack
constexpr int PF_THREADS = 448;
constexpr int PF_EPI_WARPS = 4;
constexpr int PF_TMA_WARP = 4;
constexpr int PF_MMA_WARP = 5;
constexpr int PF_UNPACK_WARP0 = 6;
constexpr int PF_UNPACK_THREADS = 256;
constexpr uint32_t PF_TMEM_COLS = 512;

// kind::i8 instruction descriptor: D = s32, A = s8, B = s8, both K-major,
// N = 256, M = 128.
constexpr uint32_t PF_IDESC = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(PF_BN >> 3) << 17) |
                              ((uint32_t)(PF_BM >> 4) << 24);

struct PrefillArgs {
    int M, N, K;
    int num_m, num_n, num_k, num_tiles;
    const float *gamma0, *gamma1;
    const float *s;       // [M] per-token scales
    void *y;              // [M][N] fp32, or bf16 when y_bf16
    float *y_amax;        // optional [M]: max |y| per row, folded in with atomicMax (zeroed beforehand)
    int32_t *acc0, *acc1; // optional [M][N]
    int y_bf16;           // store y as bf16 (nearest even of the fp32 value)
    int vec_ok;           // rows of y are 16-byte multiples: TMA stores
    int full_units;       // whole tiles (units [0, full_units))
    int tail_q;           // sub-tiles per remaining tile (1: none; 2 or 4, BitLinear only)
    int num_units;        // full_units + (num_tiles - full_units) * tail_q
};

// Unit u of the persistent loop: tile (mb, nb), output columns [col0, col0 + ncols)
// of its PF_BN (B rows of the tile).
struct PfUnit {
    int mb, nb, col0, ncols;
};

BITNET_DEVINL PfUnit pf_unit(const PrefillArgs &a, int u)
{
    PfUnit r;
    int tile;
    if (u < a.full_units) {
        tile = u;
        r.col0 = 0;
        r.ncols = PF_BN;
    } else {
        const int v = u - a.full_units;
        const int q = v % a.tail_q;
        tile = a.full_units + v / a.tail_q;
        r.ncols = PF_BN / a.tail_q;
        r.col0 = q * r.ncols;
    }
    r.mb = tile % a.num_m;
    r.nb = tile / a.num_m;
    return r;
}

// kind::i8 instruction descriptor with N = ncols (a multiple of 16, <= 256).
BITNET_DEVINL uint32_t pf_idesc(int ncols)
{
    return (PF_IDESC & ~(0x3Fu << 17)) | ((uint32_t)(ncols >> 3) << 17);
}

// codes {0,1,2} (one per byte) -> int8 {-1,0,1}: per byte (c | 0x80) - 1 cannot
// borrow across bytes, xor 0x80 restores the sign.
BITNET_DEVINL uint32_t codes_to_s8(uint32_t c)
{
    return ((c | 0x80808080u) - 0x01010101u) ^ 0x80808080u;
}

// 256 threads turn one packed stage (rows x 32 B, rows <= 256) into rows x 128 B of
// int8, 16-byte chunk c of row r stored at r*128 + ((c ^ (r & 7)) << 4).
BITNET_DEVINL void pf_unpack_stage(const unsigned char *bp, unsigned char *bu, int u, int rows)
{
    constexpr uint32_t M3 = 0x03030303u;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int t = u + PF_UNPACK_THREADS * i;
        if (t >= 2 * rows) break;
        const int row = t >> 1, half = t & 1;
        const uint4 p = *reinterpret_cast<const uint4 *>(bp + row * 32 + half * 16);
        const uint32_t wv[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            uint4 o;
            o.x = codes_to_s8(wv[w] & M3);
            o.y = codes_to_s8((wv[w] >> 2) & M3);
            o.z = codes_to_s8((wv[w] >> 4) & M3);
            o.w = codes_to_s8((wv[w] >> 6) & M3);
            const int chunk = half * 4 + w;
            *reinterpret_cast<uint4 *>(bu + row * 128 + ((chunk ^ (row & 7)) << 4)) = o;
        }
    }
}

BITNET_DEVINL void pf_store_row32(float *dst, const float (&v)[32], int ncols, bool vec)
{
    if (vec && ncols >= 32) {
#pragma unroll
        for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4 *>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (j < ncols) dst[j] = v[j];
    }
}

BITNET_DEVINL void pf_store_row32_bf16(uint16_t *dst, const uint32_t (&pk)[16], int ncols)
{
#pragma unroll
    for (int j = 0; j < 32; ++j)
        if (j < ncols) dst[j] = (uint16_t)(j & 1 ? pk[j >> 1] >> 16 : pk[j >> 1] & 0xffffu);
}

BITNET_DEVINL void pf_store_row32_i(int32_t *dst, const uint32_t (&v)[32], int ncols, bool vec, int off)
{
    if (vec && ncols >= 32) {
#pragma unroll
        for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<int4 *>(dst + j) = make_int4((int)v[j] - off, (int)v[j + 1] - off,
                                                           (int)v[j + 2] - off, (int)v[j + 3] - off);
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (j < ncols) dst[j] = (int)v[j] - off;
    }
}

template <bool FFN>
__global__ void __launch_bounds__(PF_THREADS, 1)
    k_prefill(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
              const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmY, const PrefillArgs a)
{
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem);
    uint64_t *unpacked = full + PF_STAGES;
    uint64_t *empty = unpacked + PF_STAGES;
    uint64_t *acc_full = empty + PF_STAGES;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *mma_done = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    unsigned char *stages = smem + PF_HDR;
    unsigned char *epi_bufs = stages + PF_STAGES * PF_STAGE_BYTES;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < PF_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&unpacked[s], PF_UNPACK_THREADS / 32); // one arrival per unpack warp
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], PF_EPI_WARPS); // one arrival per epilogue warp
        }
        mbar_init(mma_done, 1);
        fence_mbarrier_init();
    }
    if (warp == PF_TMA_WARP && lane == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB0);
        if (FFN) prefetch_tensormap(&tmB1);
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
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0, last_par = 0; // per stage bit flags
            bool ok = true;
            for (int unit = blockIdx.x; unit < a.num_units && ok; unit += gridDim.x) {
                const PfUnit un = pf_unit(a, unit);
                const int mb = un.mb, nb = un.nb;
                for (int kb = 0; kb < a.num_k; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1)) {
                        ok = false;
                        break;
                    }
                    unsigned char *st = stages + stage * PF_STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[stage], PF_A_BYTES + un.ncols * (PF_BK / 4));
                    tma_load_2d(st, &tmA, kb * PF_BK, mb * PF_BM, &full[stage]);
                    unsigned char *bp = st + PF_A_BYTES + PF_BU_BYTES;
                    if constexpr (FFN) {
                        tma_load_2d(bp, &tmB0, kb * (PF_BK / 4), nb * (PF_BN / 2), &full[stage]);
                        tma_load_2d(bp + PF_BP_BYTES / 2, &tmB1, kb * (PF_BK / 4), nb * (PF_BN / 2), &full[stage]);
                    } else if (un.ncols == PF_BN) {
                        tma_load_2d(bp, &tmB0, kb * (PF_BK / 4), nb * PF_BN, &full[stage]);
                    } else {
                        // a sub-tile: tmB1's box is ncols rows
                        tma_load_2d(bp, &tmB1, kb * (PF_BK / 4), nb * PF_BN + un.col0, &full[stage]);
                    }
                    issued |= 1u << stage;
                    last_par = (last_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == PF_STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            // let every copy this CTA issued land before the CTA can exit
            for (int s = 0; s < PF_STAGES; ++s)
                if (issued & (1u << s)) mbar_wait_drain(&full[s], (last_par >> s) & 1);
        }
    } else if (warp == PF_MMA_WARP) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int unit = blockIdx.x; unit < a.num_units && ok; unit += gridDim.x) {
                const PfUnit un = pf_unit(a, unit);
                if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * PF_BN);
                const uint32_t idesc = pf_idesc(un.ncols);
                for (int kb = 0; kb < a.num_k; ++kb) {
                    if (!mbar_wait(&full[stage], phase) || !mbar_wait(&unpacked[stage], phase)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    unsigned char *st = stages + stage * PF_STAGE_BYTES;
                    const uint64_t adesc = umma_desc_k_sw128(st);
                    const uint64_t bdesc = umma_desc_k_sw128(st + PF_A_BYTES);
#pragma unroll
                    for (int j = 0; j < PF_BK / 32; ++j)
                        umma_i8(d_tmem, adesc + 2 * j, bdesc + 2 * j, idesc, (kb | j) != 0);
                    umma_commit(&empty[stage]);
                    if (++stage == PF_STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                umma_commit(&acc_full[acc]);
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1;
                }
            }
            // every MMA issued must finish before TMEM / shared memory is released
            umma_commit(mma_done);
            mbar_wait_drain(mma_done, 0);
        }
        __syncwarp();
    } else if (warp >= PF_UNPACK_WARP0) {
        // ---------------- unpackers ----------------
        const int u = threadIdx.x - PF_UNPACK_WARP0 * 32;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int unit = blockIdx.x; unit < a.num_units && ok; unit += gridDim.x) {
            const PfUnit un = pf_unit(a, unit);
            for (int kb = 0; kb < a.num_k; ++kb) {
                if (!mbar_wait(&full[stage], phase)) {
                    ok = false;
                    break;
                }
                unsigned char *st = stages + stage * PF_STAGE_BYTES;
                pf_unpack_stage(st + PF_A_BYTES + PF_BU_BYTES, st + PF_A_BYTES, u, un.ncols);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&unpacked[stage]);
                if (++stage == PF_STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
    } else {
        // ---------------- epilogue (warps 0-3: TMEM lanes 32w..32w+31) ----------------
        // Chunks of 32 rows x 32 columns go through a swizzled staging buffer
        // and one TMA store; two buffers per warp.  fp32: 128-byte rows, chunk
        // j of row l at l*128 + ((j ^ (l & 7)) << 4); bf16: 64-byte rows, chunk
        // j at l*64 + ((j ^ ((l >> 1) & 3)) << 4) (the 64-byte swizzle).  Both
        // keep the eight lanes of a shared-memory wavefront on distinct banks.
        pdl_wait();
        const float g0 = a.gamma0[0];
        const float g1 = FFN ? a.gamma1[0] : 0.0f;
        const bool tma_out = a.vec_ok != 0;
        const bool obf = a.y_bf16 != 0;
        unsigned char *wbuf = epi_bufs + warp * 2 * PF_EPI_BUF;
        int nbuf = 0;
        uint32_t rmax = 0; // this lane's row: max magnitude bits of the stored values of the tile
        auto emit = [&](const float (&o)[32], int m, int n, bool mok) {
            const int nv = a.N - n; // valid columns of this chunk (the rest is never stored)
            uint32_t pk[16];
            if (obf) {
#pragma unroll
                for (int j = 0; j < 16; ++j) pk[j] = bf16_rn_bits(o[2 * j]) | (bf16_rn_bits(o[2 * j + 1]) << 16);
                if (a.y_amax) {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (j < nv) rmax = max(rmax, ((j & 1 ? pk[j >> 1] >> 16 : pk[j >> 1]) & 0x7fffu) << 16);
                }
            } else if (a.y_amax) {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (j < nv) rmax = max(rmax, __float_as_uint(o[j]) & 0x7fffffffu);
            }
            if (tma_out) {
                unsigned char *buf = wbuf + nbuf * PF_EPI_BUF;
                if (lane == 0) bulk_wait_group_read<1>(); // the store that used this buffer has read it
                __syncwarp();
                if (obf) {
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        *reinterpret_cast<uint4 *>(buf + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) =
                            make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        *reinterpret_cast<float4 *>(buf + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                            make_float4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmY, n, m - lane, buf); // rows/columns outside y are not written
                    bulk_commit_group();
                }
                nbuf ^= 1;
            } else if (mok && n < a.N) {
                if (obf)
                    pf_store_row32_bf16(static_cast<uint16_t *>(a.y) + (size_t)m * a.N + n, pk, nv);
                else
                    pf_store_row32(static_cast<float *>(a.y) + (size_t)m * a.N + n, o, nv, false);
            }
        };
        // the epilogue of one 32-column chunk (BitLinear) or of one 32-column chunk of h
        // (gate columns c, up columns c + PF_BN / 2) from its int32 sums
        auto fin_lin = [&](const uint32_t (&v)[32], int c, int nb, int m, bool mok, float r0) {
            const int n = nb * PF_BN + 32 * c;
            if (n < a.N) {
                if (a.acc0 && mok) pf_store_row32_i(a.acc0 + (size_t)m * a.N + n, v, a.N - n, false, 0);
                float o[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) o[j] = __fmul_rn((float)(int)v[j], r0);
                emit(o, m, n, mok);
            }
        };
        auto fin_ffn = [&](const uint32_t (&vg)[32], const uint32_t (&vu)[32], int c, int nb, int m, bool mok,
                           float r0, float r1) {
            const int n = nb * (PF_BN / 2) + 32 * c;
            if (n < a.N) {
                if (mok && a.acc0) pf_store_row32_i(a.acc0 + (size_t)m * a.N + n, vg, a.N - n, false, 0);
                if (mok && a.acc1) pf_store_row32_i(a.acc1 + (size_t)m * a.N + n, vu, a.N - n, false, 0);
                float o[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float gv = __fmul_rn((float)(int)vg[j], r0);
                    const float uv = __fmul_rn((float)(int)vu[j], r1);
                    const float gp = gv > 0.0f ? gv : 0.0f;
                    o[j] = __fmul_rn(__fmul_rn(gp, gp), uv);
                }
                emit(o, m, n, mok);
            }
        };
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int unit = blockIdx.x; unit < a.num_units; unit += gridDim.x) {
            const PfUnit un = pf_unit(a, unit);
            if (!mbar_wait(&acc_full[acc], acc_phase)) break;
            tc_fence_after();
            const int m = un.mb * PF_BM + warp * 32 + lane;
            const bool mok = m < a.M;
            const float sm = mok ? a.s[m] : 1.0f;
            const float r0 = __fdiv_rn(g0, sm);
            const float r1 = FFN ? __fdiv_rn(g1, sm) : 0.0f;
            const uint32_t tb = tmem_base + ((uint32_t)(warp * 32) << 16) + (uint32_t)(acc * PF_BN);
            if constexpr (!FFN) {
#pragma unroll 1
                for (int c = 0; c < un.ncols / 32; ++c) {
                    uint32_t v[32];
                    tmem_ld32(tb + 32 * c, v);
                    tmem_wait_ld(v);
                    fin_lin(v, un.col0 / 32 + c, un.nb, m, mok, r0);
                }
            } else {
#pragma unroll 1
                for (int c = 0; c < PF_BN / 64; ++c) {
                    uint32_t vg[32], vu[32];
                    tmem_ld32(tb + 32 * c, vg);
                    tmem_ld32(tb + PF_BN / 2 + 32 * c, vu);
                    tmem_wait_ld(vg);
                    tmem_regs_fence(vu);
                    fin_ffn(vg, vu, c, un.nb, m, mok, r0, r1);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
            if (a.y_amax) {
                if (mok && rmax != 0u) atomicMax(reinterpret_cast<unsigned *>(a.y_amax) + m, rmax);
                rmax = 0;
            }
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1;
            }
        }
        if (tma_out && lane == 0) bulk_wait_group_all();
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
