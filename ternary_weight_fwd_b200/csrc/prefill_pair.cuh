// prefill_pair.cuh -- large-M (prefill) BitLinear on CTA pairs: tcgen05.mma
// cta_group::2, kind::i8, one 256 x 256 int32 tile per pair in tensor memory.
//
// BitNet model page, "Model details" / "Quantization" (W1.58A8) and
// "Architecture" (BitLinear without bias, ReLU^2 in the FFN).
//
// Why pairs: the weights arrive packed (2 bits) and are expanded to int8 in
// shared memory, so every k-stage writes the B tile into shared memory and
// the tensor core reads it back.  With one CTA per 128 x 256 tile a stage
// moves ~112 KB through an SM's shared memory for 8.4 M int8 MACs, more than
// the MMA needs time for.  In a pair, each CTA holds its own 128 tokens of A
// and only half (128 rows) of B; the pair's MMA (M = 256, N = 256) reads each
// half once for both SMs.  Per SM and stage: TMA 20 KB, unpack 4 KB read +
// 16 KB write, MMA 32 KB read.
//
// Roles (448 threads per CTA, identical in both CTAs of the pair):
//   warps 0-3   epilogue: tcgen05.ld this SM's 128 token rows x 256 columns,
//               dequantise, optional ReLU^2 gate, store; then release the
//               accumulator to the leader (remote mbarrier arrive)
//   warp 4      producer: TMA (no multicast) of this CTA's x_q tile and
//               packed B half into its own stage, on its own mbarrier
//   warp 5      TMEM (cta_group::2 alloc in both CTAs); in the leader CTA
//               (rank 0) one thread issues the pair's MMAs and commits them
//               to both CTAs' barriers (multicast commit)
//   warps 6-13  unpack this CTA's B half, then arrive on the leader's
//               `ready` barrier (remote arrive for rank 1)
// B rows of a tile: rows 0-127 in rank 0, 128-255 in rank 1.  For the FFN the
// two halves are the gate rows and the up rows of the same 128 features.
#pragma once

#include "common.cuh"
#include "prefill.cuh"

namespace bitnet {

constexpr int P2_BM = 128;                  // tokens per CTA (pair tile: 256)
constexpr int P2_BN = 256;                  // B rows per pair tile (per CTA: 128)
constexpr int P2_BK = 128;                  // k bytes per stage
constexpr int P2_STAGES = 5;
constexpr int P2_A_BYTES = P2_BM * P2_BK;           // 16 KiB
constexpr int P2_BU_BYTES = (P2_BN / 2) * P2_BK;    // 16 KiB
constexpr int P2_BP_BYTES = (P2_BN / 2) * P2_BK / 4; // 4 KiB
constexpr int P2_STAGE_BYTES = P2_A_BYTES + P2_BU_BYTES + P2_BP_BYTES;
constexpr int P2_HDR = 1024;
constexpr int P2_EPI_BUF = 32 * 128;        // one warp's 32 rows x 32 fp32 columns
constexpr int P2_EPI_BYTES = 4 * 2 * P2_EPI_BUF; // 4 epilogue warps, double-buffered
constexpr int P2_SMEM = P2_HDR + P2_STAGES * P2_STAGE_BYTES + P2_EPI_BYTES + 1024;
constexpr int P2_THREADS = 448;
constexpr int P2_UNPACK_THREADS = 256;
constexpr int P2_EPI_THREADS = 128;
constexpr uint32_t P2_TMEM_COLS = 512;

// kind::i8, D = s32, A = B = s8, K-major, N = 256, M = 256 (pair).
constexpr uint32_t P2_IDESC = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(P2_BN >> 3) << 17) |
                              ((uint32_t)(256 >> 4) << 24);

BITNET_DEVINL void tmem_alloc_pair(uint32_t *slot, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
}
BITNET_DEVINL void tmem_relinquish_pair() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;"); }
BITNET_DEVINL void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

BITNET_DEVINL void umma_i8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on the barrier at this offset in every CTA of `mask` when the
// pair's previously issued MMAs have completed.
BITNET_DEVINL void umma_commit_pair_mc(uint64_t *bar, uint16_t mask)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                     smem_u32(bar)),
                 "h"(mask)
                 : "memory");
}

// Arrive once on the leader's own barrier when the pair's MMAs have completed.
BITNET_DEVINL void umma_commit_pair(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// Arrive (release, cluster scope) on the barrier at this offset in CTA `rank`.
BITNET_DEVINL void mbar_arrive_remote(uint64_t *bar, uint32_t rank)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(mapa_shared(smem_u32(bar), rank))
                 : "memory");
}

template <bool FFN>
__global__ void __launch_bounds__(P2_THREADS, 1)
    k_prefill_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmY,
                   const PrefillArgs a)
{
    extern __shared__ unsigned char p2_smem_raw[];
    unsigned char *smem =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(p2_smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem);
    uint64_t *ready = full + P2_STAGES;
    uint64_t *empty = ready + P2_STAGES;
    uint64_t *acc_full = empty + P2_STAGES;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *mma_done = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    unsigned char *stages = smem + P2_HDR;
    unsigned char *epi_bufs = stages + P2_STAGES * P2_STAGE_BYTES;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = (int)(blockIdx.x >> 1);
    const int npairs = (int)(gridDim.x >> 1);

    if (threadIdx.x == 0) {
        for (int s = 0; s < P2_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&ready[s], 2 * (P2_UNPACK_THREADS / 32)); // one arrival per unpack warp of each CTA
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 2 * (P2_EPI_THREADS / 32)); // one per epilogue warp of each CTA
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
        tmem_alloc_pair(tmem_slot, P2_TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync(); // barriers of both CTAs initialised, TMEM allocated in both
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_launch_dependents();

    if (warp == PF_TMA_WARP) {
        // ---------------- producer (both CTAs) ----------------
        if (lane == 0) {
            pdl_wait();
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0, last_par = 0;
            bool ok = true;
            for (int tile = pair; tile < a.num_tiles && ok; tile += npairs) {
                const int mb = tile % a.num_m, nb = tile / a.num_m;
                for (int kb = 0; kb < a.num_k; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1)) {
                        ok = false;
                        break;
                    }
                    unsigned char *st = stages + stage * P2_STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[stage], P2_A_BYTES + P2_BP_BYTES);
                    tma_load_2d(st, &tmA, kb * P2_BK, mb * 2 * P2_BM + (int)rank * P2_BM, &full[stage]);
                    unsigned char *bp = st + P2_A_BYTES + P2_BU_BYTES;
                    if constexpr (FFN)
                        tma_load_2d(bp, rank ? &tmB1 : &tmB0, kb * (P2_BK / 4), nb * (P2_BN / 2), &full[stage]);
                    else
                        tma_load_2d(bp, &tmB0, kb * (P2_BK / 4), nb * P2_BN + (int)rank * (P2_BN / 2),
                                    &full[stage]);
                    issued |= 1u << stage;
                    last_par = (last_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == P2_STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            for (int s = 0; s < P2_STAGES; ++s)
                if (issued & (1u << s)) mbar_wait_drain(&full[s], (last_par >> s) & 1);
        }
    } else if (warp == PF_MMA_WARP) {
        // ---------------- MMA issuer (leader CTA) ----------------
        if (leader && lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = pair; tile < a.num_tiles && ok; tile += npairs) {
                if (!mbar_wait_cluster(&acc_empty[acc], acc_phase ^ 1)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * P2_BN);
                for (int kb = 0; kb < a.num_k; ++kb) {
                    if (!mbar_wait_cluster(&ready[stage], phase)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    unsigned char *st = stages + stage * P2_STAGE_BYTES;
                    const uint64_t adesc = umma_desc_k_sw128(st);
                    const uint64_t bdesc = umma_desc_k_sw128(st + P2_A_BYTES);
#pragma unroll
                    for (int j = 0; j < P2_BK / 32; ++j)
                        umma_i8_pair(d_tmem, adesc + 2 * j, bdesc + 2 * j, P2_IDESC, (kb | j) != 0);
                    umma_commit_pair_mc(&empty[stage], 0x3);
                    if (++stage == P2_STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                umma_commit_pair_mc(&acc_full[acc], 0x3);
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1;
                }
            }
            umma_commit_pair(mma_done);
            mbar_wait_drain(mma_done, 0);
        }
        __syncwarp();
    } else if (warp >= PF_UNPACK_WARP0) {
        // ---------------- unpackers (both CTAs) ----------------
        const int u = threadIdx.x - PF_UNPACK_WARP0 * 32;
        const int row = u >> 1, half = u & 1;
        constexpr uint32_t M3 = 0x03030303u;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int tile = pair; tile < a.num_tiles && ok; tile += npairs) {
            for (int kb = 0; kb < a.num_k; ++kb) {
                if (!mbar_wait(&full[stage], phase)) {
                    ok = false;
                    break;
                }
                unsigned char *st = stages + stage * P2_STAGE_BYTES;
                const uint4 p = *reinterpret_cast<const uint4 *>(st + P2_A_BYTES + P2_BU_BYTES + row * 32 + half * 16);
                const uint32_t wv[4] = {p.x, p.y, p.z, p.w};
                unsigned char *bu = st + P2_A_BYTES + row * 128;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    uint4 o;
                    o.x = codes_to_s8(wv[w] & M3);
                    o.y = codes_to_s8((wv[w] >> 2) & M3);
                    o.z = codes_to_s8((wv[w] >> 4) & M3);
                    o.w = codes_to_s8((wv[w] >> 6) & M3);
                    const int chunk = half * 4 + w;
                    *reinterpret_cast<uint4 *>(bu + ((chunk ^ (row & 7)) << 4)) = o;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(&ready[stage], 0);
                if (++stage == P2_STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
    } else {
        // ---------------- epilogue (warps 0-3 of both CTAs) ----------------
        // y chunks of 32 rows x 32 columns are staged in a 128-byte-swizzled
        // buffer (conflict-free writes: chunk j of row l at l*128 + ((j ^ (l & 7)) << 4))
        // and written by one TMA store; two buffers per warp alternate.
        pdl_wait();
        const float g0 = a.gamma0[0];
        const float g1 = FFN ? a.gamma1[0] : 0.0f;
        const bool tma_out = a.vec_ok != 0;
        unsigned char *wbuf = epi_bufs + warp * 2 * P2_EPI_BUF;
        int nbuf = 0;
        auto emit = [&](const float (&o)[32], int m, int n, bool mok) {
            if (tma_out) {
                unsigned char *buf = wbuf + nbuf * P2_EPI_BUF;
                if (lane == 0) bulk_wait_group_read<1>(); // the store that used this buffer has read it
                __syncwarp();
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    *reinterpret_cast<float4 *>(buf + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                        make_float4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmY, n, m - lane, buf); // rows m-lane .. m-lane+31; out-of-range rows/cols skipped
                    bulk_commit_group();
                }
                nbuf ^= 1;
            } else if (mok && n < a.N) {
                pf_store_row32(a.y + (size_t)m * a.N + n, o, a.N - n, false);
            }
        };
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = pair; tile < a.num_tiles; tile += npairs) {
            const int mb = tile % a.num_m, nb = tile / a.num_m;
            if (!mbar_wait(&acc_full[acc], acc_phase)) break;
            tc_fence_after();
            const int m = mb * 2 * P2_BM + (int)rank * P2_BM + warp * 32 + lane;
            const bool mok = m < a.M;
            const float sm = mok ? a.s[m] : 1.0f;
            const float r0 = __fdiv_rn(g0, sm);
            const float r1 = FFN ? __fdiv_rn(g1, sm) : 0.0f;
            const uint32_t tb = tmem_base + ((uint32_t)(warp * 32) << 16) + (uint32_t)(acc * P2_BN);
            if constexpr (!FFN) {
#pragma unroll 1
                for (int c = 0; c < P2_BN / 32; ++c) {
                    uint32_t v[32];
                    tmem_ld32(tb + 32 * c, v);
                    tmem_wait_ld();
                    const int n = nb * P2_BN + 32 * c;
                    if (n < a.N) {
                        float o[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j) o[j] = __fmul_rn((float)(int)v[j], r0);
                        emit(o, m, n, mok);
                        if (a.acc0 && mok) pf_store_row32_i(a.acc0 + (size_t)m * a.N + n, v, a.N - n, false, 0);
                    }
                }
            } else {
#pragma unroll 1
                for (int c = 0; c < P2_BN / 64; ++c) {
                    uint32_t vg[32], vu[32];
                    tmem_ld32(tb + 32 * c, vg);
                    tmem_ld32(tb + P2_BN / 2 + 32 * c, vu);
                    tmem_wait_ld();
                    const int n = nb * (P2_BN / 2) + 32 * c;
                    if (n < a.N) {
                        float o[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const float gv = __fmul_rn((float)(int)vg[j], r0);
                            const float uv = __fmul_rn((float)(int)vu[j], r1);
                            const float gp = gv > 0.0f ? gv : 0.0f;
                            o[j] = __fmul_rn(__fmul_rn(gp, gp), uv);
                        }
                        emit(o, m, n, mok);
                        if (mok && a.acc0) pf_store_row32_i(a.acc0 + (size_t)m * a.N + n, vg, a.N - n, false, 0);
                        if (mok && a.acc1) pf_store_row32_i(a.acc1 + (size_t)m * a.N + n, vu, a.N - n, false, 0);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(&acc_empty[acc], 0);
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1;
            }
        }
        if (tma_out && lane == 0) bulk_wait_group_all();
        __syncwarp();
    }

    // every MMA of the pair has completed (leader drained mma_done) and no CTA
    // touches the other's shared memory after this point
    tc_fence_before();
    cluster_sync();
    if (warp == PF_MMA_WARP) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, P2_TMEM_COLS);
    }
}

} // namespace bitnet
