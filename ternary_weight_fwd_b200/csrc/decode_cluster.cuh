// decode_cluster.cuh -- small-M (decode) BitLinear with the absmax quantiser
// fused in, split over the K dimension inside a thread-block cluster.
//
// BitNet model page, "Model details" / "Quantization" (W1.58A8: per-token
// absmax int8 activations, absmean ternary weights) and "Architecture"
// (BitLinear without bias, ReLU^2 FFN).
//
// Why a cluster: a token's scale s = 127 / max_k |x_k| needs the whole row,
// and every output row needs the whole quantised row.  Instead of every CTA
// re-reading and re-quantising all of x, the C CTAs of a cluster split K:
//   1. each CTA copies its rows x K-slice tile of the packed weights into
//      shared memory (16-byte cp.async from every thread, issued before the
//      dependency wait) and bulk-copies its K slice of x (all tokens of the
//      tile);
//   2. it computes per-token partial maxima over its slice and pushes them to
//      every peer's shared memory (st.async, counted on the peer's mbarrier);
//   3. every CTA then knows the exact max, so it quantises only its own slice
//      (bit-identical to a whole-row quantiser: max is order-independent);
//   4. contraction on its slice with mma.m16n8k32 u8 x s8 (A = 16 weight rows
//      of codes c = w + 1, unpacked by shift-and-mask; B = 8 tokens of x_q),
//      the code offset sum_k x removed per slice;
//   5. partial int32 sums are scattered to the CTA that owns each output row
//      (st.async into its shared memory); int32 addition is exact and
//      order-free, so the result equals the single-CTA contraction;
//   6. owners finish: dequantise (acc * gamma / s), optional ReLU^2 gate, store
//      (fp32 or bf16), optionally folding the per-token maxima of the stored
//      values into a zeroed [M] vector (warp reduction, one atomicMax per CTA).
// Given per-token maxima of x (from the epilogue of the BitLinear that wrote
// x) replace step 2's reduction and exchange: every CTA reads them directly.
// All waits are bounded mbarrier waits; every CTA runs the whole exchange
// protocol even after a timeout so that no peer is left waiting.
#pragma once

#include "common.cuh"
#include "decode.cuh"
#include "pack_quant.cuh"

namespace bitnet {

constexpr int DC_THREADS = 256;
constexpr int DC_RGW_MAX = 8; // max row groups (of 16 rows) per warp

struct DcArgs {
    const void *x;
    const float *x_amax;        // optional [M]: max |x| per token, given (no reduction, no exchange)
    const uint8_t *w0, *w1;     // packed [N][K/4]
    const float *gamma0, *gamma1;
    void *y;                    // fp32, or bf16 when y_bf16
    float *y_amax;              // optional [M]: max |y| per token, atomicMax into zeroed memory
    int y_bf16;
    int32_t *acc0, *acc1;
    int8_t *xq_out;
    float *s_out;
    int M, N, K;
    int C;         // CTAs per cluster (K split)
    int rpc;       // output rows per cluster (multiple of 8)
    int ks;        // 64-wide k-steps per CTA (the last CTAs may have fewer)
    int own_rows;  // output rows finished by each CTA of the cluster
    int orp;       // row pitch (ints) of a partial-sum block, == 4 mod 8
    uint32_t w_mat_bytes;       // shared bytes per matrix (rows padded to 16)
    uint32_t xs_off, xs_row;    // x slice staging: 8 rows
    uint32_t xq_off, xq_stride; // quantised slice: 8 rows (stride == 64 mod 128)
    uint32_t part_off;          // outgoing partial sums [C owners][NMAT][8 tok][orp] int32
                                // (reuses the weight region when M <= 8: written after the contraction,
                                // and a single token tile never needs the weights again)
    uint32_t recv_off;          // incoming partial sums [C sources][NMAT][8 tok][orp] int32
    uint32_t blk_bytes;         // bytes of one [NMAT][8][orp] block
};

// Header layout (first 1024 bytes of shared memory).
constexpr int DC_HDR = 1024;

// Bulk copy of `bytes` from this CTA's shared memory into a peer's shared
// memory (same cluster), counted on the peer's mbarrier.
BITNET_DEVINL void bulk_s2peer(uint32_t dst_cluster_addr, const void *src_smem, uint32_t bytes,
                               uint32_t peer_bar)
{
    asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     dst_cluster_addr),
                 "r"(smem_u32(src_smem)), "r"(bytes), "r"(peer_bar)
                 : "memory");
}

// RGW = row groups per warp (1, 2, 3, 4, 6 or 8), chosen by the host for the shape.
template <int NMAT, bool XF32, int RGW>
__global__ void __launch_bounds__(DC_THREADS, 2) k_decode_cluster(const DcArgs a)
{
    extern __shared__ unsigned char dc_smem_raw[];
    unsigned char *smem =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(dc_smem_raw) + 127) & ~uintptr_t(127));
    uint64_t *bar_w = reinterpret_cast<uint64_t *>(smem);
    uint64_t *bar_x = bar_w + 1;
    uint64_t *bar_amax = bar_w + 2; // [2], alternating token tiles
    uint64_t *bar_red = bar_w + 4;  // [2]
    float *tok_s = reinterpret_cast<float *>(smem + 64);
    int *tok_rs = reinterpret_cast<int *>(smem + 96);
    float *tok_r = reinterpret_cast<float *>(smem + 128);     // [2][8]
    unsigned *s_amax = reinterpret_cast<unsigned *>(smem + 192); // [8] per-token max magnitude bits of y
    float *amax_slot = reinterpret_cast<float *>(smem + 256); // [C][8]
    unsigned char *sW = smem + DC_HDR;
    unsigned char *sXs = smem + a.xs_off;
    unsigned char *sXq = smem + a.xq_off;
    int *part = reinterpret_cast<int *>(smem + a.part_off);
    int *recv = reinterpret_cast<int *>(smem + a.recv_off);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t4 = lane & 3;
    const int C = a.C;
    const uint32_t r = cluster_ctarank();
    const int64_t n0 = (int64_t)(blockIdx.x / C) * a.rpc;
    const bool first_cluster = blockIdx.x < (unsigned)C;
    const int64_t rows_left = (int64_t)a.N - n0;
    const int R = rows_left <= 0 ? 0 : (int)(rows_left < a.rpc ? rows_left : a.rpc);
    const int KS = a.K / 64;
    const int ks0 = (int)r * a.ks;
    const int ksn = max(0, min(a.ks, KS - ks0));
    const int own0 = (int)r * a.own_rows;
    const int nown = max(0, min(a.own_rows, R - own0));
    const int RG = (a.rpc + 15) / 16;
    const uint32_t box_w = (uint32_t)a.ks * 16;
    constexpr int ESZ = XF32 ? 4 : 2;
    const uint32_t xrow = (uint32_t)ksn * 64 * ESZ;
    const int blk_ints = (int)(a.blk_bytes / 4);
    const char *xb = static_cast<const char *>(a.x);

    // ---- barriers, then the weight stream (independent of the previous grid) ----
    if (tid == 0) {
        mbar_init(bar_w, DC_THREADS);
        mbar_init(bar_x, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar_amax[i], 1);
            mbar_init(&bar_red[i], 1);
        }
        fence_mbarrier_init();
    }
    if (tid < 8) s_amax[tid] = 0u;
    __syncthreads();
    cluster_arrive(); // peers may send to this CTA once every CTA of the cluster has arrived here
    {
        // this cluster's rows x this CTA's K slice, 16-byte chunks spread over
        // all threads; (mat, row, chunk) advanced incrementally (no division)
        const int total = NMAT * R * ksn;
        if (total > 0) {
            const int dq = DC_THREADS / ksn, dr = DC_THREADS % ksn;
            int kc = tid % ksn, row = tid / ksn, mat = 0;
            while (row >= R && mat < NMAT) {
                row -= R;
                ++mat;
            }
            const size_t row_bytes = (size_t)a.K / 4;
            for (int c = tid; c < total; c += DC_THREADS) {
                const uint8_t *src = (mat ? a.w1 : a.w0) + (size_t)(n0 + row) * row_bytes + (size_t)(ks0 + kc) * 16;
                cp_async16(sW + mat * a.w_mat_bytes + (uint32_t)row * box_w + kc * 16, src);
                kc += dr;
                row += dq;
                if (kc >= ksn) {
                    kc -= ksn;
                    ++row;
                }
                while (row >= R && mat < NMAT) {
                    row -= R;
                    ++mat;
                }
            }
        }
        cp_async_mbar_arrive(bar_w);
    }
    pdl_launch_dependents();
    pdl_wait();

    // x slice of a token tile -> sXs (issued by thread 0)
    auto issue_x = [&](int m0, int mt) {
        if (ksn > 0) {
            mbar_arrive_expect_tx(bar_x, (uint32_t)mt * xrow);
            for (int j = 0; j < mt; ++j)
                bulk_g2s(sXs + j * a.xs_row, xb + ((size_t)(m0 + j) * a.K + (size_t)ks0 * 64) * ESZ, xrow, bar_x);
        } else {
            mbar_arrive(bar_x);
        }
    };
    if (tid == 0) issue_x(0, min(8, a.M));

    const float gam0 = a.gamma0[0];
    const float gam1 = NMAT == 2 ? a.gamma1[0] : 0.0f;
    bool ok = true, wready = false;

    // shared-memory offsets of this lane's weight rows, one per row group
    uint32_t woff[RGW];
    bool wact[RGW];
#pragma unroll
    for (int i = 0; i < RGW; ++i) {
        const int rgi = warp + 8 * i;
        wact[i] = rgi < NMAT * RG;
        const int mat = NMAT == 1 ? 0 : rgi / RG;
        const int rg = rgi - mat * RG;
        woff[i] = wact[i] ? mat * a.w_mat_bytes + (uint32_t)(rg * 16 + g) * box_w + t4 * 4 : 0;
    }

    int tile = 0;
    for (int m0 = 0; m0 < a.M; m0 += 8, ++tile) {
        const int mt = min(8, a.M - m0);
        const int pp = tile & 1;                        // which barrier of each pair
        const uint32_t ph = (uint32_t)(tile >> 1) & 1u; // its phase parity
        const bool given = a.x_amax != nullptr; // per-token maxima supplied: no reduction, no exchange
        if (tid == 0) {
            if (!given) mbar_arrive_expect_tx(&bar_amax[pp], (uint32_t)(C - 1) * 32);
            mbar_arrive_expect_tx(&bar_red[pp], (uint32_t)(C - 1) * a.blk_bytes);
            if (tile > 0) issue_x(m0, mt);
        }
        ok = mbar_wait(bar_x, (uint32_t)tile & 1u) && ok;

        // ---- partial absmax of this slice, warp j <-> token j ----
        if (!given) {
            float mx = 0.0f;
            if (warp < mt && ok) {
                const uint4 *src = reinterpret_cast<const uint4 *>(sXs + warp * a.xs_row);
                for (uint32_t c = lane; c < xrow / 16; c += 32) mx = fmaxf(mx, chunk_absmax<XF32>(src[c]));
            }
            mx = warp_max(mx);
            if (lane == 0) amax_slot[r * 8 + warp] = mx;
        }
        __syncthreads();
        if (tile == 0) cluster_wait(); // every peer's barriers exist before anyone sends to them
        if (!given) {
            if (tid < C && tid != (int)r) {
                const float *v = &amax_slot[r * 8];
                const uint32_t dst = mapa_shared(smem_u32(&amax_slot[r * 8]), tid);
                const uint32_t bar = mapa_shared(smem_u32(&bar_amax[pp]), tid);
                st_async_v4f(dst, v[0], v[1], v[2], v[3], bar);
                st_async_v4f(dst + 16, v[4], v[5], v[6], v[7], bar);
            }
            ok = mbar_wait_cluster(&bar_amax[pp], ph) && ok;
        }
        if (tid < 8) {
            float am = 0.0f;
            if (given) {
                if (tid < mt) am = a.x_amax[m0 + tid];
            } else {
                for (int src = 0; src < C; ++src) am = fmaxf(am, amax_slot[src * 8 + tid]);
            }
            tok_s[tid] = quant_scale(am);
        }
        __syncthreads();

        // ---- quantise this slice (exact scale known), partial row sums ----
        {
            int rs = 0;
            if (warp < mt) {
                const float sc = tok_s[warp];
                const uint4 *src = reinterpret_cast<const uint4 *>(sXs + warp * a.xs_row);
                unsigned char *dst = sXq + warp * a.xq_stride;
                int8_t *gdst = (a.xq_out && first_cluster) ? a.xq_out + (size_t)(m0 + warp) * a.K + ks0 * 64
                                                            : nullptr;
                for (uint32_t c = lane; c < xrow / 16; c += 32) {
                    const uint2 qv = chunk_quant<XF32>(src[c], sc, rs);
                    if constexpr (XF32) {
                        reinterpret_cast<uint32_t *>(dst)[c] = qv.x;
                        if (gdst) reinterpret_cast<uint32_t *>(gdst)[c] = qv.x;
                    } else {
                        reinterpret_cast<uint2 *>(dst)[c] = qv;
                        if (gdst) reinterpret_cast<uint2 *>(gdst)[c] = qv;
                    }
                }
            }
            rs = warp_sum(rs);
            if (lane == 0) tok_rs[warp] = rs;
        }
        if (first_cluster && r == 0 && a.s_out && tid < mt) a.s_out[m0 + tid] = tok_s[tid];
        if (tid < 16) {
            const int mat = tid >> 3, j = tid & 7;
            if (mat < NMAT) tok_r[tid] = __fdiv_rn(mat ? gam1 : gam0, tok_s[j]);
        }
        __syncthreads();
        if (!wready) {
            ok = mbar_wait(bar_w, 0) && ok;
            wready = true;
        }

        // ---- contraction over this slice; acc[i][h]: row group i, k half h ----
        int acc[RGW][2][4];
#pragma unroll
        for (int i = 0; i < RGW; ++i)
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[i][h][e] = 0;
        if (ok && ksn > 0) {
            // loads of k-step ks+1 are issued before the MMAs of k-step ks
            constexpr uint32_t M3 = 0x03030303u;
            const unsigned char *xq_lane = sXq + g * a.xq_stride + t4 * 16;
            const uint32_t hi_off = 8 * box_w;
            uint4 xv = *reinterpret_cast<const uint4 *>(xq_lane);
            uint32_t wlo[RGW], whi[RGW];
#pragma unroll
            for (int i = 0; i < RGW; ++i) {
                const unsigned char *p = sW + woff[i];
                wlo[i] = wact[i] ? *reinterpret_cast<const uint32_t *>(p) : 0u;
                whi[i] = wact[i] ? *reinterpret_cast<const uint32_t *>(p + hi_off) : 0u;
            }
#pragma unroll 1
            for (int ks = 0; ks < ksn; ++ks) {
                const bool more = ks + 1 < ksn;
                const uint4 xn = more ? *reinterpret_cast<const uint4 *>(xq_lane + (ks + 1) * 64) : xv;
                uint32_t nlo[RGW], nhi[RGW];
#pragma unroll
                for (int i = 0; i < RGW; ++i) {
                    const unsigned char *p = sW + woff[i] + (ks + 1) * 16;
                    nlo[i] = (wact[i] && more) ? *reinterpret_cast<const uint32_t *>(p) : 0u;
                    nhi[i] = (wact[i] && more) ? *reinterpret_cast<const uint32_t *>(p + hi_off) : 0u;
                }
#pragma unroll
                for (int i = 0; i < RGW; ++i) {
                    if (wact[i]) {
                        const uint32_t lo = wlo[i], hi = whi[i];
                        mma_u8s8_16832(acc[i][0], lo & M3, hi & M3, (lo >> 2) & M3, (hi >> 2) & M3, xv.x, xv.y);
                        mma_u8s8_16832(acc[i][1], (lo >> 4) & M3, (hi >> 4) & M3, (lo >> 6) & M3, (hi >> 6) & M3,
                                       xv.z, xv.w);
                    }
                }
                xv = xn;
#pragma unroll
                for (int i = 0; i < RGW; ++i) {
                    wlo[i] = nlo[i];
                    whi[i] = nhi[i];
                }
            }
        }
        __syncthreads(); // every warp is done with the weights: `part` may reuse their space

        // ---- partial sums (code offset removed) into per-owner blocks ----
        {
            const int rs0 = tok_rs[2 * t4], rs1 = tok_rs[2 * t4 + 1];
#pragma unroll
            for (int i = 0; i < RGW; ++i) {
                const int rgi = warp + 8 * i;
                if (wact[i]) {
                    const int mat = NMAT == 1 ? 0 : rgi / RG;
                    const int rg = rgi - mat * RG;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int row = rg * 16 + g + 8 * h;
                        if (row < R) {
                            const int j = row / a.own_rows, orow = row - j * a.own_rows;
                            int *blk = part + j * blk_ints + (mat * 8 + 2 * t4) * a.orp + orow;
                            blk[0] = acc[i][0][2 * h] + acc[i][1][2 * h] - rs0;
                            blk[a.orp] = acc[i][0][2 * h + 1] + acc[i][1][2 * h + 1] - rs1;
                        }
                    }
                }
            }
        }
        fence_proxy_async_smem(); // generic writes of `part` -> visible to the bulk copies
        __syncthreads();
        if (tid < C && tid != (int)r) {
            const uint32_t dst = mapa_shared(smem_u32(recv + (int)r * blk_ints), tid);
            bulk_s2peer(dst, part + tid * blk_ints, a.blk_bytes, mapa_shared(smem_u32(&bar_red[pp]), tid));
        }
        ok = mbar_wait_cluster(&bar_red[pp], ph) && ok;
        if (m0 + 8 >= a.M) cluster_arrive(); // this CTA needs nothing more from its peers

        // ---- owners: sum the C partials, dequantise, gate, store ----
        const bool obf = a.y_bf16 != 0;
        const int total = nown * mt;
        for (int base = warp * 32; base < total; base += DC_THREADS) {
            const int idx = base + lane;
            const bool act = idx < total;
            const int orow = act ? idx % nown : 0, j = act ? idx / nown : mt - 1;
            uint32_t mag = 0;
            if (act) {
                int s0 = 0, s1 = 0;
                for (int src = 0; src < C; ++src) {
                    const int *blk =
                        (src == (int)r ? part + (int)r * blk_ints : recv + src * blk_ints) + j * a.orp + orow;
                    s0 += blk[0];
                    if (NMAT == 2) s1 += blk[8 * a.orp];
                }
                const size_t o = (size_t)(m0 + j) * a.N + (size_t)(n0 + own0 + orow);
                if (a.acc0) a.acc0[o] = s0;
                float v = __fmul_rn((float)s0, tok_r[j]);
                if constexpr (NMAT == 2) {
                    if (a.acc1) a.acc1[o] = s1;
                    const float v1 = __fmul_rn((float)s1, tok_r[8 + j]);
                    const float gp = v > 0.0f ? v : 0.0f;
                    v = __fmul_rn(__fmul_rn(gp, gp), v1);
                }
                out_store(a.y, o, v, obf);
                mag = out_mag_bits(v, obf);
            }
            if (a.y_amax) warp_token_max(mag, j, s_amax);
        }
        __syncthreads();
        if (a.y_amax && tid < mt) {
            if (s_amax[tid]) atomicMax(reinterpret_cast<unsigned *>(a.y_amax) + m0 + tid, s_amax[tid]);
            s_amax[tid] = 0u;
        }
    }
    if (!wready && tid == 0) mbar_wait_drain(bar_w, 0);
    // no CTA leaves while a peer's bulk copy may still read its shared memory:
    // every peer has arrived above only after receiving all of its partial sums
    cluster_wait();
}

} // namespace bitnet
