// decode.cuh -- small-M (decode) BitLinear: stream the packed ternary weights
// once, contract against all M <= 64 tokens, dequantise in the epilogue.
//
// BitNet model page, "Model details" / "Quantization" (W1.58A8) and
// "Architecture" (BitLinear, no bias, ReLU^2 FFN).
//
// Design (one CTA per slice of output rows, 256 threads):
//  * Weight prefetch before the dependency wait.  The CTA's rows of the packed
//    matrix (or of both the gate and up matrices) are bulk-copied into shared
//    memory first thing, then the kernel waits for the previous grid
//    (programmatic dependent launch).  Weights never depend on the previous
//    kernel, so in a stream of layers the HBM weight stream of kernel i+1
//    overlaps the tail of kernel i.
//  * Activations: int8 x_q, per-token scales and row sums from the workspace
//    written by the quantiser kernel (the cluster kernel in decode_cluster.cuh
//    fuses that step instead; this kernel serves shapes it does not cover).
//  * Contraction on the legacy integer tensor path, mma.m16n8k32 u8 x s8:
//    A = 16 weight rows x 32 codes (c = w + 1 in {0,1,2}, unsigned), B = 32 k x
//    8 tokens (x_q, signed).  One packed 32-bit word gives 16 codes; the four
//    shift-and-mask results ((w >> 2j) & 0x03030303) are exactly the A
//    registers, so unpacking costs 7 integer ops per 16 weights.  The
//    code offset is removed exactly in the epilogue: sum_k x*(w+1) - sum_k x.
//  * k is split across the 8 warps in 64-wide steps; partial int32 sums are
//    combined with shared-memory atomics (exact, order-free).
#pragma once

#include "common.cuh"
#include "pack_quant.cuh"

namespace bitnet {

constexpr int DEC_THREADS = 256;
constexpr int DEC_WARPS = 8;
constexpr int DEC_RGM = 4;   // max row groups (of 16) per matrix per CTA
constexpr int DEC_HDR = 1024; // shared-memory header bytes (barriers, per-token scalars)

struct DecodeArgs {
    const int8_t *xq;       // [M][K] int8 quantised activations
    const float *s_in;      // [M] per-token scales
    const int32_t *rs_in;   // [M] per-token sums of x_q
    const uint8_t *w0, *w1; // [N][K/4] packed
    const float *gamma0, *gamma1;
    void *y;                // [M][N] fp32, or bf16 when y_bf16
    float *y_amax;          // optional [M]: max |y| per token, atomicMax into zeroed memory
    int32_t *acc0, *acc1;   // [M][N] optional
    int y_bf16;
    int M, N, K;
    int grid;               // CTAs sharing the N rows
    int rg;                 // row groups per matrix per CTA (<= DEC_RGM)
    int w_stride;           // shared bytes per weight row (== 16 mod 128)
    int rp;                 // reduction row pitch in ints (== 4 mod 32)
};

BITNET_DEVINL void mma_u8s8_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                  uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One 64-wide k-step for every row group of every matrix.  xv = this lane's 16
// activation bytes for token g, k = kbase + 16*t4 .. +15.
template <int NMAT>
BITNET_DEVINL void dec_kstep(int (&acc)[NMAT][DEC_RGM][4], const uint8_t *sW, int w_stride, int rg, int ks, int g,
                             int t4, const uint4 xv)
{
    constexpr uint32_t M3 = 0x03030303u;
#pragma unroll
    for (int mat = 0; mat < NMAT; ++mat) {
#pragma unroll
        for (int r = 0; r < DEC_RGM; ++r) {
            if (r < rg) {
                const uint8_t *p = sW + (size_t)((mat * rg + r) * 16 + g) * w_stride + ks * 16 + t4 * 4;
                const uint32_t lo = *reinterpret_cast<const uint32_t *>(p);
                const uint32_t hi = *reinterpret_cast<const uint32_t *>(p + 8 * w_stride);
                mma_u8s8_16832(acc[mat][r], lo & M3, hi & M3, (lo >> 2) & M3, (hi >> 2) & M3, xv.x, xv.y);
                mma_u8s8_16832(acc[mat][r], (lo >> 4) & M3, (hi >> 4) & M3, (lo >> 6) & M3, (hi >> 6) & M3, xv.z,
                               xv.w);
            }
        }
    }
}

// CH = k-steps per warp held in registers per chunk.
template <int NMAT, int CH>
__global__ void __launch_bounds__(DEC_THREADS, 2) k_decode(const DecodeArgs a)
{
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *bar_w = reinterpret_cast<uint64_t *>(smem);
    float *tok_s = reinterpret_cast<float *>(smem + 64);    // [8]
    int *tok_rs = reinterpret_cast<int *>(smem + 96);       // [8]
    float *tok_r = reinterpret_cast<float *>(smem + 128);   // [2][8]
    unsigned *s_amax = reinterpret_cast<unsigned *>(smem + 192); // [8] per-token max magnitude bits
    uint8_t *sW = smem + DEC_HDR;
    const int rg = a.rg;
    const size_t w_bytes = (size_t)NMAT * rg * 16 * a.w_stride;
    int *sRed = reinterpret_cast<int *>(sW + w_bytes); // [NMAT][8 tok][rp]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t4 = lane & 3;
    const int64_t r0 = (int64_t)a.N * blockIdx.x / a.grid;
    const int R = (int)((int64_t)a.N * (blockIdx.x + 1) / a.grid - r0);
    const uint32_t row_bytes = (uint32_t)(a.K / 4);

    if (tid == 0) {
        mbar_init(bar_w, 1);
        fence_mbarrier_init();
    }
    if (tid < 8) s_amax[tid] = 0u;
    __syncthreads();
    // ---- weight prefetch: independent of the previous grid ----
    if (warp == 0) {
        if (lane == 0) mbar_arrive_expect_tx(bar_w, (uint32_t)NMAT * R * row_bytes);
        __syncwarp();
        for (int i = lane; i < NMAT * R; i += 32) {
            const int mat = i / R, r = i - mat * R;
            const uint8_t *src = (mat ? a.w1 : a.w0) + (r0 + r) * row_bytes;
            bulk_g2s(sW + (size_t)(mat * rg * 16 + r) * a.w_stride, src, row_bytes, bar_w);
        }
    }
    pdl_launch_dependents();
    pdl_wait();

    const float gam0 = a.gamma0[0];
    const float gam1 = NMAT == 2 ? a.gamma1[0] : 0.0f;
    const int KS = a.K / 64;
    bool weights_ready = false;

    for (int m0 = 0; m0 < a.M; m0 += 8) {
        const int mt = min(8, a.M - m0);
        // ---- scales and row sums of this 8-token tile (from the quantiser kernel) ----
        if (tid < mt) {
            tok_s[tid] = a.s_in[m0 + tid];
            tok_rs[tid] = a.rs_in[m0 + tid];
        }
        for (int i = tid; i < NMAT * 8 * a.rp; i += DEC_THREADS) sRed[i] = 0;
        __syncthreads();
        if (tid < 16) {
            const int mat = tid >> 3, j = tid & 7;
            if (mat < NMAT) tok_r[tid] = j < mt ? __fdiv_rn(mat ? gam1 : gam0, tok_s[j]) : 0.0f;
        }
        if (!weights_ready) {
            if (!mbar_wait(bar_w, 0)) return; // timeout recorded; copies cannot still be pending
            weights_ready = true;
        }

        // ---- contraction ----
        int acc[NMAT][DEC_RGM][4];
#pragma unroll
        for (int mat = 0; mat < NMAT; ++mat)
#pragma unroll
            for (int r = 0; r < DEC_RGM; ++r)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[mat][r][e] = 0;

        {
            const bool tok_ok = g < mt;
            const int8_t *xrow = a.xq + (size_t)(m0 + (tok_ok ? g : 0)) * a.K + t4 * 16;
            for (int base = warp; base < KS; base += DEC_WARPS * CH) {
                uint4 xv[CH];
#pragma unroll
                for (int c = 0; c < CH; ++c) {
                    const int ks = base + c * DEC_WARPS;
                    xv[c] = (ks < KS && tok_ok) ? __ldg(reinterpret_cast<const uint4 *>(xrow + ks * 64))
                                                : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int c = 0; c < CH; ++c) {
                    const int ks = base + c * DEC_WARPS;
                    if (ks < KS) dec_kstep<NMAT>(acc, sW, a.w_stride, rg, ks, g, t4, xv[c]);
                }
            }
        }

        // ---- combine the warps' partial sums (exact int32 atomics) ----
#pragma unroll
        for (int mat = 0; mat < NMAT; ++mat) {
#pragma unroll
            for (int r = 0; r < DEC_RGM; ++r) {
                if (r < rg) {
                    const int row = r * 16 + g;
                    int *base = sRed + (mat * 8 + 2 * t4) * a.rp + row;
                    atomicAdd(base, acc[mat][r][0]);
                    atomicAdd(base + a.rp, acc[mat][r][1]);
                    atomicAdd(base + 8, acc[mat][r][2]);
                    atomicAdd(base + a.rp + 8, acc[mat][r][3]);
                }
            }
        }
        __syncthreads();

        // ---- epilogue: remove the code offset, dequantise, (gate), store ----
        const bool obf = a.y_bf16 != 0;
        const int total = R * mt;
        for (int base = warp * 32; base < total; base += DEC_THREADS) {
            const int idx = base + lane;
            const bool act = idx < total;
            const int row = act ? idx % R : 0, j = act ? idx / R : mt - 1;
            uint32_t mag = 0;
            if (act) {
                const size_t o = (size_t)(m0 + j) * a.N + r0 + row;
                const int a0 = sRed[j * a.rp + row] - tok_rs[j];
                if (a.acc0) a.acc0[o] = a0;
                float v = __fmul_rn((float)a0, tok_r[j]);
                if constexpr (NMAT == 2) {
                    const int a1 = sRed[(8 + j) * a.rp + row] - tok_rs[j];
                    if (a.acc1) a.acc1[o] = a1;
                    const float v1 = __fmul_rn((float)a1, tok_r[8 + j]);
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
}

} // namespace bitnet
