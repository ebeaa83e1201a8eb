// decode_seq.cuh -- a whole sequence of decode-size BitLinear / gated-FFN ops
// (for example every projection of every layer of one decode step) in ONE
// persistent kernel launch.
//
// BitNet model page, "Model details" / "Quantization" (W1.58A8: per-token
// absmax int8 activations, absmean ternary weights) and "Architecture"
// (BitLinear without bias, ReLU^2 FFN).  Each op computes exactly what
// bitnet_linear / bitnet_ffn_gate_up compute; the results are bit-identical.
//
// Why: at M <= 64 tokens one BitLinear streams 1.6-8.8 MB of packed weights,
// 0.25-1.35 us at HBM speed, while a kernel boundary plus the dependent
// quantise -> contract -> reduce -> store chain costs several microseconds.
// Here the grid stays resident for the whole sequence:
//   * every CTA streams its slice of every op's packed weights into a
//     shared-memory ring (16-byte cp.async from every thread, completion on a
//     per-slot mbarrier), as many ops ahead of the one being computed as the
//     ring holds; the copies for the next ops start as soon as an op's slice
//     is free.  Weights are read-only for the whole launch, so their stream
//     never waits for another op;
//   * eight compute warps run the ops in order with the cluster K-split of
//     decode_cluster.cuh (partial absmax exchange, local quantisation of the
//     CTA's K slice, mma.m16n8k32 u8 x s8, partial int32 sums exchanged
//     through distributed shared memory, owners dequantise and store);
//   * ordering between ops comes only from real data hazards.  The host finds,
//     for every op, the latest earlier op whose output overlaps this op's input
//     (read after write) and the latest earlier op whose input or output
//     overlaps this op's output (write after read / write).  After an op, every
//     CTA adds one to that op's completion counter (release, device scope);
//     a dependent op waits (acquire) until the counter reaches the number of
//     CTAs of its partition before it reads x, resp. before it stores y.  Ops
//     run in the same order on every CTA of a partition, so waiting for op i
//     covers every op before i;
//   * groups of ops that share no memory (connected components of the hazard
//     graph, e.g. the layers of a decode step with their own output buffers)
//     run side by side on disjoint partitions of the clusters; the host deals
//     them out by weight bytes and picks the partition count;
//   * a projection whose weights do not fit a CTA's ring on its partition is
//     cut into consecutive slices of its output rows, each one op; with one
//     token tile the later slices reuse the first slice's quantised x;
//   * an op that reads an earlier op's output reads its x slice in place from
//     L2 (no staging), which leaves that shared memory to the weight ring.
// The counters live in a caller-provided zero-filled workspace; the last CTA
// to finish zeroes them again.  Every wait is bounded (device status word).
#pragma once

#include <type_traits>

#include "common.cuh"
#include "decode.cuh"
#include "decode_cluster.cuh"
#include "pack_quant.cuh"

namespace bitnet {

constexpr int DS_MAX_OPS = 320;   // ops per launch, after row slicing (kernel-parameter space)
constexpr int DS_COMPUTE = 256;   // eight compute warps
constexpr int DS_CONTROL = 128;   // control warps: weight copies and completion signals
constexpr int DS_THREADS = DS_COMPUTE + DS_CONTROL;
constexpr int DS_SLOTS = 8;       // ops whose weights may be in the ring at once
constexpr int DS_PSLOTS = 16;     // weight pieces in the ring at once (one per matrix of an op)
constexpr int DS_HDR = 1024 + 8 * 96; // header: barriers, per-token scalars, staged op descriptors
constexpr int DS_MAX_KS = 32;     // 64-wide k-steps per CTA
constexpr int DS_MAX_PARTS = 8;   // partitions: independent groups of ops on disjoint clusters
constexpr int DS_RGW = 8;         // row groups (of 16 output rows) per compute warp (host limit)

// One op of a sequence: a BitLinear or gated FFN over N output rows.  The host
// may cut a projection into several ops over consecutive slices of its output
// rows (w0/w1 and y then point at the slice's first row / column).
struct __align__(16) DsOp {
    const void *x;               // [M][K] bf16 or fp32
    const uint8_t *w0, *w1;      // packed [N][K/4]; w1 (up) only for the gated FFN
    const float *gamma0, *gamma1;
    float *y;                    // y[m][n] at y + m * ldy + n, n < N
    int K, N;
    int ldy;                     // row pitch of y (elements)
    int wait_x;                  // earlier op that must be complete before x is read (-1: none)
    int wait_y;                  // earlier op that must be complete before y is written (-1: none)
    int nxt;                     // next op of the same partition (-1: last)
    int16_t ks;                  // 64-wide k-steps per CTA (the last CTAs may have fewer)
    int16_t rpc;                 // output rows per cluster (multiple of 16)
    int16_t own_rows;            // rows finished by each CTA of a cluster (rpc / C)
    int16_t orp;                 // row pitch (ints) of a partial-sum block, == 4 mod 8
    int16_t box_w;               // shared bytes per weight row: 16 * odd (conflict-free rows)
    int16_t cl0, ncl;            // clusters running this op: [cl0, cl0 + ncl) (its partition)
    uint8_t nmat;                // 1 = BitLinear, 2 = gate/up + ReLU^2
    uint8_t xf32;                // x is fp32 (else bf16)
    uint8_t xbuf;                // x staging buffer: 0/1 alternate among ops whose x can be
                                 // prefetched, 2 for ops that read an earlier op's output
    uint8_t reuse;               // same x as the previous op of the partition, one token tile:
                                 // its quantised slice, scales and row sums are still in place
};

struct DsProgram {
    int n_ops, M, C, n_ctas;
    int n_parts;
    int part_cl0[DS_MAX_PARTS], part_ncl[DS_MAX_PARTS], part_first[DS_MAX_PARTS];
    unsigned *counters;          // [DS_MAX_OPS] completions, then [1] exits (workspace)
    uint32_t xs_off[3];          // x staging buffers (DsOp::xbuf): 8 token rows each
    uint32_t xs_pitch[3];        // bytes per token row (the largest K slice of the ops using the buffer)
    uint32_t xq_off, xq_stride;  // quantised x slice: 8 rows (stride == 64 mod 128)
    uint32_t part_off, recv_off; // outgoing / incoming partial sums, C blocks each
    uint32_t ring_off, ring_bytes;
    DsOp ops[DS_MAX_OPS];
};

// Header offsets.
constexpr int DS_BAR_FULL = 0;                     // [DS_PSLOTS] weight piece landed (one cp.async arrival per control thread)
constexpr int DS_BAR_AMAX = DS_BAR_FULL + 8 * DS_PSLOTS; // [2]
constexpr int DS_BAR_RED = DS_BAR_AMAX + 16;       // [2]
constexpr int DS_BAR_X = DS_BAR_RED + 16;          // [3] x staging buffer landed (expect_tx + bulk bytes)
constexpr int DS_TOK_S = 256;                      // float [8]
constexpr int DS_TOK_RS = 288;                     // int [8]
constexpr int DS_TOK_R = 320;                      // float [16]
constexpr int DS_AMAX = 384;                       // float [8 ranks][8 tokens]
constexpr int DS_STARTS = 640;                     // uint32 [DS_PSLOTS] ring starts of live pieces
constexpr int DS_RELEASED = 704;                   // uint32: ops whose weight slice is free
constexpr int DS_DONE = 708;                       // uint32: ops complete on this CTA
constexpr int DS_DESC_READY = 712;                 // uint32: op descriptors staged in shared memory
constexpr int DS_Y_CLEAR = 716;                    // uint32: ops whose y-region ordering wait is satisfied
constexpr int DS_OP_P0 = 720;                      // uint32 [DS_SLOTS]: first piece of each op in the ring
constexpr int DS_GAMMA = 768;                      // float [DS_DESC_SLOTS][2]: gammas of the staged ops
constexpr int DS_DESC = 1024;                      // DsOp [DS_DESC_SLOTS]: this CTA's k-th op in slot k % DS_DESC_SLOTS
constexpr int DS_DESC_SLOTS = 8;

static_assert(sizeof(DsOp) == 96 && DS_DESC + DS_DESC_SLOTS * 96 <= DS_HDR, "staged op descriptors");

// Descriptor of this CTA's k-th op, staged in shared memory (slot k % DS_DESC_SLOTS).
BITNET_DEVINL const DsOp &ds_desc(unsigned char *smem, int k)
{
    return *reinterpret_cast<const DsOp *>(smem + DS_DESC + (k % DS_DESC_SLOTS) * (int)sizeof(DsOp));
}

// Stage op j (program index) as this CTA's k-th op (one thread), with the
// values of its gammas (read here, well ahead of the op, not on its critical path).
BITNET_DEVINL void ds_stage_desc(const DsProgram &p, unsigned char *smem, int j, int k)
{
    float *gam = reinterpret_cast<float *>(smem + DS_GAMMA) + 2 * (k % DS_DESC_SLOTS);
    gam[0] = p.ops[j].gamma0[0];
    gam[1] = p.ops[j].nmat == 2 ? p.ops[j].gamma1[0] : 0.0f;
    const uint4 *src = reinterpret_cast<const uint4 *>(&p.ops[j]);
    uint4 *dst = reinterpret_cast<uint4 *>(smem + DS_DESC + (k % DS_DESC_SLOTS) * (int)sizeof(DsOp));
#pragma unroll
    for (int i = 0; i < (int)(sizeof(DsOp) / 16); ++i) dst[i] = src[i];
}

// Where op slices go in the ring.  Positions are virtual (monotone within a
// launch); a slice never straddles the ring's end.  Producer and consumers
// compute the same sequence of starts from the same op list.
BITNET_DEVINL uint32_t ring_place(uint32_t head, uint32_t size, uint32_t ring)
{
    const uint32_t off = head % ring;
    return off + size > ring ? head - off + ring : head;
}

// Ring bytes of one weight piece: this cluster's rows of one matrix x this CTA's K slice.
__host__ __device__ __forceinline__ uint32_t ds_piece_bytes(const DsOp &op) { return (uint32_t)(op.rpc * op.box_w); }

// Barriers among the compute warps and among the control warps.
BITNET_DEVINL void compute_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
BITNET_DEVINL void control_sync() { asm volatile("bar.sync 2, 128;" ::: "memory"); }
// Hand-offs from the compute warps to the control warp: monotone counters in
// shared memory (ops whose weight slice is free / ops complete on this CTA),
// written by compute thread 0 after a compute barrier (release, CTA scope)
// and polled by the control warp (acquire, CTA scope).
BITNET_DEVINL void st_release_cta(uint32_t *p, uint32_t v)
{
    asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}
BITNET_DEVINL uint32_t ld_acquire_cta(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
    return v;
}
// Bounded wait until *c >= target (a hand-off counter of this CTA).
BITNET_DEVINL bool wait_local(const uint32_t *c, uint32_t target)
{
    if (ld_acquire_cta(c) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t spin = 1;; ++spin) {
        __nanosleep(20);
        if (ld_acquire_cta(c) >= target) return true;
        if ((spin & 255u) == 0 && globaltimer_ns() - t0 > BITNET_WAIT_LIMIT_NS) {
            record_status(BITNET_ERR_TIMEOUT);
            return false;
        }
    }
}

// Bounded spin on an mbarrier phase with the non-blocking test_wait (a warp
// suspended inside try_wait can resume well after the phase completes; here
// every wait is short and on the critical path).
BITNET_DEVINL bool mbar_test(uint32_t bar_addr, uint32_t parity, bool cluster_scope)
{
    uint32_t ok;
    if (cluster_scope)
        asm volatile("{\n\t.reg .pred p;\n\t"
                     "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}"
                     : "=r"(ok)
                     : "r"(bar_addr), "r"(parity)
                     : "memory");
    else
        asm volatile("{\n\t.reg .pred p;\n\t"
                     "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}"
                     : "=r"(ok)
                     : "r"(bar_addr), "r"(parity)
                     : "memory");
    return ok != 0;
}

BITNET_DEVINL bool mbar_spin(uint64_t *bar, uint32_t parity, bool cluster_scope = false)
{
    const uint32_t a = smem_u32(bar);
    if (mbar_test(a, parity, cluster_scope)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t spin = 1;; ++spin) {
        if (mbar_test(a, parity, cluster_scope)) return true;
        if ((spin & 1023u) == 0) {
            if (status_failed()) return false;
            if (globaltimer_ns() - t0 > BITNET_WAIT_LIMIT_NS) {
                record_status(BITNET_ERR_TIMEOUT);
                return false;
            }
        }
    }
}

// Shared-memory loads through 32-bit shared-window addresses (the operand
// pointers are built from an aligned integer address, so the compiler would
// otherwise emit generic loads).
BITNET_DEVINL uint32_t lds32(uint32_t a)
{
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
BITNET_DEVINL uint4 lds128(uint32_t a)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}

BITNET_DEVINL uint4 ld_cg_v4(const void *p)
{
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

BITNET_DEVINL unsigned ld_acquire_gpu(const unsigned *p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Bounded wait until *c >= target (completion counter of an earlier op).
BITNET_DEVINL bool wait_count(const unsigned *c, unsigned target)
{
    if (ld_acquire_gpu(c) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t spin = 1;; ++spin) {
        __nanosleep(32);
        if (ld_acquire_gpu(c) >= target) return true;
        if ((spin & 63u) == 0) {
            if (status_failed()) return false;
            if (globaltimer_ns() - t0 > BITNET_WAIT_LIMIT_NS) {
                record_status(BITNET_ERR_TIMEOUT);
                return false;
            }
        }
    }
}

// Weight issue, run by the control warps.  Ops [released, issued) hold
// ring slices; op `issued` is started while a slot is free and its slice fits
// behind the oldest live one.  The slice (this cluster's rows x this CTA's K
// slice, for each matrix) is copied in 16-byte cp.async chunks spread over the
// DS_CONTROL threads; each then arrives on the slot's mbarrier when its own
// copies have landed (cp.async.mbarrier.arrive.noinc, DS_CONTROL arrivals per
// phase).
// Called before the first op and again each time an op has released its slice.
struct DsIssue {
    uint32_t head;  // virtual ring position after the last issued piece
    int issued;     // this CTA's ops whose pieces have all been started
    int next;       // program index of the op being issued (-1: none)
    int pieces;     // pieces started so far
    int mat;        // next matrix of the op being issued
};

__device__ __forceinline__ void ds_issue(const DsProgram &p, unsigned char *smem, DsIssue &st, int released)
{
    uint64_t *bar_full = reinterpret_cast<uint64_t *>(smem + DS_BAR_FULL);
    uint32_t *starts = reinterpret_cast<uint32_t *>(smem + DS_STARTS);
    uint32_t *op_p0 = reinterpret_cast<uint32_t *>(smem + DS_OP_P0);
    const int tid = threadIdx.x - DS_COMPUTE;
    const int C = p.C;
    const int r = (int)cluster_ctarank();
    const int cl = blockIdx.x / C;
    // starts[] and op_p0[] are written by every control thread with the same values;
    // each reads back its own
    while (st.next >= 0 && st.issued - released < DS_SLOTS) {
        const int k = st.issued; // this CTA's ordinal of the op
        const DsOp &op = p.ops[st.next];
        const int q = st.pieces;
        if (st.mat == 0) op_p0[k % DS_SLOTS] = (uint32_t)q;
        const uint32_t size = ds_piece_bytes(op);
        // an op's pieces are placed back to back (no wrap between them, and the host keeps
        // a whole op within the ring): the up piece always fits once older ops are released
        const uint32_t start = st.mat == 1 ? st.head : ring_place(st.head, size * op.nmat, p.ring_bytes);
        // oldest piece still in use: the first piece of op `released`, if that op has begun
        const int live0 = released < k ? (int)op_p0[released % DS_SLOTS] : (st.mat > 0 ? (int)op_p0[k % DS_SLOTS] : q);
        if (live0 < q && start + size - starts[live0 % DS_PSLOTS] > p.ring_bytes) break; // no room yet
        // the slot's previous copies have landed (already true unless a consumer gave up
        // waiting for them): no copy is ever in flight into reused memory
        if (q >= DS_PSLOTS) mbar_wait_drain(&bar_full[q % DS_PSLOTS], (uint32_t)((q - DS_PSLOTS) / DS_PSLOTS) & 1u);
        starts[q % DS_PSLOTS] = start;
        st.head = start + size;
        ++st.pieces;
        const int mat = st.mat;
        if (++st.mat == op.nmat) {
            st.mat = 0;
            ++st.issued;
            st.next = op.nxt;
        }
        const int64_t n0 = (int64_t)(cl - op.cl0) * op.rpc;
        const int64_t rows_left = (int64_t)op.N - n0;
        const int R = rows_left <= 0 ? 0 : (int)(rows_left < op.rpc ? rows_left : op.rpc);
        const int KS = op.K / 64;
        const int ks0 = r * op.ks;
        const int ksn = max(0, min(op.ks, KS - ks0));
        const int total = R * ksn;
        if (total > 0 && !status_failed()) {
            unsigned char *dst0 = smem + p.ring_off + start % p.ring_bytes;
            const uint8_t *w = (mat ? op.w1 : op.w0) + (size_t)n0 * (op.K / 4) + (size_t)ks0 * 16;
            const size_t row_bytes = (size_t)op.K / 4;
            // (row, chunk) of chunk index c = tid + DS_CONTROL i, advanced incrementally; the
            // quotients by ksn (<= 32) of numbers below 2^11 are exact through a rounded reciprocal
            const float inv_ksn = __frcp_rn((float)ksn);
            const int dq = (int)(((float)DS_CONTROL + 0.5f) * inv_ksn), dr = DS_CONTROL - dq * ksn;
            int row = (int)(((float)tid + 0.5f) * inv_ksn), kc = tid - row * ksn;
            for (int c = tid; c < total; c += DS_CONTROL) {
                cp_async16(dst0 + (uint32_t)row * op.box_w + kc * 16, w + (size_t)row * row_bytes + (size_t)kc * 16);
                kc += dr;
                row += dq;
                if (kc >= ksn) {
                    kc -= ksn;
                    ++row;
                }
            }
        }
        cp_async_mbar_arrive(&bar_full[q % DS_PSLOTS]);
    }
}

// Publish "op j is complete on this CTA" (release, device scope).  Every
// compute thread's stores of op j precede it through the named barrier the
// control warp waits on.
BITNET_DEVINL void ds_signal(const DsProgram &p, int j)
{
    __threadfence();
    atomicAdd(&p.counters[j], 1u);
}

// Per-CTA launch state shared by the ops (uniform across the CTA's threads).
struct DsState {
    int tile;        // token tiles done in this launch (partial-sum exchange barriers and parity)
    int atile;       // token tiles whose maxima were exchanged (absmax barriers and parity)
    uint32_t xw;     // completed waits on x staging buffer b (0..2) in bit b (its next parity)
    bool ok;
};

// Bulk-copy one token tile of op `op`'s x slice into staging buffer `b`, one
// token row per lane (called by a whole warp).  Rows are this CTA's K slice of
// tokens m0 .. m0 + mt - 1; lane 0 arms the buffer's mbarrier.
BITNET_DEVINL void ds_load_x(const DsProgram &p, const DsOp &op, unsigned char *smem, int b, int m0, int mt, int ks0,
                             int ksn, int lane)
{
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + DS_BAR_X) + b;
    const int esz = op.xf32 ? 4 : 2;
    const uint32_t xrow = (uint32_t)ksn * 64 * esz;
    if (ksn <= 0) {
        if (lane == 0) mbar_arrive(bar);
        return;
    }
    if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)mt * xrow);
    if (lane < mt) {
        unsigned char *dst = smem + p.xs_off[b] + lane * p.xs_pitch[b];
        const char *src = static_cast<const char *>(op.x) + ((size_t)(m0 + lane) * op.K + (size_t)ks0 * 64) * esz;
        bulk_g2s(dst, src, xrow, bar);
    }
}

// One op on the compute warps: every token tile of 8, cluster K-split.
// `last_op` makes the final tile arrive on the exit phase of the cluster
// barrier.  The control warp is told when the op's weight slice is free and
// when the op is complete (it publishes the completion).
//
// j: the op's program index (completion counters); k: its ordinal among this
// CTA's ops (ring slot, hand-off counters, staged descriptors); prev: program
// index of this CTA's previous op (-1: none).
// q0: ring piece of the op's first matrix (the second, for the gated FFN, is
// q0 + 1); wb0 / wb1: shared-memory offsets of the two pieces.
__device__ __forceinline__ void ds_op(const DsProgram &p, const DsOp &op, int j, int k, int prev, int q0,
                                      uint32_t wb0, uint32_t wb1, unsigned char *smem, DsState &st, bool last_op)
{
    uint64_t *bar_full = reinterpret_cast<uint64_t *>(smem + DS_BAR_FULL);
    uint64_t *bar_amax = reinterpret_cast<uint64_t *>(smem + DS_BAR_AMAX);
    uint64_t *bar_red = reinterpret_cast<uint64_t *>(smem + DS_BAR_RED);
    uint64_t *bar_x = reinterpret_cast<uint64_t *>(smem + DS_BAR_X);
    float *tok_s = reinterpret_cast<float *>(smem + DS_TOK_S);
    int *tok_rs = reinterpret_cast<int *>(smem + DS_TOK_RS);
    float *tok_r = reinterpret_cast<float *>(smem + DS_TOK_R);
    float *amax_slot = reinterpret_cast<float *>(smem + DS_AMAX);
    unsigned char *sXq = smem + p.xq_off;
    int *part = reinterpret_cast<int *>(smem + p.part_off);
    int *recv = reinterpret_cast<int *>(smem + p.recv_off);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t4 = lane & 3;
    const int C = p.C;
    const uint32_t r = cluster_ctarank();
    const int cl = blockIdx.x / C;
    const int nmat = op.nmat;
    const bool xf32 = op.xf32 != 0;
    const int64_t n0 = (int64_t)(cl - op.cl0) * op.rpc;
    const int64_t rows_left = (int64_t)op.N - n0;
    const int R = rows_left <= 0 ? 0 : (int)(rows_left < op.rpc ? rows_left : op.rpc);
    const int KS = op.K / 64;
    const int ks0 = (int)r * op.ks;
    const int ksn = max(0, min(op.ks, KS - ks0));
    const int own0 = (int)r * op.own_rows;
    const int nown = max(0, min(op.own_rows, R - own0));
    // Quotients by runtime row counts without integer division: for 0 <= i <
    // 2^11 and 1 <= d <= 2^10, (i + 0.5) * fl(1/d) lies at least 0.5/d from
    // every integer while its rounding error stays below 2^-12, so truncation
    // gives floor(i / d) exactly.
    const float inv_own = __frcp_rn((float)op.own_rows); // correctly rounded, as 1.0f / x
    const float inv_nown = __frcp_rn((float)max(nown, 1));
    const int RG = op.rpc / 16;
    const int nrgi = nmat * RG; // row groups of the cluster: rgi = warp + 8 i (matrix rgi / RG)
    const uint32_t box_w = (uint32_t)op.box_w;
    const int nchunk = ksn * 4 * (xf32 ? 4 : 2); // 16-byte x chunks per token in this slice
    const int orp = op.orp;
    const int blk_ints = nmat * 8 * orp;
    const uint32_t blk_bytes = (uint32_t)blk_ints * 4;
    bool up_ready = nmat == 1; // the up projection's piece has landed (gated FFN only)
    const int xb = op.xbuf; // this op's x staging buffer
    const unsigned char *sXs = smem + p.xs_off[xb];
    const uint32_t xs_pitch = p.xs_pitch[xb];
    const unsigned target = (unsigned)(op.ncl * C); // CTAs of this partition (every op it waits for is in it)

    const float *gam = reinterpret_cast<const float *>(smem + DS_GAMMA) + 2 * (k % DS_DESC_SLOTS);
    const float gam0 = gam[0];
    const float gam1 = gam[1];
    const bool reuse = op.reuse != 0; // x_q, tok_s and tok_rs of the previous op stand
    // x written earlier in this launch (buffer 2) is read in place from L2 by both
    // passes below instead of being staged: it leaves that shared memory to the ring
    const bool direct = xb == 2;
    const int esz = xf32 ? 4 : 2;

    for (int m0 = 0; m0 < p.M; m0 += 8, ++st.tile) {
        const int mt = min(8, p.M - m0);
        const int pp = st.tile & 1;
        const uint32_t ph = (uint32_t)(st.tile >> 1) & 1u;
        const int app = st.atile & 1;
        const uint32_t aph = (uint32_t)(st.atile >> 1) & 1u;
        if (tid == 0) {
            if (!reuse) mbar_arrive_expect_tx(&bar_amax[app], (uint32_t)(C - 1) * 32);
            mbar_arrive_expect_tx(&bar_red[pp], (uint32_t)(C - 1) * blk_bytes);
        }
        // the first tile of an op that reads nothing this launch writes was fetched
        // during this CTA's previous op
        if (warp == 0 && !reuse && (m0 > 0 || k == 0 || op.wait_x >= 0)) {
            if (m0 == 0 && op.wait_x >= 0) { // x is written by an earlier op of this launch
                if (lane == 0) {
                    if (prev >= 0 && op.wait_x == prev) ds_signal(p, prev); // the previous op: publish it right here
                    st.ok = wait_count(&p.counters[op.wait_x], target) && st.ok;
                }
                __syncwarp();
            }
            if (!direct) ds_load_x(p, op, smem, xb, m0, mt, ks0, ksn, lane);
        }
        if (warp == 7 && m0 == 0 && op.nxt >= 0) {
            // the next op's first tile reads memory no op of this launch writes: fetch it now
            wait_local(reinterpret_cast<const uint32_t *>(smem + DS_DESC_READY), (uint32_t)k + 2);
            const DsOp &nx = ds_desc(smem, k + 1);
            if (nx.wait_x < 0 && !nx.reuse) { // its buffer (0/1) is not this op's and no earlier op still uses it
                const int nks0 = (int)r * nx.ks;
                ds_load_x(p, nx, smem, nx.xbuf, 0, min(8, p.M), nks0, max(0, min(nx.ks, nx.K / 64 - nks0)), lane);
            }
        }

        if (!reuse) {
            // ---- partial absmax of this warp's token over the staged (or in-place) slice ----
            if (direct) {
                compute_sync(); // warp 0's acquire of the producer's completion precedes every read
            } else {
                st.ok = mbar_spin(&bar_x[xb], (st.xw >> xb) & 1u) && st.ok;
                st.xw ^= 1u << xb;
            }
            const uint4 *src = reinterpret_cast<const uint4 *>(sXs + warp * xs_pitch);
            const char *gx = static_cast<const char *>(op.x) + ((size_t)(m0 + warp) * op.K + (size_t)ks0 * 64) * esz;
            auto xchunk = [&](int c) { return direct ? ld_cg_v4(gx + 16 * (size_t)c) : src[c]; };
            float mx = 0.0f;
            if (warp < mt) {
                if (xf32) {
#pragma unroll 4
                    for (int c = lane; c < nchunk; c += 32) mx = fmaxf(mx, chunk_absmax<true>(xchunk(c)));
                } else {
#pragma unroll 4
                    for (int c = lane; c < nchunk; c += 32) mx = fmaxf(mx, chunk_absmax<false>(xchunk(c)));
                }
            }
            mx = warp_max(mx);
            if (lane == 0) amax_slot[r * 8 + warp] = mx;
            compute_sync();
            if (st.tile == 0) cluster_wait(); // every peer's barriers exist before anyone sends to them
            if (tid < C && tid != (int)r) {
                const float *v = &amax_slot[r * 8];
                const uint32_t dst = mapa_shared(smem_u32(&amax_slot[r * 8]), tid);
                const uint32_t bar = mapa_shared(smem_u32(&bar_amax[app]), tid);
                st_async_v4f(dst, v[0], v[1], v[2], v[3], bar);
                st_async_v4f(dst + 16, v[4], v[5], v[6], v[7], bar);
            }
            st.ok = mbar_spin(&bar_amax[app], aph, true) && st.ok;
            ++st.atile;
            if (tid < 8) {
                float am = 0.0f;
                for (int src = 0; src < C; ++src) am = fmaxf(am, amax_slot[src * 8 + tid]);
                tok_s[tid] = quant_scale(am);
            }
            compute_sync();

            // ---- quantise the staged slice (exact scale known), row sums ----
            {
                int rs = 0;
                if (warp < mt) {
                    const float sc = tok_s[warp];
                    unsigned char *dst = sXq + warp * p.xq_stride;
                    if (xf32) {
#pragma unroll 4
                        for (int c = lane; c < nchunk; c += 32)
                            reinterpret_cast<uint32_t *>(dst)[c] = chunk_quant<true>(xchunk(c), sc, rs).x;
                    } else {
#pragma unroll 4
                        for (int c = lane; c < nchunk; c += 32)
                            reinterpret_cast<uint2 *>(dst)[c] = chunk_quant<false>(xchunk(c), sc, rs);
                    }
                }
                rs = warp_sum(rs);
                if (lane == 0) tok_rs[warp] = rs;
            }
        } // !reuse
        if (tid < 16) {
            const int mat = tid >> 3, jj = tid & 7;
            if (mat < nmat) tok_r[tid] = __fdiv_rn(mat ? gam1 : gam0, tok_s[jj]);
        }
        compute_sync();
        if (m0 == 0) st.ok = mbar_spin(&bar_full[q0 % DS_PSLOTS], (uint32_t)(q0 / DS_PSLOTS) & 1u) && st.ok;

        // ---- contraction, two row groups at a time; partial sums (code offset
        //      removed) into per-owner blocks ----
        {
            constexpr uint32_t M3 = 0x03030303u;
            const int rs0 = tok_rs[2 * t4], rs1 = tok_rs[2 * t4 + 1];
            const uint32_t xq_lane = smem_u32(sXq) + g * p.xq_stride + t4 * 16;
            const uint32_t hi_off = 8 * box_w;
            for (int rgi0 = warp; rgi0 < nrgi; rgi0 += 16) {
                const int rgi1 = rgi0 + 8;
                const bool two = rgi1 < nrgi;
                const int mat0 = rgi0 >= RG ? 1 : 0, mat1 = rgi1 >= RG ? 1 : 0;
                if (!up_ready && (mat0 || (two && mat1))) { // row groups of the up projection from here on
                    st.ok = mbar_spin(&bar_full[(q0 + 1) % DS_PSLOTS], (uint32_t)((q0 + 1) / DS_PSLOTS) & 1u) && st.ok;
                    up_ready = true;
                }
                const uint32_t w0 = smem_u32(smem) + (mat0 ? wb1 : wb0) + (uint32_t)((rgi0 - mat0 * RG) * 16 + g) * box_w + t4 * 4;
                const uint32_t w1 = smem_u32(smem) + (mat1 ? wb1 : wb0) + (uint32_t)((rgi1 - mat1 * RG) * 16 + g) * box_w + t4 * 4;
                // four independent accumulator chains per row group: k-step parity x k half
                int a0[4][4] = {}, a1[4][4] = {};
                if (st.ok && ksn > 0) {
                    // Branch-free bodies: one variant with the second row group (TWO) and
                    // one without, pairs of k-steps, then the odd last k-step.
                    auto kstep_pair = [&](int ks, auto two_c) {
                        constexpr bool TWO = decltype(two_c)::value;
                        const uint4 xa = lds128(xq_lane + ks * 64);
                        const uint4 xb2 = lds128(xq_lane + (ks + 1) * 64);
                        const uint32_t la0 = lds32(w0 + ks * 16);
                        const uint32_t ha0 = lds32(w0 + hi_off + ks * 16);
                        const uint32_t lb0 = lds32(w0 + (ks + 1) * 16);
                        const uint32_t hb0 = lds32(w0 + hi_off + (ks + 1) * 16);
                        uint32_t la1 = 0u, ha1 = 0u, lb1 = 0u, hb1 = 0u;
                        if constexpr (TWO) {
                            la1 = lds32(w1 + ks * 16);
                            ha1 = lds32(w1 + hi_off + ks * 16);
                            lb1 = lds32(w1 + (ks + 1) * 16);
                            hb1 = lds32(w1 + hi_off + (ks + 1) * 16);
                        }
                        mma_u8s8_16832(a0[0], la0 & M3, ha0 & M3, (la0 >> 2) & M3, (ha0 >> 2) & M3, xa.x, xa.y);
                        mma_u8s8_16832(a0[1], (la0 >> 4) & M3, (ha0 >> 4) & M3, (la0 >> 6) & M3, (ha0 >> 6) & M3,
                                       xa.z, xa.w);
                        mma_u8s8_16832(a0[2], lb0 & M3, hb0 & M3, (lb0 >> 2) & M3, (hb0 >> 2) & M3, xb2.x, xb2.y);
                        mma_u8s8_16832(a0[3], (lb0 >> 4) & M3, (hb0 >> 4) & M3, (lb0 >> 6) & M3, (hb0 >> 6) & M3,
                                       xb2.z, xb2.w);
                        if constexpr (TWO) {
                            mma_u8s8_16832(a1[0], la1 & M3, ha1 & M3, (la1 >> 2) & M3, (ha1 >> 2) & M3, xa.x, xa.y);
                            mma_u8s8_16832(a1[1], (la1 >> 4) & M3, (ha1 >> 4) & M3, (la1 >> 6) & M3,
                                           (ha1 >> 6) & M3, xa.z, xa.w);
                            mma_u8s8_16832(a1[2], lb1 & M3, hb1 & M3, (lb1 >> 2) & M3, (hb1 >> 2) & M3, xb2.x,
                                           xb2.y);
                            mma_u8s8_16832(a1[3], (lb1 >> 4) & M3, (hb1 >> 4) & M3, (lb1 >> 6) & M3,
                                           (hb1 >> 6) & M3, xb2.z, xb2.w);
                        }
                    };
                    auto kstep_last = [&](int ks, auto two_c) {
                        constexpr bool TWO = decltype(two_c)::value;
                        const uint4 xa = lds128(xq_lane + ks * 64);
                        const uint32_t la0 = lds32(w0 + ks * 16);
                        const uint32_t ha0 = lds32(w0 + hi_off + ks * 16);
                        mma_u8s8_16832(a0[0], la0 & M3, ha0 & M3, (la0 >> 2) & M3, (ha0 >> 2) & M3, xa.x, xa.y);
                        mma_u8s8_16832(a0[1], (la0 >> 4) & M3, (ha0 >> 4) & M3, (la0 >> 6) & M3, (ha0 >> 6) & M3,
                                       xa.z, xa.w);
                        if constexpr (TWO) {
                            const uint32_t la1 = lds32(w1 + ks * 16);
                            const uint32_t ha1 = lds32(w1 + hi_off + ks * 16);
                            mma_u8s8_16832(a1[0], la1 & M3, ha1 & M3, (la1 >> 2) & M3, (ha1 >> 2) & M3, xa.x, xa.y);
                            mma_u8s8_16832(a1[1], (la1 >> 4) & M3, (ha1 >> 4) & M3, (la1 >> 6) & M3,
                                           (ha1 >> 6) & M3, xa.z, xa.w);
                        }
                    };
                    auto run = [&](auto two_c) {
                        int ks = 0;
#pragma unroll 1
                        for (; ks + 1 < ksn; ks += 2) kstep_pair(ks, two_c);
                        if (ks < ksn) kstep_last(ks, two_c);
                    };
                    if (two)
                        run(std::true_type{});
                    else
                        run(std::false_type{});
                }
                auto store = [&](const int (&a)[4][4], int rgi) {
                    const int mat = rgi >= RG ? 1 : 0;
                    const int rg = rgi - mat * RG;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int row = rg * 16 + g + 8 * h;
                        if (row < R) {
                            const int jo = (int)(((float)row + 0.5f) * inv_own), orow = row - jo * op.own_rows;
                            int *blk = part + jo * blk_ints + (mat * 8 + 2 * t4) * orp + orow;
                            blk[0] = a[0][2 * h] + a[1][2 * h] + a[2][2 * h] + a[3][2 * h] - rs0;
                            blk[orp] = a[0][2 * h + 1] + a[1][2 * h + 1] + a[2][2 * h + 1] + a[3][2 * h + 1] - rs1;
                        }
                    }
                };
                store(a0, rgi0);
                if (two) store(a1, rgi1);
            }
        }
        fence_proxy_async_smem(); // generic writes of `part` -> visible to the bulk copies
        compute_sync();            // also: every warp is done with this tile's weights and x_q
        if (tid < C && tid != (int)r) {
            const uint32_t dst = mapa_shared(smem_u32(recv + (int)r * blk_ints), tid);
            bulk_s2peer(dst, part + tid * blk_ints, blk_bytes, mapa_shared(smem_u32(&bar_red[pp]), tid));
        }
        // the slice is free (every compute warp passed the barrier after the
        // contraction): the control warp refills the ring meanwhile
        if (m0 + 8 >= p.M && tid == 0) st_release_cta(reinterpret_cast<uint32_t *>(smem + DS_RELEASED), (uint32_t)k + 1);
        st.ok = mbar_spin(&bar_red[pp], ph, true) && st.ok;
        if (last_op && m0 + 8 >= p.M) cluster_arrive(); // nothing more is needed from the peers
        if (m0 == 0 && op.wait_y >= 0) { // y was read or written by an earlier op of this launch
            // the control warp acquired that op's completion counter (device scope)
            // and passed it on through this CTA's y-clear counter
            if (tid == 0)
                st.ok = wait_local(reinterpret_cast<const uint32_t *>(smem + DS_Y_CLEAR), (uint32_t)k + 1) && st.ok;
            compute_sync();
        }

        // ---- owners: sum the C partials, dequantise, gate, store ----
        for (int idx = tid; idx < nown * mt; idx += DS_COMPUTE) {
            const int jj = (int)(((float)idx + 0.5f) * inv_nown), orow = idx - jj * nown;
            int s0 = 0, s1 = 0;
            for (int src = 0; src < C; ++src) {
                const int *blk = (src == (int)r ? part + (int)r * blk_ints : recv + src * blk_ints) + jj * orp + orow;
                s0 += blk[0];
                if (nmat == 2) s1 += blk[8 * orp];
            }
            const size_t o = (size_t)(m0 + jj) * op.ldy + (size_t)(n0 + own0 + orow);
            const float v0 = __fmul_rn((float)s0, tok_r[jj]);
            if (nmat == 1) {
                op.y[o] = v0;
            } else {
                const float v1 = __fmul_rn((float)s1, tok_r[8 + jj]);
                const float gp = v0 > 0.0f ? v0 : 0.0f;
                op.y[o] = __fmul_rn(__fmul_rn(gp, gp), v1);
            }
        }
        compute_sync();
    }
    // every store of this op precedes the control warp's completion signal
    if (tid == 0) st_release_cta(reinterpret_cast<uint32_t *>(smem + DS_DONE), (uint32_t)k + 1);
}

__global__ void __launch_bounds__(DS_THREADS, 1) k_decode_seq(const __grid_constant__ DsProgram p)
{
    extern __shared__ unsigned char ds_smem_raw[];
    unsigned char *smem =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(ds_smem_raw) + 127) & ~uintptr_t(127));
    const int tid = threadIdx.x;
    if (tid == 0) {
        uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
        for (int i = 0; i < DS_PSLOTS; ++i) mbar_init(&bars[DS_BAR_FULL / 8 + i], DS_CONTROL);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars[DS_BAR_AMAX / 8 + i], 1);
            mbar_init(&bars[DS_BAR_RED / 8 + i], 1);
        }
        for (int i = 0; i < 3; ++i) mbar_init(&bars[DS_BAR_X / 8 + i], 1);
        fence_mbarrier_init();
        *reinterpret_cast<volatile uint32_t *>(smem + DS_RELEASED) = 0u;
        *reinterpret_cast<volatile uint32_t *>(smem + DS_DONE) = 0u;
        *reinterpret_cast<volatile uint32_t *>(smem + DS_DESC_READY) = 0u;
        *reinterpret_cast<volatile uint32_t *>(smem + DS_Y_CLEAR) = 0u;
    }
    __syncthreads();
    cluster_arrive(); // peers may send to this CTA once every CTA of the cluster has arrived here

    // this CTA's partition: the ops it runs, in program order, linked by DsOp::nxt
    const int cl = (int)blockIdx.x / p.C;
    int part = 0;
    for (int q = 1; q < p.n_parts; ++q)
        if (cl >= p.part_cl0[q]) part = q;
    const int first = p.part_first[part];

    if (tid >= DS_COMPUTE) {
        // control warps: keep the weight ring full, publish each op's completion
        DsIssue iss = {0u, 0, first, 0, 0};
        ds_issue(p, smem, iss, 0);
        const uint32_t *released = reinterpret_cast<const uint32_t *>(smem + DS_RELEASED);
        const uint32_t *done = reinterpret_cast<const uint32_t *>(smem + DS_DONE);
        uint32_t *desc_ready = reinterpret_cast<uint32_t *>(smem + DS_DESC_READY);
        uint32_t *y_clear = reinterpret_cast<uint32_t *>(smem + DS_Y_CLEAR);
        // y-region waits are acquired here, ahead of the compute warps' epilogues: the first
        // op's now, the next op's once the current one is done (it runs later)
        auto clear_y = [&](int j, int k) {
            const int w = p.ops[j].wait_y;
            if (w >= 0) wait_count(&p.counters[w], (unsigned)(p.ops[j].ncl * p.C));
            st_release_cta(y_clear, (uint32_t)k + 1);
        };
        // the first op descriptors, staged in shared memory (one op per thread)
        const int ctid = tid - DS_COMPUTE;
        int staged = 0, stage_next = first; // ops staged so far; program index of the next one
        {
            int j = first;
            for (int q = 0; q < ctid && j >= 0 && q < DS_DESC_SLOTS; ++q) j = p.ops[j].nxt;
            if (ctid < DS_DESC_SLOTS && j >= 0) ds_stage_desc(p, smem, j, ctid);
            while (staged < DS_DESC_SLOTS && stage_next >= 0) {
                stage_next = p.ops[stage_next].nxt;
                ++staged;
            }
        }
        control_sync();
        if (ctid == 0) {
            st_release_cta(desc_ready, (uint32_t)staged);
            clear_y(first, 0);
        }
        int k = 0;
        for (int j = first; j >= 0; j = p.ops[j].nxt, ++k) {
            wait_local(released, (uint32_t)k + 1);
            control_sync();
            ds_issue(p, smem, iss, k + 1);
            if (ctid == 0) {
                wait_local(done, (uint32_t)k + 1);
                // an op the very next op of this CTA reads is published by compute thread 0 itself
                const int nx = p.ops[j].nxt;
                if (!(nx >= 0 && p.ops[nx].wait_x == j)) ds_signal(p, j);
                // op k no longer needs its descriptor slot: stage the next unstaged op there
                if (stage_next >= 0) {
                    ds_stage_desc(p, smem, stage_next, staged);
                    st_release_cta(desc_ready, (uint32_t)++staged);
                    stage_next = p.ops[stage_next].nxt;
                }
                if (nx >= 0) clear_y(nx, k + 1);
            }
        }
        asm volatile("cp.async.wait_all;" ::: "memory"); // every weight copy has landed
        cluster_wait();
        cluster_arrive();
    } else {
        uint32_t off = 0; // ring offset where the next op's pieces may start (no wrap inside an op)
        DsState st = {0, 0, 0u, true};
        const uint32_t *desc_ready = reinterpret_cast<const uint32_t *>(smem + DS_DESC_READY);
        int prev = -1, k = 0, pieces = 0;
        for (int j = first; j >= 0; ++k) {
            st.ok = wait_local(desc_ready, (uint32_t)k + 1) && st.ok;
            const DsOp &op = ds_desc(smem, k);
            const int nxt = op.nxt; // read before the slot can be restaged (after this op)
            // ring positions of the op's pieces: the sequence the control warps place (ring_place on
            // monotone positions), kept here as the offset within the ring (no division)
            const uint32_t size = ds_piece_bytes(op);
            const uint32_t total = size * op.nmat;
            if (off + total > p.ring_bytes) off = 0; // the op would straddle the end: it starts over
            const uint32_t start0 = off, start1 = off + size; // start1: the up projection's piece (gated FFN)
            off += total;
            ds_op(p, op, j, k, prev, pieces, p.ring_off + start0, p.ring_off + start1, smem, st, nxt < 0);
            pieces += op.nmat;
            prev = j;
            j = nxt;
        }
        // every x copy has landed before the CTA may exit (already true unless a
        // wait gave up): the last phase waited on each staging buffer is drained
        if (tid == 0) {
            uint64_t *bar_x = reinterpret_cast<uint64_t *>(smem + DS_BAR_X);
            for (int b = 0; b < 3; ++b) mbar_wait_drain(&bar_x[b], ((st.xw >> b) & 1u) ^ 1u);
        }
    }
    __syncthreads();
    if (tid == 0) {
        // the last CTA out leaves the counters zeroed for the next launch
        __threadfence();
        const unsigned prev = atomicAdd(&p.counters[DS_MAX_OPS], 1u);
        if (prev == (unsigned)p.n_ctas - 1) {
            for (int i = 0; i < p.n_ops; ++i) atomicExch(&p.counters[i], 0u);
            atomicExch(&p.counters[DS_MAX_OPS], 0u);
        }
    }
    // no CTA leaves while a peer's bulk copy may still read its shared memory
    cluster_wait();
}

} // namespace bitnet
