// decode_tasks.cuh -- a decode step (many small-M BitLinear / gated-FFN ops over
// the same M <= 64 tokens) in one persistent launch: bitnet_decode_sequence.
//
// BitNet model page, "Model details" / "Architecture" (BitLinear layers, no
// bias, ReLU^2 FFN) and "Quantization" (W1.58A8: absmean ternary weights,
// per-token absmax int8 activations).  Each op computes exactly what
// bitnet_linear / bitnet_ffn_gate_up compute; this file only changes how the
// work of many ops is laid out on the GPU.
//
// Work is cut into tasks, claimed in a fixed global order by the CTAs through
// one atomic counter (dynamic scheduling: a CTA that finishes early takes the
// next task):
//   * quant task (op j, token m for M <= 8, else tokens 8 i .. 8 i + 7):
//     per-token absmax quantisation of the op's x (optionally RMS-normalised
//     first) on all compute warps (one token), or one compute warp per token,
//     written to the workspace as int8 in the fragment layout [K/64][Mp][64]
//     plus the scale and row sum.
//   * row task (op j, block b): 128 RG rows of the packed weights (RG = 2 for
//     M <= 8, else 1; a BitLinear: output rows 128 RG b ..; a gated FFN: 64 RG
//     gate rows and the same up rows), full K, against all tokens.  Compute
//     warp w owns RG 16-row groups: rows g and g + 8 of the mma fragment are
//     two output rows (BitLinear) or the gate and the up row of one output
//     (FFN), so each lane ends with complete sums and the epilogue needs no
//     exchange between warps or CTAs.
// Tasks wait only on earlier tasks of the order (an op's rows on its quant
// tasks; a quant task on the rows of the op that wrote its x; outputs on the
// readers / writers of the same bytes before them), and every task a CTA
// holds was claimed by a running CTA, so progress does not depend on how many
// CTAs are resident at once.
//
// Roles in a CTA (352 threads):
//   warp 8  weight producer: claims tasks, writes them to a 4-entry queue in
//           shared memory, streams each row task's packed weights into a ring of
//           pieces (128 rows x 512 k: two TMA boxes of 64 rows x 128 bytes, with
//           the 128-byte swizzle so the fragment loads hit 32 distinct banks).
//           The tensor maps are made on the device by a small kernel launched
//           before this one, from a template map (the matrix's address, extent
//           and row pitch put in with tensormap.replace).  Weights never wait
//           for any other task.
//   warp 9  activation producer: for a row task, waits for its dependencies,
//           copies the per-token scales and row sums and the gammas, and streams
//           the matching x_q chunk ([8][Mp][64] bytes) next to each weight piece
//           (all with cp.async: it never waits for its own loads).
//   warps 0-7 compute: quant tasks; for row tasks the contraction with
//           mma.m16n8k32 u8 x s8 (codes c = w + 1 in {0,1,2}; the offset is
//           removed exactly with the row sum: sum c*x - sum x) and the epilogue.
//           They only arrive on a shared-memory barrier when a task's stores
//           are issued.
//   warp 10 completion: per task, once the compute warps arrived, makes their
//           stores visible device-wide (fence) and counts the task done, so
//           the fence's round trip stays off the compute warps.
// Completion counters live in the caller's workspace; the last CTA out zeroes
// them.  Every wait is bounded (device status word), and after a timeout every
// wait returns at once, so the launch always ends.
#pragma once

#include "common.cuh"
#include "decode.cuh"
#include "exact_sumsq.cuh"

namespace bitnet {

constexpr int DT_COMPUTE = 256;                 // compute threads (warps 0-7)
constexpr int DT_THREADS = 352;                 // + weight producer (8), activation producer (9), completion (10)
constexpr int DT_ROWS = 128;                    // packed rows per row task and 16-row group per warp
constexpr int DT_KC = 512;                      // k per piece
constexpr int DT_KB = DT_KC / 64;               // 64-k blocks per piece
constexpr int DT_PITCH = DT_KC / 4;             // 128-byte rows, 16-byte chunk c of row r at chunk c ^ (r & 7)
constexpr int DT_WBYTES = DT_ROWS * DT_PITCH;   // 16384 weight bytes of a piece in shared memory, per row-group set
constexpr int DT_BOX_ROWS = 64;                 // rows of one TMA box of weights
constexpr int DT_QUEUE = 4;                     // tasks claimed ahead of the compute warps (at most)
constexpr int DT_MAX_OPS = 128;
constexpr int DT_MAX_SEGS = 512;
constexpr int DT_MAX_DEPS = 8;
constexpr int DT_MAX_SLOTS = 16;
constexpr int DT_MAX_M = 64;
// 16-byte chunks of a row of x per compute thread (K <= 8192): 8 for fp32, 4 for bf16
template <bool XF32> __host__ __device__ constexpr int dt_quant_ch() { return XF32 ? 8 : 4; }

// counters (uint32) at the start of the workspace
constexpr int DT_CNT_TASK = 0;  // next task to claim
constexpr int DT_CNT_EXIT = 1;  // CTAs finished
constexpr int DT_CNT_OPS = 2;   // then per op: quant tasks done, row tasks done

constexpr uint16_t DT_DEP_QUANT = 0x8000u; // dependency on an op's quant tasks (else its row tasks)
constexpr int DT_QEND = 0x7fffffff;         // queue entry: no more tasks

struct DtOp {
    const void *x;                 // [M][K] bf16 or fp32 (read by the quant tasks)
    const uint8_t *w0, *w1;        // [N][K/4] packed (w1: up projection of a gated FFN)
    const float *gamma0, *gamma1;
    const float *norm_g;           // [K] RMS normalisation weight, or null
    float *y;                      // [M][N] fp32 output
    int8_t *xq;                    // workspace: [K/64][Mp][64]
    float *s;                      // workspace: [Mp]
    int32_t *rs;                   // workspace: [Mp]
    float norm_eps;
    int K, N;
    int nmat, xf32;
    int rtasks;                    // row tasks (blocks of 128 packed rows)
    int stall;                     // tests only: 1 = the row tasks wait for one quant task too many
    int nq, nr;                    // dependencies of the quant tasks, of the row outputs
    uint16_t deps[DT_MAX_DEPS];    // deps[0 .. nq): ops whose rows precede the quant tasks;
                                   // deps[nq .. nq+nr): op | DT_DEP_QUANT, or op (its rows)
};

struct DtSeg {        // consecutive tasks of one op in the global order
    int start;        // global index of the segment's first task
    uint16_t op;
    uint16_t first;   // first token (quant) or row block (rows); bit 15: 1 = quant segment
};

struct DtProgram {
    CUtensorMap wtmpl;   // template of the weight maps: uint8 [N][K/4], box 64 rows x 128 bytes, 128-byte swizzle
    int n_ops, n_segs, n_tasks, M, Mp, n_slots, slot_bytes;
    unsigned *counters;
    CUtensorMap *wmaps;  // workspace: [n_ops][2] maps of w0, w1 (made by k_decode_maps)
    DtOp ops[DT_MAX_OPS];
    DtSeg segs[DT_MAX_SEGS];
};

// ---- shared-memory map ------------------------------------------------------
constexpr int DT_BAR_FULL = 0;                        // [DT_MAX_SLOTS]
constexpr int DT_BAR_EMPTY = DT_BAR_FULL + 8 * DT_MAX_SLOTS;
constexpr int DT_BAR_QFULL = DT_BAR_EMPTY + 8 * DT_MAX_SLOTS;
constexpr int DT_BAR_QINFO = DT_BAR_QFULL + 8 * DT_QUEUE;
constexpr int DT_BAR_QEMPTY = DT_BAR_QINFO + 8 * DT_QUEUE;
constexpr int DT_BAR_CDONE = DT_BAR_QEMPTY + 8 * DT_QUEUE; // compute warps done with the entry's task
constexpr int DT_QTASK = DT_BAR_CDONE + 8 * DT_QUEUE; // int[DT_QUEUE]
constexpr int DT_QOP = DT_QTASK + 4 * DT_QUEUE;       // DtEntry[DT_QUEUE]: the row task's op fields
constexpr int DT_RED = 512;                           // quant-task reductions (512 bytes)
// per queue entry (row tasks): fl(gamma0 / s[m]), rowsum[m], fl(gamma1 / s[m]) for m < M
constexpr int DT_INFO = 1024;
constexpr int DT_INFO_R0 = 0, DT_INFO_RS = 4 * DT_MAX_M, DT_INFO_R1 = 8 * DT_MAX_M;
constexpr int DT_INFO_BYTES = 12 * DT_MAX_M;
constexpr int DT_DIG = 4096;                          // [8 warps][20] long accumulators (quant tasks)
constexpr int DT_HDR = 6144; // the piece ring starts here

// The fields of a row task's op that the compute warps use, written into the
// queue entry by the weight producer (which reads the op anyway), so that the
// compute warps read shared memory at a task's start instead of the op table
// in kernel-parameter space.
struct DtEntry {
    float *y;
    int K, N, nmat, pad;
};
static_assert(DT_INFO + DT_QUEUE * DT_INFO_BYTES <= DT_DIG, "shared header");
static_assert(DT_DIG + 8 * 8 * SS_LONG_DIGITS <= DT_HDR && DT_DIG % 8 == 0, "shared header");
static_assert(DT_QOP % 8 == 0 && DT_QOP + (int)sizeof(DtEntry) * DT_QUEUE <= DT_RED, "shared header");
static_assert(DT_HDR % 1024 == 0 && DT_WBYTES % 1024 == 0, "ring alignment (128-byte swizzle)");

// task t -> (op, kind, index)
struct DtTask {
    int op, idx;
    bool quant;
};

BITNET_DEVINL DtTask dt_decode(const DtProgram &p, int t)
{
    int lo = 0, hi = p.n_segs - 1;
    while (lo < hi) { // last segment with start <= t
        const int mid = (lo + hi + 1) >> 1;
        if (p.segs[mid].start <= t) lo = mid;
        else hi = mid - 1;
    }
    const DtSeg sg = p.segs[lo];
    DtTask r;
    r.op = sg.op;
    r.quant = (sg.first & 0x8000u) != 0;
    r.idx = (int)(sg.first & 0x7fffu) + (t - sg.start);
    return r;
}

// Queue entries hold the decoded task (the weight producer decodes each claim
// once): quant << 31 | op << 24 | idx; -1 ends the queue.
BITNET_DEVINL int dt_pack(const DtTask &k) { return (k.quant ? (int)0x80000000u : 0) | (k.op << 24) | k.idx; }
BITNET_DEVINL DtTask dt_unpack(int w)
{
    DtTask r;
    r.quant = w < 0;
    r.op = (w >> 24) & 0x7f;
    r.idx = w & 0xffffff;
    return r;
}

BITNET_DEVINL unsigned dt_ld_acquire(const unsigned *c)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(c) : "memory");
    return v;
}

// Bounded wait until *c >= target; false after a timeout (recorded) or once
// another wait gave up.
BITNET_DEVINL bool dt_wait_count(const unsigned *c, unsigned target)
{
    if (dt_ld_acquire(c) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    const uint64_t limit = wait_limit_ns();
    for (uint32_t spin = 1;; ++spin) {
        __nanosleep(64);
        if (dt_ld_acquire(c) >= target) return true;
        if ((spin & 31u) == 0) {
            if (status_failed()) return false;
            if (globaltimer_ns() - t0 > limit) {
                record_status(BITNET_ERR_TIMEOUT);
                return false;
            }
        }
    }
}

// named barrier of the eight compute warps
BITNET_DEVINL void dt_bar_compute() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

BITNET_DEVINL unsigned *dt_qdone(const DtProgram &p, int j) { return p.counters + DT_CNT_OPS + 2 * j; }
BITNET_DEVINL unsigned *dt_rdone(const DtProgram &p, int j) { return p.counters + DT_CNT_OPS + 2 * j + 1; }

// Completion targets: one count per quant task (token) and per row task.
// quant tasks of an op: one per token for M <= 8, else one per 8 tokens (a warp per token)
BITNET_DEVINL unsigned dt_qtarget(const DtProgram &p, int) { return (unsigned)(p.M <= 8 ? p.M : (p.M + 7) / 8); }
BITNET_DEVINL unsigned dt_rtarget(const DtProgram &p, int j) { return (unsigned)p.ops[j].rtasks; }


// 16-byte asynchronous copy; zero-fills the destination when !valid (nothing is read).
BITNET_DEVINL void dt_cp16(uint32_t dst, const void *src, bool valid)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}

BITNET_DEVINL void dt_cp4(uint32_t dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

BITNET_DEVINL void dt_cp_arrive(uint32_t bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

BITNET_DEVINL uint4 dt_ld_cg16(const void *p)
{
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

BITNET_DEVINL float dt_ld_cg_f32(const float *p)
{
    float v;
    asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}

BITNET_DEVINL int dt_ld_cg_s32(const int32_t *p)
{
    int v;
    asm volatile("ld.global.cg.s32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

BITNET_DEVINL int dt_pieces(int K) { return (K + DT_KC - 1) / DT_KC; }

// Position in the piece ring: slot and the parity of its current use.
struct DtRing {
    int slot = 0;
    uint32_t par = 0;
    BITNET_DEVINL void next(int n_slots)
    {
        if (++slot == n_slots) {
            slot = 0;
            par ^= 1u;
        }
    }
};

// ---- tensor maps of the weights -------------------------------------------
// Made on the device, by a small kernel launched just before the sequence
// kernel (k_decode_maps, one CTA per op): the template with the matrix's
// address, extent and row pitch put in, published to the workspace with a
// release fence for the tensor-map proxy.  The sequence kernel's weight
// producer acquires an op's maps once before its first copy with them.
BITNET_DEVINL void dt_tmap_set(uint32_t sm, const void *w, int K, int N)
{
    asm volatile("tensormap.replace.tile.global_address.shared::cta.b1024.b64 [%0], %1;" ::"r"(sm), "l"(w)
                 : "memory");
    asm volatile("tensormap.replace.tile.global_dim.shared::cta.b1024.b32 [%0], 0, %1;" ::"r"(sm), "r"(K / 4)
                 : "memory");
    asm volatile("tensormap.replace.tile.global_dim.shared::cta.b1024.b32 [%0], 1, %1;" ::"r"(sm), "r"(N)
                 : "memory");
    asm volatile("tensormap.replace.tile.global_stride.shared::cta.b1024.b64 [%0], 0, %1;" ::"r"(sm),
                 "l"((unsigned long long)(K / 4))
                 : "memory");
}

__global__ void __launch_bounds__(32) k_decode_maps(const __grid_constant__ DtProgram p)
{
    __shared__ alignas(128) unsigned char sm[2][128];
    const int j = blockIdx.x, lane = threadIdx.x;
    pdl_launch_dependents(); // the sequence kernel starts now; its weight producer waits for this grid
    // block 0 zeroes the completion counters: every counter access of the sequence kernel follows
    // its weight producer's wait for this grid, and this grid starts after all earlier work on the
    // stream, so the launch never depends on what an earlier call left in these bytes
    if (j == 0)
        for (int i = lane; i < DT_CNT_OPS + 2 * p.n_ops; i += 32) p.counters[i] = 0u;
    if (j >= p.n_ops) return;
    const DtOp &op = p.ops[j];
    for (int m = 0; m < op.nmat; ++m) {
        if (lane < 8) reinterpret_cast<uint4 *>(sm[m])[lane] = reinterpret_cast<const uint4 *>(&p.wtmpl)[lane];
        __syncwarp();
        if (lane == 0) dt_tmap_set(smem_u32(sm[m]), m ? op.w1 : op.w0, op.K, op.N);
        __syncwarp();
        asm volatile("tensormap.cp_fenceproxy.global.shared::cta.tensormap::generic.release.gpu.sync.aligned [%0], "
                     "[%1], 128;" ::"l"(p.wmaps + 2 * j + m),
                     "r"(smem_u32(sm[m]))
                     : "memory");
    }
}

// Lane 0: acquire op j's maps (once per op and CTA).
BITNET_DEVINL void dt_maps_acquire(const DtProgram &p, int j, uint32_t (&have)[DT_MAX_OPS / 32])
{
    if (have[j >> 5] & (1u << (j & 31))) return;
    for (int m = 0; m < p.ops[j].nmat; ++m)
        asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(p.wmaps + 2 * j + m) : "memory");
    have[j >> 5] |= 1u << (j & 31);
}

// ---- weight producer (warp 8) -------------------------------------------------
// A piece of a row task: for each of its RG 128-row groups, two boxes of 64
// rows x 128 bytes at k-bytes 128 pc (rows past N and bytes past K/4 read as
// zero).  BitLinear: rows 128 q .. of the task's block; gated FFN: the group's
// 64 gate rows, then the same 64 up rows.
template <int RG>
BITNET_DEVINL void dt_weight_producer(const DtProgram &p, unsigned char *smem)
{
    const int lane = threadIdx.x & 31;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + DT_BAR_FULL);
    uint64_t *empty = reinterpret_cast<uint64_t *>(smem + DT_BAR_EMPTY);
    uint64_t *qfull = reinterpret_cast<uint64_t *>(smem + DT_BAR_QFULL);
    uint64_t *qempty = reinterpret_cast<uint64_t *>(smem + DT_BAR_QEMPTY);
    volatile int *qtask = reinterpret_cast<volatile int *>(smem + DT_QTASK);
    unsigned char *ring = smem + DT_HDR;
    uint32_t seq = 0;
    DtRing ring_pos;
    uint32_t have[DT_MAX_OPS / 32] = {0u, 0u, 0u, 0u}; // ops whose maps this warp has acquired
    uint32_t issued = 0, last_par = 0;               // slots with copies issued, and their last phase
    pdl_wait(); // the tensor maps written by k_decode_maps are visible
    // the claim of the next task is issued one task ahead, so its latency overlaps the copies
    unsigned claim = 0;
    if (lane == 0) claim = atomicAdd(&p.counters[DT_CNT_TASK], 1u);
    for (;;) {
        int t = (int)__shfl_sync(0xffffffffu, claim, 0);
        if (t >= p.n_tasks) t = -1;
        DtTask tk = {0, 0, false};
        if (t >= 0) tk = dt_decode(p, t);
        const int e = (int)(seq % DT_QUEUE);
        mbar_wait(&qempty[e], ((seq / DT_QUEUE) & 1u) ^ 1u);
        if (lane == 0) {
            qtask[e] = t < 0 ? DT_QEND : dt_pack(tk);
            if (t >= 0 && !tk.quant) {
                const DtOp &op = p.ops[tk.op];
                DtEntry *en = reinterpret_cast<DtEntry *>(smem + DT_QOP) + e;
                en->y = op.y;
                en->K = op.K;
                en->N = op.N;
                en->nmat = op.nmat;
            }
            mbar_arrive(&qfull[e]);
        }
        ++seq;
        if (t < 0) break;
        if (lane == 0) claim = atomicAdd(&p.counters[DT_CNT_TASK], 1u);
        if (tk.quant) continue;
        const DtOp &op = p.ops[tk.op];
        if (lane == 0) dt_maps_acquire(p, tk.op, have);
        const CUtensorMap *g0 = p.wmaps + 2 * tk.op;
        const bool ffn = op.nmat == 2;
        const int np = dt_pieces(op.K);
        for (int pc = 0; pc < np; ++pc, ring_pos.next(p.n_slots)) {
            const int s = ring_pos.slot;
            mbar_wait(&empty[s], ring_pos.par ^ 1u);
            if (lane == 0) {
                {
                    unsigned char *dst = ring + (size_t)s * (size_t)p.slot_bytes;
                    mbar_arrive_expect_tx(&full[s], RG * DT_WBYTES);
                    const int x = pc * (DT_KC / 4);
#pragma unroll
                    for (int q = 0; q < RG; ++q) {
                        unsigned char *d = dst + q * DT_WBYTES;
                        if (ffn) {
                            const int row = tk.idx * (RG * DT_ROWS / 2) + q * (DT_ROWS / 2);
                            tma_load_2d(d, g0, x, row, &full[s]);
                            tma_load_2d(d + DT_BOX_ROWS * DT_PITCH, g0 + 1, x, row, &full[s]);
                        } else {
                            const int row = tk.idx * (RG * DT_ROWS) + q * DT_ROWS;
                            tma_load_2d(d, g0, x, row, &full[s]);
                            tma_load_2d(d + DT_BOX_ROWS * DT_PITCH, g0, x, row + DT_BOX_ROWS, &full[s]);
                        }
                    }
                }
                issued |= 1u << s;
                last_par = (last_par & ~(1u << s)) | (ring_pos.par << s);
            }
        }
    }
    // every copy this warp issued has landed before the CTA can exit
    if (lane == 0)
        for (int s = 0; s < p.n_slots; ++s)
            if (issued & (1u << s)) mbar_wait_drain(&full[s], (last_par >> s) & 1u);
    __syncwarp();
}

// ---- activation producer (warp 9) -------------------------------------------
template <int RG>
BITNET_DEVINL void dt_act_producer(const DtProgram &p, unsigned char *smem)
{
    const int lane = threadIdx.x & 31;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + DT_BAR_FULL);
    uint64_t *empty = reinterpret_cast<uint64_t *>(smem + DT_BAR_EMPTY);
    uint64_t *qfull = reinterpret_cast<uint64_t *>(smem + DT_BAR_QFULL);
    uint64_t *qinfo = reinterpret_cast<uint64_t *>(smem + DT_BAR_QINFO);
    uint64_t *qempty = reinterpret_cast<uint64_t *>(smem + DT_BAR_QEMPTY);
    const volatile int *qtask = reinterpret_cast<const volatile int *>(smem + DT_QTASK);
    const uint32_t ring = smem_u32(smem + DT_HDR);
    const int Mp = p.Mp;
    uint32_t seq = 0;
    DtRing ring_pos;
    for (;;) {
        const int e = (int)(seq % DT_QUEUE);
        mbar_wait(&qfull[e], (seq / DT_QUEUE) & 1u);
        const int t = qtask[e];
        bool rows = false;
        DtTask tk = {0, 0, true};
        if (t != DT_QEND) {
            tk = dt_unpack(t);
            rows = !tk.quant;
        }
        if (rows) {
            const DtOp &op = p.ops[tk.op];
            // dependencies: the op's own quant tasks, then the readers / writers of its output bytes
            if (lane == 0) {
                dt_wait_count(dt_qdone(p, tk.op), dt_qtarget(p, tk.op) + (unsigned)op.stall);
                for (int d = op.nq; d < op.nq + op.nr; ++d) {
                    const int o = op.deps[d] & 0x7fff;
                    if (op.deps[d] & DT_DEP_QUANT) dt_wait_count(dt_qdone(p, o), dt_qtarget(p, o));
                    else dt_wait_count(dt_rdone(p, o), dt_rtarget(p, o));
                }
            }
            __syncwarp();
            // the epilogue's factors fl(gamma / s[m]) and the row sums of this task's op into the
            // entry (this warp runs a task ahead of the compute warps, so the divisions and the
            // loads leave their path); every lane arrives on the entry's info barrier
            {
                unsigned char *inf = smem + DT_INFO + e * DT_INFO_BYTES;
                const float g0 = dt_ld_cg_f32(op.gamma0);
                const float g1 = op.nmat == 2 ? dt_ld_cg_f32(op.gamma1) : 0.0f;
                for (int m = lane; m < p.M; m += 32) {
                    const float sm = dt_ld_cg_f32(op.s + m);
                    reinterpret_cast<int *>(inf + DT_INFO_RS)[m] = dt_ld_cg_s32(op.rs + m);
                    reinterpret_cast<float *>(inf + DT_INFO_R0)[m] = __fdiv_rn(g0, sm);
                    if (op.nmat == 2) reinterpret_cast<float *>(inf + DT_INFO_R1)[m] = __fdiv_rn(g1, sm);
                }
                mbar_arrive(&qinfo[e]);
            }
            // the x_q chunk of every piece: [8 k-blocks][Mp][64] bytes, contiguous in the workspace
            const int np = dt_pieces(op.K);
            for (int pc = 0; pc < np; ++pc, ring_pos.next(p.n_slots)) {
                const int s = ring_pos.slot;
                mbar_wait(&empty[s], ring_pos.par ^ 1u);
                const int nkb = min(DT_KB, (op.K - pc * DT_KC) / 64);
                const int chunks = nkb * Mp * 4; // 16-byte chunks
                const uint8_t *src = reinterpret_cast<const uint8_t *>(op.xq) + (size_t)pc * DT_KB * Mp * 64;
                const uint32_t dst = ring + (uint32_t)s * (uint32_t)p.slot_bytes + RG * DT_WBYTES;
                for (int c = lane; c < chunks; c += 32) dt_cp16(dst + 16u * c, src + 16 * c, true);
                dt_cp_arrive(smem_u32(&full[s]));
            }
        } else {
            mbar_arrive(&qinfo[e]); // keeps the entry's phases in step (every lane: the count is 32)
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&qempty[e]);
        ++seq;
        if (t == DT_QEND) break;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// Byte offset of x_q element k of token m in the fragment layout.  A k-block
// (64 bytes per token) holds, at 16 t4 .. 16 t4 + 15, the 16 values that lane
// group t4 of an mma over that block multiplies.  Ragged last piece (fewer than
// 512 k): block k / 64, position k % 64.  Full piece pc: block 8 pc + kb of the
// piece holds, at 16 t4, the values of packed word 8 t4 + kb of the piece (k =
// 512 pc + 128 t4 + 16 kb ..), so that lane group t4 reads the weight words
// 8 t4 .. 8 t4 + 7 of a row as two 16-byte chunks (both operands use the same
// order of k inside the piece, which leaves the dot product unchanged).
BITNET_DEVINL size_t dt_xq_offset(int k, int m, int Mp, int K)
{
    const int pc = k >> 9, kk = k & 511;
    int blk, pos;
    if ((pc + 1) * DT_KC <= K) {
        blk = 8 * pc + ((kk >> 4) & 7);
        pos = ((kk >> 7) << 4) | (kk & 15);
    } else {
        blk = k >> 6;
        pos = k & 63;
    }
    return ((size_t)blk * Mp + m) * 64 + pos;
}

// ---- quant task (compute warps): tokens 8 i .. 8 i + 7 of op j, one per warp --
// Warp w quantises token m = 8 i + w (m < M).  The row is read from L2 in
// passes, so any K <= 8192 fits and no barrier between warps is needed: the
// absmax pass and the quantise pass; with the RMS normalisation first, a pass
// for the exponent of the row maximum and one for the exact sum of squares
// (128-bit window, or the warp's long accumulator in shared memory for a row
// of very wide range), and the normalised values are recomputed in the later
// passes.  x_q goes to the fragment layout: byte k of token m at
// ((k / 64) * Mp + m) * 64 + k % 64.
template <bool XF32>
BITNET_DEVINL void dt_chunk_vals(const uint4 q, float (&f)[XF32 ? 4 : 8])
{
    if constexpr (XF32) {
        f[0] = __uint_as_float(q.x), f[1] = __uint_as_float(q.y), f[2] = __uint_as_float(q.z);
        f[3] = __uint_as_float(q.w);
    } else {
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            f[2 * h] = bf16_bits_lo(w[h]);
            f[2 * h + 1] = bf16_bits_hi(w[h]);
        }
    }
}

// A batch of QB chunks c0 + 32 b of the row (b < QB, c < nch), loaded before any
// is used (one L2 round trip per batch), as fp32 values; normalised when g is
// set: fl(fl(x r) g).  Chunks past the row are left zero.
template <bool XF32, bool NORM, int QB>
BITNET_DEVINL void dt_batch(const char *row, int c0, int nch, const float *g, float r,
                            float (&f)[QB][XF32 ? 4 : 8])
{
    constexpr int EPC = XF32 ? 4 : 8;
    uint4 q[QB];
    float4 gv[NORM ? QB * (EPC / 4) : 1];
#pragma unroll
    for (int b = 0; b < QB; ++b) {
        const int c = c0 + 32 * b;
        q[b] = make_uint4(0u, 0u, 0u, 0u);
        if (c < nch) {
            q[b] = dt_ld_cg16(row + 16 * (size_t)c);
            if constexpr (NORM) {
#pragma unroll
                for (int u = 0; u < EPC / 4; ++u)
                    gv[b * (EPC / 4) + u] = __ldg(reinterpret_cast<const float4 *>(g) + (EPC / 4) * c + u);
            }
        }
    }
#pragma unroll
    for (int b = 0; b < QB; ++b) {
        dt_chunk_vals<XF32>(q[b], f[b]);
        if constexpr (NORM) {
            if (c0 + 32 * b < nch) {
#pragma unroll
                for (int h = 0; h < EPC; ++h) {
                    const float4 gq = gv[b * (EPC / 4) + h / 4];
                    const float gh = (h & 3) == 0 ? gq.x : (h & 3) == 1 ? gq.y : (h & 3) == 2 ? gq.z : gq.w;
                    f[b][h] = __fmul_rn(__fmul_rn(f[b][h], r), gh);
                }
            }
        }
    }
}

// The absmax pass and the quantise pass over the (normalised) row of token m.
template <bool XF32, bool NORM, int QB>
BITNET_DEVINL void dt_quant_pass(const DtProgram &p, const DtOp &op, int m, const char *row, int nch, float r)
{
    const int lane = threadIdx.x & 31;
    constexpr int EPC = XF32 ? 4 : 8;
    float mx = 0.0f;
    for (int c0 = lane; c0 < nch; c0 += 32 * QB) {
        float fr[QB][EPC];
        dt_batch<XF32, NORM, QB>(row, c0, nch, op.norm_g, r, fr);
#pragma unroll
        for (int b = 0; b < QB; ++b)
#pragma unroll
            for (int h = 0; h < EPC; ++h) mx = fmaxf(mx, fabsf(fr[b][h]));
    }
    mx = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(mx)));
    const float sc = quant_scale(mx);
    int rsum = 0;
    int8_t *xq = op.xq;
    for (int c0 = lane; c0 < nch; c0 += 32 * QB) {
        float fr[QB][EPC];
        dt_batch<XF32, NORM, QB>(row, c0, nch, op.norm_g, r, fr);
#pragma unroll
        for (int b = 0; b < QB; ++b) {
            const int c = c0 + 32 * b;
            if (c < nch) {
                int q[EPC];
#pragma unroll
                for (int h = 0; h < EPC; ++h) {
                    q[h] = quant_one(fr[b][h], sc);
                    rsum += q[h];
                }
                const int k0 = c * EPC;
                int8_t *dst = xq + dt_xq_offset(k0, m, p.Mp, op.K);
                if constexpr (XF32) {
                    *reinterpret_cast<uint32_t *>(dst) = pack4_s8(q[0], q[1], q[2], q[3]);
                } else {
                    *reinterpret_cast<uint2 *>(dst) =
                        make_uint2(pack4_s8(q[0], q[1], q[2], q[3]), pack4_s8(q[4], q[5], q[6], q[7]));
                }
            }
        }
    }
    rsum = warp_sum(rsum);
    if (lane == 0) {
        op.s[m] = sc;
        op.rs[m] = rsum;
    }
}

template <bool XF32, int SHRINK>
BITNET_DEVINL void dt_quant_warp(const DtProgram &p, const DtOp &op, int m, unsigned char *smem)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int EPC = XF32 ? 4 : 8; // elements per 16-byte chunk
    // chunks per lane per batch: 32 values in the absmax and quantise passes, 16 in the sum-of-squares
    // and normalised ones; halved (SHRINK = 2) where the contraction of many token tiles holds more registers
    constexpr int QB = (XF32 ? 8 : 4) / SHRINK;
    constexpr int QS = (XF32 ? 4 : 2) / SHRINK;
    const int K = op.K, nch = K / EPC;
    const char *row = static_cast<const char *>(op.x) + (size_t)m * K * (XF32 ? 4 : 2);
    float r = 1.0f;
    if (op.norm_g) {
        // RMS normalisation: exact sum of squares (rounded once), r in binary64 -> binary32
        float xm = 0.0f;
        for (int c0 = lane; c0 < nch; c0 += 32 * QS) {
            float f[QS][EPC];
            dt_batch<XF32, false, QS>(row, c0, nch, nullptr, 1.0f, f);
#pragma unroll
            for (int b = 0; b < QB; ++b)
#pragma unroll
                for (int h = 0; h < EPC; ++h) xm = fmaxf(xm, fabsf(f[b][h]));
        }
        xm = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(xm)));
        const uint32_t E = ss_exponent(xm); // the largest exponent of the row
        SsWindow acc;
        if (E != 0)
            for (int c0 = lane; c0 < nch; c0 += 32 * QS) {
                float f[QS][EPC];
                dt_batch<XF32, false, QS>(row, c0, nch, nullptr, 1.0f, f);
#pragma unroll
                for (int b = 0; b < QS; ++b)
#pragma unroll
                    for (int h = 0; h < EPC; ++h) ss_window_add(acc, f[b][h], E);
            }
        ss_warp_sum(acc.lo, acc.hi);
        double ss;
        if (!__all_sync(0xffffffffu, acc.fits)) { // warp-uniform
            unsigned long long *dig = reinterpret_cast<unsigned long long *>(smem + DT_DIG) + warp * SS_LONG_DIGITS;
            if (lane < SS_LONG_DIGITS) dig[lane] = 0ull;
            __syncwarp();
            for (int c0 = lane; c0 < nch; c0 += 32 * QS) {
                float f[QS][EPC];
                dt_batch<XF32, false, QS>(row, c0, nch, nullptr, 1.0f, f);
#pragma unroll
                for (int b = 0; b < QS; ++b)
#pragma unroll
                    for (int h = 0; h < EPC; ++h) ss_long_add(dig, f[b][h]);
            }
            __syncwarp();
            ss = ss_long_round(dig);
        } else {
            ss = E ? ss_window_round(acc.lo, acc.hi, E) : 0.0;
        }
        r = __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(__ddiv_rn(ss, (double)K), (double)op.norm_eps))));
    }
    if (op.norm_g) dt_quant_pass<XF32, true, QS>(p, op, m, row, nch, r); // + the weights: smaller batches
    else dt_quant_pass<XF32, false, QB>(p, op, m, row, nch, r);
}

// ---- quant task of one token on all compute warps (M <= 8) --------------------
// Thread t holds 16-byte chunks c = t + 256 i of the row (x read once, from L2,
// in one round trip): the shortest latency for a single row, which is what a
// decode step of few tokens waits on.
template <bool XF32>
BITNET_DEVINL void dt_quant_row(const DtProgram &p, const DtOp &op, int m, unsigned char *smem)
{
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int EPC = XF32 ? 4 : 8; // elements per chunk
    constexpr int DT_QUANT_CH = dt_quant_ch<XF32>();
    const int K = op.K, nch = K / EPC;
    float *red = reinterpret_cast<float *>(smem + DT_RED);           // [8] maxima / scratch
    int *redi = reinterpret_cast<int *>(smem + DT_RED + 32);         // [8] row sums
    uint32_t *rede = reinterpret_cast<uint32_t *>(smem + DT_RED + 64);  // [8] exponents
    int *redf = reinterpret_cast<int *>(smem + DT_RED + 96);         // [8] window fits
    uint64_t *redw = reinterpret_cast<uint64_t *>(smem + DT_RED + 128); // [8][2] window sums
    unsigned long long *dig = reinterpret_cast<unsigned long long *>(smem + DT_RED + 256); // [20]
    float *bc = reinterpret_cast<float *>(smem + DT_RED + 416);     // broadcasts
    const char *row = static_cast<const char *>(op.x) + (size_t)m * K * (XF32 ? 4 : 2);
    float v[DT_QUANT_CH * EPC];
#pragma unroll
    for (int i = 0; i < DT_QUANT_CH; ++i) {
        const int c = tid + 256 * i;
        uint4 q = make_uint4(0u, 0u, 0u, 0u);
        if (c < nch) q = dt_ld_cg16(row + 16 * (size_t)c);
        if constexpr (XF32) {
            v[4 * i + 0] = __uint_as_float(q.x);
            v[4 * i + 1] = __uint_as_float(q.y);
            v[4 * i + 2] = __uint_as_float(q.z);
            v[4 * i + 3] = __uint_as_float(q.w);
        } else {
            const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                v[8 * i + 2 * h] = bf16_bits_lo(w[h]);
                v[8 * i + 2 * h + 1] = bf16_bits_hi(w[h]);
            }
        }
    }
    if (op.norm_g) {
        // RMS normalisation: exact sum of squares (rounded once), r in binary64 -> binary32
        uint32_t em = 0;
#pragma unroll
        for (int e = 0; e < DT_QUANT_CH * EPC; ++e) em = max(em, ss_exponent(v[e]));
        em = __reduce_max_sync(0xffffffffu, em);
        if (lane == 0) rede[warp] = em;
        if (tid < SS_LONG_DIGITS) dig[tid] = 0ull;
        dt_bar_compute();
        uint32_t E = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) E = max(E, rede[w]);
        SsWindow acc;
        if (E != 0) {
#pragma unroll
            for (int e = 0; e < DT_QUANT_CH * EPC; ++e) ss_window_add(acc, v[e], E);
        }
        ss_warp_sum(acc.lo, acc.hi);
        const bool fits = __all_sync(0xffffffffu, acc.fits);
        if (lane == 0) {
            redw[2 * warp] = acc.lo;
            redw[2 * warp + 1] = acc.hi;
            redf[warp] = fits ? 1 : 0;
        }
        dt_bar_compute();
        bool slow = false;
#pragma unroll
        for (int w = 0; w < 8; ++w) slow = slow || redf[w] == 0;
        if (slow) {
#pragma unroll
            for (int e = 0; e < DT_QUANT_CH * EPC; ++e) ss_long_add(dig, v[e]);
            dt_bar_compute();
        }
        if (tid == 0) {
            double ss;
            if (slow) {
                ss = ss_long_round(dig);
            } else {
                uint64_t lo = 0, hi = 0;
                for (int w = 0; w < 8; ++w) ss_add128(lo, hi, redw[2 * w], redw[2 * w + 1]);
                ss = E ? ss_window_round(lo, hi, E) : 0.0;
            }
            const double mean = __ddiv_rn(ss, (double)K);
            bc[0] = __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(mean, (double)op.norm_eps))));
        }
        dt_bar_compute();
        const float r = bc[0];
#pragma unroll
        for (int i = 0; i < DT_QUANT_CH; ++i) {
#pragma unroll
            for (int h = 0; h < EPC; ++h) {
                const int k = (tid + 256 * i) * EPC + h;
                if (k < K) v[EPC * i + h] = __fmul_rn(__fmul_rn(v[EPC * i + h], r), __ldg(op.norm_g + k));
            }
        }
    }
    // per-token absmax (padding elements are zero)
    float mx = 0.0f;
#pragma unroll
    for (int e = 0; e < DT_QUANT_CH * EPC; ++e) mx = fmaxf(mx, fabsf(v[e]));
    mx = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(mx)));
    if (lane == 0) red[warp] = mx;
    dt_bar_compute();
    float amax = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) amax = fmaxf(amax, red[w]);
    const float sc = quant_scale(amax);
    // quantise into the fragment layout: byte k of token m at ((k / 64) * Mp + m) * 64 + k % 64
    int rsum = 0;
    int8_t *xq = op.xq;
#pragma unroll
    for (int i = 0; i < DT_QUANT_CH; ++i) {
        const int c = tid + 256 * i;
        if (c < nch) {
            int q[EPC];
#pragma unroll
            for (int h = 0; h < EPC; ++h) {
                q[h] = quant_one(v[EPC * i + h], sc);
                rsum += q[h];
            }
            const int k0 = c * EPC;
            int8_t *dst = xq + dt_xq_offset(k0, m, p.Mp, K);
            if constexpr (XF32) {
                *reinterpret_cast<uint32_t *>(dst) = pack4_s8(q[0], q[1], q[2], q[3]);
            } else {
                *reinterpret_cast<uint2 *>(dst) =
                    make_uint2(pack4_s8(q[0], q[1], q[2], q[3]), pack4_s8(q[4], q[5], q[6], q[7]));
            }
        }
    }
    rsum = warp_sum(rsum);
    if (lane == 0) redi[warp] = rsum;
    dt_bar_compute();
    if (tid == 0) {
        int tot = 0;
        for (int w = 0; w < 8; ++w) tot += redi[w];
        op.s[m] = sc;
        op.rs[m] = tot;
    }
}

// ---- row task contraction over one piece (compute warp w) ------------------
// The A fragments are the packed words masked in place, without shifting:
// (w & (0x03030303 << 2j)) holds the codes of position j of each byte scaled
// by 4^j (at most 2 * 64 = 128: still a u8 operand).  Accumulator set
// acc[r][j] (SC = 4) therefore collects 4^j * sum c*x, exactly (|sum c*x| <
// 2^21 for K <= 8192, so 64 * it fits int32), and the sets are combined with
// exact arithmetic shifts at the end of the task.  With SC = 2 (many token
// tiles, fewer registers) the word is used as is for positions 0, 1 and
// shifted by 4 for positions 2, 3: set j & 1 holds 4^(j & 1) * its sum.
// One mma covers a pair of k-blocks (its two k halves) at one position j.
// acc[r][j][tt][4]: row group r of the warp, set j, token tile tt.  The
// fragment's rows g and g + 8 are slot rows lo and hi of row group 0 (row
// group r is 128 rows further): BitLinear 16 w + g and 16 w + g + 8, gated FFN
// 8 w + g (gate) and 64 + 8 w + g (up).  Rows are 128 bytes with the 16-byte
// chunks swizzled by (row & 7) = g, so k-block kb of a row is its chunk
// kb ^ g; wlo / whi: this lane's word in chunk 0 of rows lo / hi, g16 = g << 4.
template <int SC>
BITNET_DEVINL uint32_t dt_code_bits(uint32_t w, uint32_t w4, int j)
{
    if constexpr (SC == 4) return w & (0x03030303u << (2 * j));
    else return (j < 2 ? w : w4) & (0x03030303u << (2 * (j & 1)));
}

template <int TT, int SC, int RG>
BITNET_DEVINL void dt_kpair(int (&acc)[RG][SC][TT][4], const uint32_t (&l0)[RG], const uint32_t (&h0)[RG],
                            const uint32_t (&l1)[RG], const uint32_t (&h1)[RG], const uint4 (&b0)[TT],
                            const uint4 (&b1)[TT])
{
#pragma unroll
    for (int r = 0; r < RG; ++r) {
        const uint32_t L0 = l0[r], H0 = h0[r], L1 = l1[r], H1 = h1[r];
        const uint32_t L04 = SC == 4 ? 0u : L0 >> 4, H04 = SC == 4 ? 0u : H0 >> 4;
        const uint32_t L14 = SC == 4 ? 0u : L1 >> 4, H14 = SC == 4 ? 0u : H1 >> 4;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t a0 = dt_code_bits<SC>(L0, L04, j), a1 = dt_code_bits<SC>(H0, H04, j);
            const uint32_t a2 = dt_code_bits<SC>(L1, L14, j), a3 = dt_code_bits<SC>(H1, H14, j);
#pragma unroll
            for (int tt = 0; tt < TT; ++tt) {
                const uint32_t bj0 = j == 0 ? b0[tt].x : j == 1 ? b0[tt].y : j == 2 ? b0[tt].z : b0[tt].w;
                const uint32_t bj1 = j == 0 ? b1[tt].x : j == 1 ? b1[tt].y : j == 2 ? b1[tt].z : b1[tt].w;
                mma_u8s8_16832(acc[r][SC == 4 ? j : (j & 1)][tt], a0, a1, a2, a3, bj0, bj1);
            }
        }
    }
}

BITNET_DEVINL uint4 dt_ld_b(uint32_t addr)
{
    uint4 b;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w) : "r"(addr));
    return b;
}

struct DtArow {
    uint32_t lo, hi, g16;
};

template <int RG>
BITNET_DEVINL void dt_ld_a(uint32_t (&lo)[RG], uint32_t (&hi)[RG], const DtArow &w, int kb)
{
    const uint32_t kx = ((uint32_t)kb << 4) ^ w.g16;
#pragma unroll
    for (int r = 0; r < RG; ++r) {
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(lo[r]) : "r"(w.lo + (uint32_t)(r * DT_WBYTES) + kx));
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(hi[r]) : "r"(w.hi + (uint32_t)(r * DT_WBYTES) + kx));
    }
}

// A ragged piece (fewer than 8 k-blocks; an odd last block is paired with zeros).
template <int TT, int SC, int RG>
BITNET_DEVINL void dt_piece(int (&acc)[RG][SC][TT][4], const DtArow &wrow, uint32_t xrow, int Mp, int nkb)
{
#pragma unroll
    for (int kp = 0; kp < DT_KB / 2; ++kp) {
        if (2 * kp < nkb) {
            const bool two = 2 * kp + 1 < nkb;
            uint32_t l0[RG], h0[RG], l1[RG], h1[RG];
            uint4 b0[TT], b1[TT];
            dt_ld_a<RG>(l0, h0, wrow, 2 * kp);
            if (two) {
                dt_ld_a<RG>(l1, h1, wrow, 2 * kp + 1);
            } else {
#pragma unroll
                for (int r = 0; r < RG; ++r) l1[r] = h1[r] = 0u;
            }
#pragma unroll
            for (int tt = 0; tt < TT; ++tt) {
                b0[tt] = dt_ld_b(xrow + (uint32_t)((2 * kp * Mp + tt * 8) * 64));
                b1[tt] = two ? dt_ld_b(xrow + (uint32_t)(((2 * kp + 1) * Mp + tt * 8) * 64)) : make_uint4(0, 0, 0, 0);
            }
            dt_kpair<TT, SC, RG>(acc, l0, h0, l1, h1, b0, b1);
        }
    }
}

// A full piece (8 k-blocks) in the permuted order of dt_xq_offset: lane group
// t4 of k-block kb uses word 8 t4 + kb of each row, so a row's eight words for
// the lane are its chunks 2 t4 and 2 t4 + 1 (two 16-byte loads; chunk c sits
// at c ^ g).  Every weight fragment (and, for one token tile, every activation
// fragment) is loaded before the first mma.
template <int RG>
BITNET_DEVINL void dt_ld_a_full(uint32_t (&lo)[DT_KB][RG], uint32_t (&hi)[DT_KB][RG], const DtArow &w, uint32_t t4)
{
    const uint32_t base_lo = w.lo - 4 * t4, base_hi = w.hi - 4 * t4; // chunk 0 of rows lo / hi
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t cx = ((2 * t4 + h) << 4) ^ w.g16;
#pragma unroll
        for (int r = 0; r < RG; ++r) {
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(lo[4 * h][r]), "=r"(lo[4 * h + 1][r]), "=r"(lo[4 * h + 2][r]), "=r"(lo[4 * h + 3][r])
                         : "r"(base_lo + (uint32_t)(r * DT_WBYTES) + cx));
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(hi[4 * h][r]), "=r"(hi[4 * h + 1][r]), "=r"(hi[4 * h + 2][r]), "=r"(hi[4 * h + 3][r])
                         : "r"(base_hi + (uint32_t)(r * DT_WBYTES) + cx));
        }
    }
}

template <int TT, int SC, int RG>
BITNET_DEVINL void dt_piece_full(int (&acc)[RG][SC][TT][4], const DtArow &wrow, uint32_t xrow, int Mp, uint32_t t4)
{
    uint32_t lo[DT_KB][RG], hi[DT_KB][RG];
    dt_ld_a_full<RG>(lo, hi, wrow, t4);
    if constexpr (TT == 1) {
        uint4 bq[DT_KB][1];
#pragma unroll
        for (int kb = 0; kb < DT_KB; ++kb) bq[kb][0] = dt_ld_b(xrow + (uint32_t)(kb * Mp * 64));
#pragma unroll
        for (int kp = 0; kp < DT_KB / 2; ++kp)
            dt_kpair<TT, SC, RG>(acc, lo[2 * kp], hi[2 * kp], lo[2 * kp + 1], hi[2 * kp + 1], bq[2 * kp],
                                 bq[2 * kp + 1]);
    } else {
#pragma unroll
        for (int kp = 0; kp < DT_KB / 2; ++kp) {
            uint4 b0[TT], b1[TT];
#pragma unroll
            for (int tt = 0; tt < TT; ++tt) {
                b0[tt] = dt_ld_b(xrow + (uint32_t)((2 * kp * Mp + tt * 8) * 64));
                b1[tt] = dt_ld_b(xrow + (uint32_t)(((2 * kp + 1) * Mp + tt * 8) * 64));
            }
            dt_kpair<TT, SC, RG>(acc, lo[2 * kp], hi[2 * kp], lo[2 * kp + 1], hi[2 * kp + 1], b0, b1);
        }
    }
}

template <int TT, int RG>
BITNET_DEVINL void dt_compute(const DtProgram &p, unsigned char *smem)
{
    constexpr int SC = TT <= 2 ? 4 : 2; // accumulator sets (scales of the masked codes)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t4 = lane & 3;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + DT_BAR_FULL);
    uint64_t *empty = reinterpret_cast<uint64_t *>(smem + DT_BAR_EMPTY);
    uint64_t *qfull = reinterpret_cast<uint64_t *>(smem + DT_BAR_QFULL);
    uint64_t *qinfo = reinterpret_cast<uint64_t *>(smem + DT_BAR_QINFO);
    uint64_t *qempty = reinterpret_cast<uint64_t *>(smem + DT_BAR_QEMPTY);
    uint64_t *cdone = reinterpret_cast<uint64_t *>(smem + DT_BAR_CDONE);
    const volatile int *qtask = reinterpret_cast<const volatile int *>(smem + DT_QTASK);
    const uint32_t ring = smem_u32(smem + DT_HDR);
    const int Mp = p.Mp, M = p.M;
    uint32_t seq = 0;
    DtRing ring_pos;
    for (;;) {
        const int e = (int)(seq % DT_QUEUE);
        mbar_wait(&qfull[e], (seq / DT_QUEUE) & 1u);
        const int t = qtask[e];
        if (t == DT_QEND) break;
        const DtTask tk = dt_unpack(t);
        if (tk.quant) {
            const DtOp &op = p.ops[tk.op];
            if constexpr (TT == 1) {
                // one token on all compute warps; the op that wrote x (read after write) is complete
                if (tid == 0)
                    for (int d = 0; d < op.nq; ++d)
                        dt_wait_count(dt_rdone(p, op.deps[d]), dt_rtarget(p, op.deps[d]));
                dt_bar_compute();
                if (op.xf32) dt_quant_row<true>(p, op, tk.idx, smem);
                else dt_quant_row<false>(p, op, tk.idx, smem);
            } else {
                const int m = tk.idx * 8 + warp;
                if (m < M) {
                    // the op that wrote x (read after write) is complete
                    if (lane == 0)
                        for (int d = 0; d < op.nq; ++d)
                            dt_wait_count(dt_rdone(p, op.deps[d]), dt_rtarget(p, op.deps[d]));
                    __syncwarp();
                    if (op.xf32) dt_quant_warp<true, TT >= 8 ? 2 : 1>(p, op, m, smem);
                    else dt_quant_warp<false, TT >= 8 ? 2 : 1>(p, op, m, smem);
                }
            }
            // every lane's stores precede lane 0's arrival; the completion warp counts the
            // task once every warp arrived
            __syncwarp();
            if (lane == 0) mbar_arrive(&cdone[e]);
        } else {
            int acc[RG][SC][TT][4];
#pragma unroll
            for (int r = 0; r < RG; ++r)
#pragma unroll
                for (int a = 0; a < SC; ++a)
#pragma unroll
                    for (int tt = 0; tt < TT; ++tt)
#pragma unroll
                        for (int c = 0; c < 4; ++c) acc[r][a][tt][c] = 0;
            // the entry's op fields (valid until this task's qempty arrival)
            const int K = reinterpret_cast<const DtEntry *>(smem + DT_QOP)[e].K;
            const int np = dt_pieces(K);
            const bool ffn = reinterpret_cast<const DtEntry *>(smem + DT_QOP)[e].nmat == 2;
            const uint32_t row_lo = ffn ? (uint32_t)(warp * 8 + g) : (uint32_t)(warp * 16 + g);
            const uint32_t row_hi = row_lo + (ffn ? (uint32_t)DT_BOX_ROWS : 8u);
            const uint32_t xlane = (uint32_t)(RG * DT_WBYTES + g * 64 + t4 * 16);
            for (int pc = 0; pc < np; ++pc, ring_pos.next(p.n_slots)) {
                const int s = ring_pos.slot;
                mbar_wait(&full[s], ring_pos.par);
                const uint32_t base = ring + (uint32_t)s * (uint32_t)p.slot_bytes;
                const int nkb = min(DT_KB, (K - pc * DT_KC) >> 6);
                const DtArow wr = {base + row_lo * DT_PITCH + t4 * 4, base + row_hi * DT_PITCH + t4 * 4,
                                   (uint32_t)g << 4};
                if (nkb == DT_KB)
                    dt_piece_full<TT, SC, RG>(acc, wr, base + xlane, Mp, (uint32_t)t4);
                else
                    dt_piece<TT, SC, RG>(acc, wr, base + xlane, Mp, nkb);
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
            }
            // set a holds 4^a times its sum: exact arithmetic shifts
#pragma unroll
            for (int r = 0; r < RG; ++r)
#pragma unroll
                for (int a = 1; a < SC; ++a)
#pragma unroll
                    for (int tt = 0; tt < TT; ++tt)
#pragma unroll
                        for (int c = 0; c < 4; ++c) acc[r][0][tt][c] += acc[r][a][tt][c] >> (2 * a);
            // epilogue: y = fl((float)(sum c*x - sum x) * fl(gamma / s))
            mbar_wait(&qinfo[e], (seq / DT_QUEUE) & 1u);
            const unsigned char *inf = smem + DT_INFO + e * DT_INFO_BYTES;
            const float *ir0 = reinterpret_cast<const float *>(inf + DT_INFO_R0);
            const float *ir1 = reinterpret_cast<const float *>(inf + DT_INFO_R1);
            const int *irs = reinterpret_cast<const int *>(inf + DT_INFO_RS);
            const int N = reinterpret_cast<const DtEntry *>(smem + DT_QOP)[e].N;
            float *y = reinterpret_cast<const DtEntry *>(smem + DT_QOP)[e].y;
            if (ffn) {
#pragma unroll
                for (int tt = 0; tt < TT; ++tt)
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int m = tt * 8 + 2 * t4 + q;
                        if (m < M) {
                            const int rsm = irs[m];
                            const float rg0 = ir0[m], rg1 = ir1[m];
#pragma unroll
                            for (int r = 0; r < RG; ++r) {
                                const int n = tk.idx * (RG * DT_ROWS / 2) + (warp + 8 * r) * 8 + g;
                                if (n < N) {
                                    const float gv = __fmul_rn((float)(acc[r][0][tt][q] - rsm), rg0);
                                    const float uv = __fmul_rn((float)(acc[r][0][tt][2 + q] - rsm), rg1);
                                    const float pg = gv > 0.0f ? gv : 0.0f;
                                    y[(size_t)m * N + n] = __fmul_rn(__fmul_rn(pg, pg), uv);
                                }
                            }
                        }
                    }
            } else {
#pragma unroll
                for (int tt = 0; tt < TT; ++tt)
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const int m = tt * 8 + 2 * t4 + q;
                        if (m < M) {
                            const int rsm = irs[m];
                            const float rsc = ir0[m];
#pragma unroll
                            for (int r = 0; r < RG; ++r) {
                                const int n0 = tk.idx * (RG * DT_ROWS) + (warp + 8 * r) * 16 + g;
#pragma unroll
                                for (int h = 0; h < 2; ++h) {
                                    const int n = n0 + 8 * h;
                                    if (n < N)
                                        y[(size_t)m * N + n] = __fmul_rn((float)(acc[r][0][tt][2 * h + q] - rsm), rsc);
                                }
                            }
                        }
                    }
            }
            // every lane's stores precede (warp barrier) lane 0's arrival; the completion warp
            // makes them visible device-wide and counts the task
            __syncwarp();
            if (lane == 0) mbar_arrive(&cdone[e]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&qempty[e]);
        ++seq;
    }
}

// ---- completion warp (warp 10) ----------------------------------------------
// Tasks in queue order: once the eight compute warps arrived (their stores are
// issued and ordered before the arrival), one fence makes the stores visible
// at device scope and one atomic counts the task.
BITNET_DEVINL void dt_completion(const DtProgram &p, unsigned char *smem)
{
    const int lane = threadIdx.x & 31;
    uint64_t *qfull = reinterpret_cast<uint64_t *>(smem + DT_BAR_QFULL);
    uint64_t *qempty = reinterpret_cast<uint64_t *>(smem + DT_BAR_QEMPTY);
    uint64_t *cdone = reinterpret_cast<uint64_t *>(smem + DT_BAR_CDONE);
    const volatile int *qtask = reinterpret_cast<const volatile int *>(smem + DT_QTASK);
    for (uint32_t seq = 0;; ++seq) {
        const int e = (int)(seq % DT_QUEUE);
        const uint32_t par = (seq / DT_QUEUE) & 1u;
        mbar_wait(&qfull[e], par);
        const int t = qtask[e];
        if (t == DT_QEND) break;
        const DtTask tk = dt_unpack(t);
        mbar_wait(&cdone[e], par);
        if (lane == 0) {
            __threadfence();
            atomicAdd(tk.quant ? dt_qdone(p, tk.op) : dt_rdone(p, tk.op), 1u);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&qempty[e]);
    }
}

template <int TT, int RG>
__global__ void __launch_bounds__(DT_THREADS, 1) k_decode_tasks(const __grid_constant__ DtProgram p)
{
    extern __shared__ unsigned char dt_smem_raw[];
    unsigned char *smem =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(dt_smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x;
    if (tid == 0) {
        uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
        for (int i = 0; i < p.n_slots; ++i) {
            mbar_init(&bars[DT_BAR_FULL / 8 + i], 33); // weight producer (expect_tx) + 32 activation lanes (cp.async, noinc)
            mbar_init(&bars[DT_BAR_EMPTY / 8 + i], 8); // compute warps
        }
        for (int i = 0; i < DT_QUEUE; ++i) {
            mbar_init(&bars[DT_BAR_QFULL / 8 + i], 1);
            mbar_init(&bars[DT_BAR_QINFO / 8 + i], 32);  // activation producer lanes
            mbar_init(&bars[DT_BAR_QEMPTY / 8 + i], 10); // compute warps, activation producer, completion warp
            mbar_init(&bars[DT_BAR_CDONE / 8 + i], 8);   // compute warps
        }
        fence_mbarrier_init();
    }
    __syncthreads();
    const int warp = tid >> 5;
    if (warp == 8) dt_weight_producer<RG>(p, smem);
    else if (warp == 9) dt_act_producer<RG>(p, smem);
    else if (warp == 10) dt_completion(p, smem);
    else dt_compute<TT, RG>(p, smem);
    __syncthreads();
    if (tid == 0) {
        // the last CTA out leaves the counters zeroed for the next launch
        __threadfence();
        const unsigned prev = atomicAdd(&p.counters[DT_CNT_EXIT], 1u);
        if (prev == gridDim.x - 1) {
            __threadfence();
            for (int i = 0; i < DT_CNT_OPS + 2 * p.n_ops; ++i) atomicExch(&p.counters[i], 0u);
        }
    }
}

} // namespace bitnet
