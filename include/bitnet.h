/*
 * bitnet.h -- C ABI of the B200 (sm_100a) BitLinear forward library.
 *
 * The operation is the BitLinear layer of BitNet b1.58 as the "BitNet" model
 * page of the transformers documentation describes it (section "Model
 * details", items "Architecture" and "Quantization"): weights quantised to
 * {-1, 0, +1} by absmean quantisation, activations quantised to 8-bit integers
 * by per-token absmax quantisation (W1.58A8), no bias, and a squared-ReLU FFN
 * (BitNetConfig: hidden_act = "relu2").  The page gives no formulas; the ones
 * implemented here are
 *
 *   gamma = mean |W|                       (one per weight matrix, fp32)
 *   W_q   = clamp(rne(W / (gamma + eps)), -1, 1)
 *   s_m   = 127 / max(max_k |x_mk|, 1e-5)  (one per token = row of x, fp32)
 *   x_q   = clamp(rne(x * s_m), -128, 127)
 *   acc   = x_q . W_q^T                    (exact int32)
 *   y     = (float)acc * (gamma / s_m)     (fp32)
 *   h     = (g > 0 ? g*g : 0) * u          (gate/up FFN, g and u two BitLinear outputs)
 *
 * rne = round half to even.  The quantisers use IEEE fp32 division and one
 * rounded fp32 product, so their integer results are reproducible exactly.
 *
 * Layouts (all row-major, C order):
 *   x         [M][K]   bf16 or fp32 activations (M tokens, K input features)
 *   W latent  [N][K]   fp32 (N output features)
 *   w_packed  [N][K/4] uint8: code c = W_q + 1 in {0,1,2}; within row n the
 *             little-endian 32-bit word at byte 4*g holds weights
 *             k = 16g .. 16g+15, weight 16g + 4j + b in byte b, bits 2j..2j+1
 *   x_q       [M][K]   int8
 *   y, h      [M][N]   fp32
 *   acc       [M][N]   int32
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers unless stated otherwise; the caller owns all
 *     memory.  The library never allocates or frees device memory and never
 *     synchronises the stream; work is enqueued on `stream` and runs
 *     asynchronously.
 *   - Arguments are validated on the host before anything is launched; on any
 *     error nothing is launched and the status says why.  After launching,
 *     a launch error reported by the CUDA runtime is returned as
 *     BITNET_ERR_CUDA.  Faults that happen later, while the kernels run, are
 *     reported by the CUDA runtime on the next synchronising call.
 *   - Shapes: M >= 1, N >= 1, K >= 64 with K % 64 == 0.  Every pointer must be
 *     16-byte aligned.
 *   - Inputs must be finite (not checked).
 *   - Reads of w_packed and gamma may begin before earlier work on the same
 *     stream has finished (programmatic dependent launch): they must not be
 *     written by work still in flight on that stream.  Pack, then synchronise
 *     (or wait on an event) before the first call that reads the result.
 *     Everything else obeys normal stream order.
 */
#ifndef BITNET_H
#define BITNET_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BITNET_OK = 0,
    BITNET_ERR_INVALID_ARG = 1,       /* null pointer, non-positive size, bad enum */
    BITNET_ERR_UNSUPPORTED_SHAPE = 2, /* K not a positive multiple of 64, sizes too large */
    BITNET_ERR_MISALIGNED = 3,        /* a pointer is not 16-byte aligned */
    BITNET_ERR_CUDA = 4,              /* the CUDA runtime reported an error */
    BITNET_ERR_TIMEOUT = 5,           /* a device-side wait gave up (see bitnet_device_status) */
    BITNET_ERR_WORKSPACE = 6          /* workspace pointer null or too small */
} bitnet_status_t;

typedef enum {
    BITNET_DTYPE_BF16 = 0,
    BITNET_DTYPE_F32 = 1
} bitnet_dtype_t;

/* Kernel selection for bitnet_linear / bitnet_ffn_gate_up. */
typedef enum {
    BITNET_DISPATCH_AUTO = 0,         /* by M: decode kernels for M <= 64, else prefill */
    BITNET_DISPATCH_DECODE_FUSED = 1, /* decode kernel quantising x itself (M <= 64) */
    BITNET_DISPATCH_DECODE = 2,       /* quantiser kernel + decode kernel (M <= 64) */
    BITNET_DISPATCH_PREFILL = 3       /* quantiser kernel + tcgen05 GEMM (any M) */
} bitnet_dispatch_t;

/* Human-readable name of a status code (static string, never NULL). */
const char *bitnet_status_string(bitnet_status_t status);

/* ABI version of this library: major * 10000 + minor * 100 + patch. */
int bitnet_version(void);

/*
 * Workspace needed by bitnet_pack_weights for an [N][K] matrix: N * 8 bytes
 * (one fp64 partial sum per row).
 */
size_t bitnet_pack_workspace_size(int64_t N, int64_t K);

/*
 * Offline absmean ternarisation and 2-bit packing of one weight matrix
 * (page: "Quantization" -- ternary {-1, 0, +1} weights by absmean; "Model
 * variants" -- the deployable weights are stored packed).
 *
 *   w          [N][K] fp32 latent weights (device, read)
 *   eps        additive epsilon of gamma + eps (1e-5 in BitNet b1.58)
 *   w_packed   [N][K/4] uint8 packed codes (device, written)
 *   gamma      [1] fp32 (device, written): mean |W|, accumulated in fp64 in a
 *              fixed order (each row left to right, then the rows top to
 *              bottom) and rounded once to fp32
 *   workspace  device scratch of bitnet_pack_workspace_size(N, K) bytes
 *
 * Deterministic: identical inputs give identical bytes on every run.
 */
bitnet_status_t bitnet_pack_weights(const float *w, int64_t N, int64_t K, float eps,
                                    uint8_t *w_packed, float *gamma,
                                    void *workspace, size_t ws_bytes,
                                    cudaStream_t stream);

/*
 * Per-token absmax int8 quantisation of activations (page: "Quantization" --
 * 8-bit activations by absmax, per token).
 *
 *   x        [M][K] activations of type x_dtype (device, read)
 *   x_q      [M][K] int8 (device, written)
 *   s        [M] fp32 per-token scales s_m = 127 / max(max|x_m|, 1e-5) (device, written)
 *   rowsum   [M] int32 sum_k x_q[m][k] (device, written; may be NULL)
 */
bitnet_status_t bitnet_quant_act(const void *x, bitnet_dtype_t x_dtype, int64_t M, int64_t K,
                                 int8_t *x_q, float *s, int32_t *rowsum,
                                 cudaStream_t stream);

/*
 * Workspace needed by bitnet_linear / bitnet_ffn_gate_up for the given shape
 * (holds the quantised activations, scales and row sums between kernels).
 */
size_t bitnet_workspace_size(int64_t M, int64_t N, int64_t K);

/*
 * BitLinear forward y = dequant(quant(x) . W_q^T) (page: "Architecture" --
 * BitLinear layers without bias; "Quantization" -- W1.58A8).
 *
 *   x          [M][K] activations of type x_dtype (device, read)
 *   w_packed   [N][K/4] packed ternary weights from bitnet_pack_weights
 *   gamma      [1] fp32 weight scale from bitnet_pack_weights (device)
 *   y          [M][N] fp32 output (device, written)
 *   x_q_out    [M][K] int8 quantised activations (optional, may be NULL)
 *   s_out      [M] fp32 per-token scales (optional, may be NULL)
 *   acc_out    [M][N] int32 exact accumulators (optional, may be NULL)
 *   workspace  device scratch of at least bitnet_workspace_size(M, N, K) bytes
 *
 * Small M (decode) streams the packed weights through a GEMV-style kernel;
 * large M (prefill) runs a tcgen05 int8 tensor-core GEMM.  Both give
 * bit-identical results.
 */
bitnet_status_t bitnet_linear(const void *x, bitnet_dtype_t x_dtype, int64_t M, int64_t K,
                              const uint8_t *w_packed, const float *gamma, int64_t N,
                              float *y, int8_t *x_q_out, float *s_out, int32_t *acc_out,
                              void *workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * bitnet_linear without a caller-provided workspace, for callers that cannot
 * allocate device memory when they call: a serving engine that has already
 * reserved all free HBM for its own pool (KV cache) and hands kernels only
 * their inputs and outputs, plugin hosts that forbid allocation after
 * start-up, and latency-critical loops where an allocation's implicit device
 * synchronisation would stall the pipeline.  The BitNet page has no
 * counterpart to this call; it is a deployment convenience.
 *
 * Arguments and results are those of bitnet_linear without the optional
 * outputs and the workspace.  Scratch (quantised activations, scales, row
 * sums) lives in a fixed 8 MiB device array inside this library, held on
 * every GPU that loads the library until the process exits.  Shapes whose
 * scratch exceeds it, i.e. M * K + 2 * (M * 4) (each rounded up to 256 bytes)
 * > 8 MiB, are rejected with BITNET_ERR_WORKSPACE before anything is launched.
 *
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current), and so does the first
 * call after the device's context has been destroyed and created again
 * (cudaDeviceReset); make those calls before any stream capture.  No call allocates or frees memory.  All calls
 * share the one array and it keeps the last call's contents (nothing in it
 * needs to start at zero): calls that can overlap on the GPU -- on different
 * streams, or on different host threads -- race on it and give wrong
 * results; order them on one stream or use bitnet_linear.
 */
bitnet_status_t bitnet_linear_noalloc(const void *x, bitnet_dtype_t x_dtype, int64_t M, int64_t K,
                                      const uint8_t *w_packed, const float *gamma, int64_t N,
                                      float *y, cudaStream_t stream);

/*
 * Gate/up half of the BitNet FFN with the squared-ReLU gate fused in the
 * epilogue (page: "Architecture" -- ReLU^2 in the FFN; BitNetConfig
 * hidden_act = "relu2"):
 *   g = BitLinear_gate(x), u = BitLinear_up(x), h = relu(g)^2 * u.
 * Both projections share one quantisation of x.
 *
 *   x            [M][K] activations (device, read)
 *   wg_packed    [N][K/4], gamma_g [1]: gate projection
 *   wu_packed    [N][K/4], gamma_u [1]: up projection
 *   h            [M][N] fp32 output (device, written)
 *   acc_g_out, acc_u_out  [M][N] int32 accumulators (optional, may be NULL)
 *   workspace    as for bitnet_linear
 *
 * The down projection is a plain bitnet_linear call with x = h
 * (x_dtype = BITNET_DTYPE_F32), which quantises h per token again.
 */
bitnet_status_t bitnet_ffn_gate_up(const void *x, bitnet_dtype_t x_dtype, int64_t M, int64_t K,
                                   const uint8_t *wg_packed, const float *gamma_g,
                                   const uint8_t *wu_packed, const float *gamma_u, int64_t N,
                                   float *h, int32_t *acc_g_out, int32_t *acc_u_out,
                                   void *workspace, size_t ws_bytes, cudaStream_t stream);

/* ---- RMS normalisation (subln) fused in front of the quantiser ------------ */

/*
 * x_q = quant(RMSNorm(x)) in one pass over x (page: "Architecture" -- subln
 * normalisation, no bias in the normalisation layers; BitNetConfig
 * rms_norm_eps = 1e-5):
 *   y_k = (x_k * r) * g_k,  r = 1 / sqrt(mean_k(x_k^2) + eps)
 * followed by the per-token absmax quantiser of bitnet_quant_act applied to y.
 * Precision is fixed so that results are reproducible: the sum of squares
 * is the exact sum of the (exact) squares rounded once to the nearest fp64,
 * ties to even -- independent of any summation order; r is computed in fp64
 * with correctly rounded division and square root and rounded once to fp32;
 * y is two fp32 products in the order shown.
 *
 *   x      [M][K] activations of type x_dtype (device, read); K <= 8192
 *   g      [K] fp32 normalisation weight (device, read)
 *   eps    >= 0 (1e-5 in BitNet b1.58)
 *   x_q, s, rowsum   as bitnet_quant_act, for y
 */
bitnet_status_t bitnet_rmsnorm_quant(const void *x, bitnet_dtype_t x_dtype, int64_t M, int64_t K,
                                     const float *g, float eps, int8_t *x_q, float *s, int32_t *rowsum,
                                     cudaStream_t stream);

/*
 * bitnet_linear / bitnet_ffn_gate_up applied to RMSNorm(x) (weight g, epsilon
 * eps, as bitnet_rmsnorm_quant): the normalisation runs inside the
 * quantisation pass, so x is read once and never written back normalised.
 * Same arguments, results and workspace as bitnet_linear /
 * bitnet_ffn_gate_up otherwise (K <= 8192).  For M <= 64 the quantiser and
 * the decode GEMV are separate kernels (the fused-quantiser decode kernel is
 * not used); BITNET_DISPATCH_DECODE_FUSED gives BITNET_ERR_UNSUPPORTED_SHAPE.
 */
bitnet_status_t bitnet_linear_norm(const void *x, bitnet_dtype_t x_dtype, int64_t M, int64_t K,
                                   const float *g, float eps, const uint8_t *w_packed, const float *gamma,
                                   int64_t N, float *y, int8_t *x_q_out, float *s_out, int32_t *acc_out,
                                   void *workspace, size_t ws_bytes, cudaStream_t stream);

bitnet_status_t bitnet_ffn_gate_up_norm(const void *x, bitnet_dtype_t x_dtype, int64_t M, int64_t K,
                                        const float *g, float eps,
                                        const uint8_t *wg_packed, const float *gamma_g,
                                        const uint8_t *wu_packed, const float *gamma_u, int64_t N,
                                        float *h, int32_t *acc_g_out, int32_t *acc_u_out,
                                        void *workspace, size_t ws_bytes, cudaStream_t stream);

/* ---- output options: bf16 outputs, emitted and given per-token maxima ---- */

/*
 * bitnet_linear / bitnet_ffn_gate_up with options for chaining BitLinears
 * (page: "Quantization" -- every BitLinear quantises its input per token by
 * absmax, so the maximum of each output row is what the next BitLinear's
 * quantiser needs first).
 *
 *   x, x_dtype, M, K, weights, N, workspace, stream: as bitnet_linear /
 *              bitnet_ffn_gate_up
 *   x_amax     [M] fp32 (device, read; may be NULL): max_k |x[m][k]| given by
 *              the caller, typically the y_amax of the BitLinear that wrote x.
 *              The quantiser uses it instead of reducing the row (and the
 *              decode kernel skips the exchange of partial maxima between the
 *              CTAs of a cluster); the result is identical when it is the
 *              true maximum.  Not allowed together with norm_g (the maxima of
 *              x are not those of RMSNorm(x)): BITNET_ERR_INVALID_ARG.
 *   norm_g, norm_eps  optional RMS normalisation in front of the quantiser, as
 *              bitnet_linear_norm (norm_g NULL: none)
 *   y (h)      [M][N] output of type y_dtype (h_dtype): BITNET_DTYPE_F32, or
 *              BITNET_DTYPE_BF16 = the fp32 value rounded to the nearest bf16,
 *              ties to even.  The fp32 value is fl(acc * fl(gamma / s)) (and
 *              fl(fl(p * p) * u), p = max(g, 0), for the gated FFN), exactly
 *              as bitnet_linear / bitnet_ffn_gate_up store it.
 *   y_amax     [M] fp32 (device, written; may be NULL): max_n |y[m][n]| of the
 *              values as stored (after bf16 rounding), folded in by the
 *              epilogues with integer atomicMax on the bit patterns (exact and
 *              order-independent).  The library zeroes it first (inside the
 *              quantiser kernel, or with one small kernel ahead of the fused
 *              decode kernel).  Must not overlap x_amax (BITNET_ERR_INVALID_ARG).
 *
 * All pointers 16-byte aligned.  A bf16 y whose rows are not 16-byte
 * multiples (N % 8 != 0) is written with plain stores instead of tensor
 * stores.
 */
bitnet_status_t bitnet_linear_ex(const void *x, bitnet_dtype_t x_dtype, const float *x_amax, const float *norm_g,
                                 float norm_eps, int64_t M, int64_t K, const uint8_t *w_packed, const float *gamma,
                                 int64_t N, void *y, bitnet_dtype_t y_dtype, float *y_amax, void *workspace,
                                 size_t ws_bytes, cudaStream_t stream);

bitnet_status_t bitnet_ffn_gate_up_ex(const void *x, bitnet_dtype_t x_dtype, const float *x_amax,
                                      const float *norm_g, float norm_eps, int64_t M, int64_t K,
                                      const uint8_t *wg_packed, const float *gamma_g, const uint8_t *wu_packed,
                                      const float *gamma_u, int64_t N, void *h, bitnet_dtype_t h_dtype,
                                      float *h_amax, void *workspace, size_t ws_bytes, cudaStream_t stream);

/* ---- decode sequences: many small-M ops in one persistent launch ---------- */

typedef enum {
    BITNET_OP_LINEAR = 0,     /* y = BitLinear(x), as bitnet_linear */
    BITNET_OP_FFN_GATE_UP = 1 /* y = relu(BitLinear_gate(x))^2 * BitLinear_up(x), as bitnet_ffn_gate_up */
} bitnet_op_kind_t;

/* One op of a sequence.  All pointers are device pointers, 16-byte aligned. */
typedef struct bitnet_op {
    int32_t kind;          /* bitnet_op_kind_t */
    int32_t x_dtype;       /* bitnet_dtype_t of x */
    const void *x;         /* [M][K] activations (read) */
    int64_t K;             /* in features: multiple of 64, at most 8192 */
    int64_t N;             /* out features */
    const uint8_t *w0;     /* [N][K/4] packed: W, or W_gate for the FFN */
    const float *gamma0;   /* [1] */
    const uint8_t *w1;     /* [N][K/4] packed W_up (FFN only, else NULL) */
    const float *gamma1;   /* [1] (FFN only, else NULL) */
    float *y;              /* [M][N] fp32 output (written): y, or h for the FFN */
    const float *norm_g;   /* [K] RMS normalisation weight applied to x first (as bitnet_linear_norm), or NULL */
    float norm_eps;        /* its epsilon (>= 0; used only with norm_g) */
} bitnet_op_t;

#define BITNET_SEQ_MAX_OPS 128        /* ops of one launch (and of the host planning calls) */
#define BITNET_SEQ_MAX_OPS_TOTAL 1024 /* ops of one bitnet_decode_sequence call */
#define BITNET_SEQ_MAX_M 64

/*
 * Workspace of bitnet_decode_sequence for up to n_ops ops over M tokens whose
 * K are at most K_max: completion counters, the TMA tensor maps of the ops'
 * weights (made by the kernel), then per op the quantised activations
 * ([K/64][Mp][64] int8, Mp = M rounded up to 8, 16, 32 or 64), scales and row
 * sums.  A list of n ops needs exactly
 *   up256(4 * (2 + 2n)) + up256(256n + 128) + sum over ops of (up256(K * Mp) + 512)
 * bytes (up256 = rounded up to a multiple of 256); this returns that for
 * n_ops ops of K = K_max.  A list longer than BITNET_SEQ_MAX_OPS runs as
 * launches of BITNET_SEQ_MAX_OPS ops (the last one shorter), each with its own
 * consecutive part of the workspace laid out as above for its ops, every op
 * sized for the largest K of the whole list; the size is the sum of the parts.
 * 1 <= n_ops <= BITNET_SEQ_MAX_OPS_TOTAL; 0 for arguments out of range.
 */
size_t bitnet_sequence_workspace_size(int32_t n_ops, int64_t M, int64_t K_max);

/*
 * Host-only planning step of bitnet_decode_sequence (launches nothing, needs
 * no GPU): validates the ops exactly as bitnet_decode_sequence does and
 * writes, per op j, the ordering that the sequence kernel will enforce:
 *   wait_x[j]  latest i < j whose y overlaps op j's x (read after write), or -1
 *   wait_y[j]  latest i < j whose x or y overlaps op j's y (write after read /
 *              write after write), or -1
 * Byte ranges: x covers M*K elements of x_dtype, y covers M*N floats.
 */
bitnet_status_t bitnet_sequence_plan(const bitnet_op_t *ops, int32_t n_ops, int64_t M,
                                     int32_t *wait_x, int32_t *wait_y);

/*
 * Host-only: the order in which bitnet_decode_sequence takes the ops up
 * (launches nothing, needs no GPU).  order[k] = index into ops of the k-th op.
 * The order keeps every pair of ops whose byte ranges conflict (see
 * bitnet_sequence_plan) in list order, so every op reads, and every output
 * ends up holding, exactly what running the ops in list order gives; only
 * independent ops move.
 */
bitnet_status_t bitnet_sequence_schedule(const bitnet_op_t *ops, int32_t n_ops, int64_t M, int32_t *order);

/*
 * Run ops[0..n_ops) -- every one a decode-size BitLinear or gated FFN over
 * the same M tokens, optionally RMS-normalising its input first -- in ONE
 * persistent kernel launch (preceded by a one-wave kernel that writes the
 * weights' TMA tensor maps into the workspace: two launches per call).  The
 * results are bit-identical to calling
 * bitnet_linear / bitnet_ffn_gate_up (bitnet_linear_norm /
 * bitnet_ffn_gate_up_norm when norm_g is set) for each op in order on
 * `stream`: an op whose x is an earlier op's y reads that y, and every output
 * holds what the last op that writes it stored.  The page has no counterpart
 * to this call: it is the decode-step execution of the BitLinear layers that
 * the page's model stacks (page: "Architecture").
 *
 * Execution: every op is cut into tasks -- quantisation tasks (absmax, after
 * the optional RMS normalisation: one per token for M <= 8, else one per 8
 * tokens with a warp per token) and one
 * task per 128 packed weight rows (256 when M <= 8; half of them output rows
 * of a gated FFN) over all of K -- and the CTAs of
 * the launch (one per SM) claim tasks in a fixed order through a counter in
 * the workspace.  A task waits only for the tasks it depends on: an op's
 * weight rows for its quantisation tasks, a quantisation task for the rows of
 * the op that wrote its x, and an op's outputs for the earlier readers and
 * writers of the same bytes (see bitnet_sequence_tasks).  Weights are
 * streamed ahead of every wait.  Progress does not depend on how many CTAs
 * are resident at the same time.
 *
 *   ops, n_ops  1 <= n_ops <= BITNET_SEQ_MAX_OPS_TOTAL ops (host array,
 *               read during the call only; the launch keeps its own copy).
 *               Lists longer than BITNET_SEQ_MAX_OPS run as consecutive
 *               launches of BITNET_SEQ_MAX_OPS ops in list order (two kernels
 *               each); a later launch starts once the earlier one has
 *               finished, so ops in different launches are ordered as in the
 *               list.  All parts are validated before the first launch.
 *   M           tokens, 1 <= M <= BITNET_SEQ_MAX_M, the same for every op
 *   workspace   device memory of at least
 *               bitnet_sequence_workspace_size(n_ops, M, max K) bytes, any
 *               contents: each launch zeroes its own completion counters (the
 *               first 4 * (2 + 2 * n) bytes of its part) before its sequence
 *               kernel uses them, and leaves them zero again (also after a
 *               device-side timeout), so one workspace may serve different op
 *               lists one after the other.  Calls that may run at the same time
 *               need separate workspaces.
 *
 * Errors (nothing is launched): BITNET_ERR_INVALID_ARG for a null pointer, a
 * bad kind or dtype, a negative or non-finite norm_eps, an op whose y overlaps
 * its own x, any op's weights, gammas or norm weight, or the workspace;
 * BITNET_ERR_UNSUPPORTED_SHAPE for K not a multiple of 64 or above 8192, or an
 * op that would wait on more than 8 groups of tasks; BITNET_ERR_MISALIGNED;
 * BITNET_ERR_WORKSPACE.  The launch is stream-ordered (it starts once earlier
 * work on `stream` has finished).  Weights, gammas and norm weights must not be
 * written by other work while it runs: they are read ahead of every ordering
 * wait.
 */
bitnet_status_t bitnet_decode_sequence(const bitnet_op_t *ops, int32_t n_ops, int64_t M,
                                       void *workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * Host-only: the task order bitnet_decode_sequence would launch for `ctas`
 * CTAs (no device is touched).  The 2 * n_ops task groups -- per op, its
 * quantisation tasks (kind 0: M tasks for M <= 8, else ceil(M / 8)) and its weight-row
 * tasks (kind 1) --
 * in the order the CTAs claim them; for group k:
 *   group_op[k]     index into ops
 *   group_kind[k]   0 = quantisation, 1 = weight rows
 *   group_tasks[k]  number of tasks
 *   dep_count[k], deps[9k .. 9k + 9)  positions (< k) of the groups that must
 *                   be complete before it (reduced: none implied by another;
 *                   a rows group's own quantisation group is always among
 *                   them, besides at most 8 others), unused entries -1
 * All arrays have 2 * n_ops entries (deps: 18 * n_ops).
 */
bitnet_status_t bitnet_sequence_tasks(const bitnet_op_t *ops, int32_t n_ops, int64_t M, int32_t ctas,
                                      int32_t *group_op, int32_t *group_kind, int32_t *group_tasks,
                                      int32_t *dep_count, int32_t *deps);

/*
 * Tests only (host-armed failure injection, no GPU fault): make the weight-row
 * tasks of op `op` (index into the whole list of later bitnet_decode_sequence
 * calls, 0 <= op < BITNET_SEQ_MAX_OPS_TOTAL)
 * wait for one quantisation task more than exist, so that the wait runs out
 * after the wait limit and the launch ends with BITNET_ERR_TIMEOUT in the
 * device status word; -1 turns it off.  Returns the previous value (-2 if
 * op is out of range).
 */
int bitnet_set_sequence_test_stall(int op);

/*
 * Limit of every bounded device-side wait of this library, in nanoseconds (0
 * restores the default of two seconds).  Returns the previous value, or 0 if
 * it could not be set.  For tests of the timeout path; synchronises with the
 * device (a plain copy to device memory).
 */
uint64_t bitnet_set_wait_limit_ns(uint64_t ns);

/*
 * Device-side status word.  Kernels whose waits are bounded record
 * BITNET_ERR_TIMEOUT there (and exit) instead of spinning forever.  This call
 * synchronises `stream`, copies the word to *status_out and, if clear != 0,
 * resets it to BITNET_OK.  Returns BITNET_ERR_CUDA if the copy fails.
 */
bitnet_status_t bitnet_device_status(int clear, bitnet_status_t *status_out, cudaStream_t stream);

/*
 * Number of SMs the library sizes its grids for on the current device
 * (queried once per device).  Returns 0 on error.
 */
int bitnet_num_sms(void);

/*
 * Process-wide kernel selection (a bitnet_dispatch_t value); every selection
 * computes bit-identical results.  Returns the previous value, or -1 if the
 * value is not a bitnet_dispatch_t (nothing changed).  A forced decode
 * selection makes calls with M > 64 (or a K too large for the decode
 * kernel) return BITNET_ERR_UNSUPPORTED_SHAPE.  Intended for tests and
 * benchmarks; not synchronised with calls running in other threads.
 */
int bitnet_set_dispatch(int dispatch);

/*
 * Number of kernel launches this library has issued in this process (all
 * devices, including launches recorded into CUDA graphs during capture).
 * Monotonic; for measuring how many kernels a sequence of calls enqueues.
 */
uint64_t bitnet_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* BITNET_H */
