// common.cuh -- sm_100a PTX helpers shared by the BitLinear kernels.
//
// Everything here is a thin wrapper over one documented PTX instruction
// (mbarrier, bulk/tensor copies, programmatic dependent launch, tcgen05).
// Every wait on a barrier is bounded: after g_wait_limit_ns of wall time
// the wait records BITNET_ERR_TIMEOUT in the device status word and returns
// false, and the caller unwinds instead of spinning forever.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "bitnet.h"

#define BITNET_DEVINL __device__ __forceinline__

namespace bitnet {

// Two seconds: far above any legitimate wait in these kernels.
constexpr unsigned long long kDefaultWaitLimitNs = 2000000000ull;

// Device status word (one per device).  The library is one translation unit,
// so this is its only definition.
__device__ int g_device_status = 0;

// Limit of every bounded wait, in nanoseconds of wall time (one per device;
// lowered only by tests, through bitnet_set_wait_limit_ns).
__device__ unsigned long long g_wait_limit_ns = kDefaultWaitLimitNs;

BITNET_DEVINL uint64_t wait_limit_ns() { return *(volatile unsigned long long *)&g_wait_limit_ns; }

BITNET_DEVINL void record_status(int code) { atomicCAS(&g_device_status, 0, code); }
BITNET_DEVINL bool status_failed() { return *(volatile int *)&g_device_status != 0; }

BITNET_DEVINL uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

BITNET_DEVINL uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier ------------------------------------------------------------

BITNET_DEVINL void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

BITNET_DEVINL void fence_mbarrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

BITNET_DEVINL void mbar_arrive(uint64_t *bar)
{
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
                 : "memory");
}

BITNET_DEVINL void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

BITNET_DEVINL bool mbar_try_wait(uint32_t bar_addr, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar_addr), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait until the phase with the given parity has completed.  Bounded: returns
// false (after recording a timeout) if it does not complete in time or if
// another wait on the device already gave up.
BITNET_DEVINL bool mbar_wait(uint64_t *bar, uint32_t parity)
{
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t spin = 1;; ++spin) {
        if (mbar_try_wait(a, parity)) return true;
        if ((spin & 255u) == 0) {
            if (status_failed()) return false;
            if (globaltimer_ns() - t0 > wait_limit_ns()) {
                record_status(BITNET_ERR_TIMEOUT);
                return false;
            }
        }
    }
}

// Cluster-scope variant: waits until a phase completed by remote arrivals or
// remote st.async transactions, and makes the peers' writes visible.
BITNET_DEVINL bool mbar_try_wait_cluster(uint32_t bar_addr, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar_addr), "r"(parity)
        : "memory");
    return ok != 0;
}

BITNET_DEVINL bool mbar_wait_cluster(uint64_t *bar, uint32_t parity)
{
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait_cluster(a, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t spin = 1;; ++spin) {
        if (mbar_try_wait_cluster(a, parity)) return true;
        if ((spin & 255u) == 0) {
            if (status_failed()) return false;
            if (globaltimer_ns() - t0 > wait_limit_ns()) {
                record_status(BITNET_ERR_TIMEOUT);
                return false;
            }
        }
    }
}

// ---- thread-block clusters / distributed shared memory ------------------

BITNET_DEVINL uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

BITNET_DEVINL uint32_t cluster_id_x()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}

// Whole-cluster barrier (every thread of every CTA), release/acquire.  Used
// once at kernel start, before any CTA has anything to wait for.
BITNET_DEVINL void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Split-phase cluster barrier: every thread arrives (release) and later waits
// (acquire); work between the two overlaps the barrier's latency.
BITNET_DEVINL void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
BITNET_DEVINL void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

// Address of the same shared-memory location in CTA `rank` of this cluster.
BITNET_DEVINL uint32_t mapa_shared(uint32_t local_addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_addr), "r"(rank));
    return r;
}

// Asynchronous 8-byte store into a peer CTA's shared memory; the peer's
// mbarrier (same cluster) counts the bytes on arrival.
BITNET_DEVINL void st_async_v2(uint32_t remote_addr, int a, int b, uint32_t remote_bar)
{
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.s32 [%0], {%1, %2}, [%3];" ::"r"(
                     remote_addr),
                 "r"(a), "r"(b), "r"(remote_bar)
                 : "memory");
}

BITNET_DEVINL void st_async_v4f(uint32_t remote_addr, float a, float b, float c, float d, uint32_t remote_bar)
{
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                     remote_addr),
                 "f"(a), "f"(b), "f"(c), "f"(d), "r"(remote_bar)
                 : "memory");
}

// ---- bulk / tensor copies (async proxy) ----------------------------------

// 1-D bulk copy global -> shared, completion counted on `bar` (bytes % 16 == 0,
// both addresses 16-byte aligned).
BITNET_DEVINL void bulk_g2s(void *dst_smem, const void *src_gmem, uint32_t bytes, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// 16-byte asynchronous copy global -> shared (L2 only), Ampere-style.
BITNET_DEVINL void cp_async16(void *dst_smem, const void *src_gmem)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst_smem)), "l"(src_gmem) : "memory");
}

// Arrive on `bar` once every cp.async this thread issued so far has landed
// (the arrival is counted in the barrier's expected count: .noinc).
BITNET_DEVINL void cp_async_mbar_arrive(uint64_t *bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// 2-D tiled tensor copy global -> shared (no multicast).  c0 is the innermost
// coordinate in elements; callers keep c0 * elem_size a multiple of 16 bytes.
BITNET_DEVINL void tma_load_2d(void *dst_smem, const CUtensorMap *map, int32_t c0, int32_t c1, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst_smem)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}

// 2-D tiled tensor copy shared -> global (bulk-group completion).
BITNET_DEVINL void tma_store_2d(const CUtensorMap *map, int32_t c0, int32_t c1, const void *src_smem)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(smem_u32(src_smem))
                 : "memory");
}
BITNET_DEVINL void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N committed bulk groups still read their shared source.
template <int N>
BITNET_DEVINL void bulk_wait_group_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until every committed bulk group has completed (writes performed).
BITNET_DEVINL void bulk_wait_group_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

BITNET_DEVINL void prefetch_tensormap(const CUtensorMap *map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Order this thread's generic-proxy shared-memory writes before later
// async-proxy (tensor core / TMA) accesses.
BITNET_DEVINL void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- programmatic dependent launch -------------------------------------

// Block until the grids this grid depends on have completed and their memory
// is visible (a no-op when launched without a programmatic dependency).
BITNET_DEVINL void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Allow the next grid in the stream to start launching.
BITNET_DEVINL void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---- small utilities -----------------------------------------------------

// 16-byte load through L2 only (data written by other CTAs during the kernel).
BITNET_DEVINL uint4 ld_cg_v4(const void *p)
{
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

BITNET_DEVINL float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

BITNET_DEVINL int warp_sum(int v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Quantise one value: rne(x * s) clamped to [-128, 127], fp32 product rounded once.
BITNET_DEVINL int quant_one(float x, float s)
{
    int q = __float2int_rn(__fmul_rn(x, s));
    return max(-128, min(127, q));
}

// s = 127 / max(amax, 1e-5), IEEE fp32 division.
BITNET_DEVINL float quant_scale(float amax) { return __fdiv_rn(127.0f, fmaxf(amax, 1e-5f)); }

BITNET_DEVINL uint32_t pack4_s8(int a, int b, int c, int d)
{
    return (uint32_t)(a & 0xff) | ((uint32_t)(b & 0xff) << 8) | ((uint32_t)(c & 0xff) << 16) |
           ((uint32_t)(d & 0xff) << 24);
}

BITNET_DEVINL float bf16_bits_lo(uint32_t w) { return __uint_as_float(w << 16); }
BITNET_DEVINL float bf16_bits_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// ---- output stage: fp32, or bf16 = the fp32 value rounded to nearest even ----

BITNET_DEVINL uint32_t bf16_rn_bits(float v) { return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v)); }

// Magnitude of the value as stored, as the bit pattern of a non-negative fp32
// (non-negative floats order like their bit patterns, so maxima are integer
// maxima and atomicMax on the bits is exact and order-free).
BITNET_DEVINL uint32_t out_mag_bits(float v, bool bf16)
{
    return bf16 ? (bf16_rn_bits(v) & 0x7fffu) << 16 : __float_as_uint(v) & 0x7fffffffu;
}

BITNET_DEVINL void out_store(void *y, size_t o, float v, bool bf16)
{
    if (bf16)
        static_cast<uint16_t *>(y)[o] = (uint16_t)bf16_rn_bits(v);
    else
        static_cast<float *>(y)[o] = v;
}

// Fold each lane's magnitude bits into per-token maxima (shared memory, bits
// of non-negative floats).  Lanes hold consecutive elements of an epilogue
// whose token index j does not decrease from lane to lane; a lane without an
// element passes bits 0 and a j no smaller than any active lane's.
BITNET_DEVINL void warp_token_max(uint32_t bits, int j, unsigned *smax)
{
    const int jlo = __shfl_sync(0xffffffffu, j, 0), jhi = __shfl_sync(0xffffffffu, j, 31);
    for (int t = jlo; t <= jhi; ++t) {
        const unsigned m = __reduce_max_sync(0xffffffffu, j == t ? bits : 0u);
        if ((threadIdx.x & 31) == 0 && m != 0u) atomicMax(&smax[t], m);
    }
}

// ---- tcgen05 (5th-generation tensor cores, tensor memory) ----------------

BITNET_DEVINL void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
BITNET_DEVINL void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Whole warp: allocate `ncols` TMEM columns, address written to *slot.
BITNET_DEVINL void tmem_alloc(uint32_t *slot, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
}
BITNET_DEVINL void tmem_relinquish() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;"); }
BITNET_DEVINL void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 bytes, 8-row core groups 1024 bytes apart (SBO), LBO unused (1), sm100
// descriptor version 1.
BITNET_DEVINL uint64_t umma_desc_k_sw128(const void *smem_ptr)
{
    const uint64_t addr = smem_u32(smem_ptr);
    return ((addr >> 4) & 0x3FFFull) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) |
           (2ull << 61);
}

// D[tmem] (+)= A[smem] . B[smem]^T, int8 inputs, int32 accumulators.
BITNET_DEVINL void umma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when every tcgen05 operation issued so far by this
// thread has completed.
BITNET_DEVINL void umma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// Warp-collective: 32 lanes x 32 consecutive 32-bit columns.
BITNET_DEVINL void tmem_ld32(uint32_t taddr, uint32_t (&v)[32])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
                   "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
                   "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]),
                   "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]),
                   "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
                 : "r"(taddr)
                 : "memory");
}
// The registers a tcgen05.ld writes are valid only after tcgen05.wait::ld, but
// the compiler does not know that: these forms name them as operands of the
// wait (or of an empty statement right after it), so no use of them can be
// scheduled before the wait.
BITNET_DEVINL void tmem_regs_fence(uint32_t (&v)[32])
{
    asm volatile(""
                 : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]), "+r"(v[7]),
                   "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]), "+r"(v[14]),
                   "+r"(v[15]), "+r"(v[16]), "+r"(v[17]), "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]),
                   "+r"(v[22]), "+r"(v[23]), "+r"(v[24]), "+r"(v[25]), "+r"(v[26]), "+r"(v[27]), "+r"(v[28]),
                   "+r"(v[29]), "+r"(v[30]), "+r"(v[31])
                 :
                 : "memory");
}

BITNET_DEVINL void tmem_wait_ld(uint32_t (&v)[32])
{
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]), "+r"(v[7]),
                   "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]), "+r"(v[14]),
                   "+r"(v[15]), "+r"(v[16]), "+r"(v[17]), "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]),
                   "+r"(v[22]), "+r"(v[23]), "+r"(v[24]), "+r"(v[25]), "+r"(v[26]), "+r"(v[27]), "+r"(v[28]),
                   "+r"(v[29]), "+r"(v[30]), "+r"(v[31])
                 :
                 : "memory");
}

// Bounded wait that ignores the failure flag: used only to let this CTA's own
// in-flight copies / MMAs land before it releases shared or tensor memory.
BITNET_DEVINL bool mbar_wait_drain(uint64_t *bar, uint32_t parity)
{
    const uint32_t a = smem_u32(bar);
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(a, parity))
        if (globaltimer_ns() - t0 > wait_limit_ns()) return false;
    return true;
}

} // namespace bitnet
