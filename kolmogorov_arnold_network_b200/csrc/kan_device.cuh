// kan_device.cuh -- device-side building blocks shared by the kernels:
// the span/weight evaluation of uniform cubic B-splines, bounded waits, and
// thin wrappers over the sm_100a PTX used by the tensor-core kernels
// (mbarrier, TMA, tcgen05).  All PTX is written from the public PTX ISA.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kan_internal.h"

namespace kan {

// ---------------------------------------------------------------------------
// Span and local weights (steps S1, S2)
//
// For the uniform grid t_j = lo + (j-k)h of degree k, h = (hi-lo)/G, an input
// x lies in knot interval floor(u)+k with u = (x-lo)/h.  With s = floor(u)
// and the local coordinate t = u - s in [0,1), exactly B_s..B_{s+k} can be
// non-zero (the "local 4-basis lookup" of the InKAN landing page, "Why
// InKAN?", for k = 3), and those with index outside 0..G+k-1 do not exist.
// The input is inside the extended knots iff -k <= u < G+k; NaN and +-inf
// fail that test, so they contribute nothing and never reach an index
// computation (the FlashKAN abstract's clamp of the normalised coordinate to
// [0, k+1] gives the same zeros).
//
// Cubic weights: the four pieces of the uniform cubic B-spline written in a
// form without cancellation on the bounded coordinate t in [0,1) (the
// "stable piecewise polynomial evaluation" with non-negative output of the
// InKAN page, "Numerically Stable"):
//   w0 = (1-t)^3/6            w3 = t^3/6
//   w1 = 2/3 - t^2 (2-t)/2    w2 = 2/3 - (1-t)^2 (1+t)/2     (w2(t) = w1(1-t))
// and their derivatives with respect to x (factor 1/h):
//   w0' = -(1-t)^2/2   w1' = (3t^2-4t)/2   w2' = -(3(1-t)^2-4(1-t))/2   w3' = t^2/2
//
// Any degree k (1..5): the k+1 weights are built in k passes of the local
// triangle on the unit-spaced knots (the FlashKAN abstract's "k sequential
// passes for degree-k splines", done on k+1 registers instead of the whole
// knot vector):
//   b^0 = (1);  b^d_r = ((t + d - r) b^{d-1}_{r-1} + (r + 1 - t) b^{d-1}_r) / d,  r = 0..d
// (b^{d-1}_{-1} = b^{d-1}_d = 0).  Every factor is non-negative for t in
// [0,1), so no cancellation occurs.  The derivatives come from the degree
// k-1 weights: w'_r = (b^{k-1}_{r-1} - b^{k-1}_r) / h.
// ---------------------------------------------------------------------------
constexpr int KAN_MAX_DEGREE = 5;
constexpr int KAN_MAX_NW = KAN_MAX_DEGREE + 1;   // local weights of the highest degree

struct Span {
    int s;       // first of the k+1 basis indices
    float t;     // local coordinate in [0,1)
    bool valid;  // inside the extended knots
};

__device__ __forceinline__ Span span_of(float x, float lo, float inv_h, int G, int k)
{
    Span r;
    float u = (x - lo) * inv_h;
    r.valid = (u >= -(float)k) && (u < (float)(G + k));
    float f = floorf(r.valid ? u : 0.0f);
    r.s = (int)f;
    r.t = r.valid ? (u - f) : 0.0f;
    return r;
}

__device__ __forceinline__ void weights(float t, float w[4])
{
    const float s = 1.0f - t;
    const float t2 = t * t, s2 = s * s;
    w[0] = s2 * s * (1.0f / 6.0f);
    w[1] = (2.0f / 3.0f) - 0.5f * t2 * (1.0f + s);
    w[2] = (2.0f / 3.0f) - 0.5f * s2 * (1.0f + t);
    w[3] = t2 * t * (1.0f / 6.0f);
}

__device__ __forceinline__ void dweights(float t, float inv_h, float d[4])
{
    const float s = 1.0f - t;
    d[0] = -0.5f * s * s * inv_h;
    d[1] = (1.5f * t - 2.0f) * t * inv_h;
    d[2] = -(1.5f * s - 2.0f) * s * inv_h;
    d[3] = 0.5f * t * t * inv_h;
}

// Degree-k weights b[0..k] (entries past k are 0) by the local triangle; with
// DERIV, also the derivatives d[0..k] (times inv_h).  k is warp-uniform in
// every caller, so the early exit does not diverge.
template <bool DERIV>
__device__ __forceinline__ void weights_k(float t, int k, float inv_h, float (&b)[KAN_MAX_NW], float (&d)[KAN_MAX_NW])
{
#pragma unroll
    for (int r = 0; r < KAN_MAX_NW; ++r) b[r] = r == 0 ? 1.0f : 0.0f;
#pragma unroll
    for (int dg = 1; dg <= KAN_MAX_DEGREE; ++dg) {
        if (dg > k) break;
        if (DERIV && dg == k) {
            // degree k-1 values are in b[0..k-1]: w'_r = (b_{r-1} - b_r) / h
#pragma unroll
            for (int r = 0; r < KAN_MAX_NW; ++r) {
                const float left = r > 0 ? b[r - 1] : 0.0f;
                const float right = r < dg ? b[r] : 0.0f;
                d[r] = r <= dg ? (left - right) * inv_h : 0.0f;
            }
        }
        const float inv_d = 1.0f / (float)dg;
        // in place, from the top: b[r] still holds degree dg-1 when it is read
#pragma unroll
        for (int r = KAN_MAX_NW - 1; r >= 0; --r) {
            if (r > dg) continue;
            const float left = r > 0 ? (t + (float)(dg - r)) * b[r - 1] : 0.0f;
            const float right = r < dg ? ((float)(r + 1) - t) * b[r] : 0.0f;
            b[r] = (left + right) * inv_d;
        }
    }
}

// silu(x) = x sigma(x) and silu'(x) = sigma(x) (1 + x (1 - sigma(x))), with
// sigma(x) = 1 / (1 + e^-x) through the correctly rounded reciprocal (no
// division sequence); sigma -> 0 as e^-x -> inf, and x = -inf gives 0.
__device__ __forceinline__ float sigmoid_f(float x) { return __frcp_rn(1.0f + __expf(-x)); }

__device__ __forceinline__ float silu_f(float x) { return x * sigmoid_f(x); }

__device__ __forceinline__ float dsilu_f(float x)
{
    const float sg = sigmoid_f(x);
    return sg * (1.0f + x * (1.0f - sg));
}

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// ---------------------------------------------------------------------------
// Device status word and bounded waits
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Record an error code (any writer wins; every writer writes a non-zero code).
__device__ __forceinline__ void record_status(unsigned int* status, unsigned int code)
{
    if (status) *(volatile unsigned int*)status = code;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of the mbarrier to complete, giving up after
// limit_ns nanoseconds: then records KAN_ERR_TIMEOUT and returns false.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, unsigned int* status,
                                          uint64_t limit_ns = KAN_WAIT_LIMIT_NS)
{
    if (mbar_test(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_test(bar, parity)) return true;
        if (globaltimer_ns() - t0 > limit_ns) {
            record_status(status, KAN_ERR_TIMEOUT);
            return false;
        }
    }
}

// ---------------------------------------------------------------------------
// TMA (per-CTA tiled loads, no multicast)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, uint32_t bar, int c0, int c1)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            dst),
        "l"(tmap), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}

// Tiled 2-D TMA store of a shared-memory box (issued by one thread, completed
// as a bulk group); the box's smem may be reused once bulk_wait_read allows.
__device__ __forceinline__ void tma_store_2d(const void* tmap, uint32_t src, int c0, int c1)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(tmap), "r"(src),
                 "r"(c0), "r"(c1)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until at most N bulk groups of this thread still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: TMEM allocation, MMA, commit, loads
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, 16-bit operands (bf16 or fp16, per the
// instruction descriptor), fp32 accumulation.
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on the mbarrier when every tcgen05 op issued so far by this
// thread has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns: lane l of the warp gets row
// (lane base + l), columns col..col+15.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 16 consecutive 32-bit columns, the store direction.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Barrier among `count` threads (a multiple of 32) of the CTA on hardware barrier `id` (1..15).
__device__ __forceinline__ void named_bar_sync(int id, int count)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ---------------------------------------------------------------------------
// CTA pairs (a cluster of two CTAs sharing one tcgen05.mma.cta_group::2)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// The shared::cluster address of the same shared-memory location in CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

// Arrive on an mbarrier of another CTA of the cluster (release at cluster scope).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// Arrivals without release semantics, for signals that publish no memory data:
// "this warp has read the accumulator into registers" (its tcgen05 loads have
// completed, tcgen05.wait::ld, and tcgen05.fence::before_thread_sync precedes
// the arrival).  A release at cluster scope would first wait for every earlier
// global store of the thread to complete (measured ~0.9 us per arrival after
// a tile's dx stores, on the critical path of the pair's epilogue).
__device__ __forceinline__ void mbar_arrive_relaxed(uint32_t bar)
{
    asm volatile("mbarrier.arrive.relaxed.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// try_wait with acquire at cluster scope (for barriers that CTAs of the pair arrive on).
__device__ __forceinline__ bool mbar_test_cluster(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, unsigned int* status,
                                                  uint64_t limit_ns = KAN_WAIT_LIMIT_NS)
{
    if (mbar_test_cluster(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_test_cluster(bar, parity)) return true;
        if (globaltimer_ns() - t0 > limit_ns) {
            record_status(status, KAN_ERR_TIMEOUT);
            return false;
        }
    }
}

// Every thread of both CTAs of the cluster (release / acquire).
__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Tiled 2-D TMA load by either CTA of a pair, completing on the mbarrier at
// shared::cluster address `bar` (the leader CTA's barrier).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const void* tmap, uint32_t bar, int c0, int c1)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
        "[%2];" ::"r"(dst),
        "l"(tmap), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D (M = 256 over the pair) (+)= A * B^T: A's rows 0-127 from the leader's shared
// memory and 128-255 from the peer's (same address), B's N columns split the
// same way; each CTA's TMEM receives its 128 rows.  Issued by the leader only.
__device__ __forceinline__ void mma_f16_ss_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on the mbarrier at the same offset in both CTAs of the pair when
// every tcgen05 op issued so far by this thread has completed.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
        "h"((uint16_t)3)
        : "memory");
}

// ---------------------------------------------------------------------------
// Operand descriptors
// ---------------------------------------------------------------------------
// Shared-memory matrix descriptor (tcgen05 "matrix descriptor"):
//   bits  0-13  start address >> 4
//   bits 16-29  leading-dimension byte offset >> 4
//   bits 32-45  stride-dimension byte offset >> 4
//   bits 46-47  descriptor version (1 on sm_100)
//   bits 49-51  base offset (0: every swizzle atom here is 1024-byte aligned)
//   bit  52     leading-dimension offset mode (0: relative)
//   bits 61-63  swizzle mode (2 = 128-byte swizzle)
// With the 128-byte swizzle, a K-major tile is a stack of 8-row x 128-byte
// atoms (SBO = 1024, LBO unused); an MN-major tile is a set of
// [K rows x 128 bytes] column blocks, LBO apart, whose 8-row groups are
// SBO = 1024 apart.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes, uint32_t layout)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)(layout & 7u) << 61;
    return d;
}

__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes)
{
    return smem_desc(saddr, lbo_bytes, sbo_bytes, 2u);
}

// Instruction descriptor for kind::f16 with fp32 accumulation:
//   bits 4-5 D format (1 = f32), bits 7-9 A format, bits 10-12 B format
//   (fp16 = 0, bf16 = 1), bit 15 A major, bit 16 B major (0 = K, 1 = MN),
//   bits 17-22 N >> 3, bits 24-28 M >> 4.
__host__ __device__ constexpr uint32_t instr_desc(uint32_t ab_format, uint32_t a_mn_major, uint32_t b_mn_major,
                                                  uint32_t M, uint32_t N)
{
    return (1u << 4) | (ab_format << 7) | (ab_format << 10) | (a_mn_major << 15) | (b_mn_major << 16) |
           ((N >> 3) << 17) | ((M >> 4) << 24);
}

// Byte offset of 16-byte chunk `chunk` of row `row` inside a 128-byte
// swizzled tile (the layout TMA writes with CU_TENSOR_MAP_SWIZZLE_128B).
__device__ __forceinline__ uint32_t sw128_chunk(uint32_t row, uint32_t chunk)
{
    return row * 128u + (((chunk ^ (row & 7u)) & 7u) << 4);
}

// Byte offset of the element at byte column `colb` (0..127) of row `row`.
__device__ __forceinline__ uint32_t sw128_byte(uint32_t row, uint32_t colb)
{
    return sw128_chunk(row, colb >> 4) | (colb & 15u);
}

}  // namespace kan
