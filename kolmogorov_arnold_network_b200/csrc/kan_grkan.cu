// kan_grkan.cu -- the group-rational KAN (GR-KAN) activation, forward and
// backward, with a deterministic, atomic-free gradient reduction.
//
// GR-KAN is the Group-Rational KAN of the Kolmogorov-Arnold Transformer; the
// FlashKAT abstract ("FlashKAT: Understanding and Addressing Performance
// Bottlenecks in the Kolmogorov-Arnold Transformer") traces its slow training
// to the gradient accumulation of the backward pass (memory stalls, atomic
// adds to slow memory) and fixes it with a kernel that keeps partial sums on
// chip.  The rational function is the Pade activation unit of that page's
// reference list, in the form whose denominator cannot vanish:
//   phi(x) = P(x) / Q(x),  P(x) = sum_{p=0..m} a_p x^p,  Q(x) = 1 + |S(x)|,
//   S(x) = sum_{q=1..n} b_q x^q,
// with one coefficient set (a[g, :], b[g, :]) per group g of C / G
// contiguous channels.  Backward, for upstream gradient dY (sign(0) = 0):
//   dx       = dY (P' - phi sign(S) S') / Q
//   da[g, p] = sum over the group's elements of dY x^p / Q
//   db[g, q] = sum over the group's elements of -dY phi sign(S) x^q / Q
//
// Layout and work split (B200): x, y, dY, dx are [rows, C] row-major in the
// operand dtype.  A block owns the columns of one group (or a 256-thread strip
// of them) and a contiguous chunk of rows; each thread reads 16-byte vectors
// of one fixed column position, so every element a thread sees belongs to
// the same group and its m+1+n gradient terms stay in registers.  At the end
// the block reduces them with warp shuffles and one shared-memory pass in a
// fixed order and writes one partial per block; a second kernel adds the
// partials of every group in row-chunk order in fp64.  No atomics, and the
// result is the same bit for bit on every run.  Two elements of a vector
// share their group's coefficients, so the arithmetic runs on element pairs
// with the packed f32x2 instructions (half the FMA-pipe instructions).  Every pass over HBM is a
// streaming read or write of whole 16-byte vectors: the kernels are bound by
// HBM bandwidth.
#include <cuda_bf16.h>

#include <algorithm>

#include "kan_internal.h"

namespace kan {
namespace {

constexpr int kMaxNum = 8;        // at most 8 numerator coefficients (m <= 7)
constexpr int kMaxDen = 8;        // at most 8 denominator coefficients (n <= 8)
constexpr int kAcc = kMaxNum + kMaxDen;
constexpr int kThreads = 256;

struct GrArgs {
    const void* x;
    const void* dY;
    void* y;                  // forward output, or dx
    const float* a;           // [G, m+1]
    const float* b;           // [G, n]
    float* part;              // backward: [row_chunks][G * strips][kAcc] block partials (null: no gradients)
    int64_t rows, C;
    int G, cg;                // groups, channels per group
    int m1, n;                // numerator coefficients (m+1), denominator coefficients (n)
    int vpg;                  // vectors per group row (cg / VEC)
    int strips;               // column strips per group (ceil(vpg / kThreads))
    int tps;                  // threads per strip row (min(vpg, kThreads))
    int rb;                   // rows per block iteration (kThreads / tps, at least 1)
    int64_t rows_per_chunk;
};

// 16-byte vectors of the operand dtype: raw loads (kept packed while they are
// in flight) and their conversion to fp32.
template <typename T> struct Vec;
template <> struct Vec<float> {
    static constexpr int N = 4;
    __device__ static void unpack(const uint4& q, float (&v)[4])
    {
        v[0] = __uint_as_float(q.x); v[1] = __uint_as_float(q.y);
        v[2] = __uint_as_float(q.z); v[3] = __uint_as_float(q.w);
    }
    __device__ static void store(void* p, const float (&v)[4])
    {
        *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
};
template <> struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ static void unpack(const uint4& q, float (&v)[8])
    {
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            v[2 * e] = __uint_as_float(w[e] << 16);
            v[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
        }
    }
    __device__ static void store(void* p, const float (&v)[8])
    {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
            w[e] = *reinterpret_cast<uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
};

__device__ __forceinline__ uint4 ld_vec(const void* p) { return *reinterpret_cast<const uint4*>(p); }

// Two fp32 lanes in one 64-bit register pair, operated on by the packed
// f32x2 instructions of sm_100 (one instruction, two independent
// round-to-nearest results): two elements of the same group share their
// coefficients, so their arithmetic runs pairwise.
using f2 = uint64_t;
__device__ __forceinline__ f2 pk2(float a, float b)
{
    f2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void unpk2(f2 v, float& a, float& b) { asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v)); }
__device__ __forceinline__ f2 fma2(f2 a, f2 b, f2 c)
{
    f2 r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ f2 mul2(f2 a, f2 b)
{
    f2 r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// Value and derivative of sum_i c_i x^i (i = 0..deg) by Horner's rule (the
// better-conditioned order for the wide range of x^i), for two elements at
// once; DMAX bounds the unrolled loop, every index is a compile-time constant
// (c stays in registers).
template <int DMAX, int NCO>
__device__ __forceinline__ void horner_d2(const f2 (&c)[NCO], int deg, f2 x, f2& v, f2& d)
{
    static_assert(DMAX < NCO, "coefficient array too short");
    v = 0ull;
    d = 0ull;
#pragma unroll
    for (int i = DMAX; i >= 0; --i) {
        if (i <= deg) {
            d = fma2(d, x, v);
            v = fma2(v, x, c[i]);
        }
    }
}

// M1, N: compile-time numerator / denominator coefficient counts (the KAT
// choice m = 5, n = 4 is instantiated on its own), or 0 for the runtime
// counts in the arguments.  Each step handles RIF rows; the next step's
// vectors are loaded (and kept packed) before this step's arithmetic, so the
// loads' latency hides behind it.
template <typename T, bool BWD, int M1, int N>
__global__ void __launch_bounds__(kThreads, BWD ? (M1 ? 3 : 2) : 4) grkan_kernel(const GrArgs a)
{
    constexpr int VEC = Vec<T>::N;
    // rows per step and thread (the backward's fp32 rows, with half the elements per vector, take two
    // rows per step to keep enough bytes in flight; measured faster than one on B200)
    constexpr int RIF = BWD ? (sizeof(T) == 4 ? 2 : 1) : 2;
    const int m1 = M1 ? M1 : a.m1, n = N ? N : a.n;
    constexpr int MC = M1 ? M1 : kMaxNum;            // numerator coefficients, unroll bound
    constexpr int NC = N ? N : kMaxDen;              // denominator coefficients, unroll bound
    constexpr int PW = MC - 1 > NC ? MC - 1 : NC;    // highest power a gradient term needs
    const int gs = blockIdx.x;                       // group * strips + strip
    const int g = gs / a.strips, strip = gs - g * a.strips;
    const int tid = threadIdx.x;
    const int rr = tid / a.tps, cv = tid - rr * a.tps;           // row within the iteration, vector column
    const int vcol = strip * kThreads + cv;                      // vector index within the group row
    const bool active = rr < a.rb && vcol < a.vpg;
    // the group's coefficients (zero past the runtime counts); S has no constant term
    __shared__ float sa[kMaxNum], sb[kMaxDen + 1];
    if (tid < kMaxNum) sa[tid] = tid < m1 ? a.a[g * m1 + tid] : 0.0f;
    if (tid <= kMaxDen) sb[tid] = (tid >= 1 && tid <= n) ? a.b[g * n + tid - 1] : 0.0f;
    __syncthreads();
    f2 ca[MC], cb[NC + 1];
#pragma unroll
    for (int i = 0; i < MC; ++i) ca[i] = pk2(sa[i], sa[i]);
#pragma unroll
    for (int i = 0; i <= NC; ++i) cb[i] = pk2(sb[i], sb[i]);

    // gradient terms, per lane of the element pairs (summed in a fixed order at the end)
    f2 acc2[MC + NC];
#pragma unroll
    for (int i = 0; i < MC + NC; ++i) acc2[i] = 0ull;

    const int64_t r_begin = (int64_t)blockIdx.y * a.rows_per_chunk;
    const int64_t r_end = min(a.rows, r_begin + a.rows_per_chunk);
    const int64_t col = (int64_t)g * a.cg + (int64_t)vcol * VEC;
    const T* X = reinterpret_cast<const T*>(a.x);
    const T* G = reinterpret_cast<const T*>(a.dY);
    T* Y = reinterpret_cast<T*>(a.y);
    const int64_t step = (int64_t)RIF * a.rb;
    if (active) {
        uint4 xq[RIF], gq[RIF];
        auto fetch = [&](int64_t r0) {
#pragma unroll
            for (int h = 0; h < RIF; ++h) {
                const int64_t rh = r0 + (int64_t)h * a.rb;
                if (rh < r_end) {
                    xq[h] = ld_vec(X + rh * a.C + col);
                    if (BWD) gq[h] = ld_vec(G + rh * a.C + col);
                }
            }
        };
        fetch(r_begin + rr);
        for (int64_t r = r_begin + rr; r < r_end; r += step) {
            float xv[RIF][VEC], gv[RIF][VEC];
#pragma unroll
            for (int h = 0; h < RIF; ++h) {
                Vec<T>::unpack(xq[h], xv[h]);
                if (BWD) Vec<T>::unpack(gq[h], gv[h]);
            }
            if (r + step < r_end) fetch(r + step);
#pragma unroll
            for (int h = 0; h < RIF; ++h) {
                const int64_t rh = r + (int64_t)h * a.rb;
                if (rh >= r_end) break;
                float ov[VEC];
#pragma unroll
                for (int e = 0; e < VEC; e += 2) {
                    const f2 x = pk2(xv[h][e], xv[h][e + 1]);
                    f2 P, dP, S, dS;
                    horner_d2<MC - 1>(ca, m1 - 1, x, P, dP);
                    horner_d2<NC>(cb, n, x, S, dS);
                    float s0, s1;
                    unpk2(S, s0, s1);
                    const f2 iQ = pk2(__fdividef(1.0f, 1.0f + fabsf(s0)), __fdividef(1.0f, 1.0f + fabsf(s1)));
                    const f2 phi = mul2(P, iQ);
                    if (!BWD) {
                        unpk2(phi, ov[e], ov[e + 1]);
                        continue;
                    }
                    // nps = -phi sign(S)
                    float p0, p1;
                    unpk2(phi, p0, p1);
                    const f2 nps = pk2(s0 > 0.0f ? -p0 : (s0 < 0.0f ? p0 : 0.0f), s1 > 0.0f ? -p1 : (s1 < 0.0f ? p1 : 0.0f));
                    const f2 ga = mul2(pk2(gv[h][e], gv[h][e + 1]), iQ);   // d phi / d a_p = x^p / Q
                    unpk2(mul2(ga, fma2(nps, dS, dP)), ov[e], ov[e + 1]);
                    if (a.part) {
                        const f2 gb = mul2(ga, nps);                     // d phi / d b_q = -phi sign(S) x^q / Q
                        f2 xp = pk2(1.0f, 1.0f);
#pragma unroll
                        for (int i = 0; i <= PW; ++i) {
                            if (i < MC) acc2[i] = fma2(ga, xp, acc2[i]);
                            if (i >= 1 && i <= NC) acc2[MC + i - 1] = fma2(gb, xp, acc2[MC + i - 1]);
                            if (i < PW) xp = mul2(xp, x);
                        }
                    }
                }
                if (Y) Vec<T>::store(Y + rh * a.C + col, ov);
            }
        }
    }
    if (!BWD || !a.part) return;
    float acc[MC + NC];
#pragma unroll
    for (int i = 0; i < MC + NC; ++i) {
        float lo, hi;
        unpk2(acc2[i], lo, hi);
        acc[i] = lo + hi;
    }
    // block reduction in a fixed order: lanes by shuffles (inactive lanes hold zeros), then the
    // warps' sums in warp order; entries past the runtime counts are zero
    __shared__ float wsum[kThreads / 32][kAcc];
    const int warp = tid >> 5, lane = tid & 31;
#pragma unroll
    for (int i = 0; i < kAcc; ++i) {
        // (slot i of the partial: numerator terms 0..kMaxNum-1, then denominator terms)
        const int src = i < kMaxNum ? i : MC + (i - kMaxNum);
        float v = 0.0f;
        if (i < kMaxNum ? i < MC : i - kMaxNum < NC) {
#pragma unroll
            for (int j = 0; j < MC + NC; ++j) v = j == src ? acc[j] : v;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) wsum[warp][i] = v;
    }
    __syncthreads();
    if (tid < kAcc) {
        float v = 0.0f;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) v += wsum[w][tid];
        a.part[((int64_t)blockIdx.y * gridDim.x + gs) * kAcc + tid] = v;
    }
}

// da[g, p], db[g, q] from the block partials: for each group, its strips and
// row chunks summed in a fixed order, in fp64.
__global__ void grkan_reduce_kernel(const float* __restrict__ part, int chunks, int G, int strips, int m1, int n,
                                    float* __restrict__ da, float* __restrict__ db)
{
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= G * kAcc) return;
    const int g = t / kAcc, i = t - g * kAcc;
    const bool is_a = i < kMaxNum;
    const int idx = is_a ? i : i - kMaxNum;
    if (is_a ? (idx >= m1 || !da) : (idx >= n || !db)) return;
    double s = 0.0;
    for (int c = 0; c < chunks; ++c)
        for (int st = 0; st < strips; ++st) s += (double)part[((int64_t)c * G * strips + g * strips + st) * kAcc + i];
    if (is_a) da[g * m1 + idx] = (float)s;
    else db[g * n + idx] = (float)s;
}

struct GrPlan {
    int vec, vpg, strips, tps, rb, threads, chunks;
    int64_t rows_per_chunk;
};

template <typename T, bool BWD>
const void* kernel_of(int m1, int n)
{
    if (m1 == 6 && n == 4) return reinterpret_cast<const void*>(&grkan_kernel<T, BWD, 6, 4>);
    return reinterpret_cast<const void*>(&grkan_kernel<T, BWD, 0, 0>);
}

// Blocks: one per (group, strip) and row chunk, with as many row chunks as
// fill one wave of resident blocks exactly (the rows split evenly), so that
// no second, partial wave trails the first.
GrPlan plan_of(const kan_grkan_shape& s, bool bwd)
{
    GrPlan P{};
    const bool f32 = s.dtype == KAN_F32;
    P.vec = f32 ? 4 : 8;
    const int cg = (int)(s.channels / s.groups);
    P.vpg = cg / P.vec;
    P.tps = std::min(P.vpg, kThreads);
    P.strips = (P.vpg + kThreads - 1) / kThreads;
    P.rb = std::max(1, kThreads / P.tps);
    P.threads = std::min(kThreads, ((P.tps * P.rb + 31) / 32) * 32);
    int dev = 0, sms = 148, occ = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int m1 = s.num_degree + 1, n = s.den_degree;
    const void* fn = f32 ? (bwd ? kernel_of<float, true>(m1, n) : kernel_of<float, false>(m1, n))
                         : (bwd ? kernel_of<__nv_bfloat16, true>(m1, n) : kernel_of<__nv_bfloat16, false>(m1, n));
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, P.threads, 0) != cudaSuccess || occ < 1) {
        cudaGetLastError();
        occ = 4;
    }
    const int64_t wave = (int64_t)std::max(1, sms) * occ;
    const int64_t per_chunk_blocks = (int64_t)s.groups * P.strips;
    int64_t chunks = std::max<int64_t>(1, wave / per_chunk_blocks);
    chunks = std::min<int64_t>(chunks, std::max<int64_t>(1, (s.rows + P.rb - 1) / P.rb));
    chunks = std::min<int64_t>(chunks, 65535);
    P.rows_per_chunk = std::max<int64_t>(1, (s.rows + chunks - 1) / chunks);
    P.chunks = (int)std::max<int64_t>(1, (s.rows + P.rows_per_chunk - 1) / P.rows_per_chunk);
    return P;
}

kan_status gr_fail(kan_status st, const char* msg) { return set_last_error(st, msg); }

kan_status validate(const kan_grkan_shape* s)
{
    if (!s) return gr_fail(KAN_ERR_INVALID_ARG, "shape is NULL");
    if (s->rows < 0 || s->channels < 1 || s->groups < 1) return gr_fail(KAN_ERR_INVALID_ARG, "rows >= 0, channels >= 1, groups >= 1");
    if (s->channels % s->groups != 0) return gr_fail(KAN_ERR_INVALID_ARG, "channels must be a multiple of groups");
    if (s->num_degree < 1 || s->num_degree > kMaxNum - 1) return gr_fail(KAN_ERR_INVALID_ARG, "num_degree must be 1..7");
    if (s->den_degree < 1 || s->den_degree > kMaxDen) return gr_fail(KAN_ERR_INVALID_ARG, "den_degree must be 1..8");
    if (s->dtype != KAN_F32 && s->dtype != KAN_BF16) return gr_fail(KAN_ERR_INVALID_ARG, "unknown dtype");
    const int esz = s->dtype == KAN_F32 ? 4 : 2;
    const int64_t cg = s->channels / s->groups;
    if ((cg * esz) % 16 != 0)
        return gr_fail(KAN_ERR_UNSUPPORTED, "channels per group times the element size must be a multiple of 16 bytes");
    if (s->groups > 65535 || s->channels > ((int64_t)1 << 30)) return gr_fail(KAN_ERR_UNSUPPORTED, "sizes too large");
    return KAN_OK;
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <typename T, bool BWD>
cudaError_t launch_gr(const kan_grkan_shape& s, const GrPlan& P, GrArgs a, cudaStream_t st)
{
    a.rows = s.rows;
    a.C = s.channels;
    a.G = s.groups;
    a.cg = (int)(s.channels / s.groups);
    a.m1 = s.num_degree + 1;
    a.n = s.den_degree;
    a.vpg = P.vpg;
    a.strips = P.strips;
    a.tps = P.tps;
    a.rb = P.rb;
    a.rows_per_chunk = P.rows_per_chunk;
    const dim3 grid((unsigned)(s.groups * P.strips), (unsigned)P.chunks);
    if (a.m1 == 6 && a.n == 4) grkan_kernel<T, BWD, 6, 4><<<grid, P.threads, 0, st>>>(a);
    else grkan_kernel<T, BWD, 0, 0><<<grid, P.threads, 0, st>>>(a);
    count_launch();
    return cudaGetLastError();
}

}  // namespace
}  // namespace kan

using namespace kan;

extern "C" {

kan_status kan_grkan_workspace_size(const kan_grkan_shape* s, size_t* bytes)
{
    kan_status st = validate(s);
    if (st != KAN_OK) return st;
    if (!bytes) return gr_fail(KAN_ERR_INVALID_ARG, "bytes is NULL");
    const GrPlan P = plan_of(*s, true);
    *bytes = (size_t)P.chunks * s->groups * P.strips * kAcc * sizeof(float);
    return KAN_OK;
}

kan_status kan_grkan_forward(const kan_grkan_shape* s, const void* x, const float* a, const float* b, void* y,
                             void* stream)
{
    kan_status st = validate(s);
    if (st != KAN_OK) return st;
    if (!a || !b || (s->rows > 0 && (!x || !y))) return gr_fail(KAN_ERR_INVALID_ARG, "a null pointer");
    if ((x && !al16(x)) || (y && !al16(y))) return gr_fail(KAN_ERR_UNSUPPORTED, "x and y must be 16-byte aligned");
    if (s->rows == 0) return KAN_OK;
    const GrPlan P = plan_of(*s, false);
    GrArgs g{};
    g.x = x;
    g.y = y;
    g.a = a;
    g.b = b;
    const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = record_mark(timing_marks().after_prep, cs);
    if (e == cudaSuccess)
        e = s->dtype == KAN_F32 ? launch_gr<float, false>(*s, P, g, cs) : launch_gr<__nv_bfloat16, false>(*s, P, g, cs);
    if (e != cudaSuccess) return gr_fail(KAN_ERR_CUDA, cudaGetErrorString(e));
    return KAN_OK;
}

kan_status kan_grkan_backward(const kan_grkan_shape* s, const void* x, const float* a, const float* b, const void* dY,
                              void* dx, float* da, float* db, void* workspace, size_t ws_bytes, void* stream)
{
    kan_status st = validate(s);
    if (st != KAN_OK) return st;
    if (!a || !b || (s->rows > 0 && (!x || !dY))) return gr_fail(KAN_ERR_INVALID_ARG, "a null pointer");
    if ((x && !al16(x)) || (dY && !al16(dY)) || (dx && !al16(dx)) || (workspace && !al16(workspace)))
        return gr_fail(KAN_ERR_UNSUPPORTED, "x, dY, dx and the workspace must be 16-byte aligned");
    if (!dx && !da && !db) return KAN_OK;
    const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const int m1 = s->num_degree + 1, n = s->den_degree;
    cudaError_t e = cudaSuccess;
    if (s->rows == 0) {
        if (da) e = cudaMemsetAsync(da, 0, sizeof(float) * s->groups * m1, cs);
        if (e == cudaSuccess && db) e = cudaMemsetAsync(db, 0, sizeof(float) * s->groups * n, cs);
        return e == cudaSuccess ? KAN_OK : gr_fail(KAN_ERR_CUDA, cudaGetErrorString(e));
    }
    const GrPlan P = plan_of(*s, true);
    const size_t need = (size_t)P.chunks * s->groups * P.strips * kAcc * sizeof(float);
    const bool grads = da || db;
    if (grads && (ws_bytes < need || !workspace)) return gr_fail(KAN_ERR_WORKSPACE, "workspace too small");
    GrArgs g{};
    g.x = x;
    g.dY = dY;
    g.y = dx;
    g.a = a;
    g.b = b;
    g.part = grads ? reinterpret_cast<float*>(workspace) : nullptr;
    e = record_mark(timing_marks().after_prep, cs);
    if (e == cudaSuccess)
        e = s->dtype == KAN_F32 ? launch_gr<float, true>(*s, P, g, cs) : launch_gr<__nv_bfloat16, true>(*s, P, g, cs);
    if (e == cudaSuccess && grads) {
        const int total = s->groups * kAcc;
        grkan_reduce_kernel<<<(total + 127) / 128, 128, 0, cs>>>(g.part, P.chunks, s->groups, P.strips, m1, n, da, db);
        count_launch();
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) return gr_fail(KAN_ERR_CUDA, cudaGetErrorString(e));
    return KAN_OK;
}

}  // extern "C"
