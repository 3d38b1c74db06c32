// kan_ukan.cu -- the coefficient generator of UKAN layers (KAN layers on an
// unbounded grid), forward and backward, and the input range that sizes the
// generated window.
//
// "Want to train KANS at scale? Now UKAN!" (Abstract): a coefficient-generator
// (CG) model produces, on the fly, only the B-spline coefficients needed
// locally on an unbounded symmetric grid, fed with the positional encoding of
// grid groups.  Here: knots j h for every integer j, cubic B-splines, group q
// = the g basis indices q g .. q g + g - 1, encoding PE(q) = (sin q w_l,
// cos q w_l), w_l = 10000^(-2l/d), and the generator
//   hid(q) = silu(W1 PE(q) + b1),  c(q) = W2 hid(q) + b2  (out * in * g values)
// whose output for groups q0 .. q0+nq-1 is written as the coefficient window
// coef[out][in][nq g] (window index ql g + r for basis q g + r) in the operand
// dtype, exactly the layout of the KAN layer's coefficients.  The layer then
// runs on that window as a bounded grid with G = nq g - 3 intervals and
// lo = (q0 g + 3) h: its basis index 0 is the unbounded basis q0 g.
//
// Backward: dc(q) = dcoef of the window; dW2 = sum_q dc(q) hid(q)^T and
// db2 = sum_q dc(q) row by row; dhid(q) = W2^T dc(q) reduced over all out*in*g
// rows by blocks (fp32 partials, then one fixed-order fp64 pass: no atomics);
// then dpre = dhid silu'(pre), dW1 = sum_q dpre PE(q)^T, db1 = sum_q dpre.
// Every kernel here streams W2 / coef / dcoef from HBM once.
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>

#include "kan_device.cuh"

namespace kan {
namespace {

constexpr int kUkThreads = 256;
constexpr int kMaxHidden = 256;
constexpr int kMaxHidTerms = 12288;        // nq * H held in shared memory (48 KiB)
constexpr int kTq = 4, kTh = 4;            // dhid register tile: 4 groups x 4 hidden units per thread

__device__ __forceinline__ float silu_pre(float z) { return z * __frcp_rn(1.0f + __expf(-z)); }

// pre[ql, h] = W1[h, :] . PE(q0 + ql) + b1[h], computed by a block into shared memory.
__device__ void hidden_pre(const float* __restrict__ W1, const float* __restrict__ b1, int q0, int nq, int d, int H,
                           float* pre)
{
    for (int t = threadIdx.x; t < nq * H; t += blockDim.x) {
        const int ql = t / H, h = t - ql * H;
        const float q = (float)(q0 + ql);
        float acc = b1[h];
        for (int l = 0; l < d / 2; ++l) {
            const float w = exp2f(-(2.0f * l / (float)d) * 13.287712379549449f);   // 10000^(-2l/d), log2(10000)
            float sv, cv;
            sincosf(q * w, &sv, &cv);
            acc = fmaf(W1[h * d + 2 * l], sv, acc);
            acc = fmaf(W1[h * d + 2 * l + 1], cv, acc);
        }
        pre[t] = acc;
    }
}

template <typename T> __device__ __forceinline__ T cvt_out(float v);
template <> __device__ __forceinline__ float cvt_out<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 cvt_out<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// Chunks of kCE edges per block iteration: the chunk's W2 rows (kCE * g rows
// of H floats, contiguous in W2) are staged in shared memory by coalesced
// loads (rows padded to H + 4 floats: 16-byte aligned, conflict-free 16-byte
// reads across rows), then every thread computes four window entries (one W2
// row, four groups) with 16-byte shared loads and writes them into the edges'
// contiguous window rows.  H is a multiple of 4.
constexpr int kCE = 32;

__device__ __forceinline__ float4 lds4(const float* p) { return *reinterpret_cast<const float4*>(p); }

template <typename T>
__global__ void __launch_bounds__(kUkThreads) ukan_generate_kernel(const float* __restrict__ W1,
                                                                    const float* __restrict__ b1,
                                                                    const float* __restrict__ W2,
                                                                    const float* __restrict__ b2, T* __restrict__ coef,
                                                                    float* __restrict__ pre_out, int64_t edges, int g,
                                                                    int d, int H, int q0, int nq)
{
    extern __shared__ __align__(16) float sh[];
    const int hp = H + 4;
    const int nqp = (nq + 3) / 4 * 4;           // hidden rows padded to whole blocks of four groups
    float* hid = sh;                             // [nqp][hp] (rows past nq are zero)
    float* sw = sh + nqp * hp;                   // [kCE * g][hp]
    {
        float* pre = sw;                         // scratch: [nq * H] fits in the W2 staging area
        hidden_pre(W1, b1, q0, nq, d, H, pre);
        __syncthreads();
        for (int t = threadIdx.x; t < nqp * H; t += blockDim.x) {
            const int ql = t / H, h = t - ql * H;
            const float v = ql < nq ? pre[t] : 0.0f;
            if (blockIdx.x == 0 && ql < nq) pre_out[t] = v;
            hid[ql * hp + h] = ql < nq ? silu_pre(v) : 0.0f;
        }
        __syncthreads();
    }
    const int nqb = nqp / 4;
    for (int64_t c0 = (int64_t)blockIdx.x * kCE; c0 < edges; c0 += (int64_t)gridDim.x * kCE) {
        const int ne = (int)(edges - c0 < kCE ? edges - c0 : kCE);
        __syncthreads();
        for (int t = threadIdx.x; t < ne * g * (H / 4); t += blockDim.x) {
            const int row = t / (H / 4), h4 = t - row * (H / 4);
            *reinterpret_cast<float4*>(sw + row * hp + 4 * h4) =
                *reinterpret_cast<const float4*>(W2 + (c0 * g + row) * H + 4 * h4);
        }
        __syncthreads();
        // work items: (edge, group block, row r) with r fastest
        for (int it = threadIdx.x; it < ne * nqb * g; it += blockDim.x) {
            const int r = it % g, rest = it / g;
            const int qb = rest % nqb, e = rest / nqb;
            const float* w = sw + (e * g + r) * hp;
            const float* hq = hid + (qb * 4) * hp;
            const float bias = b2[(c0 + e) * g + r];
            float acc[4] = {bias, bias, bias, bias};
            for (int h = 0; h < H; h += 4) {
                const float4 wv = lds4(w + h);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float4 hv = lds4(hq + u * hp + h);
                    acc[u] = fmaf(wv.x, hv.x, fmaf(wv.y, hv.y, fmaf(wv.z, hv.z, fmaf(wv.w, hv.w, acc[u]))));
                }
            }
            T* crow = coef + (c0 + e) * (int64_t)nq * g;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int ql = qb * 4 + u;
                if (ql < nq) crow[ql * g + r] = cvt_out<T>(acc[u]);
            }
        }
    }
}

// dW2[e, :] = sum_q dc(q)[e] hid(q), db2[e] = sum_q dc(q)[e]: chunks of kCE edges
// (their dcoef window rows staged in shared memory), each thread four hidden
// units of one W2 row (16-byte loads and stores).
__global__ void __launch_bounds__(kUkThreads) ukan_dw2_kernel(const float* __restrict__ pre,
                                                               const float* __restrict__ dcoef,
                                                               float* __restrict__ dW2, float* __restrict__ db2,
                                                               int64_t edges, int g, int H, int nq)
{
    extern __shared__ __align__(16) float sh[];
    float* hid = sh;                             // [nq][H]
    float* sd = sh + nq * H;                     // [kCE][nq * g]
    for (int t = threadIdx.x; t < nq * H; t += blockDim.x) hid[t] = silu_pre(pre[t]);
    const int nw = nq * g;
    const int hb_n = H / 4;
    for (int64_t c0 = (int64_t)blockIdx.x * kCE; c0 < edges; c0 += (int64_t)gridDim.x * kCE) {
        const int ne = (int)(edges - c0 < kCE ? edges - c0 : kCE);
        __syncthreads();
        for (int t = threadIdx.x; t < ne * nw; t += blockDim.x) sd[t] = dcoef[c0 * nw + t];
        __syncthreads();
        if (db2)
            for (int t = threadIdx.x; t < ne * g; t += blockDim.x) {
                const int e = t / g, r = t - e * g;
                float sb = 0.0f;
                for (int ql = 0; ql < nq; ++ql) sb += sd[e * nw + ql * g + r];
                db2[(c0 + e) * g + r] = sb;
            }
        if (!dW2) continue;
        // work items: (row = edge * g + r, hidden block) with the hidden block fastest
        for (int it = threadIdx.x; it < ne * g * hb_n; it += blockDim.x) {
            const int hb = it % hb_n, row = it / hb_n;
            const int e = row / g, r = row - e * g;
            float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            for (int ql = 0; ql < nq; ++ql) {
                const float dv = sd[e * nw + ql * g + r];
                const float4 hv = lds4(hid + ql * H + 4 * hb);
                acc.x = fmaf(dv, hv.x, acc.x);
                acc.y = fmaf(dv, hv.y, acc.y);
                acc.z = fmaf(dv, hv.z, acc.z);
                acc.w = fmaf(dv, hv.w, acc.w);
            }
            *reinterpret_cast<float4*>(dW2 + ((c0 + e) * g + r) * H + 4 * hb) = acc;
        }
    }
}

// Block partials of dhid[ql, h] = sum_e dc(ql)[e] W2[e, h] over a contiguous
// range of edges: chunks of 64 edges (64 g rows of W2 and the matching dcoef
// values) staged in shared memory; a thread accumulates a 4 x 4 tile of
// (group, hidden unit) pairs over one of RG interleaved subsets of the rows,
// and the RG partial tiles are added in subset order at the end; one partial
// row per block.
__global__ void __launch_bounds__(kUkThreads) ukan_dhid_kernel(const float* __restrict__ W2,
                                                                const float* __restrict__ dcoef,
                                                                float* __restrict__ part, int64_t edges, int g, int H,
                                                                int nq, int64_t edges_per_block)
{
    constexpr int CE = 64;                                    // edges per chunk
    extern __shared__ __align__(16) float sh[];
    const int rows = CE * g;                                  // W2 rows per chunk
    const int hp = H + 4;
    float* sw = sh;                                           // [rows][hp]
    float* sd = sh + rows * hp;                               // [nq][rows]
    const int tq_n = (nq + kTq - 1) / kTq, th_n = H / kTh;
    const int tiles = tq_n * th_n;
    const int RG = tiles >= kUkThreads ? 1 : kUkThreads / tiles;   // row subsets
    const int rg = threadIdx.x / tiles;                       // (>= RG: idle; tiles > 256: see the s loop)
    const int64_t e_begin = (int64_t)blockIdx.x * edges_per_block;
    const int64_t e_end = min(edges, e_begin + edges_per_block);
    float acc[4][kTq][kTh];
#pragma unroll
    for (int s = 0; s < 4; ++s)
#pragma unroll
        for (int a = 0; a < kTq; ++a)
#pragma unroll
            for (int b = 0; b < kTh; ++b) acc[s][a][b] = 0.0f;
    for (int64_t c0 = e_begin; c0 < e_end; c0 += CE) {
        const int ne = (int)(e_end - c0 < CE ? e_end - c0 : CE);
        __syncthreads();
        for (int t = threadIdx.x; t < ne * g * (H / 4); t += blockDim.x) {
            const int row = t / (H / 4), h4 = t - row * (H / 4);
            *reinterpret_cast<float4*>(sw + row * hp + 4 * h4) =
                *reinterpret_cast<const float4*>(W2 + (c0 * g + row) * H + 4 * h4);
        }
        for (int t = threadIdx.x; t < nq * ne * g; t += blockDim.x) {
            const int ql = t / (ne * g), rr = t - ql * (ne * g);
            const int e = rr / g, r = rr - e * g;
            sd[ql * rows + rr] = dcoef[(c0 + e) * (int64_t)nq * g + ql * g + r];
        }
        __syncthreads();
        if (RG > 1) {
            if (rg >= RG) continue;
            const int tile = threadIdx.x - rg * tiles;
            const int tq = tile / th_n, th = tile - tq * th_n;
            for (int rr = rg; rr < ne * g; rr += RG) {
                float dv[kTq];
#pragma unroll
                for (int a = 0; a < kTq; ++a) dv[a] = tq * kTq + a < nq ? sd[(tq * kTq + a) * rows + rr] : 0.0f;
                const float4 wv = lds4(sw + rr * hp + th * kTh);
#pragma unroll
                for (int a = 0; a < kTq; ++a) {
                    acc[0][a][0] = fmaf(dv[a], wv.x, acc[0][a][0]);
                    acc[0][a][1] = fmaf(dv[a], wv.y, acc[0][a][1]);
                    acc[0][a][2] = fmaf(dv[a], wv.z, acc[0][a][2]);
                    acc[0][a][3] = fmaf(dv[a], wv.w, acc[0][a][3]);
                }
            }
        } else {
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const int tile = threadIdx.x + s * blockDim.x;
                if (tile >= tiles) break;
                const int tq = tile / th_n, th = tile - tq * th_n;
                for (int rr = 0; rr < ne * g; ++rr) {
                    float dv[kTq];
#pragma unroll
                    for (int a = 0; a < kTq; ++a) dv[a] = tq * kTq + a < nq ? sd[(tq * kTq + a) * rows + rr] : 0.0f;
                    const float4 wv = lds4(sw + rr * hp + th * kTh);
#pragma unroll
                    for (int a = 0; a < kTq; ++a) {
                        acc[s][a][0] = fmaf(dv[a], wv.x, acc[s][a][0]);
                        acc[s][a][1] = fmaf(dv[a], wv.y, acc[s][a][1]);
                        acc[s][a][2] = fmaf(dv[a], wv.z, acc[s][a][2]);
                        acc[s][a][3] = fmaf(dv[a], wv.w, acc[s][a][3]);
                    }
                }
            }
        }
    }
    if (RG > 1) {
        // the RG subsets' tiles, added in subset order
        __syncthreads();
        float* red = sh;                                      // [RG][tiles][16]
        if (rg < RG) {
            const int tile = threadIdx.x - rg * tiles;
#pragma unroll
            for (int a = 0; a < kTq; ++a)
#pragma unroll
                for (int b = 0; b < kTh; ++b) red[(rg * tiles + tile) * 16 + a * kTh + b] = acc[0][a][b];
        }
        __syncthreads();
        for (int t = threadIdx.x; t < tiles * 16; t += blockDim.x) {
            const int tile = t / 16, ab = t - tile * 16, a = ab / kTh, b = ab - a * kTh;
            float v = 0.0f;
            for (int q = 0; q < RG; ++q) v += red[(q * tiles + tile) * 16 + ab];
            const int tq = tile / th_n, th = tile - tq * th_n;
            const int ql = tq * kTq + a, h = th * kTh + b;
            if (ql < nq) part[(int64_t)blockIdx.x * nq * H + ql * H + h] = v;
        }
        return;
    }
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        const int tile = threadIdx.x + s * blockDim.x;
        if (tile >= tiles) break;
        const int tq = tile / th_n, th = tile - tq * th_n;
#pragma unroll
        for (int a = 0; a < kTq; ++a)
#pragma unroll
            for (int b = 0; b < kTh; ++b) {
                const int ql = tq * kTq + a, h = th * kTh + b;
                if (ql < nq) part[(int64_t)blockIdx.x * nq * H + ql * H + h] = acc[s][a][b];
            }
    }
}

// Sums of the block partials for every (group, hidden unit), split into kSub
// contiguous runs of blocks summed in parallel, the runs then added in order
// (fp64 throughout): dhid.
constexpr int kSub = 8;

__global__ void __launch_bounds__(kUkThreads) ukan_dhid_sum_kernel(const float* __restrict__ part, int nblocks,
                                                                    int n, double* __restrict__ sub)
{
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= n * kSub) return;
    const int o = t / kSub, k = t - o * kSub;
    const int per = (nblocks + kSub - 1) / kSub;
    double v = 0.0;
    for (int b = k * per; b < min(nblocks, (k + 1) * per); ++b) v += (double)part[(int64_t)b * n + o];
    sub[t] = v;
}

// dhid from the run sums (added in run order), then dpre = dhid silu'(pre),
// dW1[h, :] = sum_q dpre[q, h] PE(q), db1[h] = sum_q dpre[q, h].  One block.
__global__ void __launch_bounds__(kUkThreads) ukan_dw1_kernel(const double* __restrict__ sub,
                                                               const float* __restrict__ pre, int q0, int nq, int d,
                                                               int H, float* __restrict__ dW1, float* __restrict__ db1)
{
    extern __shared__ float sh[];
    float* dpre = sh;                                         // [nq][H]
    for (int t = threadIdx.x; t < nq * H; t += blockDim.x) {
        double s = 0.0;
        for (int k = 0; k < kSub; ++k) s += sub[t * kSub + k];
        const float z = pre[t];
        const float sg = __frcp_rn(1.0f + __expf(-z));
        dpre[t] = (float)s * (sg * (1.0f + z * (1.0f - sg)));
    }
    __syncthreads();
    for (int t = threadIdx.x; t < H * d; t += blockDim.x) {
        const int h = t / d, c = t - h * d;
        const int l = c / 2;
        const float w = exp2f(-(2.0f * l / (float)d) * 13.287712379549449f);
        float acc = 0.0f;
        for (int ql = 0; ql < nq; ++ql) {
            float sv, cv;
            sincosf((float)(q0 + ql) * w, &sv, &cv);
            acc = fmaf(dpre[ql * H + h], (c & 1) ? cv : sv, acc);
        }
        if (dW1) dW1[t] = acc;
    }
    if (db1)
        for (int h = threadIdx.x; h < H; h += blockDim.x) {
            float acc = 0.0f;
            for (int ql = 0; ql < nq; ++ql) acc += dpre[ql * H + h];
            db1[h] = acc;
        }
}

// Minimum and maximum of n values: block partials, then one block in order (no atomics).
template <typename T>
__global__ void range_kernel(const T* __restrict__ x, int64_t n, float* __restrict__ part)
{
    float lo = INFINITY, hi = -INFINITY;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
        const float v = to_f(x[e]);
        lo = fminf(lo, v);
        hi = fmaxf(hi, v);
    }
    for (int o = 16; o > 0; o >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    __shared__ float sl[32], shh[32];
    if ((threadIdx.x & 31) == 0) {
        sl[threadIdx.x >> 5] = lo;
        shh[threadIdx.x >> 5] = hi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w) {
            lo = fminf(lo, sl[w]);
            hi = fmaxf(hi, shh[w]);
        }
        part[2 * blockIdx.x] = lo;
        part[2 * blockIdx.x + 1] = hi;
    }
}

__global__ void range_final_kernel(const float* __restrict__ part, int nblocks, float* __restrict__ out)
{
    if (threadIdx.x != 0) return;
    float lo = INFINITY, hi = -INFINITY;
    for (int b = 0; b < nblocks; ++b) {
        lo = fminf(lo, part[2 * b]);
        hi = fmaxf(hi, part[2 * b + 1]);
    }
    out[0] = lo;
    out[1] = hi;
}

constexpr int kRangeBlocks = 296;

kan_status uk_fail(kan_status st, const char* msg) { return set_last_error(st, msg); }

kan_status validate(const kan_ukan_shape* s)
{
    if (!s) return uk_fail(KAN_ERR_INVALID_ARG, "shape is NULL");
    if (s->in < 1 || s->out < 1 || s->group < 1) return uk_fail(KAN_ERR_INVALID_ARG, "in, out, group must be >= 1");
    if (s->pe_dim < 2 || s->pe_dim % 2 || s->pe_dim > 256) return uk_fail(KAN_ERR_INVALID_ARG, "pe_dim must be even, 2..256");
    if (s->hidden < 4 || s->hidden > kMaxHidden || s->hidden % 4)
        return uk_fail(KAN_ERR_INVALID_ARG, "hidden must be a multiple of 4 in 4..256");
    if (s->nq < 1 || (int64_t)s->nq * s->group < 4) return uk_fail(KAN_ERR_INVALID_ARG, "nq * group must be >= 4");
    if ((int64_t)s->nq * s->hidden > kMaxHidTerms) return uk_fail(KAN_ERR_UNSUPPORTED, "nq * hidden > 12288");
    if (s->dtype != KAN_F32 && s->dtype != KAN_BF16) return uk_fail(KAN_ERR_INVALID_ARG, "unknown dtype");
    if (s->in * s->out > ((int64_t)1 << 36)) return uk_fail(KAN_ERR_UNSUPPORTED, "sizes too large");
    return KAN_OK;
}

int dhid_blocks(int64_t edges)
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return (int)std::max<int64_t>(1, std::min<int64_t>((edges + 63) / 64, (int64_t)sms * 2));
}

int chunk_blocks(int64_t edges)
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return (int)std::max<int64_t>(1, std::min<int64_t>((edges + kCE - 1) / kCE, (int64_t)sms * 4));
}

size_t gen_smem(const kan_ukan_shape& s)
{
    const int hp = s.hidden + 4, nqp = (s.nq + 3) / 4 * 4;
    return (size_t)(nqp * hp + std::max(kCE * s.group * hp, s.nq * s.hidden)) * sizeof(float);
}

size_t dw2_smem(const kan_ukan_shape& s) { return (size_t)(s.nq * s.hidden + kCE * s.nq * s.group) * sizeof(float); }

// workspace: the dhid block partials (float), then the run sums (double)
size_t part_bytes(const kan_ukan_shape& s)
{
    return ((size_t)dhid_blocks(s.in * s.out) * s.nq * s.hidden * sizeof(float) + 255) & ~(size_t)255;
}
size_t ukan_ws_bytes(const kan_ukan_shape& s) { return part_bytes(s) + (size_t)s.nq * s.hidden * kSub * sizeof(double); }

size_t dhid_smem(const kan_ukan_shape& s)
{
    // staging, or the final combine of the row subsets ([RG][tiles][16] <= 256 * 16 floats)
    const size_t stage = (size_t)(64 * s.group * (s.hidden + 4) + s.nq * 64 * s.group);
    return std::max<size_t>(stage, 256 * 16) * sizeof(float);
}

}  // namespace
}  // namespace kan

using namespace kan;

extern "C" {

kan_status kan_ukan_layer_shape(const kan_ukan_shape* s, int64_t batch, float h, kan_shape* out)
{
    kan_status st = validate(s);
    if (st != KAN_OK) return st;
    if (!out) return uk_fail(KAN_ERR_INVALID_ARG, "out is NULL");
    if (!(h > 0.0f) || !isfinite(h)) return uk_fail(KAN_ERR_INVALID_ARG, "h must be finite and > 0");
    const int G = s->nq * s->group - 3;
    if (G > 250) return uk_fail(KAN_ERR_UNSUPPORTED, "nq * group - 3 > 250 (the layer's grid limit)");
    out->batch = batch;
    out->in = s->in;
    out->out = s->out;
    out->G = G;
    // the window's basis 0 is the unbounded basis q0 g, supported from (q0 g) h = lo - 3 h
    out->lo = (float)(((double)s->q0 * s->group + 3.0) * (double)h);
    out->hi = (float)((double)out->lo + (double)G * (double)h);
    out->dtype = s->dtype;
    out->has_base = 0;
    out->path = KAN_PATH_AUTO;
    out->degree = 3;
    out->dims = 1;
    return KAN_OK;
}

kan_status kan_ukan_generate(const kan_ukan_shape* s, const float* W1, const float* b1, const float* W2,
                             const float* b2, void* coef, float* pre, void* stream)
{
    kan_status st = validate(s);
    if (st != KAN_OK) return st;
    if (!W1 || !b1 || !W2 || !b2 || !coef || !pre) return uk_fail(KAN_ERR_INVALID_ARG, "a null pointer");
    const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const int64_t edges = s->in * s->out;
    const size_t smem = gen_smem(*s);
    if (smem > 227 * 1024) return uk_fail(KAN_ERR_UNSUPPORTED, "group * hidden too large for the generator stage");
    static size_t configured = 0;
    if (smem > 48 * 1024 && configured < smem) {
        cudaFuncSetAttribute(ukan_generate_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        cudaFuncSetAttribute(ukan_generate_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             227 * 1024);
        configured = 227 * 1024;
    }
    const int blocks = chunk_blocks(edges);
    if (s->dtype == KAN_F32)
        ukan_generate_kernel<float><<<blocks, kUkThreads, smem, cs>>>(W1, b1, W2, b2, (float*)coef, pre, edges,
                                                                      s->group, s->pe_dim, s->hidden, s->q0, s->nq);
    else
        ukan_generate_kernel<__nv_bfloat16><<<blocks, kUkThreads, smem, cs>>>(
            W1, b1, W2, b2, (__nv_bfloat16*)coef, pre, edges, s->group, s->pe_dim, s->hidden, s->q0, s->nq);
    count_launch();
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? KAN_OK : uk_fail(KAN_ERR_CUDA, cudaGetErrorString(e));
}

kan_status kan_ukan_workspace_size(const kan_ukan_shape* s, size_t* bytes)
{
    kan_status st = validate(s);
    if (st != KAN_OK) return st;
    if (!bytes) return uk_fail(KAN_ERR_INVALID_ARG, "bytes is NULL");
    *bytes = ukan_ws_bytes(*s);
    return KAN_OK;
}

kan_status kan_ukan_generate_backward(const kan_ukan_shape* s, const float* W1, const float* W2, const float* pre,
                                      const float* dcoef, float* dW1, float* db1, float* dW2, float* db2,
                                      void* workspace, size_t ws_bytes, void* stream)
{
    kan_status st = validate(s);
    if (st != KAN_OK) return st;
    if (!W1 || !W2 || !pre || !dcoef) return uk_fail(KAN_ERR_INVALID_ARG, "a null pointer");
    const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const int64_t edges = s->in * s->out;
    cudaError_t e = cudaSuccess;
    if (dW2 || db2) {
        const size_t smem = dw2_smem(*s);
        if (smem > 227 * 1024) return uk_fail(KAN_ERR_UNSUPPORTED, "nq * group too large for the dW2 stage");
        static size_t configured2 = 0;
        if (smem > 48 * 1024 && configured2 < smem) {
            cudaFuncSetAttribute(ukan_dw2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
            configured2 = 227 * 1024;
        }
        ukan_dw2_kernel<<<chunk_blocks(edges), kUkThreads, smem, cs>>>(pre, dcoef, dW2, db2, edges, s->group,
                                                                          s->hidden, s->nq);
        count_launch();
        e = cudaGetLastError();
    }
    if (e == cudaSuccess && (dW1 || db1)) {
        const int nb = dhid_blocks(edges);
        const size_t need = ukan_ws_bytes(*s);
        if (ws_bytes < need || !workspace) return uk_fail(KAN_ERR_WORKSPACE, "workspace too small");
        const int64_t per = (edges + nb - 1) / nb;
        float* part = reinterpret_cast<float*>(workspace);
        double* sub = reinterpret_cast<double*>(reinterpret_cast<char*>(workspace) + part_bytes(*s));
        {
            const int tiles = ((s->nq + kTq - 1) / kTq) * ((s->hidden + kTh - 1) / kTh);
            if (tiles > 4 * kUkThreads) return uk_fail(KAN_ERR_UNSUPPORTED, "nq * hidden too large for the dhid tiles");
            const size_t smem = dhid_smem(*s);
            if (smem > 227 * 1024) return uk_fail(KAN_ERR_UNSUPPORTED, "group * hidden too large for the dhid stage");
            static size_t configured = 0;
            if (smem > 48 * 1024 && configured < smem) {
                cudaFuncSetAttribute(ukan_dhid_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
                configured = 227 * 1024;
            }
            ukan_dhid_kernel<<<nb, kUkThreads, smem, cs>>>(W2, dcoef, part, edges, s->group, s->hidden, s->nq, per);
        }
        count_launch();
        e = cudaGetLastError();
        if (e == cudaSuccess) {
            const int n = s->nq * s->hidden;
            ukan_dhid_sum_kernel<<<(n * kSub + kUkThreads - 1) / kUkThreads, kUkThreads, 0, cs>>>(part, nb, n, sub);
            ukan_dw1_kernel<<<1, kUkThreads, (size_t)n * sizeof(float), cs>>>(sub, pre, s->q0, s->nq, s->pe_dim,
                                                                            s->hidden, dW1, db1);
            count_launch(2);
            e = cudaGetLastError();
        }
    }
    return e == cudaSuccess ? KAN_OK : uk_fail(KAN_ERR_CUDA, cudaGetErrorString(e));
}

kan_status kan_input_range(int64_t n, const void* x, int32_t dtype, float* minmax, void* workspace, size_t ws_bytes,
                           void* stream)
{
    if (n < 1 || !x || !minmax) return uk_fail(KAN_ERR_INVALID_ARG, "n >= 1 and non-null pointers");
    if (dtype != KAN_F32 && dtype != KAN_BF16) return uk_fail(KAN_ERR_INVALID_ARG, "unknown dtype");
    if (ws_bytes < 2 * kRangeBlocks * sizeof(float) || !workspace)
        return uk_fail(KAN_ERR_WORKSPACE, "workspace too small (2368 bytes)");
    const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    float* part = reinterpret_cast<float*>(workspace);
    if (dtype == KAN_F32) range_kernel<float><<<kRangeBlocks, 256, 0, cs>>>((const float*)x, n, part);
    else range_kernel<__nv_bfloat16><<<kRangeBlocks, 256, 0, cs>>>((const __nv_bfloat16*)x, n, part);
    range_final_kernel<<<1, 32, 0, cs>>>(part, kRangeBlocks, minmax);
    count_launch(2);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? KAN_OK : uk_fail(KAN_ERR_CUDA, cudaGetErrorString(e));
}

}  // extern "C"
