// kan_simt.cu -- CUDA-core kernels of the KAN layer: the basis step on its
// own, and a complete forward/backward for shapes the tensor-core path does
// not take (tiny layers, strides TMA cannot address).  Each output element
// is produced by one thread with a fixed summation order, so results are
// deterministic; no atomics.
#include "kan_device.cuh"

namespace kan {
namespace {

constexpr int kFwdRows = 4;       // batch rows per forward block
constexpr int kFwdChunk = 256;    // inputs staged per pass in the forward block

// Weights (and derivatives) of an input on its local coordinate: the cubic
// closed form for k = 3, the local triangle otherwise (entries past k are 0).
__device__ __forceinline__ void local_weights(float t, int k, float inv_h, float (&w)[KAN_MAX_NW],
                                              float (&d)[KAN_MAX_NW], bool want_d)
{
    if (k == 3) {
        float w4[4], d4[4];
        weights(t, w4);
        if (want_d) dweights(t, inv_h, d4);
#pragma unroll
        for (int r = 0; r < KAN_MAX_NW; ++r) {
            w[r] = r < 4 ? w4[r] : 0.0f;
            d[r] = (want_d && r < 4) ? d4[r] : 0.0f;
        }
    } else if (want_d) {
        weights_k<true>(t, k, inv_h, w, d);
    } else {
        weights_k<false>(t, k, inv_h, w, d);
    }
}

template <typename T>
__global__ void basis_kernel(const T* __restrict__ x, int64_t n, float lo, float inv_h, int G, int k, int32_t* span,
                             float* w, float* dw)
{
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
        Span sp = span_of(to_f(x[e]), lo, inv_h, G, k);
        float wv[KAN_MAX_NW], dv[KAN_MAX_NW];
        local_weights(sp.t, k, inv_h, wv, dv, true);
        if (span) span[e] = sp.valid ? sp.s : INT32_MIN;
#pragma unroll
        for (int r = 0; r < KAN_MAX_NW; ++r) {
            if (r > k) break;
            if (w) w[e * (k + 1) + r] = sp.valid ? wv[r] : 0.0f;
            if (dw) dw[e * (k + 1) + r] = sp.valid ? dv[r] : 0.0f;
        }
    }
}

// y[b, j]: block = kFwdRows rows, threads stride over j.  The rows' spans
// and weights for a chunk of inputs are staged in shared memory.
template <typename T>
__global__ void forward_kernel(const T* __restrict__ x, const T* __restrict__ coef, const T* __restrict__ w_base,
                               T* __restrict__ y, int64_t batch, int64_t in, int64_t out, int G, int k, float lo,
                               float inv_h)
{
    __shared__ int s_span[kFwdRows][kFwdChunk];
    __shared__ float s_w[kFwdRows][kFwdChunk][KAN_MAX_NW];
    __shared__ float s_silu[kFwdRows][kFwdChunk];
    const int nb = G + k;
    const int64_t b0 = (int64_t)blockIdx.x * kFwdRows;
    const int nrows = (int)(batch - b0 < kFwdRows ? batch - b0 : kFwdRows);

    for (int64_t jb = 0; jb < out; jb += blockDim.x) {
        const int64_t j = jb + threadIdx.x;
        float acc[kFwdRows], accb[kFwdRows];
#pragma unroll
        for (int r = 0; r < kFwdRows; ++r) acc[r] = accb[r] = 0.f;

        for (int64_t i0 = 0; i0 < in; i0 += kFwdChunk) {
            const int ni = (int)(in - i0 < kFwdChunk ? in - i0 : kFwdChunk);
            __syncthreads();
            for (int e = threadIdx.x; e < kFwdRows * ni; e += blockDim.x) {
                int r = e / ni, ii = e % ni;
                float xv = r < nrows ? to_f(x[(b0 + r) * in + i0 + ii]) : 0.f;
                Span sp = span_of(xv, lo, inv_h, G, k);
                float wv[KAN_MAX_NW], dv[KAN_MAX_NW];
                local_weights(sp.t, k, inv_h, wv, dv, false);
                const bool use = sp.valid && r < nrows;
                s_span[r][ii] = use ? sp.s : -1000;
#pragma unroll
                for (int q = 0; q < KAN_MAX_NW; ++q) s_w[r][ii][q] = use ? wv[q] : 0.f;
                s_silu[r][ii] = (w_base && r < nrows) ? silu_f(xv) : 0.f;
            }
            __syncthreads();
            if (j < out) {
                const T* cj = coef + (j * in + i0) * nb;
                for (int ii = 0; ii < ni; ++ii) {
                    const T* cji = cj + (int64_t)ii * nb;
#pragma unroll
                    for (int r = 0; r < kFwdRows; ++r) {
                        int s = s_span[r][ii];
#pragma unroll
                        for (int q = 0; q < KAN_MAX_NW; ++q) {
                            int m = s + q;
                            if (q <= k && m >= 0 && m < nb) acc[r] += to_f(cji[m]) * s_w[r][ii][q];
                        }
                    }
                    if (w_base) {
                        float wb = to_f(w_base[j * in + i0 + ii]);
#pragma unroll
                        for (int r = 0; r < kFwdRows; ++r) accb[r] += wb * s_silu[r][ii];
                    }
                }
            }
        }
        if (j < out)
            for (int r = 0; r < nrows; ++r) y[(b0 + r) * out + j] = from_f<T>(acc[r] + accb[r]);
    }
}

// dcoef[j, i, m] (m < nb) and dw_base[j, i] (m == nb): one thread per
// (j, i, m), batch summed in order; each thread keeps one accumulator and adds
// the weight of its own basis function when the input's span covers it.
template <typename T>
__global__ void dcoef_kernel(const T* __restrict__ x, const T* __restrict__ dY, float* __restrict__ dcoef,
                             float* __restrict__ dw_base, int64_t batch, int64_t in, int64_t out, int G, int k,
                             float lo, float inv_h)
{
    const int nb = G + k;
    const int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (e >= in * out * (nb + 1)) return;
    const int m = (int)(e % (nb + 1));
    const int64_t ji = e / (nb + 1);
    const int64_t j = ji / in, i = ji % in;
    if (m == nb ? !dw_base : !dcoef) return;
    float acc = 0.f;
    for (int64_t b = 0; b < batch; ++b) {
        const float xv = to_f(x[b * in + i]);
        const float g = to_f(dY[b * out + j]);
        if (m == nb) {
            acc += silu_f(xv) * g;
            continue;
        }
        const Span sp = span_of(xv, lo, inv_h, G, k);
        const int q = m - sp.s;
        if (sp.valid && q >= 0 && q <= k) {
            float wv[KAN_MAX_NW], dv[KAN_MAX_NW];
            local_weights(sp.t, k, inv_h, wv, dv, false);
            float wq = 0.0f;   // (selected without indexing registers)
#pragma unroll
            for (int r = 0; r < KAN_MAX_NW; ++r) wq = r == q ? wv[r] : wq;
            acc += wq * g;
        }
    }
    if (m == nb) dw_base[ji] = acc;
    else dcoef[ji * nb + m] = acc;
}

// dx[b, i]: one thread per (b, i), j summed in order.
template <typename T>
__global__ void dx_kernel(const T* __restrict__ x, const T* __restrict__ coef, const T* __restrict__ w_base,
                          const T* __restrict__ dY, T* __restrict__ dx, int64_t batch, int64_t in, int64_t out,
                          int G, int k, float lo, float inv_h)
{
    const int nb = G + k;
    const int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (e >= batch * in) return;
    const int64_t b = e / in, i = e % in;
    float xv = to_f(x[e]);
    Span sp = span_of(xv, lo, inv_h, G, k);
    float wv[KAN_MAX_NW], dv[KAN_MAX_NW];
    local_weights(sp.t, k, inv_h, wv, dv, true);
    const float ds = w_base ? dsilu_f(xv) : 0.f;
    float acc = 0.f;
    for (int64_t j = 0; j < out; ++j) {
        const T* cji = coef + (j * in + i) * nb;
        float d = 0.f;
        if (sp.valid) {
#pragma unroll
            for (int q = 0; q < KAN_MAX_NW; ++q) {
                int m = sp.s + q;
                if (q <= k && m >= 0 && m < nb) d += to_f(cji[m]) * dv[q];
            }
        }
        if (w_base) d += to_f(w_base[j * in + i]) * ds;
        acc += to_f(dY[b * out + j]) * d;
    }
    dx[e] = from_f<T>(acc);
}

__global__ void zero_kernel(float* p, int64_t n)
{
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x)
        p[e] = 0.f;
}

// One thread waits on an mbarrier that nothing arrives at; the bounded wait
// gives up after limit_ns and records KAN_ERR_TIMEOUT.
__global__ void wait_selftest_kernel(uint64_t limit_ns, unsigned int* status)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_addr(&bar), 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(smem_addr(&bar), 0, status, limit_ns);
}

inline int blocks_for(int64_t n, int threads)
{
    int64_t b = (n + threads - 1) / threads;
    return (int)(b < 1 ? 1 : (b > 65535LL * 32 ? 65535LL * 32 : b));
}

}  // namespace

cudaError_t simt_basis(const Problem& p, const void* x, int32_t* span, float* w, float* dw, cudaStream_t st)
{
    const int64_t n = p.batch * p.in;
    if (n == 0) return cudaSuccess;
    if (p.dtype == KAN_F32) {
        basis_kernel<float><<<blocks_for(n, 256), 256, 0, st>>>((const float*)x, n, p.lo, p.inv_h, p.G, p.k, span, w, dw);
        count_launch();
    } else {
        basis_kernel<__nv_bfloat16><<<blocks_for(n, 256), 256, 0, st>>>((const __nv_bfloat16*)x, n, p.lo, p.inv_h,
                                                                         p.G, p.k, span, w, dw);
        count_launch();
    }
    return cudaGetLastError();
}

cudaError_t simt_forward(const Problem& p, const void* x, const void* coef, const void* w_base, void* y,
                         cudaStream_t st)
{
    if (p.batch == 0) return cudaSuccess;
    cudaError_t e = record_mark(timing_marks().after_prep, st);
    if (e != cudaSuccess) return e;
    const int blocks = (int)((p.batch + kFwdRows - 1) / kFwdRows);
    const int threads = p.out >= 128 ? 128 : (int)((p.out + 31) / 32 * 32);
    if (p.dtype == KAN_F32) {
        forward_kernel<float><<<blocks, threads, 0, st>>>((const float*)x, (const float*)coef, (const float*)w_base,
                                                          (float*)y, p.batch, p.in, p.out, p.G, p.k, p.lo, p.inv_h);
        count_launch();
    } else {
        forward_kernel<__nv_bfloat16><<<blocks, threads, 0, st>>>(
            (const __nv_bfloat16*)x, (const __nv_bfloat16*)coef, (const __nv_bfloat16*)w_base, (__nv_bfloat16*)y,
            p.batch, p.in, p.out, p.G, p.k, p.lo, p.inv_h);
        count_launch();
    }
    return cudaGetLastError();
}

cudaError_t simt_backward(const Problem& p, const void* x, const void* coef, const void* w_base, const void* dY,
                          void* dx, float* dcoef, float* dw_base, cudaStream_t st)
{
    cudaError_t e;
    if (p.batch == 0) {
        if (dcoef && (e = zero_f32(dcoef, p.out * p.Kt, st)) != cudaSuccess) return e;
        if (dw_base && (e = zero_f32(dw_base, p.out * p.in, st)) != cudaSuccess) return e;
        return cudaSuccess;
    }
    if ((e = record_mark(timing_marks().after_prep, st)) != cudaSuccess) return e;
    if (dcoef || dw_base) {
        const int64_t n = p.in * p.out * (p.nb + 1);
        if (p.dtype == KAN_F32) {
            dcoef_kernel<float><<<blocks_for(n, 128), 128, 0, st>>>((const float*)x, (const float*)dY, dcoef, dw_base,
                                                                     p.batch, p.in, p.out, p.G, p.k, p.lo, p.inv_h);
            count_launch();
        } else {
            dcoef_kernel<__nv_bfloat16><<<blocks_for(n, 128), 128, 0, st>>>(
                (const __nv_bfloat16*)x, (const __nv_bfloat16*)dY, dcoef, dw_base, p.batch, p.in, p.out, p.G, p.k,
                p.lo, p.inv_h);
            count_launch();
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if ((e = record_mark(timing_marks().after_dcoef, st)) != cudaSuccess) return e;
    if (dx) {
        const int64_t n = p.batch * p.in;
        if (p.dtype == KAN_F32) {
            dx_kernel<float><<<blocks_for(n, 128), 128, 0, st>>>((const float*)x, (const float*)coef,
                                                                  (const float*)w_base, (const float*)dY, (float*)dx,
                                                                  p.batch, p.in, p.out, p.G, p.k, p.lo, p.inv_h);
            count_launch();
        } else {
            dx_kernel<__nv_bfloat16><<<blocks_for(n, 128), 128, 0, st>>>(
                (const __nv_bfloat16*)x, (const __nv_bfloat16*)coef, (const __nv_bfloat16*)w_base,
                (const __nv_bfloat16*)dY, (__nv_bfloat16*)dx, p.batch, p.in, p.out, p.G, p.k, p.lo, p.inv_h);
            count_launch();
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t zero_f32(float* p, int64_t n, cudaStream_t st)
{
    if (n <= 0) return cudaSuccess; {
    zero_kernel<<<blocks_for(n, 256) > 4096 ? 4096 : blocks_for(n, 256), 256, 0, st>>>(p, n);
    count_launch();
    }
    return cudaGetLastError();
}

cudaError_t simt_wait_selftest(int64_t limit_ns, unsigned int* status, cudaStream_t st)
{
    wait_selftest_kernel<<<1, 32, 0, st>>>((uint64_t)limit_ns, status);
    count_launch();
    return cudaGetLastError();
}

}  // namespace kan
