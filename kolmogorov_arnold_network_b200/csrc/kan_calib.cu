// kan_calib.cu -- calibration kernel for the CUDA-core fp32 roofline.
//
// The fp32 path's bound counts algorithmic FMAs (4 per edge per GEMM) at the
// GPU's fp32 FMA rate, which no vendor table on this machine gives as a
// measured number.  kan_ffma_probe runs a kernel that does nothing but
// independent FMA chains, so that events around it measure that rate on the
// GPU at hand, at the clock it runs at.
#include "kan_internal.h"

namespace kan {
namespace {

constexpr int kProbeThreads = 256;
constexpr int kChains = 8;     // independent chains per thread (covers the FMA latency)
constexpr int kUnroll = 32;    // steps per loop iteration

// c_k <- c_k * m + a, kChains chains, iters * kUnroll steps; m and a arrive as
// kernel arguments so that nothing folds at compile time.
__global__ void __launch_bounds__(kProbeThreads) ffma_probe_kernel(int64_t iters, float m, float a, float* sink)
{
    float c[kChains];
#pragma unroll
    for (int k = 0; k < kChains; ++k) c[k] = (float)(threadIdx.x + k) * 1.0e-3f;
    for (int64_t it = 0; it < iters; ++it) {
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
#pragma unroll
            for (int k = 0; k < kChains; ++k) c[k] = fmaf(c[k], m, a);
    }
    float s = 0.0f;
#pragma unroll
    for (int k = 0; k < kChains; ++k) s += c[k];
    sink[(int64_t)blockIdx.x * kProbeThreads + threadIdx.x] = s;
}

}  // namespace
}  // namespace kan

extern "C" kan_status kan_ffma_probe(int32_t blocks, int64_t iters, float* sink, double* flops, void* stream)
{
    if (blocks < 1 || iters < 1 || !sink || !flops)
        return kan::set_last_error(KAN_ERR_INVALID_ARG, "kan_ffma_probe: blocks, iters >= 1 and non-null pointers");
    *flops = 2.0 * (double)blocks * kan::kProbeThreads * (double)iters * kan::kUnroll * kan::kChains;
    kan::ffma_probe_kernel<<<blocks, kan::kProbeThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        iters, 0.999999f, 1.0e-6f, sink);
    kan::count_launch();
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return kan::set_last_error(KAN_ERR_CUDA, cudaGetErrorString(e));
    return KAN_OK;
}
