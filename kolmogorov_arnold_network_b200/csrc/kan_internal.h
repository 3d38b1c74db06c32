// kan_internal.h -- declarations shared by the library's translation units
// (not part of the public ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/kan_b200.h"

#define KAN_WAIT_LIMIT_NS 1000000000ull  // every device-side wait gives up after ~1 s
#define KAN_MAX_G 250

namespace kan {

// Validated problem description passed from the C-ABI layer to launchers.
struct Problem {
    int64_t batch, in, out;
    int G;
    int k;           // spline degree (1..5)
    int dims;        // 1: univariate; 2: tensor-product surfaces over consecutive input pairs
    int nb1;         // G + k univariate basis functions
    int nb;          // columns of the dense expansion per unit: nb1 (1-D) or nb1^2 (2-D, one unit = one pair)
    int64_t x_ld;    // row length of x and dx (the layer's input count)
    int64_t Kt;      // in * nb (spline columns of the dense expansion); `in` counts units (pairs for 2-D)
    float lo, hi, inv_h;
    int dtype;       // KAN_F32 / KAN_BF16
    bool base;
    int path;
};

// Device status word (defined in kan_api.cu).
unsigned int* device_status_ptr();

// Count one kernel launch (defined in kan_api.cu).
void count_launch(int n = 1);

// Record the detail string that kan_last_error() returns on this thread.
kan_status set_last_error(kan_status st, const char* msg);

// Caller-provided timing marks (kan_set_timing_marks), per host thread:
// events recorded on the call's stream after the operand preparation and, in
// the backward, after the dcoef kernels.  Null members record nothing.
struct TimingMarks {
    cudaEvent_t after_prep = nullptr;
    cudaEvent_t after_dcoef = nullptr;
};
const TimingMarks& timing_marks();
inline cudaError_t record_mark(cudaEvent_t ev, cudaStream_t st) { return ev ? cudaEventRecord(ev, st) : cudaSuccess; }

// ---- CUDA-core kernels (kan_simt.cu) ----
cudaError_t simt_basis(const Problem& p, const void* x, int32_t* span, float* w, float* dw, cudaStream_t st);
cudaError_t simt_forward(const Problem& p, const void* x, const void* coef, const void* w_base, void* y,
                         cudaStream_t st);
cudaError_t simt_backward(const Problem& p, const void* x, const void* coef, const void* w_base, const void* dY,
                          void* dx, float* dcoef, float* dw_base, cudaStream_t st);
cudaError_t simt_wait_selftest(int64_t limit_ns, unsigned int* status, cudaStream_t st);
cudaError_t zero_f32(float* p, int64_t n, cudaStream_t st);

// ---- tensor-core kernels (kan_tc.cu) ----
// Returns true when the tensor-core path can run this problem (alignment of
// the strides that TMA needs, sizes); `why` receives the reason otherwise.
bool tc_supported(const Problem& p, bool backward, const char** why);
size_t tc_workspace_forward(const Problem& p, int num_sms);
size_t tc_workspace_backward(const Problem& p, int num_sms);
// Return cudaSuccess or an error; a driver-level failure (tensor map encode)
// is mapped to cudaErrorInvalidValue with detail in *detail.
cudaError_t tc_forward(const Problem& p, const void* x, const void* coef, const void* w_base, void* y, void* ws,
                       int num_sms, cudaStream_t st, const char** detail);
cudaError_t tc_backward(const Problem& p, const void* x, const void* coef, const void* w_base, const void* dY,
                        void* dx, float* dcoef, float* dw_base, void* ws, int num_sms, cudaStream_t st,
                        const char** detail);

}  // namespace kan
