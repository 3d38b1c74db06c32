// kan_api.cu -- the C ABI of libkan_b200.so: argument validation, workspace
// sizing, kernel-family dispatch and error reporting.  Declarations and the
// contract of every entry point are in include/kan_b200.h.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "kan_internal.h"

namespace kan {

static std::atomic<uint64_t> g_launches{0};
void count_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

__device__ unsigned int g_device_status = 0;

unsigned int* device_status_ptr()
{
    // Resolved per device on first use; the symbol is per-context.
    static unsigned int* ptrs[64] = {nullptr};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
        ptrs[dev] = reinterpret_cast<unsigned int*>(p);
    }
    return ptrs[dev];
}

namespace {
thread_local char g_last_error[512] = "";
thread_local TimingMarks g_marks;
}

const TimingMarks& timing_marks() { return g_marks; }

void set_timing_marks(void* after_prep, void* after_dcoef)
{
    g_marks.after_prep = reinterpret_cast<cudaEvent_t>(after_prep);
    g_marks.after_dcoef = reinterpret_cast<cudaEvent_t>(after_dcoef);
}

kan_status set_last_error(kan_status st, const char* msg)
{
    snprintf(g_last_error, sizeof(g_last_error), "%s", msg);
    return st;
}

namespace {

kan_status fail(kan_status st, const char* fmt, const char* arg = nullptr)
{
    if (arg)
        snprintf(g_last_error, sizeof(g_last_error), fmt, arg);
    else
        snprintf(g_last_error, sizeof(g_last_error), "%s", fmt);
    return st;
}

kan_status cuda_fail(cudaError_t e, const char* where)
{
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s", where, cudaGetErrorString(e));
    return KAN_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

kan_status validate(const kan_shape* s, Problem* p)
{
    if (!s) return fail(KAN_ERR_INVALID_ARG, "shape is NULL");
    if (s->batch < 0) return fail(KAN_ERR_INVALID_ARG, "batch < 0");
    if (s->in < 1 || s->out < 1) return fail(KAN_ERR_INVALID_ARG, "in and out must be >= 1");
    if (s->G < 1) return fail(KAN_ERR_INVALID_ARG, "G must be >= 1");
    if (s->G > KAN_MAX_G) return fail(KAN_ERR_UNSUPPORTED, "G > 250 is not supported");
    if (!isfinite(s->lo) || !isfinite(s->hi) || !(s->hi > s->lo))
        return fail(KAN_ERR_INVALID_ARG, "grid range needs finite lo < hi");
    if (s->dtype != KAN_F32 && s->dtype != KAN_BF16) return fail(KAN_ERR_INVALID_ARG, "unknown dtype");
    if (s->has_base != 0 && s->has_base != 1) return fail(KAN_ERR_INVALID_ARG, "has_base must be 0 or 1");
    if (s->path < KAN_PATH_AUTO || s->path > KAN_PATH_SIMT) return fail(KAN_ERR_INVALID_ARG, "unknown path");
    if (s->degree < 1 || s->degree > 5) return fail(KAN_ERR_INVALID_ARG, "degree must be 1..5");
    if (s->dims != 1 && s->dims != 2) return fail(KAN_ERR_INVALID_ARG, "dims must be 1 or 2");
    if (s->dims == 2) {
        if (s->in % 2 != 0) return fail(KAN_ERR_INVALID_ARG, "2-D surfaces need an even input count");
        if (s->has_base) return fail(KAN_ERR_INVALID_ARG, "2-D surfaces have no SiLU branch");
        if (s->degree != 3) return fail(KAN_ERR_UNSUPPORTED, "2-D surfaces are cubic (degree 3) only");
        if (s->path == KAN_PATH_SIMT) return fail(KAN_ERR_UNSUPPORTED, "2-D surfaces run on the tensor-core path only");
    }
    const int64_t nb1 = s->G + s->degree;
    const int64_t nb = s->dims == 2 ? nb1 * nb1 : nb1;
    const int64_t units = s->dims == 2 ? s->in / 2 : s->in;
    if (units > ((int64_t)1 << 40) / nb || s->out > ((int64_t)1 << 40) || s->batch > ((int64_t)1 << 40))
        return fail(KAN_ERR_UNSUPPORTED, "sizes too large");
    p->batch = s->batch;
    p->in = units;
    p->x_ld = s->in;
    p->out = s->out;
    p->G = s->G;
    p->k = s->degree;
    p->dims = s->dims;
    p->nb1 = (int)nb1;
    p->nb = (int)nb;
    p->Kt = units * nb;
    p->lo = s->lo;
    p->hi = s->hi;
    p->inv_h = (float)((double)s->G / ((double)s->hi - (double)s->lo));
    p->dtype = s->dtype;
    p->base = s->has_base != 0;
    p->path = s->path;
    return KAN_OK;
}

int num_sms()
{
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

// Which family runs this call; KAN_OK or KAN_ERR_UNSUPPORTED (forced tensor path impossible).
kan_status choose(const Problem& p, bool backward, bool* use_tc)
{
    const char* why = nullptr;
    bool ok = tc_supported(p, backward, &why);
    if (p.path == KAN_PATH_SIMT) {
        *use_tc = false;
        return KAN_OK;
    }
    if (p.path == KAN_PATH_TENSOR) {
        if (!ok) return fail(KAN_ERR_UNSUPPORTED, "tensor-core path not possible: %s", why);
        *use_tc = true;
        return KAN_OK;
    }
    // automatic: the tensor-core kernels for every shape whose strides TMA can
    // address; the CUDA-core kernels only for the others (1-D layers)
    if (!ok && p.dims == 2) return fail(KAN_ERR_UNSUPPORTED, "2-D surfaces: tensor-core path not possible: %s", why);
    *use_tc = ok;
    return KAN_OK;
}

}  // namespace
}  // namespace kan

using namespace kan;

extern "C" {

int kan_abi_version(void) { return KAN_ABI_VERSION; }

kan_status kan_workspace_size(const kan_shape* s, int for_backward, size_t* bytes)
{
    Problem p;
    kan_status st = validate(s, &p);
    if (st != KAN_OK) return st;
    if (!bytes) return fail(KAN_ERR_INVALID_ARG, "bytes is NULL");
    bool use_tc = false;
    if ((st = choose(p, for_backward != 0, &use_tc)) != KAN_OK) return st;
    *bytes = 0;
    if (use_tc) *bytes = for_backward ? tc_workspace_backward(p, num_sms()) : tc_workspace_forward(p, num_sms());
    return KAN_OK;
}

kan_status kan_forward(const kan_shape* s, const void* x, const void* coef, const void* w_base, void* y,
                       void* workspace, size_t ws_bytes, void* stream)
{
    Problem p;
    kan_status st = validate(s, &p);
    if (st != KAN_OK) return st;
    if (p.batch > 0 && (!x || !y)) return fail(KAN_ERR_INVALID_ARG, "x or y is NULL");
    if (!coef) return fail(KAN_ERR_INVALID_ARG, "coef is NULL");
    if (p.base != (w_base != nullptr)) return fail(KAN_ERR_INVALID_ARG, "w_base must be non-NULL iff has_base");
    if ((x && !aligned16(x)) || !aligned16(coef) || (w_base && !aligned16(w_base)) || (y && !aligned16(y)))
        return fail(KAN_ERR_UNSUPPORTED, "pointers must be 16-byte aligned");
    bool use_tc = false;
    if ((st = choose(p, false, &use_tc)) != KAN_OK) return st;
    const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (use_tc) {
        const int sms = num_sms();
        const size_t need = tc_workspace_forward(p, sms);
        if (ws_bytes < need || (need > 0 && !workspace)) return fail(KAN_ERR_WORKSPACE, "workspace too small");
        if (workspace && !aligned16(workspace)) return fail(KAN_ERR_UNSUPPORTED, "workspace must be 16-byte aligned");
        const char* detail = nullptr;
        e = tc_forward(p, x, coef, w_base, y, workspace, sms, cs, &detail);
        if (e != cudaSuccess) return detail ? fail(KAN_ERR_CUDA, "%s", detail) : cuda_fail(e, "kan_forward");
    } else {
        e = simt_forward(p, x, coef, w_base, y, cs);
        if (e != cudaSuccess) return cuda_fail(e, "kan_forward");
    }
    return KAN_OK;
}

kan_status kan_backward(const kan_shape* s, const void* x, const void* coef, const void* w_base, const void* dY,
                        void* dx, float* dcoef, float* dw_base, void* workspace, size_t ws_bytes, void* stream)
{
    Problem p;
    kan_status st = validate(s, &p);
    if (st != KAN_OK) return st;
    if (p.batch > 0 && (!x || !dY)) return fail(KAN_ERR_INVALID_ARG, "x or dY is NULL");
    if (!coef) return fail(KAN_ERR_INVALID_ARG, "coef is NULL");
    if (p.base != (w_base != nullptr)) return fail(KAN_ERR_INVALID_ARG, "w_base must be non-NULL iff has_base");
    if (!p.base && dw_base) return fail(KAN_ERR_INVALID_ARG, "dw_base given without the base branch");
    if ((x && !aligned16(x)) || !aligned16(coef) || (w_base && !aligned16(w_base)) || (dY && !aligned16(dY)) ||
        (dx && !aligned16(dx)) || (dcoef && !aligned16(dcoef)) || (dw_base && !aligned16(dw_base)))
        return fail(KAN_ERR_UNSUPPORTED, "pointers must be 16-byte aligned");
    if (!dx && !dcoef && !dw_base) return KAN_OK;
    bool use_tc = false;
    if ((st = choose(p, true, &use_tc)) != KAN_OK) return st;
    const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (use_tc) {
        const int sms = num_sms();
        const size_t need = tc_workspace_backward(p, sms);
        if (ws_bytes < need || (need > 0 && !workspace)) return fail(KAN_ERR_WORKSPACE, "workspace too small");
        if (workspace && !aligned16(workspace)) return fail(KAN_ERR_UNSUPPORTED, "workspace must be 16-byte aligned");
        const char* detail = nullptr;
        e = tc_backward(p, x, coef, w_base, dY, dx, dcoef, dw_base, workspace, sms, cs, &detail);
        if (e != cudaSuccess) return detail ? fail(KAN_ERR_CUDA, "%s", detail) : cuda_fail(e, "kan_backward");
    } else {
        e = simt_backward(p, x, coef, w_base, dY, dx, dcoef, dw_base, cs);
        if (e != cudaSuccess) return cuda_fail(e, "kan_backward");
    }
    return KAN_OK;
}

kan_status kan_basis(const kan_shape* s, const void* x, int32_t* span, float* w, float* dw, void* stream)
{
    Problem p;
    kan_status st = validate(s, &p);
    if (st != KAN_OK) return st;
    if (p.batch > 0 && !x) return fail(KAN_ERR_INVALID_ARG, "x is NULL");
    cudaError_t e = simt_basis(p, x, span, w, dw, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "kan_basis");
    return KAN_OK;
}

kan_status kan_sync_status(void* stream)
{
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "kan_sync_status");
    unsigned int* dp = device_status_ptr();
    if (!dp) return fail(KAN_ERR_CUDA, "device status word not available");
    unsigned int v = 0;
    e = cudaMemcpy(&v, dp, sizeof(v), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "kan_sync_status");
    if (v != 0) {
        const unsigned int zero = 0;
        e = cudaMemcpy(dp, &zero, sizeof(zero), cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return cuda_fail(e, "kan_sync_status");
        if (v == KAN_ERR_TIMEOUT) return fail(KAN_ERR_TIMEOUT, "a device-side wait gave up");
        return fail(KAN_ERR_DEVICE_CHECK, "a device-side check failed");
    }
    return KAN_OK;
}

kan_status kan_selftest_wait_timeout(int64_t limit_ns, void* stream)
{
    if (limit_ns < 1 || limit_ns > 2000000000LL) return fail(KAN_ERR_INVALID_ARG, "limit_ns must be in 1..2e9");
    unsigned int* dp = device_status_ptr();
    if (!dp) return fail(KAN_ERR_CUDA, "device status word not available");
    cudaError_t e = simt_wait_selftest(limit_ns, dp, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "kan_selftest_wait_timeout");
    return KAN_OK;
}

kan_status kan_set_timing_marks(void* after_prep, void* after_dcoef)
{
    set_timing_marks(after_prep, after_dcoef);
    return KAN_OK;
}

const char* kan_status_string(kan_status st)
{
    switch (st) {
    case KAN_OK: return "ok";
    case KAN_ERR_INVALID_ARG: return "invalid argument";
    case KAN_ERR_UNSUPPORTED: return "unsupported";
    case KAN_ERR_WORKSPACE: return "workspace too small";
    case KAN_ERR_CUDA: return "CUDA error";
    case KAN_ERR_TIMEOUT: return "device wait timed out";
    case KAN_ERR_DEVICE_CHECK: return "device check failed";
    }
    return "unknown status";
}

const char* kan_last_error(void) { return g_last_error; }

uint64_t kan_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
