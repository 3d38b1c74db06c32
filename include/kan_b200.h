/*
 * kan_b200.h -- C ABI of libkan_b200.so: forward and backward pass of a
 * B-spline Kolmogorov-Arnold (KAN) layer on one NVIDIA B200 (sm_100a).
 *
 * The operation (sources):
 *   y[b,j] = sum_i phi_ji(x[b,i])                  InKAN landing page, "What is a KAN?"
 *   phi_ji(x) = sum_m coef[j,i,m] B_m(x)            B-spline with local support
 *                                                   (same page and section)
 *             (+ w_base[j,i] silu(x) when has_base) optional SiLU base branch
 *   B_m: uniform B-splines of degree k (kan_shape.degree, 1..5; cubic, k = 3,
 *   is the InKAN page's layer) on G intervals of [lo,hi], the grid extended
 *   by k knots on each side, m = 0..G+k-1 ("predefined, bounded grids": UKAN
 *   abstract, "Want to train KANS at scale? Now UKAN!"; degree-k splines and
 *   the normalised coordinate bounded to [0, k+1]: FlashKAN abstract, mlsift
 *   "GPU kernel" listing).  Knots t_j = lo + (j-k)(hi-lo)/G, j = 0..G+2k;
 *   supp B_m = [t_m, t_{m+k+1}).  An input outside [t_0, t_{G+2k}) (and any
 *   NaN or inf) has all B_m = 0.  Each input touches only k+1 basis
 *   functions (for k = 3 the "local 4-basis lookup": InKAN landing page,
 *   "Why InKAN?"), evaluated on the bounded local coordinate with
 *   non-negative arithmetic only (same page, "Numerically Stable"): the cubic
 *   pieces in closed form, other degrees by k passes of the recursion over
 *   those k+1 values alone.
 *
 * Gradients (backward):
 *   dcoef[j,i,m]  = sum_b B_m(x[b,i]) dY[b,j]
 *   dw_base[j,i]  = sum_b silu(x[b,i]) dY[b,j]
 *   dx[b,i]       = sum_j dY[b,j] (sum_m coef[j,i,m] B'_m(x[b,i]) + w_base[j,i] silu'(x[b,i]))
 *   Batch reductions are deterministic: fixed order, no atomic adds (the
 *   FlashKAT abstract names atomic gradient accumulation as a bottleneck and
 *   a source of rounding error).
 *
 * Layouts: every tensor is dense row-major (C order) in device memory.
 *   x       [batch, in]          operand dtype
 *   coef    [out, in, G+k]       operand dtype (k = degree)
 *   w_base  [out, in]            operand dtype (only when has_base)
 *   y       [batch, out]         operand dtype
 *   dY      [batch, out]         operand dtype
 *   dx      [batch, in]          operand dtype
 *   dcoef   [out, in, G+k]       float32, overwritten
 *   dw_base [out, in]            float32, overwritten
 * The operand dtype is float32 or bfloat16; accumulation is always fp32.
 * Pointers must be 16-byte aligned.
 *
 * 2-D surfaces (kan_shape.dims = 2): "tensor-product B-spline surfaces for
 * joint function approximation" (InKAN landing page, "Why InKAN?", item "1D
 * and 2D Splines").  The inputs are taken in consecutive pairs (u, v) =
 * (x[b,2p], x[b,2p+1]) and each edge (j, p) carries a surface on the same
 * knot grid in both coordinates:
 *   y[b,j] = sum_p sum_{m1,m2} coef[j,p,m1,m2] B_m1(u) B_m2(v)
 *   dcoef[j,p,m1,m2] = sum_b dY[b,j] B_m1(u) B_m2(v)
 *   dx[b,2p]   = sum_j dY[b,j] sum coef[j,p,m1,m2] B'_m1(u) B_m2(v)
 *   dx[b,2p+1] = sum_j dY[b,j] sum coef[j,p,m1,m2] B_m1(u) B'_m2(v)
 * with coef and dcoef [out, in/2, G+k, G+k].  Requires in even, no SiLU
 * branch, cubic splines (degree 3), and the tensor-core path: (G+3)^2 at most
 * 249 columns per pair for bf16 and 121 for fp32 (KAN_ERR_UNSUPPORTED else).
 *
 * Ownership: the caller owns every buffer, the workspace included.  The
 * library allocates no memory per call.  It holds two fixed device arrays in
 * its own image, which every GPU that loads it keeps until the process exits:
 * a 4-byte status word, and the KAN_FIXED_SCRATCH_BYTES workspace used only by
 * kan_forward_fixed_scratch.  Their device addresses are looked up once per
 * device and kept: do not use the library across a cudaDeviceReset (or any
 * other teardown of the device's primary context) in the same process.
 *
 * Streams: every compute call is asynchronous on `stream` (a cudaStream_t
 * passed as void*, NULL = legacy default stream).  Errors found on the host
 * are returned before anything is launched.  A device-side wait that gives up
 * (every wait inside a kernel has a time limit of about one second) records
 * KAN_ERR_TIMEOUT in a device status word, which kan_sync_status() reports.
 *
 * Threading: calls may come from several host threads; kan_last_error() is
 * per thread.
 */
#ifndef KAN_B200_H
#define KAN_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KAN_API __attribute__((visibility("default")))
#else
#define KAN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define KAN_ABI_VERSION 2

typedef enum { KAN_F32 = 0, KAN_BF16 = 1 } kan_dtype;

typedef enum {
    KAN_OK = 0,
    KAN_ERR_INVALID_ARG = 1,   /* a null pointer, a non-positive size, G < 1, hi <= lo, degree not 1..5, ... */
    KAN_ERR_UNSUPPORTED = 2,   /* valid but not handled: misaligned pointer, G > 250, forced path not possible */
    KAN_ERR_WORKSPACE = 3,     /* workspace smaller than kan_workspace_size() */
    KAN_ERR_CUDA = 4,          /* a CUDA runtime or driver call failed (detail in kan_last_error) */
    KAN_ERR_TIMEOUT = 5,       /* a device-side wait gave up (reported by kan_sync_status) */
    KAN_ERR_DEVICE_CHECK = 6   /* a device-side consistency check failed (reported by kan_sync_status) */
} kan_status;

/* Kernel family selection (kan_shape.path). */
#define KAN_PATH_AUTO 0    /* tensor-core kernels when TMA can address the shape's rows, else CUDA-core kernels */
#define KAN_PATH_TENSOR 1  /* tcgen05/TMEM GEMM kernels with TMA-staged operands; KAN_ERR_UNSUPPORTED if not possible */
#define KAN_PATH_SIMT 2    /* CUDA-core kernels (any shape) */

typedef struct {
    int64_t batch;     /* rows of x; 0 is allowed (nothing to compute, dcoef/dw_base zeroed) */
    int64_t in;        /* input features, >= 1 */
    int64_t out;       /* output features, >= 1 */
    int32_t G;         /* grid intervals on [lo,hi], 1..250 */
    float lo, hi;      /* grid range, hi > lo, both finite */
    int32_t dtype;     /* kan_dtype of x, coef, w_base, y, dY, dx */
    int32_t has_base;  /* 1: add the SiLU base branch w_base[j,i] silu(x[b,i]) */
    int32_t path;      /* KAN_PATH_* */
    int32_t degree;    /* spline degree k, 1..5 (3: cubic) */
    int32_t dims;      /* 1: univariate splines; 2: tensor-product surfaces over input pairs (below) */
} kan_shape;

/* ABI version of the loaded library (KAN_ABI_VERSION it was built with). */
KAN_API int kan_abi_version(void);

/* Bytes of device workspace that kan_forward (for_backward = 0) or
 * kan_backward (for_backward = 1) needs for this shape on the current
 * device.  *bytes may be 0.  Pure host computation. */
KAN_API kan_status kan_workspace_size(const kan_shape* s, int for_backward, size_t* bytes);

/* Forward pass: y = sum_i sum_m coef[j,i,m] B_m(x[b,i]) (+ w_base silu).
 * w_base must be NULL when has_base = 0 and non-NULL otherwise.
 * workspace may be NULL when the required size is 0. */
KAN_API kan_status kan_forward(const kan_shape* s, const void* x, const void* coef, const void* w_base, void* y,
                       void* workspace, size_t ws_bytes, void* stream);

/* Backward pass for upstream gradient dY.  dx, dcoef, dw_base may each be
 * NULL to skip that output (dw_base must be NULL when has_base = 0).
 * dcoef and dw_base are float32 and overwritten (not accumulated). */
KAN_API kan_status kan_backward(const kan_shape* s, const void* x, const void* coef, const void* w_base, const void* dY,
                        void* dx, float* dcoef, float* dw_base, void* workspace, size_t ws_bytes, void* stream);

/* Size of the fixed device workspace used by kan_forward_fixed_scratch (32 MiB). */
#define KAN_FIXED_SCRATCH_BYTES (32u << 20)

/* kan_forward for callers that cannot allocate device memory when they run
 * the layer (their memory comes only from a framework's own allocator, or a
 * serving loop must not stall on cudaMalloc, or all memory is budgeted up
 * front).  Same arguments and results as kan_forward, minus the workspace:
 * the workspace is a fixed KAN_FIXED_SCRATCH_BYTES array in the library's
 * device image, which every GPU that loads the library holds until the
 * process exits.  Allocates nothing.  No counterpart on the pages this layer
 * follows: it exists for deployment only.
 *   - Shapes whose kan_workspace_size exceeds KAN_FIXED_SCRATCH_BYTES return
 *     KAN_ERR_WORKSPACE (use kan_forward with your own workspace then).
 *   - All calls share the one array: calls whose kernels overlap on the GPU
 *     (unordered streams) race; order them on one stream or with events.
 *   - The array keeps the last call's contents; the forward reads nothing
 *     from it that it did not write earlier in the same call.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress with that device current); make that first call
 *     before any stream capture begins. */
KAN_API kan_status kan_forward_fixed_scratch(const kan_shape* s, const void* x, const void* coef, const void* w_base,
                                             void* y, void* stream);

/* The basis step alone, for inspection and tests: for each x[b,i] (batch*in
 * values) the span s (int32; the k+1 non-zero functions are B_s..B_{s+k},
 * some of which may fall outside 0..G+k-1 and are then absent; s = INT32_MIN
 * when the input is outside the extended knots), the k+1 weights
 * w[., k+1] = B_{s+r}(x) and the k+1 derivatives dw[., k+1] = B'_{s+r}(x)
 * (k = s->degree).  Any output may be NULL. */
KAN_API kan_status kan_basis(const kan_shape* s, const void* x, int32_t* span, float* w, float* dw, void* stream);

/* Synchronises `stream`, then returns and clears the device status word that
 * kernels of this library set when a wait gives up (KAN_ERR_TIMEOUT) or a
 * device check fails (KAN_ERR_DEVICE_CHECK).  KAN_OK if none did. */
KAN_API kan_status kan_sync_status(void* stream);

/* Failure-path self test: launches one kernel whose thread waits on an
 * mbarrier that nothing completes, with a limit of limit_ns nanoseconds
 * (1 .. 2e9).  The wait gives up and records KAN_ERR_TIMEOUT, which the next
 * kan_sync_status() returns.  Faults and hangs nothing. */
KAN_API kan_status kan_selftest_wait_timeout(int64_t limit_ns, void* stream);

/* Number of kernels this library has launched in this process (all entry
 * points, all devices), for accounting of the launches inside a timed region. */
KAN_API uint64_t kan_launch_count(void);

/* Optional timing marks for benchmarks.  While set, the kan_forward and
 * kan_backward calls made on this host thread record the given CUDA events
 * (cudaEvent_t passed as void*, created and owned by the caller) on their
 * stream at the boundaries between their kernel groups:
 *   after_prep  : after the operand preparation (fp32: operand maxima and the
 *                 fp16 hi/lo copies; bf16: nothing precedes it), before the
 *                 first GEMM kernel (forward and backward);
 *   after_dcoef : kan_backward only, after the dcoef / dw_base kernels and
 *                 before the dx kernels.
 * An event recorded before and one after the call then split the call into
 * preparation, dcoef and dx time.  NULL arguments record nothing; call with
 * (NULL, NULL) to turn the marks off.  No counterpart on the pages: a
 * measurement aid.  Always KAN_OK. */
KAN_API kan_status kan_set_timing_marks(void* after_prep, void* after_dcoef);

/* Calibration kernel for the CUDA-core fp32 roofline (the bound of the fp32
 * path counts algorithmic FMAs): launches `blocks` blocks of 256 threads, each
 * thread running 8 independent fp32 FMA chains for iters * 32 steps, and
 * writes one float per thread to `sink` (device memory, blocks * 256 floats,
 * so that the work is not optimised away).  *flops receives the FLOPs the
 * launch executes (2 per FMA).  Asynchronous on `stream`; time it with events.
 * No counterpart on the pages: a measurement aid.  KAN_ERR_INVALID_ARG for
 * blocks < 1, iters < 1 or a null pointer. */
KAN_API kan_status kan_ffma_probe(int32_t blocks, int64_t iters, float* sink, double* flops, void* stream);

/* ------------------------------------------------------------------------
 * GR-KAN: the group-rational activation of the Kolmogorov-Arnold Transformer.
 *
 * The FlashKAT abstract ("FlashKAT: Understanding and Addressing Performance
 * Bottlenecks in the Kolmogorov-Arnold Transformer", Abstract) traces the slow
 * training of GR-KAN to the gradient accumulation of its backward pass (memory
 * stalls, atomic adds) and fixes it by keeping the accumulation on chip.  The
 * rational function is the Pade activation unit of that page's reference list,
 * in the form whose denominator cannot vanish:
 *   y[r,c] = phi_g(x[r,c]),  phi_g(x) = P_g(x) / (1 + |S_g(x)|),
 *   P_g(x) = sum_{p=0..m} a[g,p] x^p,  S_g(x) = sum_{q=1..n} b[g,q-1] x^q,
 *   g = c / (channels / groups)   (contiguous, equal channel groups).
 * Backward for upstream gradient dY (sign(0) = 0):
 *   dx[r,c]  = dY (P' - phi sign(S) S') / (1 + |S|)
 *   da[g,p]  = sum over the group's elements of dY x^p / (1 + |S|)
 *   db[g,q-1]= sum over the group's elements of -dY phi sign(S) x^q / (1 + |S|)
 * The sums are reduced without atomics in a fixed order (per-block partials
 * in the caller's workspace, then one pass in fp64): bitwise reproducible.
 *
 * Layouts (row-major): x, y, dY, dx [rows, channels] in the operand dtype
 * (KAN_F32 or KAN_BF16); a [groups, m+1], b [groups, n], da, db float32
 * (da, db overwritten).  Pointers 16-byte aligned; channels / groups times the
 * element size must be a multiple of 16 bytes (else KAN_ERR_UNSUPPORTED).
 * ------------------------------------------------------------------------ */
typedef struct {
    int64_t rows;        /* tokens, >= 0 */
    int64_t channels;    /* >= 1, a multiple of groups */
    int32_t groups;      /* >= 1 */
    int32_t num_degree;  /* m, 1..7: P has m+1 coefficients */
    int32_t den_degree;  /* n, 1..8: S has n coefficients (no constant term) */
    int32_t dtype;       /* kan_dtype of x, y, dY, dx */
} kan_grkan_shape;

/* Bytes of workspace kan_grkan_backward needs for da / db on the current device. */
KAN_API kan_status kan_grkan_workspace_size(const kan_grkan_shape* s, size_t* bytes);

/* y = phi(x).  Asynchronous on stream; host errors return before any launch. */
KAN_API kan_status kan_grkan_forward(const kan_grkan_shape* s, const void* x, const float* a, const float* b, void* y,
                                     void* stream);

/* dx, da, db for upstream gradient dY; any of the three may be NULL to skip
 * it.  The workspace (kan_grkan_workspace_size bytes) is needed only when da
 * or db is requested.  KAN_ERR_WORKSPACE if it is too small. */
KAN_API kan_status kan_grkan_backward(const kan_grkan_shape* s, const void* x, const float* a, const float* b,
                                      const void* dY, void* dx, float* da, float* db, void* workspace,
                                      size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * UKAN: KAN layers on an unbounded grid with generated coefficients.
 *
 * "Want to train KANS at scale? Now UKAN!" (Abstract): a coefficient-generator
 * (CG) model produces, on the fly, only the B-spline coefficients required
 * locally on an unbounded symmetric grid, fed with the positional encoding of
 * grid groups.  Reading taken here: knots j h for every integer j, cubic
 * B-splines B_m(x) = N(x/h - m); group q holds the basis indices
 * q*group .. q*group + group - 1; PE(q)[2l] = sin(q w_l), PE(q)[2l+1] =
 * cos(q w_l), w_l = 10000^(-2l/pe_dim) (the sinusoidal encoding of the page's
 * "Attention Is All You Need" reference); the generator is
 *   hid(q) = silu(W1 PE(q) + b1),  c(q) = W2 hid(q) + b2,
 *   coef[j, i, m] = c(q)[(j*in + i)*group + (m - q*group)],  q = floor(m / group),
 * with W1 [hidden, pe_dim], b1 [hidden], W2 [out*in*group, hidden],
 * b2 [out*in*group], all float32.
 *
 * A step: kan_input_range gives the batch's min / max (device), from which
 * the caller picks the groups q0 .. q0+nq-1 that its inputs reach (basis
 * floor(x/h) - 3 .. floor(x/h)); kan_ukan_generate writes those groups'
 * coefficients as the window coef [out, in, nq*group] (operand dtype); the
 * layer runs through kan_forward / kan_backward with the kan_shape that
 * kan_ukan_layer_shape returns (G = nq*group - 3, lo = (q0*group + 3) h: the
 * window's basis 0 is the unbounded basis q0*group; inputs outside the window
 * see no basis); kan_ukan_generate_backward takes the layer's dcoef back
 * through the generator.
 * ------------------------------------------------------------------------ */
typedef struct {
    int64_t in, out;     /* layer inputs and outputs, >= 1 */
    int32_t group;       /* basis functions per grid group, >= 1 */
    int32_t pe_dim;      /* encoding width, even, 2..256 */
    int32_t hidden;      /* generator hidden width, a multiple of 4 in 4..256 */
    int32_t q0, nq;      /* first group of the window and number of groups (nq*group >= 4, nq*hidden <= 12288) */
    int32_t dtype;       /* kan_dtype of the generated window (the layer's operand dtype) */
} kan_ukan_shape;

/* The kan_shape of the layer on the window (host only; h > 0 the knot spacing). */
KAN_API kan_status kan_ukan_layer_shape(const kan_ukan_shape* s, int64_t batch, float h, kan_shape* out);

/* coef [out, in, nq*group] (operand dtype) from the generator; pre [nq, hidden]
 * float32 receives the hidden pre-activations W1 PE(q) + b1 (kept for the
 * backward).  Asynchronous on stream. */
KAN_API kan_status kan_ukan_generate(const kan_ukan_shape* s, const float* W1, const float* b1, const float* W2,
                                     const float* b2, void* coef, float* pre, void* stream);

/* Bytes of workspace kan_ukan_generate_backward needs for dW1 / db1. */
KAN_API kan_status kan_ukan_workspace_size(const kan_ukan_shape* s, size_t* bytes);

/* Gradients of the generator's parameters from the window's dcoef [out, in,
 * nq*group] float32 (kan_backward's output) and the pre-activations of
 * kan_ukan_generate: dW2, db2 row by row, dW1, db1 through a fixed-order
 * reduction (block partials in the workspace, no atomics).  Any output may be
 * NULL; the workspace is needed only for dW1 / db1.  Outputs overwritten. */
KAN_API kan_status kan_ukan_generate_backward(const kan_ukan_shape* s, const float* W1, const float* W2,
                                              const float* pre, const float* dcoef, float* dW1, float* db1,
                                              float* dW2, float* db2, void* workspace, size_t ws_bytes, void* stream);

/* minmax[0..1] (device float32) = min and max of the n values x (KAN_F32 or
 * KAN_BF16), through block partials in the workspace (at least 2368 bytes).
 * Asynchronous on stream.  No counterpart on the pages: it sizes the UKAN
 * window. */
KAN_API kan_status kan_input_range(int64_t n, const void* x, int32_t dtype, float* minmax, void* workspace,
                                   size_t ws_bytes, void* stream);

/* Static description of a status code. */
KAN_API const char* kan_status_string(kan_status st);

/* Detail of the last non-OK status returned on this host thread ("" if none). */
KAN_API const char* kan_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* KAN_B200_H */
