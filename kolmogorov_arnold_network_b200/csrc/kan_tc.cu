// kan_tc.cu -- tensor-core (tcgen05 / TMEM / TMA) kernels of the KAN layer.
//
// The layer is a contraction over the dense basis expansion
//   A[b, i*(G+3)+m] = B_m(x[b,i])            (4 non-zeros per (b,i))
// with coef viewed as a [out, in*(G+3)] matrix:
//   y      = A . coef^T       (+ silu(x) . w_base^T)
//   dcoef  = dY^T . A         (dw_base = dY^T . silu(x))
//   dx     = gather of dY . coef at each input's 4 columns, times B'.
// A never exists in global memory: producer warps evaluate the span and the
// four weights of each input (the InKAN page's "local 4-basis lookup" and
// stable piecewise form) and write the dense, mostly-zero A tile straight
// into shared memory in the 128-byte-swizzled layout the tensor core reads.
// The dense expansion is cheap on tensor cores; the per-input work stays
// O(4) whatever G is.
//
// fp32 operands use three tf32 products (hi*hi + hi*lo + lo*hi) per term,
// which keeps about 21 significant bits per product; bf16 operands use one
// kind::f16 product.  Accumulation is fp32 in TMEM in both cases.
//
// Deterministic by construction: every output element is reduced by one
// CTA in a fixed order, and split-K partials are summed by a separate
// kernel in split order.  No atomics.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "kan_device.cuh"

namespace kan {
namespace {

constexpr int kBM = 128;                  // MMA M (rows of A / TMEM lanes)
constexpr int kThreads = 320;             // warp 0: TMA, warp 1: MMA + TMEM, warps 2-9: producers/epilogue
constexpr int kProducers = 256;
constexpr int kSmemBudget = 227 * 1024 - 2048;

template <int DT> struct Cfg;
template <> struct Cfg<KAN_BF16> {
    using T = __nv_bfloat16;
    static constexpr int BK = 64;         // elements per 128-byte row
    static constexpr int ESZ = 2;
    static constexpr int SPLIT = 1;       // operand copies per tile (1: plain)
    static constexpr uint32_t FMT = 1;    // bf16
};
template <> struct Cfg<KAN_F32> {
    using T = float;
    static constexpr int BK = 32;
    static constexpr int ESZ = 4;
    static constexpr int SPLIT = 2;       // hi and lo tf32 parts
    static constexpr uint32_t FMT = 2;    // tf32
};

struct FwdArgs {
    const void* x;
    void* y;                   // [batch,out] operand dtype, or fp32 partials [splits,batch,out]
    unsigned int* status;
    int64_t batch, in, out;
    int G, nb;
    float lo, inv_h;
    int Kt;                    // in * nb
    int nkb_spline;            // k-blocks covering the spline columns
    int nkb_total;             // + k-blocks of the SiLU columns
    int kb_per_split;
    int partial;
    int BN;
    int stages;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p)
{
    return (uint8_t*)(((uintptr_t)p + 1023) & ~(uintptr_t)1023);
}

__device__ __forceinline__ void st_shared_zero16(uint32_t addr)
{
    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0u) : "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

__device__ __forceinline__ void st_shared_u16(uint32_t addr, uint16_t v)
{
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

__device__ __forceinline__ void st_shared_f32(uint32_t addr, float v)
{
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Store one A element (row, column col of the k-block) into the swizzled
// tile(s): bf16 value, or the tf32 hi/lo pair.
template <int DT>
__device__ __forceinline__ void put_a(uint32_t a_hi, uint32_t a_lo, uint32_t row, int col, float v)
{
    const uint32_t off = sw128_byte(row, (uint32_t)col * Cfg<DT>::ESZ);
    if constexpr (DT == KAN_BF16) {
        __nv_bfloat16 h = __float2bfloat16_rn(v);
        st_shared_u16(a_hi + off, *reinterpret_cast<uint16_t*>(&h));
    } else {
        float hi = tf32_hi(v);
        st_shared_f32(a_hi + off, hi);
        st_shared_f32(a_lo + off, v - hi);
    }
}

// ---------------------------------------------------------------------------
// Forward: y[m0:m0+128, n0:n0+BN] over k-blocks [kb_begin, kb_end).
// ---------------------------------------------------------------------------
template <int DT>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_c_hi, const __grid_constant__ CUtensorMap tm_c_lo,
               const __grid_constant__ CUtensorMap tm_w_hi, const __grid_constant__ CUtensorMap tm_w_lo,
               const FwdArgs a)
{
    using C = Cfg<DT>;
    using T = typename C::T;
    constexpr int BK = C::BK;
    constexpr int HALF = BK / 2;          // elements per producer thread per k-block (64 bytes)
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);

    const int BN = a.BN, stages = a.stages;
    const uint32_t a_bytes = kBM * 128, b_bytes = (uint32_t)BN * 128;
    const uint32_t stage_bytes = (a_bytes + b_bytes) * C::SPLIT;
    const uint32_t sbase = smem_addr(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + stages * stage_bytes);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * stages + 1);
    auto full_a = [&](int s) { return smem_addr(&bars[s]); };
    auto full_b = [&](int s) { return smem_addr(&bars[stages + s]); };
    auto empty = [&](int s) { return smem_addr(&bars[2 * stages + s]); };
    const uint32_t accum_bar = smem_addr(&bars[3 * stages]);
    auto A_hi = [&](int s) { return sbase + s * stage_bytes; };
    auto A_lo = [&](int s) { return sbase + s * stage_bytes + a_bytes; };
    auto B_hi = [&](int s) { return sbase + s * stage_bytes + a_bytes * C::SPLIT; };
    auto B_lo = [&](int s) { return sbase + s * stage_bytes + a_bytes * C::SPLIT + b_bytes; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t m0 = (int64_t)blockIdx.y * kBM;
    const int n0 = blockIdx.x * BN;
    const int kb_begin = blockIdx.z * a.kb_per_split;
    const int kb_end = min(a.nkb_total, kb_begin + a.kb_per_split);
    const int nk = kb_end - kb_begin;
    const uint32_t tmem_cols = BN < 32 ? 32 : BN;

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(full_a(s), kProducers);
            mbar_init(full_b(s), 1);
            mbar_init(empty(s), 1);
        }
        mbar_init(accum_bar, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_slot), tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0 && nk > 0) {
            prefetch_tmap(&tm_c_hi);
            if (C::SPLIT == 2) prefetch_tmap(&tm_c_lo);
            int issued = 0;
            for (int it = 0; it < nk; ++it) {
                const int s = it % stages;
                const uint32_t ph = (it / stages) & 1;
                if (!mbar_wait(empty(s), ph ^ 1, a.status)) break;
                const int kb = kb_begin + it;
                mbar_arrive_expect_tx(full_b(s), b_bytes * C::SPLIT);
                if (kb < a.nkb_spline) {
                    tma_load_2d(B_hi(s), &tm_c_hi, full_b(s), kb * BK, n0);
                    if (C::SPLIT == 2) tma_load_2d(B_lo(s), &tm_c_lo, full_b(s), kb * BK, n0);
                } else {
                    const int kc = (kb - a.nkb_spline) * BK;
                    tma_load_2d(B_hi(s), &tm_w_hi, full_b(s), kc, n0);
                    if (C::SPLIT == 2) tma_load_2d(B_lo(s), &tm_w_lo, full_b(s), kc, n0);
                }
                ++issued;
            }
            // Drain: every load issued has landed before the CTA can exit.
            for (int it = max(0, issued - stages); it < issued; ++it)
                mbar_wait(full_b(it % stages), (it / stages) & 1, a.status);
        }
    } else if (warp == 1) {
        if (lane == 0 && nk > 0) {
            const uint32_t idesc = instr_desc(C::FMT, 0, 0, kBM, BN);
            bool ok = true;
            for (int it = 0; it < nk && ok; ++it) {
                const int s = it % stages;
                const uint32_t ph = (it / stages) & 1;
                if (!mbar_wait(full_a(s), ph, a.status) || !mbar_wait(full_b(s), ph, a.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {   // 4 x 32 bytes of K per 128-byte row
                    const uint64_t ad = smem_desc_sw128(A_hi(s) + ks * 32, 16, 1024);
                    const uint64_t bd = smem_desc_sw128(B_hi(s) + ks * 32, 16, 1024);
                    const uint32_t acc = (it > 0 || ks > 0) ? 1u : 0u;
                    if constexpr (DT == KAN_BF16) {
                        mma_bf16_ss(tmem_base, ad, bd, idesc, acc);
                    } else {
                        const uint64_t adl = smem_desc_sw128(A_lo(s) + ks * 32, 16, 1024);
                        const uint64_t bdl = smem_desc_sw128(B_lo(s) + ks * 32, 16, 1024);
                        mma_tf32_ss(tmem_base, adl, bd, idesc, acc);
                        mma_tf32_ss(tmem_base, ad, bdl, idesc, 1u);
                        mma_tf32_ss(tmem_base, ad, bd, idesc, 1u);
                    }
                }
                mma_commit(empty(s));
            }
            if (ok) mma_commit(accum_bar);
        }
    } else {
        // ---------------- producers: the A tile ----------------
        const int p = threadIdx.x - 64;
        const uint32_t row = p & (kBM - 1);
        const int half = p >> 7;
        const int64_t b = m0 + row;
        const bool row_ok = b < a.batch;
        const T* xrow = reinterpret_cast<const T*>(a.x) + (row_ok ? b : 0) * a.in;
        bool ok = true;
        for (int it = 0; it < nk; ++it) {
            const int s = it % stages;
            const uint32_t ph = (it / stages) & 1;
            if (!mbar_wait(empty(s), ph ^ 1, a.status)) {
                ok = false;
                break;
            }
            const int kb = kb_begin + it;
            const uint32_t ahi = A_hi(s), alo = A_lo(s);
            if (kb < a.nkb_spline) {
                // zero this thread's 64 bytes, then place the non-zero weights
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t off = sw128_chunk(row, half * 4 + c);
                    st_shared_zero16(ahi + off);
                    if (C::SPLIT == 2) st_shared_zero16(alo + off);
                }
                const int c_lo = kb * BK + half * HALF;       // first spline column of this thread
                const int c_hi = min(c_lo + HALF, a.Kt);      // one past the last
                if (row_ok && c_lo < c_hi) {
                    const int i_first = c_lo / a.nb, i_last = (c_hi - 1) / a.nb;
                    for (int i = i_first; i <= i_last; ++i) {
                        const Span sp = span_of(to_f(xrow[i]), a.lo, a.inv_h, a.G);
                        if (!sp.valid) continue;
                        float w[4];
                        weights(sp.t, w);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int m = sp.s + q;
                            const int col = i * a.nb + m;
                            if (m >= 0 && m < a.nb && col >= c_lo && col < c_hi)
                                put_a<DT>(ahi, alo, row, col - kb * BK, w[q]);
                        }
                    }
                }
            } else {
                // SiLU columns: dense
                const int i0 = (kb - a.nkb_spline) * BK + half * HALF;
                float v[HALF];
#pragma unroll
                for (int c = 0; c < HALF; ++c) {
                    const int i = i0 + c;
                    v[c] = (row_ok && i < a.in) ? silu_f(to_f(xrow[i])) : 0.0f;
                }
                if constexpr (DT == KAN_BF16) {
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        st_shared_v4(ahi + sw128_chunk(row, half * 4 + c), pack_bf16(v[8 * c], v[8 * c + 1]),
                                     pack_bf16(v[8 * c + 2], v[8 * c + 3]), pack_bf16(v[8 * c + 4], v[8 * c + 5]),
                                     pack_bf16(v[8 * c + 6], v[8 * c + 7]));
                } else {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        float h[4], l[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            h[e] = tf32_hi(v[4 * c + e]);
                            l[e] = v[4 * c + e] - h[e];
                        }
                        const uint32_t off = sw128_chunk(row, half * 4 + c);
                        st_shared_v4(ahi + off, __float_as_uint(h[0]), __float_as_uint(h[1]), __float_as_uint(h[2]),
                                     __float_as_uint(h[3]));
                        st_shared_v4(alo + off, __float_as_uint(l[0]), __float_as_uint(l[1]), __float_as_uint(l[2]),
                                     __float_as_uint(l[3]));
                    }
                }
            }
            fence_async_smem();
            mbar_arrive(full_a(s));
        }

        // ---------------- epilogue: TMEM -> y ----------------
        // tcgen05.ld is warp-collective: decide per warp, not per lane
        bool go = __all_sync(0xffffffffu, ok && nk > 0);
        if (go) go = __all_sync(0xffffffffu, mbar_wait(accum_bar, 0, a.status));
        if (go) {
            tc_fence_after();
            const int q = warp & 3;                 // TMEM lane quarter of this warp
            const int chalf = (warp - 2) >> 2;      // which half of the columns
            const uint32_t r = 32 * q + lane;
            const int64_t bo = m0 + r;
            const int cbeg = chalf * (BN / 2), cend = cbeg + BN / 2;
            for (int c0 = cbeg; c0 < cend; c0 += 16) {
                uint32_t v[16];
                tmem_ld16(tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
                tmem_ld_wait();
                if (bo >= a.batch) continue;
                const int64_t j0 = n0 + c0;
                if (a.partial) {
                    float* dst = reinterpret_cast<float*>(a.y) + ((int64_t)blockIdx.z * a.batch + bo) * a.out + j0;
                    if (j0 + 16 <= a.out) {
#pragma unroll
                        for (int e = 0; e < 16; e += 4)
                            *reinterpret_cast<uint4*>(dst + e) = make_uint4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                    } else {
                        for (int e = 0; e < 16 && j0 + e < a.out; ++e) dst[e] = __uint_as_float(v[e]);
                    }
                } else {
                    T* dst = reinterpret_cast<T*>(a.y) + bo * a.out + j0;
                    if constexpr (DT == KAN_BF16) {
                        if (j0 + 16 <= a.out) {
                            uint32_t pk[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                pk[e] = pack_bf16(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
                            *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                            *reinterpret_cast<uint4*>(dst + 8) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                        } else {
                            for (int e = 0; e < 16 && j0 + e < a.out; ++e)
                                dst[e] = __float2bfloat16_rn(__uint_as_float(v[e]));
                        }
                    } else {
                        if (j0 + 16 <= a.out) {
#pragma unroll
                            for (int e = 0; e < 16; e += 4)
                                *reinterpret_cast<uint4*>(dst + e) = make_uint4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                        } else {
                            for (int e = 0; e < 16 && j0 + e < a.out; ++e) dst[e] = __uint_as_float(v[e]);
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, tmem_cols);
    }
}

// y[b, j] = sum over splits z (ascending) of part[z, b, j].
template <typename T>
__global__ void reduce_splits_kernel(const float* __restrict__ part, T* __restrict__ y, int64_t n, int splits)
{
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
        float acc = 0.f;
        for (int z = 0; z < splits; ++z) acc += part[(int64_t)z * n + e];
        y[e] = from_f<T>(acc);
    }
}

// hi/lo tf32 split of an fp32 array.
__global__ void split_tf32_kernel(const float* __restrict__ src, float* __restrict__ hi, float* __restrict__ lo,
                                  int64_t n)
{
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
        float v = src[e];
        float h = tf32_hi(v);
        hi[e] = h;
        lo[e] = v - h;
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 get_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D tiled map over a row-major [rows, cols] matrix; box = [box_rows, box_cols],
// 128-byte swizzle (box_cols * esize must be 128), zero fill out of bounds.
bool make_map_2d(CUtensorMap* m, const void* base, bool f32, int64_t rows, int64_t cols, int box_rows, int box_cols,
                 const char** detail)
{
    auto enc = get_encoder();
    if (!enc) {
        *detail = "cuTensorMapEncodeTiled is not available from the driver";
        return false;
    }
    const int esz = f32 ? 4 : 2;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(cols * esz)};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                     const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        *detail = "cuTensorMapEncodeTiled rejected a tensor map";
        return false;
    }
    return true;
}

inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

struct FwdPlan {
    int BN, stages, n_tiles, m_tiles, splits, kb_per_split, nkb_spline, nkb_total;
    size_t ws_split_coef;   // bytes of tf32 hi/lo copies of coef and w_base
    size_t ws_partial;      // bytes of split partials
};

int pick_bn(int64_t out)
{
    if (out <= 32) return 32;
    if (out <= 64) return 64;
    if (out <= 128) return 128;
    return 256;
}

FwdPlan plan_forward(const Problem& p, int num_sms)
{
    FwdPlan f{};
    const bool f32 = p.dtype == KAN_F32;
    const int BK = f32 ? 32 : 64;
    const int split = f32 ? 2 : 1;
    f.BN = pick_bn(p.out);
    const int stage_bytes = (kBM * 128 + f.BN * 128) * split;
    f.stages = std::min(8, (kSmemBudget - 1024 - 256) / stage_bytes);
    f.n_tiles = (int)cdiv(p.out, f.BN);
    f.m_tiles = (int)cdiv(p.batch, kBM);
    f.nkb_spline = (int)cdiv(p.Kt, BK);
    f.nkb_total = f.nkb_spline + (p.base ? (int)cdiv(p.in, BK) : 0);
    const int64_t tiles = (int64_t)f.n_tiles * f.m_tiles;
    int splits = 1;
    if (tiles < num_sms) {
        splits = (int)std::max<int64_t>(1, num_sms / std::max<int64_t>(1, tiles));
        splits = std::min<int>(splits, std::max(1, f.nkb_total / 4));
    }
    f.kb_per_split = (int)cdiv(f.nkb_total, splits);
    f.splits = (int)cdiv(f.nkb_total, f.kb_per_split);
    f.ws_split_coef = f32 ? align256((size_t)p.out * p.Kt * 4) * 2 + (p.base ? align256((size_t)p.out * p.in * 4) * 2 : 0)
                          : 0;
    f.ws_partial = f.splits > 1 ? align256((size_t)f.splits * p.batch * p.out * 4) : 0;
    return f;
}

int smem_bytes_for(const FwdPlan& f, bool f32)
{
    const int split = f32 ? 2 : 1;
    return f.stages * (kBM * 128 + f.BN * 128) * split + 1024 + 256;
}

template <int DT>
cudaError_t launch_fwd(const FwdPlan& f, const CUtensorMap& ch, const CUtensorMap& cl, const CUtensorMap& wh,
                       const CUtensorMap& wl, const FwdArgs& args, cudaStream_t st)
{
    const int smem = smem_bytes_for(f, DT == KAN_F32);
    cudaError_t e = cudaFuncSetAttribute(fwd_kernel<DT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(f.n_tiles, f.m_tiles, f.splits);
    fwd_kernel<DT><<<grid, kThreads, smem, st>>>(ch, cl, wh, wl, args);
    return cudaGetLastError();
}

inline int grid_for(int64_t n) { return (int)std::min<int64_t>(std::max<int64_t>(1, (n + 255) / 256), 148 * 8); }

}  // namespace

bool tc_supported(const Problem& p, bool backward, const char** why)
{
    const int esz = p.dtype == KAN_F32 ? 4 : 2;
    if ((p.Kt * esz) % 16 != 0) {
        *why = "in*(G+3)*sizeof(dtype) is not a multiple of 16 bytes (TMA row stride)";
        return false;
    }
    if (p.base && (p.in * esz) % 16 != 0) {
        *why = "in*sizeof(dtype) is not a multiple of 16 bytes (TMA row stride of w_base)";
        return false;
    }
    if ((p.out * esz) % 16 != 0) {
        *why = "out*sizeof(dtype) is not a multiple of 16 bytes";
        return false;
    }
    if (p.Kt > (int64_t)1 << 30 || p.batch > ((int64_t)1 << 31) - 256) {
        *why = "problem too large for 32-bit tile coordinates";
        return false;
    }
    (void)backward;
    return true;
}

size_t tc_workspace_forward(const Problem& p, int num_sms)
{
    FwdPlan f = plan_forward(p, num_sms);
    return f.ws_split_coef + f.ws_partial;
}

cudaError_t tc_forward(const Problem& p, const void* x, const void* coef, const void* w_base, void* y, void* ws,
                       int num_sms, cudaStream_t st, const char** detail)
{
    if (p.batch == 0) return cudaSuccess;
    const bool f32 = p.dtype == KAN_F32;
    FwdPlan f = plan_forward(p, num_sms);
    uint8_t* wsp = reinterpret_cast<uint8_t*>(ws);
    const void *c_hi = coef, *c_lo = coef, *w_hi = w_base ? w_base : coef, *w_lo = w_hi;
    cudaError_t e;
    if (f32) {
        float* ch = reinterpret_cast<float*>(wsp);
        float* cl = reinterpret_cast<float*>(wsp + align256((size_t)p.out * p.Kt * 4));
        split_tf32_kernel<<<grid_for(p.out * p.Kt), 256, 0, st>>>((const float*)coef, ch, cl, p.out * p.Kt);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        c_hi = ch;
        c_lo = cl;
        w_hi = ch;
        w_lo = cl;
        if (p.base) {
            uint8_t* wb0 = wsp + align256((size_t)p.out * p.Kt * 4) * 2;
            float* wh = reinterpret_cast<float*>(wb0);
            float* wl = reinterpret_cast<float*>(wb0 + align256((size_t)p.out * p.in * 4));
            split_tf32_kernel<<<grid_for(p.out * p.in), 256, 0, st>>>((const float*)w_base, wh, wl, p.out * p.in);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
            w_hi = wh;
            w_lo = wl;
        }
        wsp += f.ws_split_coef;
    }
    const int BK = f32 ? 32 : 64;
    CUtensorMap m_ch, m_cl, m_wh, m_wl;
    if (!make_map_2d(&m_ch, c_hi, f32, p.out, p.Kt, f.BN, BK, detail) ||
        !make_map_2d(&m_cl, c_lo, f32, p.out, p.Kt, f.BN, BK, detail))
        return cudaErrorInvalidValue;
    if (p.base) {
        if (!make_map_2d(&m_wh, w_hi, f32, p.out, p.in, f.BN, BK, detail) ||
            !make_map_2d(&m_wl, w_lo, f32, p.out, p.in, f.BN, BK, detail))
            return cudaErrorInvalidValue;
    } else {
        m_wh = m_ch;
        m_wl = m_cl;
    }
    FwdArgs args{};
    args.x = x;
    args.y = f.splits > 1 ? (void*)wsp : y;
    args.status = device_status_ptr();
    args.batch = p.batch;
    args.in = p.in;
    args.out = p.out;
    args.G = p.G;
    args.nb = p.nb;
    args.lo = p.lo;
    args.inv_h = p.inv_h;
    args.Kt = (int)p.Kt;
    args.nkb_spline = f.nkb_spline;
    args.nkb_total = f.nkb_total;
    args.kb_per_split = f.kb_per_split;
    args.partial = f.splits > 1;
    args.BN = f.BN;
    args.stages = f.stages;
    e = f32 ? launch_fwd<KAN_F32>(f, m_ch, m_cl, m_wh, m_wl, args, st)
            : launch_fwd<KAN_BF16>(f, m_ch, m_cl, m_wh, m_wl, args, st);
    if (e != cudaSuccess) return e;
    if (f.splits > 1) {
        const int64_t n = p.batch * p.out;
        if (f32)
            reduce_splits_kernel<float><<<grid_for(n), 256, 0, st>>>((const float*)wsp, (float*)y, n, f.splits);
        else
            reduce_splits_kernel<__nv_bfloat16><<<grid_for(n), 256, 0, st>>>((const float*)wsp, (__nv_bfloat16*)y, n,
                                                                              f.splits);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

size_t tc_workspace_backward(const Problem& p, int num_sms)
{
    (void)p;
    (void)num_sms;
    return 0;
}

cudaError_t tc_backward(const Problem& p, const void* x, const void* coef, const void* w_base, const void* dY,
                        void* dx, float* dcoef, float* dw_base, void* ws, int num_sms, cudaStream_t st,
                        const char** detail)
{
    (void)num_sms;
    (void)ws;
    (void)detail;
    return simt_backward(p, x, coef, w_base, dY, dx, dcoef, dw_base, st);
}

}  // namespace kan
