// kan_tc.cu -- tensor-core (tcgen05 / TMEM / TMA) kernels of the KAN layer.
//
// The layer is a contraction over the dense basis expansion
//   A[b, i*(G+k)+m] = B_m(x[b,i])            (at most k+1 non-zeros per (b,i))
// with coef viewed as a [out, in*(G+k)] matrix (k: spline degree, 3 = cubic):
//   forward  y     = A . coef^T        (+ silu(x) . w_base^T)
//   dcoef          = dY^T . A          (dw_base = dY^T . silu(x))
//   dx             = sum over each input's k+1 columns of (dY . coef) times B'
//                    (+ silu'(x) * (dY . w_base))
// A never exists in global memory: producer warps evaluate each input's span
// and k+1 weights (the InKAN page's "local 4-basis lookup" in its stable
// piecewise form, for cubic splines) and write the dense, mostly-zero A tile
// (or its transpose) straight into shared memory in the 128-byte-swizzled
// layout the tensor core reads.  The dense expansion costs little on tensor
// cores, and the per-input work stays O(k+1) whatever G is.
//
// One kernel template serves five GEMMs:
//   FWD    A = basis rows (producers)  B = coef / w_base, K-major (TMA)
//   DCA    A = basis^T (producers)     B = dY (TMA)
//   DCB    A = dY^T, MN-major (TMA)    B = basis^T (producers): dcoef with
//          the outputs on M and the spline columns on N (bf16, no SiLU
//          branch), for `out` that wide N tiles would pad or split unevenly
//   DX     A = dY, K-major (TMA)       B = coef, MN-major (TMA); B'-gather epilogue
//   GEMM   A = dY, K-major (TMA)       B = w_base, MN-major (TMA); fp32 store
// Warp roles: 0 TMA, 1 MMA issue + TMEM allocation, then the A producers
// (FWD, DCA: 16 warps in 4 groups; the TMA-fed modes: 8 idle warps), then 4
// epilogue warps (which also promote the fp32 accumulators).
//
// fp32 with the SiLU branch: silu(x_i) is one more basis function of input i,
// with coefficient w_base[j, i].  Its column sits right after input i's G+k
// spline columns (column stride G+4) in the fp16 copies of the coefficients
// that the fp32 path makes anyway, so the SiLU terms ride along in every GEMM:
// the forward sums them, dcoef's epilogue writes dw_base, and the dx epilogue
// finds dY.w_base in its own accumulator.
//
// fp32 operands: every operand value v (times a per-call power-of-two scale
// taken from the operands' absolute maxima, so that it sits well inside the
// fp16 range) is split into two fp16 parts, hi = fp16(v) and lo =
// fp16((v - hi) * 2^11), which together carry about 22 significant bits.
// Three fp16 tensor-core products per term, hi*hi + (hi*lo + lo*hi) * 2^-11,
// keep about 21 bits of each product; the basis values need no scale (they
// lie in [0, 2/3]).  The tensor core's fp32 accumulation truncates, so long
// accumulations drift; the kernel therefore (a) accumulates the small hi*lo +
// lo*hi products in their own TMEM accumulator, and (b) accumulates hi*hi in
// short segments of kSegKb k-blocks, alternating between two TMEM buffers,
// which the epilogue warps add into a running fp32 total (round-to-nearest)
// while the next segment runs.
// bf16 operands: one kind::f16 product, fp32 accumulation in TMEM.
//
// Deterministic by construction: every output element is reduced by one CTA
// in a fixed order; split-K partials are summed by a separate kernel in
// split order.  No atomics.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <type_traits>
#include <mutex>

#include <cuda_fp16.h>

#include "kan_device.cuh"

namespace kan {
namespace {

constexpr int kBM = 128;          // MMA M: rows of A, TMEM lanes

// Producer warps per mode: the row producers (FWD, DCA) run 4 groups of 4
// warps that take every 4th k-block; the TMA-fed modes keep 8 idle warps.
template <int MODE> struct Warps {
    static constexpr int kProd = (MODE == 0 || MODE == 4 || MODE == 5) ? 16 : 8;   // FWD, DCA, DCB : others
    static constexpr int kGroups = kProd / 4;
    static constexpr int kEpi0 = 2 + kProd;                            // first epilogue warp
    static constexpr int kThreads = (kEpi0 + 4) * 32;
};
constexpr int kSegKb = 2;         // fp32: k-blocks per promoted accumulation segment
constexpr int kEpi = 128;         // epilogue threads (the last 4 warps)
constexpr int kSmemBudget = 227 * 1024 - 2048;

// DCA (bf16): dcoef = A^T . dY with M = spline columns (then SiLU rows), N =
// outputs, K = batch; the basis operand is written MN-major by the producers
// (rows = batch, 64-column atoms of spline columns), dY is read MN-major.
enum Mode { FWD = 0, DX = 2, GEMM = 3, DCA = 4, DCB = 5 };

template <int DT> struct Cfg;
template <> struct Cfg<KAN_BF16> {
    using T = __nv_bfloat16;
    static constexpr int BK = 64;          // K elements per 128-byte row
    static constexpr int ESZ = 2;
    static constexpr int SPLIT = 1;        // operand copies (hi only)
    static constexpr int UMMA_K = 16;
    static constexpr uint32_t FMT = 1;     // bf16
};
// fp32 operands: each value v (times a power-of-two scale) as two fp16
// parts, hi = fp16(v) and lo = fp16((v - hi) * 2^11); the tensor core sums
// hi*hi and, in a separate accumulator, hi*lo + lo*hi (scaled back by 2^-11).
template <> struct Cfg<KAN_F32> {
    using T = float;                       // x, y, dx element
    static constexpr int BK = 64;          // K elements per 128-byte operand row
    static constexpr int ESZ = 2;          // operand element size (fp16)
    static constexpr int SPLIT = 2;        // hi and lo fp16 parts
    static constexpr int UMMA_K = 16;
    static constexpr uint32_t FMT = 0;     // f16
};

// Scale of the lo part of a split operand, and its inverse.
constexpr float kLoScale = 2048.0f;
constexpr float kLoInv = 1.0f / 2048.0f;

// v -> (hi, lo) fp16 bit patterns with v ~= hi + lo * 2^-11 (about 22
// significant bits; v - hi is exact in fp32).
__device__ __forceinline__ void split_f16(float v, uint16_t& hi, uint16_t& lo)
{
    const __half h = __float2half_rn(v);
    const __half l = __float2half_rn((v - __half2float(h)) * kLoScale);
    hi = __half_as_ushort(h);
    lo = __half_as_ushort(l);
}

// Power-of-two scale s with m * s in [2^12, 2^13) (1 when m is 0, NaN or inf):
// scaled values stay well inside the fp16 range, and their lo parts too.
__host__ __device__ __forceinline__ float pow2_scale(float m)
{
    if (!(m > 0.0f) || !(m <= 3.0e38f)) return 1.0f;
    int ex;
    (void)frexpf(m, &ex);                  // m = f * 2^ex, f in [0.5, 1)
    const int e = min(100, max(-100, 13 - ex));
    return ldexpf(1.0f, e);
}

// Per-call operand scales of the fp32 path, from the absolute maxima that
// absmax_kernel leaves in the workspace: amax[0] coef, [1] w_base, [2] x, [3] dY.
//   x: silu(x) values (|silu(x)| <= |x|)
//   c: coef, and w_base times c / x (so that silu * w_base carries the same scale c)
//   d: dY
struct Scales {
    float c, x, d;
};
__device__ __forceinline__ Scales scales_of(const unsigned int* amax)
{
    Scales sc;
    sc.x = pow2_scale(__uint_as_float(amax[2]));
    sc.c = pow2_scale(fmaxf(__uint_as_float(amax[0]), __uint_as_float(amax[1]) / sc.x));
    sc.d = pow2_scale(__uint_as_float(amax[3]));
    return sc;
}

struct TcArgs {
    const void* x;             // [batch, in] operand dtype (FWD, DCA, DX epilogue)
    void* out;                 // FWD: y or partials; DCA: dcoef or partials; DX: dx; GEMM: fp32 [batch, in]
    float* out2;               // DCA: dw_base (non-partial); DX: Gb = dY.w_base (fp32 [batch,in]) or null
    unsigned int* status;
    int64_t batch, in, out_f;
    int G, nb;                 // nb: columns per input (G+k, or G+k+1 with an interleaved SiLU column)
    int nbs;                   // spline functions per input (G+k)
    int k;                     // spline degree
    int nb1;                   // univariate basis functions (G+k); 2-D: nb = nbs = nb1^2
    int64_t x_ld;              // row length of x and dx (2 * in for 2-D surfaces, whose units are input pairs)
    int twod;                  // 1: 2-D surfaces
    int ext;                   // 1: input i's SiLU column is column nbs of its group
    float lo, inv_h;
    int Kt;                    // in * nb
    int BN, stages;            // stages: pipeline depth of B (and of A when A also arrives by TMA)
    int stages_a;              // FWD, DCA: depth of the produced-A ring (its own barriers)
    int nkb_main;              // FWD: spline k-blocks; others: k-blocks over K
    int nkb_total;             // FWD: + SiLU k-blocks; others: = nkb_main
    int kb_per_split;
    int partial;
    int n_kt_tiles;            // DCA: M tiles over spline rows (separate SiLU tiles follow)
    int64_t part_ld;           // DCA partial row length
    int n_in_tile;             // DX: inputs per N tile
    int has_base;
    int x_vec;                 // 1: rows of x are 16-byte aligned (in * sizeof(T) % 16 == 0), vector loads allowed
    const unsigned int* amax;  // fp32: absolute maxima of the operands (scales_of)
    uint32_t nb_magic;         // ceil(2^32 / nb): c / nb == umulhi(c, nb_magic) for c < 2^32 / nb
    int fbox;                  // FWD: rows per B box
    int pair;                  // FWD, DCA (bf16): CTA pairs sharing cta_group::2 MMAs
    int m_tiles;               // FWD, DCA: M tiles holding work (a pair grid may have one more)
    int store_tma;             // FWD (unsplit), DCB: the output tile leaves through TMA stores of
                               // 128-row x 128-byte boxes (tensor map tA_hi over y or dcoef)
};

// (offset arithmetic on the shared array itself, not an integer round trip, so
// that accesses through the result stay shared-memory loads and stores rather
// than generic ones)
__device__ __forceinline__ uint8_t* align1024(uint8_t* p)
{
    const uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
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


__device__ __forceinline__ uint32_t pack_bf16(float a, float b)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}

// 16 bytes of dense A values (8 operand elements) at 16-byte chunk `chunk` of `row`.
template <int DT>
__device__ __forceinline__ void put_a_chunk(uint32_t a_hi, uint32_t a_lo, uint32_t row, uint32_t chunk, const float* v)
{
    const uint32_t off = sw128_chunk(row, chunk);
    if constexpr (DT == KAN_BF16) {
        st_shared_v4(a_hi + off, pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                     pack_bf16(v[6], v[7]));
    } else {
        uint32_t h[4], l[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            uint16_t h0, l0, h1, l1;
            split_f16(v[2 * e], h0, l0);
            split_f16(v[2 * e + 1], h1, l1);
            h[e] = (uint32_t)h0 | ((uint32_t)h1 << 16);
            l[e] = (uint32_t)l0 | ((uint32_t)l1 << 16);
        }
        st_shared_v4(a_hi + off, h[0], h[1], h[2], h[3]);
        st_shared_v4(a_lo + off, l[0], l[1], l[2], l[3]);
    }
}

// Floor of u (|u| < 2^22) without the conversion unit: adding 1.5*2^23 with
// round-down leaves floor(u) in the low mantissa bits.
__device__ __forceinline__ void floor_split(float u, int& s, float& f)
{
    const float r = __fadd_rd(u, 12582912.0f);
    f = r - 12582912.0f;
    s = __float_as_int(r) - 0x4B400000;
}

// Byte offset of element column c inside one 128-byte swizzled row (row & 7 = rx).
template <int ESZ>
__device__ __forceinline__ uint32_t sw_col(int c, uint32_t rx)
{
    const uint32_t cb = (uint32_t)c * ESZ;
    return ((((cb >> 4) ^ rx) & 7u) << 4) | (cb & 15u);
}

// The local weights of one input whose B_0 sits at column `base` of a
// 128-byte swizzled row: entry q (basis index s+q, q <= kq) goes to column
// base+s+q when mlo <= s+q < mhi (the caller's range keeps the column inside
// the row and the basis index inside 0..nb-1; an empty range stores nothing).
// One predicated store per entry keeps the warp convergent.  NW = 4 with
// kq = 3 for cubic splines; NW = KAN_MAX_NW with the runtime degree otherwise.
template <int DT, int NW>
__device__ __forceinline__ void scatter_win(uint32_t rb_hi, uint32_t rb_lo, uint32_t rx, int base, int s, int mlo,
                                            int mhi, const float (&w)[NW], int kq)
{
    constexpr int ESZ = 2;   // operand element size, both dtypes
    const uint32_t width = (uint32_t)(mhi - mlo);
    if constexpr (DT == KAN_BF16) {
        uint16_t h[NW];
#pragma unroll
        for (int q = 0; q < NW; q += 2) {
            const uint32_t p = pack_bf16(w[q], q + 1 < NW ? w[q + 1] : 0.0f);
            h[q] = (uint16_t)(p & 0xFFFFu);
            if (q + 1 < NW) h[q + 1] = (uint16_t)(p >> 16);
        }
#pragma unroll
        for (int q = 0; q < NW; ++q)
            if (q <= kq && (uint32_t)(s + q - mlo) < width) st_shared_u16(rb_hi + sw_col<ESZ>(base + s + q, rx), h[q]);
    } else {
#pragma unroll
        for (int q = 0; q < NW; ++q)
            if (q <= kq && (uint32_t)(s + q - mlo) < width) {
                const uint32_t off = sw_col<ESZ>(base + s + q, rx);
                uint16_t h, l;
                split_f16(w[q], h, l);
                st_shared_u16(rb_hi + off, h);
                st_shared_u16(rb_lo + off, l);
            }
    }
}

// The 16 products w1[r1] w2[r2] of one input pair's surface, whose B_{0,0}
// sits at column `base` of a 128-byte swizzled row: entry (r1, r2) goes to
// column base + (s1+r1) nb1 + s2 + r2 when both basis indices lie in 0..nb1-1
// and the column in [0, width).  Four runs of four consecutive columns, one
// scatter_win each; an empty range stores nothing.
template <int DT>
__device__ __forceinline__ void scatter_surface(uint32_t rb_hi, uint32_t rb_lo, uint32_t rx, int base, int s1, int s2,
                                                int nb1, int width, bool ok, const float (&w1)[4],
                                                const float (&w2)[4])
{
#pragma unroll
    for (int r1 = 0; r1 < 4; ++r1) {
        const int m1 = s1 + r1;
        const bool v = ok && m1 >= 0 && m1 < nb1;
        const int b1 = base + m1 * nb1;
        const int mlo = v ? max(0, -b1) : 0;
        const int mhi = v ? max(mlo, min(nb1, width - b1)) : 0;
        float wr[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) wr[q] = w1[r1] * w2[q];
        scatter_win<DT, 4>(rb_hi, rb_lo, rx, b1, s2, mlo, mhi, wr, 3);
    }
}

// Zero one 128-byte row of a produced tile (and of its lo copy for fp32).
// Store c writes 16-byte chunk c ^ rx (rx = row & 7), so the 8 consecutive
// rows of a quarter-warp hit 8 different chunks: no bank conflicts.
template <int DT>
__device__ __forceinline__ void zero_row(uint32_t rb_hi, uint32_t rb_lo, uint32_t rx)
{
#pragma unroll
    for (uint32_t c = 0; c < 8; ++c) {
        st_shared_zero16(rb_hi + 16u * (c ^ rx));
        if constexpr (DT == KAN_F32) st_shared_zero16(rb_lo + 16u * (c ^ rx));
    }
}

// A window of x[i0 .. i0 + MAXI) from one row of x, fetched in two steps so
// that the load latency can hide behind other work: issue() starts the loads
// into raw registers, values() shifts them into place (values at or past `in`
// read as 0; only the first n, n <= MAXI warp-uniform, are used by the caller).
// With vec, the row is read as 16-byte vectors starting at the aligned element
// below i0: a warp's lanes each read their own row, so every load instruction
// costs one L1 sector lookup per lane, and one vector replaces up to 8 (bf16)
// or 4 (fp32) scalar loads.  The window is shifted into place by the
// warp-uniform offset o = i0 mod (16 / sizeof(T)) through a small select /
// funnel-shift network (no dynamically indexed registers).
template <typename T, int MAXI>
struct XWindow {
    static constexpr int EPV = 16 / (int)sizeof(T);              // elements per 16-byte vector
    static constexpr int NV = (EPV - 1 + MAXI + EPV - 1) / EPV;  // vectors covering any window
    static constexpr int NR = 4 * NV + 4;
    uint32_t raw[NR];
    int o;                                                       // -1: raw already holds the values

    __device__ __forceinline__ void issue(const T* __restrict__ row, int i0, int n, int in, bool vec)
    {
        if (!vec) {
            o = -1;
#pragma unroll
            for (int k = 0; k < MAXI; ++k)
                raw[k] = __float_as_uint((k < n && i0 + k < in) ? to_f(row[i0 + k]) : 0.0f);
            return;
        }
        const int ia = i0 & ~(EPV - 1);
        o = i0 - ia;                                             // 0 .. EPV-1, uniform across the warp
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            uint4 q = make_uint4(0u, 0u, 0u, 0u);
            // (a vector holding none of the n values is skipped; in % EPV == 0)
            if (v * EPV < o + n && ia + v * EPV < in) q = *reinterpret_cast<const uint4*>(row + ia + v * EPV);
            raw[4 * v] = q.x;
            raw[4 * v + 1] = q.y;
            raw[4 * v + 2] = q.z;
            raw[4 * v + 3] = q.w;
        }
#pragma unroll
        for (int j = 4 * NV; j < NR; ++j) raw[j] = 0u;
    }

    __device__ __forceinline__ void values(float (&xv)[MAXI]) const
    {
        if (o < 0) {
#pragma unroll
            for (int k = 0; k < MAXI; ++k) xv[k] = __uint_as_float(raw[k]);
            return;
        }
        if constexpr (sizeof(T) == 4) {
            // shift by o words: two select levels
            uint32_t t[NR - 2];
#pragma unroll
            for (int j = 0; j < NR - 2; ++j) t[j] = (o & 1) ? raw[j + 1] : raw[j];
#pragma unroll
            for (int k = 0; k < MAXI; ++k) xv[k] = __uint_as_float((o & 2) ? t[k + 2] : t[k]);
        } else {
            // shift by o halves: o >> 1 words by two select levels, then o & 1 halves by a funnel shift
            const int r = o >> 1;
            uint32_t t[NR - 1], u[NR - 3];
#pragma unroll
            for (int j = 0; j < NR - 1; ++j) t[j] = (r & 1) ? raw[j + 1] : raw[j];
#pragma unroll
            for (int j = 0; j < NR - 3; ++j) u[j] = (r & 2) ? t[j + 2] : t[j];
            const uint32_t sh = (uint32_t)(o & 1) * 16u;
#pragma unroll
            for (int k = 0; k < MAXI; k += 2) {
                const uint32_t w = __funnelshift_r(u[k / 2], u[k / 2 + 1], sh);
                xv[k] = __uint_as_float(w << 16);
                if (k + 1 < MAXI) xv[k + 1] = __uint_as_float(w & 0xFFFF0000u);
            }
        }
    }
};

// One basis value at column `col` of a produced K-major row.
template <int DT>
__device__ __forceinline__ void put1(uint32_t rb_hi, uint32_t rb_lo, uint32_t rx, int col, float v)
{
    constexpr int ESZ = 2;
    if constexpr (DT == KAN_BF16) {
        st_shared_u16(rb_hi + sw_col<ESZ>(col, rx), __bfloat16_as_ushort(__float2bfloat16_rn(v)));
    } else {
        uint16_t h, l;
        split_f16(v, h, l);
        st_shared_u16(rb_hi + sw_col<ESZ>(col, rx), h);
        st_shared_u16(rb_lo + sw_col<ESZ>(col, rx), l);
    }
}

// The four local weights on the bounded coordinate t in [0,1) (see weights()).
__device__ __forceinline__ void weights_fma(float t, float (&w)[4])
{
    const float sm = 1.0f - t;
    const float t2 = t * t, s2 = sm * sm;
    w[0] = s2 * sm * (1.0f / 6.0f);
    w[1] = fmaf(t2, fmaf(t, 0.5f, -1.0f), 2.0f / 3.0f);
    w[2] = fmaf(s2, fmaf(sm, 0.5f, -1.0f), 2.0f / 3.0f);
    w[3] = t2 * t * (1.0f / 6.0f);
}

// 64-bit shifts whose amounts past 63 (including negative amounts read as
// unsigned) give 0, as the PTX shift instructions clamp them.
__device__ __forceinline__ uint64_t shl64(uint64_t v, int n)
{
    uint64_t r;
    asm("shl.b64 %0, %1, %2;" : "=l"(r) : "l"(v), "r"(n));
    return r;
}
__device__ __forceinline__ uint64_t shr64(uint64_t v, int n)
{
    uint64_t r;
    asm("shr.b64 %0, %1, %2;" : "=l"(r) : "l"(v), "r"(n));
    return r;
}

// One input's eight basis columns as a 16-byte chunk (G + 3 = 8, so that the
// columns of input i are exactly chunk i of the operand row): the four packed
// 16-bit weights P (w0 in the low bits) placed at columns s..s+3, the columns
// outside 0..7 dropped.  Branch-free for s in -3..7 (P = 0 stores zeros).
__device__ __forceinline__ uint4 chunk8(uint64_t P, int s)
{
    const int b = 16 * s;
    const uint64_t lo = shl64(P, b) | shr64(P, -b);
    const uint64_t hi = shl64(P, b - 64) | shr64(P, 64 - b);
    return make_uint4((uint32_t)lo, (uint32_t)(lo >> 32), (uint32_t)hi, (uint32_t)(hi >> 32));
}

// bf16 placement by byte permutes: the packed weights of an input sit in two
// words (w0, w1 | w2, w3), and each 32-bit word of the input's 16-byte chunk
// is one prmt of those two words under a selector that depends on the span s
// alone.  The selectors of span s are entry s + 3 (s in -3..7) of a 12-entry
// table in shared memory; entry 11 stores zeros (an input outside the
// extended knots).  A selector nibble with its top bit set copies the sign
// bit of the byte it names into the whole byte, and nibble 9 names the high
// byte of w0, whose sign is clear (the weights are nonnegative): a zero byte.
constexpr int kSelEntries = 12;

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// Selector of output word e (columns 2e, 2e+1) for table entry t.
__device__ __forceinline__ uint32_t sel_word(int t, int e)
{
    if (t >= kSelEntries - 1) return 0x9999u;
    const int s = t - 3;
    uint32_t sel = 0;
    for (int h = 0; h < 2; ++h) {
        const int q = 2 * e + h - s;   // weight index landing in column 2e + h
        const bool in = q >= 0 && q <= 3;
        const uint32_t lo = in ? 2u * q : 9u, hi = in ? 2u * q + 1u : 9u;
        sel |= (lo | (hi << 4)) << (8 * h);
    }
    return sel;
}

// bf16 weights of one input as two packed words and its selector-table entry
// (kSelEntries - 1 when the input is outside the extended knots or not real).
__device__ __forceinline__ void input_prmt(float x, bool act, float inv_h, float u0, float u_hi, uint32_t& entry,
                                           uint32_t& p0, uint32_t& p1)
{
    float u = fmaf(x, inv_h, u0);
    const bool ok = act && u >= -3.0f && u < u_hi;
    u = ok ? u : 0.0f;   // (keeps w0 nonnegative, whose sign byte the zero selectors read)
    int s;
    float f;
    floor_split(u, s, f);
    float w[4];
    weights_fma(u - f, w);
    p0 = pack_bf16(w[0], w[1]);
    p1 = pack_bf16(w[2], w[3]);
    entry = ok ? (uint32_t)(s + 3) : (uint32_t)(kSelEntries - 1);
}

// The packed weights of one input for chunk8 (bf16, or the fp16 hi / lo parts
// of the fp32 path): span s and, when the input is outside the extended knots
// (or not a real input), P = 0.
template <int DT>
__device__ __forceinline__ void input_chunk(float x, bool act, float inv_h, float u0, float u_hi, int& s,
                                            uint64_t& P_hi, uint64_t& P_lo)
{
    float u = fmaf(x, inv_h, u0);
    const bool ok = act && u >= -3.0f && u < u_hi;
    u = ok ? u : 0.0f;
    float f;
    floor_split(u, s, f);
    float w[4];
    weights_fma(u - f, w);
    if constexpr (DT == KAN_BF16) {
        const uint64_t p = (uint64_t)pack_bf16(w[0], w[1]) | ((uint64_t)pack_bf16(w[2], w[3]) << 32);
        P_hi = ok ? p : 0ull;
        P_lo = 0ull;
    } else {
        uint16_t h[4], l[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) split_f16(w[q], h[q], l[q]);
        const uint64_t ph = (uint64_t)h[0] | ((uint64_t)h[1] << 16) | ((uint64_t)h[2] << 32) | ((uint64_t)h[3] << 48);
        const uint64_t pl = (uint64_t)l[0] | ((uint64_t)l[1] << 16) | ((uint64_t)l[2] << 32) | ((uint64_t)l[3] << 48);
        P_hi = ok ? ph : 0ull;
        P_lo = ok ? pl : 0ull;
    }
}

// The eight x values of a window that starts on a 16-byte boundary, straight
// from the raw registers of an XWindow (no shift needed).
template <typename T, int MAXI>
__device__ __forceinline__ void aligned8(const XWindow<T, MAXI>& w, float (&xv)[8])
{
    if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            xv[2 * e] = __uint_as_float(w.raw[e] << 16);
            xv[2 * e + 1] = __uint_as_float(w.raw[e] & 0xFFFF0000u);
        }
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) xv[e] = __uint_as_float(w.raw[e]);
    }
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------
// PAIR: two CTAs (a cluster of 2 x 1, adjacent M tiles along x) share each MMA
// (tcgen05 cta_group::2, M = 256): each keeps its own 128 produced A rows and
// holds half of the B tile, so each SM streams half the B bytes.  The leader
// (rank 0) issues the MMAs; the follower's B loads complete on the leader's
// barriers and its producers arrive there remotely; commits reach both CTAs.
// KD: 3 for cubic splines (closed-form weights, 4 per input), 0 for any
// other degree (the runtime degree a.k; weights by the local triangle), 32
// for cubic 2-D surfaces (a unit is an input pair with nb1^2 columns; MAXI
// then counts x values, two per unit).
template <int MODE, int DT, int MAXI, bool PAIR = false, int KD = 3>
__global__ void __launch_bounds__(Warps<MODE>::kThreads, 1)
    tc_kernel(const __grid_constant__ CUtensorMap tA_hi, const __grid_constant__ CUtensorMap tA_lo,
              const __grid_constant__ CUtensorMap tB_hi, const __grid_constant__ CUtensorMap tB_lo,
              const __grid_constant__ CUtensorMap tB2_hi, const __grid_constant__ CUtensorMap tB2_lo,
              const TcArgs a)
{
    using C = Cfg<DT>;
    using T = typename C::T;
    constexpr int BK = C::BK;
    constexpr int EPB = 128 / C::ESZ;               // elements per 128-byte row
    constexpr bool F32 = DT == KAN_F32;
    constexpr bool PRODUCE = MODE == FWD || MODE == DCA || MODE == DCB;
    // DCB: the produced ring holds the B operand and the TMA ring the A operand
    constexpr bool SWAP = MODE == DCB;
    static_assert(!SWAP || (PAIR && DT == KAN_BF16 && KD == 3), "DCB: bf16 cubic 1-D, CTA pairs");
    constexpr bool TWOD = KD == 32;
    static_assert(!TWOD || PRODUCE, "2-D surfaces: produced-A kernels only");
    constexpr bool A_BY_TMA = MODE == DX || MODE == GEMM;
    static_assert(!PAIR || (PRODUCE && DT == KAN_BF16), "CTA pairs: bf16 forward and dcoef only");
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    constexpr bool A_MN = MODE == DCA || MODE == DCB;   // producer-written basis^T, or dY^T (DCB)
    constexpr bool A_SW32 = false;                   // (2-byte operands: the plain 128-byte swizzle)
    // B stored MN-major (dY for dcoef, coef / w_base for dx), for both dtypes
    // (the fp32 path's fp16 split copies keep the source layout)
    constexpr bool B_MN = MODE != FWD;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    __shared__ uint4 sel_tab[kSelEntries];   // bf16 chunk placement (see input_prmt)

    // Two rings of pipeline stages: B (TMA) with `stages` slots, and A with
    // `sa_n` slots.  A produced tile (FWD, DCA) is small next to a wide B tile,
    // so its ring is deeper: the producer groups fill A tiles several k-blocks
    // ahead of the MMA while the B ring only has to cover the TMA latency.  When
    // A arrives by TMA too (DX, GEMM) the two rings advance together (sa_n = stages).
    const int BN = a.BN, stages = a.stages;
    const int sa_n = PRODUCE ? a.stages_a : a.stages;
    // (a CTA of a pair holds half of each N = 256 MMA's B rows)
    // (DCB: the produced A ring carries the B operand, bn_cta columns, and the TMA ring dY^T, kBM rows)
    const uint32_t bn_cta = (uint32_t)(PAIR ? BN / 2 : BN) * 128;
    const uint32_t a_bytes = SWAP ? bn_cta : kBM * 128, b_bytes = SWAP ? kBM * 128 : bn_cta;
    const uint32_t a_stage = a_bytes * C::SPLIT, b_stage = b_bytes * C::SPLIT;
    const uint32_t sbase = smem_addr(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + sa_n * a_stage + stages * b_stage);
    // barrier block: full[S] empty[S] afull[SA] aempty[SA] seg_full[2] seg_empty[2] accum
    // (full[s]: B slot s (and, TMA-fed, A slot s) has landed; afull[s]: every
    // producer thread of a group has written its row of A slot s)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * stages + 2 * sa_n + 5);
    auto full = [&](int s) { return smem_addr(&bars[s]); };
    auto empty = [&](int s) { return smem_addr(&bars[stages + s]); };
    auto afull = [&](int s) { return smem_addr(&bars[2 * stages + s]); };
    auto aempty = [&](int s) { return smem_addr(&bars[2 * stages + sa_n + s]); };
    const int sb0 = 2 * stages + 2 * sa_n;
    auto seg_full = [&](int g) { return smem_addr(&bars[sb0 + g]); };
    auto seg_empty = [&](int g) { return smem_addr(&bars[sb0 + 2 + g]); };
    const uint32_t accum_bar = smem_addr(&bars[sb0 + 4]);
    auto A_hi = [&](int s) { return sbase + s * a_stage; };
    auto A_lo = [&](int s) { return sbase + s * a_stage + a_bytes; };
    auto B_hi = [&](int s) { return sbase + sa_n * a_stage + s * b_stage; };
    auto B_lo = [&](int s) { return sbase + sa_n * a_stage + s * b_stage + b_bytes; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kb_begin = blockIdx.z * a.kb_per_split;
    const int kb_end = min(a.nkb_total, kb_begin + a.kb_per_split);
    const int nk = kb_end - kb_begin;
    const int nseg = F32 ? (nk + kSegKb - 1) / kSegKb : 1;
    // TMEM columns: bf16 [acc]; fp32 [main0 | main1 | corr | total]
    const uint32_t tmem_cols =
        F32 ? 512u : (BN <= 32 ? 32u : (BN <= 64 ? 64u : (BN <= 128 ? 128u : (BN <= 256 ? 256u : 512u))));

    if (threadIdx.x == 0) {
        if constexpr (PRODUCE && !F32)
            for (int t = 0; t < kSelEntries; ++t)
                sel_tab[t] = make_uint4(sel_word(t, 0), sel_word(t, 1), sel_word(t, 2), sel_word(t, 3));
        for (int s = 0; s < stages; ++s) {
            mbar_init(full(s), 1);          // the TMA thread's expect-tx arrival
            mbar_init(empty(s), 1);         // the MMA thread's commit
        }
        for (int s = 0; s < sa_n; ++s) {
            mbar_init(afull(s), PAIR ? 256 : 128);   // every thread of one producer group (of both CTAs)
            mbar_init(aempty(s), 1);                 // the MMA thread's commit
        }
        mbar_init(seg_full(0), 1);
        mbar_init(seg_full(1), 1);
        mbar_init(seg_empty(0), kEpi);
        mbar_init(seg_empty(1), kEpi);
        mbar_init(accum_bar, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        if constexpr (PAIR) {
            tmem_alloc_pair(smem_addr(tmem_slot), tmem_cols);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_addr(tmem_slot), tmem_cols);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) cluster_sync();   // both CTAs' barriers exist before any remote arrival
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // fp32 with BN <= 64: B_hi and B_lo sit back to back in a stage, so one N = 2*BN
    // product per k-step gives hi*hi and hi*lo together ([main | hi*lo] segment
    // buffers, both promoted), and lo*hi is a second N = BN product into corr --
    // two tensor-core instructions per k-step instead of three, and A_hi read once
    const bool merged = F32 && BN <= 64;
    const uint32_t wseg = merged ? 2u * BN : (uint32_t)BN;   // columns of one segment buffer
    const uint32_t t_main0 = tmem, t_main1 = tmem + wseg, t_corr = tmem + 2u * wseg, t_total = t_corr + BN;

    // tile coordinates
    // (a pair grid runs the M tiles along x: its clusters are 2 x 1)
    const int tile_m = PAIR ? (int)blockIdx.x : (int)blockIdx.y;
    const int tile_n = PAIR ? (int)blockIdx.y : (int)blockIdx.x;
    const int64_t m0 = (int64_t)tile_m * kBM;         // FWD/DX/GEMM: batch rows; DCA: see below
    const int n0 = tile_n * BN;                       // FWD/DCA/GEMM: output columns

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0 && nk > 0) {
            prefetch_tmap(&tB_hi);
            if (A_BY_TMA) prefetch_tmap(&tA_hi);
            int dx_kt0 = 0;
            if (MODE == DX) {
                const int i0 = blockIdx.x * a.n_in_tile;
                // a TMA column start must be 16-byte aligned; a row start need not
                dx_kt0 = B_MN ? (i0 * a.nb) / (16 / C::ESZ) * (16 / C::ESZ) : i0 * a.nb;
            }
            int issued = 0;
            int s = 0;
            uint32_t ph = 0;
            for (int it = 0; it < nk; ++it, s = (s + 1 == stages) ? 0 : s + 1, ph ^= (s == 0)) {
                if (!mbar_wait(empty(s), ph ^ 1, a.status)) break;
                const int kb = kb_begin + it;
                if constexpr (PAIR) {
                    // this CTA's half of the B columns of each MMA (N = 256, then N = BN - 256),
                    // landing on the leader's full barrier (which expects both halves): local
                    // column lc < 128 is tile column 128 * rank + lc, the rest 256 + h2 * rank + lc - 128
                    const uint32_t fl = mapa_shared(full(s), 0);
                    if (leader) mbar_arrive_expect_tx(full(s), 2u * b_bytes);
                    const int h2 = (BN - 256) / 2;
                    auto tile_col = [&](int lc) { return lc < 128 ? 128 * (int)rank + lc : 256 + h2 * (int)rank + lc - 128; };
                    if (SWAP) {
                        // this CTA's 128 rows of dY^T: two 64-output atoms of BK batch rows
                        for (int c = 0; c < kBM / EPB; ++c)
                            tma_load_2d_pair(B_hi(s) + (uint32_t)c * BK * 128u, &tB_hi, fl, (int)m0 + c * EPB, kb * BK);
                    } else if (MODE == FWD) {
                        const bool spline = kb < a.nkb_main;   // (then the SiLU k-blocks, w_base)
                        for (int lc = 0; lc < BN / 2; lc += a.fbox)
                            tma_load_2d_pair(B_hi(s) + (uint32_t)lc * 128u,
                                             spline ? (const void*)&tB_hi : (const void*)&tB2_hi, fl,
                                             spline ? kb * BK : (kb - a.nkb_main) * BK, n0 + tile_col(lc));
                    } else {
                        for (int lc = 0; lc < BN / 2; lc += EPB)   // 64-column atoms
                            tma_load_2d_pair(B_hi(s) + (uint32_t)(lc / EPB) * BK * 128u, &tB_hi, fl, n0 + tile_col(lc),
                                             kb * BK);
                    }
                    ++issued;
                    continue;
                }
                const uint32_t bytes = (b_bytes + (A_BY_TMA ? a_bytes : 0u)) * C::SPLIT;
                mbar_arrive_expect_tx(full(s), bytes);
                if (MODE == FWD) {
                    // boxes of at most 128 rows (a.fbox): a wide tile is several of them
                    const bool spline = kb < a.nkb_main;
                    const int kc = spline ? kb * BK : (kb - a.nkb_main) * BK;
                    for (int h = 0; h * a.fbox < BN; ++h) {
                        const uint32_t off = (uint32_t)(h * a.fbox) * 128u;
                        tma_load_2d(B_hi(s) + off, spline ? (const void*)&tB_hi : (const void*)&tB2_hi, full(s), kc,
                                    n0 + h * a.fbox);
                        if (F32)
                            tma_load_2d(B_lo(s) + off, spline ? (const void*)&tB_lo : (const void*)&tB2_lo, full(s),
                                        kc, n0 + h * a.fbox);
                    }
                } else {
                    if (A_BY_TMA) {
                        tma_load_2d(A_hi(s), &tA_hi, full(s), kb * BK, (int)m0);
                        if (F32) tma_load_2d(A_lo(s), &tA_lo, full(s), kb * BK, (int)m0);
                    }
                    const int nbase = MODE == DX ? dx_kt0 : n0;
                    if (B_MN) {
                        for (int c = 0; c < BN / EPB; ++c) {
                            const uint32_t off = (uint32_t)c * BK * 128;
                            tma_load_2d(B_hi(s) + off, &tB_hi, full(s), nbase + c * EPB, kb * BK);
                            if (F32) tma_load_2d(B_lo(s) + off, &tB_lo, full(s), nbase + c * EPB, kb * BK);
                        }
                    } else {
                        tma_load_2d(B_hi(s), &tB_hi, full(s), kb * BK, nbase);
                        if (F32) tma_load_2d(B_lo(s), &tB_lo, full(s), kb * BK, nbase);
                    }
                }
                ++issued;
            }
            // every load issued lands before the CTA can exit (a pair's follower
            // sees that through its slots being released after the MMA used them)
            for (int it = max(0, issued - stages); it < issued; ++it) {
                if (PAIR && !leader) mbar_wait(empty(it % stages), (it / stages) & 1, a.status);
                else mbar_wait(full(it % stages), (it / stages) & 1, a.status);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issue ----------------
        if (lane == 0 && nk > 0 && leader) {
            // a 384- or 512-wide bf16 tile runs as an N=256 MMA plus an N=BN-256 MMA
            // into consecutive TMEM columns
            const int mma_n = BN > 256 ? 256 : BN;
            const uint32_t idesc = instr_desc(C::FMT, A_MN ? 1u : 0u, B_MN ? 1u : 0u, kBM, mma_n);
            const uint32_t idesc2 = instr_desc(C::FMT, A_MN ? 1u : 0u, B_MN ? 1u : 0u, kBM, BN > 256 ? BN - 256 : 16);
            const uint32_t idesc_w = instr_desc(C::FMT, A_MN ? 1u : 0u, B_MN ? 1u : 0u, kBM, merged ? 2 * BN : 16);
            // offset of B's columns 256..: 256 rows (K-major) or four 64-column atoms (MN-major);
            // a pair's CTA holds 128 of the first 256: 128 rows or two atoms
            const uint32_t b_half = B_MN ? (PAIR ? 2u : 4u) * BK * 128u : (PAIR ? 128u : 256u) * 128u;
            const uint32_t idesc_p = instr_desc(C::FMT, A_MN ? 1u : 0u, B_MN ? 1u : 0u, 2 * kBM, 256);
            const uint32_t idesc_p2 = instr_desc(C::FMT, A_MN ? 1u : 0u, B_MN ? 1u : 0u, 2 * kBM, BN > 256 ? BN - 256 : 16);
            const uint32_t b_lbo = B_MN ? (uint32_t)BK * 128u : 16u;
            const uint32_t b_step = B_MN ? (uint32_t)C::UMMA_K * 128u : 32u;
            const uint32_t a_lbo = A_MN ? (uint32_t)BK * 128u : 16u;
            const uint32_t a_step = A_MN ? (uint32_t)C::UMMA_K * 128u : 32u;
            const uint32_t a_sbo = A_SW32 ? 512u : 1024u;
            const uint32_t a_layout = A_SW32 ? 1u : 2u;
            bool ok = true;
            int s = 0, sa = 0;            // B and A ring positions (equal when A arrives by TMA)
            uint32_t ph = 0, pha = 0;
            for (int it = 0; it < nk; ++it) {
                if (PAIR) {
                    // (the follower's bytes and producer arrivals land here from the other CTA)
                    if (!mbar_wait_cluster(full(s), ph, a.status)) { ok = false; break; }
                    if (!mbar_wait_cluster(afull(sa), pha, a.status)) { ok = false; break; }
                } else {
                    if (!mbar_wait(full(s), ph, a.status)) { ok = false; break; }
                    if (PRODUCE && !mbar_wait(afull(sa), pha, a.status)) { ok = false; break; }
                }
                const int g = F32 ? it / kSegKb : 0;
                const bool seg_start = F32 && (it % kSegKb == 0);
                if (seg_start && g >= 2 && !mbar_wait(seg_empty(g & 1), ((g >> 1) - 1) & 1, a.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t t_main = (g & 1) ? t_main1 : t_main0;
                // descriptors of the stage's tiles; the k-steps advance the start address
                // field (addresses stay below 2^18, so the field never carries)
                const int sA = PRODUCE ? sa : s;
                const uint64_t ad0 = smem_desc(SWAP ? B_hi(s) : A_hi(sA), a_lbo, a_sbo, a_layout);
                const uint64_t bd0 = smem_desc_sw128(SWAP ? A_hi(sa) : B_hi(s), b_lbo, 1024);
                const uint64_t adl0 = F32 ? smem_desc(A_lo(sA), a_lbo, a_sbo, a_layout) : 0;
                const uint64_t bdl0 = F32 ? smem_desc_sw128(B_lo(s), b_lbo, 1024) : 0;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t ad = ad0 + (uint64_t)((ks * a_step) >> 4);
                    const uint64_t bd = bd0 + (uint64_t)((ks * b_step) >> 4);
                    if constexpr (PAIR) {
                        mma_f16_ss_pair(t_main0, ad, bd, idesc_p, (it > 0 || ks > 0) ? 1u : 0u);
                        if (BN > 256) {
                            const uint64_t bd2 = bd0 + (uint64_t)((b_half + ks * b_step) >> 4);
                            mma_f16_ss_pair(t_main0 + 256u, ad, bd2, idesc_p2, (it > 0 || ks > 0) ? 1u : 0u);
                        }
                    } else if constexpr (!F32) {
                        mma_bf16_ss(t_main0, ad, bd, idesc, (it > 0 || ks > 0) ? 1u : 0u);
                        if (BN > 256) {
                            const uint64_t bd2 = bd0 + (uint64_t)((b_half + ks * b_step) >> 4);
                            mma_bf16_ss(t_main0 + 256u, ad, bd2, idesc2, (it > 0 || ks > 0) ? 1u : 0u);
                        }
                    } else if (merged) {
                        const uint64_t adl = adl0 + (uint64_t)((ks * a_step) >> 4);
                        mma_bf16_ss(t_main, ad, bd, idesc_w, (!seg_start || ks > 0) ? 1u : 0u);
                        mma_bf16_ss(t_corr, adl, bd, idesc, (it > 0 || ks > 0) ? 1u : 0u);
                    } else {
                        const uint64_t adl = adl0 + (uint64_t)((ks * a_step) >> 4);
                        const uint64_t bdl = bdl0 + (uint64_t)((ks * b_step) >> 4);
                        mma_bf16_ss(t_corr, adl, bd, idesc, (it > 0 || ks > 0) ? 1u : 0u);
                        mma_bf16_ss(t_corr, ad, bdl, idesc, 1u);
                        mma_bf16_ss(t_main, ad, bd, idesc, (!seg_start || ks > 0) ? 1u : 0u);
                    }
                }
                if constexpr (PAIR) {
                    mma_commit_pair(empty(s));
                    mma_commit_pair(aempty(sa));
                } else {
                    mma_commit(empty(s));
                    if (PRODUCE) mma_commit(aempty(sa));
                }
                if (F32 && ((it + 1) % kSegKb == 0 || it + 1 == nk)) mma_commit(seg_full(g & 1));
                if (++s == stages) {
                    s = 0;
                    ph ^= 1;
                }
                if (PRODUCE && ++sa == sa_n) {
                    sa = 0;
                    pha ^= 1;
                }
            }
            if (ok) {
                if constexpr (PAIR) mma_commit_pair(accum_bar);
                else mma_commit(accum_bar);
            }
        }
    } else {
        // ---------------- A producers ----------------
        // Warps 2 .. kEpi0-1 in groups of four and, with bf16 operands, the
        // epilogue warps as one more group until the last k-block is filled
        // (they have nothing else to do before the accumulator is complete; the
        // fp32 epilogue promotes accumulator segments meanwhile).
        // Each thread fetches the x values of its next k-block into registers
        // right after it has handed over the current one, so the global-load
        // latency overlaps the other groups' k-blocks.
        const bool producer_warp = warp < Warps<MODE>::kEpi0;
        if constexpr (PRODUCE) if (producer_warp || !F32) {
            const int p = threadIdx.x - 64;
            const T* X = reinterpret_cast<const T*>(a.x);
            const float sx = F32 ? scales_of(a.amax).x : 1.0f;   // scale of the SiLU values (fp32)
            // Take A slot sa for a k-block: wait until the MMA has consumed its
            // previous contents.  Each thread then zeroes the one 128-byte row it
            // fills (16-byte stores, conflict-free under the swizzle) before it
            // writes the row's non-zero basis values: no zero traffic from L2.
            auto acquire = [&](int sa, uint32_t pha) -> bool { return mbar_wait(aempty(sa), pha ^ 1, a.status); };
            if constexpr (MODE == FWD) {
                // rows = batch m0..m0+127.  kGroups groups of 128 threads take
                // k-blocks in turn; a thread fills one whole row.  Per row and
                // k-block at most MAXI inputs have columns in the block.
                const uint32_t row = p & (kBM - 1);
                const int grp = p >> 7;                // warp-uniform
                const int64_t b = m0 + row;
                const bool row_ok = b < a.batch;
                const T* xrow = X + (row_ok ? b : 0) * a.x_ld;
                const float u0 = -a.lo * a.inv_h;      // u = x * inv_h + u0
                const float u_lo = -(float)a.k, u_hi = (float)(a.G + a.k);
                auto first_input = [&](int kb) { return (int)__umulhi((uint32_t)(kb * BK), a.nb_magic); };
                auto last_input = [&](int kb) {
                    const int c_end = min(kb * BK + BK, a.Kt);
                    return (int)__umulhi((uint32_t)(c_end - 1), a.nb_magic);
                };
                // the x window of the group's next k-block: loads issued one
                // iteration ahead, shifted into place when that k-block starts
                XWindow<T, MAXI> nxw;
                nxw.o = -1;
#pragma unroll
                for (int j = 0; j < XWindow<T, MAXI>::NR; ++j) nxw.raw[j] = 0u;
                auto fetch = [&](int kb) {
                    if (kb >= a.nkb_main || !row_ok) return;
                    const int i0 = first_input(kb);
                    // (2-D: a unit's two x values; MAXI counts values)
                    if constexpr (TWOD) nxw.issue(xrow, 2 * i0, 2 * (last_input(kb) - i0 + 1), (int)a.x_ld, a.x_vec != 0);
                    else nxw.issue(xrow, i0, last_input(kb) - i0 + 1, (int)a.in, a.x_vec != 0);
                };
                // At most sa_n groups: then a group's previous k-block is no older
                // than the previous use of the A slot it waits for, so neither the
                // aempty barrier nor any other can be two phases behind (a parity
                // wait on such a barrier would pass early).
                const int NG = min(Warps<MODE>::kGroups + (F32 ? 0 : 1), sa_n);
                if (grp < NG && grp < nk) fetch(kb_begin + grp);
                int uses = 0;                               // k-blocks this group has filled
                for (int it = grp; grp < NG && it < nk; it += NG, ++uses) {
                    float cur[MAXI];
                    const XWindow<T, MAXI> cur_raw = nxw;   // this k-block's window (the next one is fetched below)
                    const int kb = kb_begin + it;
                    const int s = it % sa_n;
                    const uint32_t ph = (it / sa_n) & 1;
                    // the slot is free (its previous use consumed)
                    if (!acquire(s, ph)) break;
                    const uint32_t ahi = A_hi(s), alo = A_lo(s);
                    const uint32_t rbase = row * 128u, rx = row & 7u;
                    // G + 3 = 8 (bf16 or fp32, no SiLU column, x rows 16-byte aligned): every
                    // input of the k-block owns one whole 16-byte chunk of the row, built in
                    // registers and stored at once (no zeroing pass, no scattered stores)
                    bool chunked = false;
                    if constexpr (MAXI == 9 && KD == 3) chunked = a.nb == 8 && !a.ext && a.x_vec && kb < a.nkb_main;
                    if (chunked) {
                        float xv[8];
                        aligned8(cur_raw, xv);
                        const int n8 = row_ok ? min(8, (int)a.in - first_input(kb)) : 0;
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            const uint32_t off = sw128_chunk(row, (uint32_t)c);
                            if constexpr (F32) {
                                int sidx;
                                uint64_t Ph, Pl;
                                input_chunk<DT>(xv[c], c < n8, a.inv_h, u0, u_hi, sidx, Ph, Pl);
                                const uint4 vh = chunk8(Ph, sidx), vl = chunk8(Pl, sidx);
                                st_shared_v4(ahi + off, vh.x, vh.y, vh.z, vh.w);
                                st_shared_v4(alo + off, vl.x, vl.y, vl.z, vl.w);
                            } else {
                                uint32_t t, p0, p1;
                                input_prmt(xv[c], c < n8, a.inv_h, u0, u_hi, t, p0, p1);
                                const uint4 sel = sel_tab[t];
                                st_shared_v4(ahi + off, prmt(p0, p1, sel.x), prmt(p0, p1, sel.y), prmt(p0, p1, sel.z),
                                             prmt(p0, p1, sel.w));
                            }
                        }
                    } else if (kb < a.nkb_main) {
                        cur_raw.values(cur);
                        zero_row<DT>(ahi + rbase, alo + rbase, rx);
                        if (row_ok) {
                            const int i0 = first_input(kb), n = last_input(kb) - i0 + 1;
                            const int cbase = i0 * a.nb - kb * BK;   // column of input i0's B_0 in this block
                            if constexpr (TWOD) {
                                // surfaces: MAXI / 2 pair slots, 16 products each
#pragma unroll
                                for (int k = 0; k < MAXI / 2; ++k) {
                                    const int base = cbase + k * a.nb;
                                    float uu = fmaf(cur[2 * k], a.inv_h, u0), uv = fmaf(cur[2 * k + 1], a.inv_h, u0);
                                    const bool ok = k < n && uu >= u_lo && uu < u_hi && uv >= u_lo && uv < u_hi;
                                    uu = ok ? uu : 0.0f;
                                    uv = ok ? uv : 0.0f;
                                    int s1, s2;
                                    float f1, f2, w1[4], w2[4];
                                    floor_split(uu, s1, f1);
                                    floor_split(uv, s2, f2);
                                    weights_fma(uu - f1, w1);
                                    weights_fma(uv - f2, w2);
                                    scatter_surface<DT>(ahi + rbase, alo + rbase, rx, base, s1, s2, a.nb1, BK, ok, w1,
                                                        w2);
                                }
                            } else {
                            // Straight-line over the MAXI input slots (the slots past n
                            // store nothing), so the inputs' arithmetic can interleave.
#pragma unroll
                            for (int k = 0; k < MAXI; ++k) {
                                const int base = cbase + k * a.nb;   // column of this input's B_0 (uniform)
                                const bool act = k < n;
                                if (F32 && a.ext) {   // input i0+k's SiLU column, when it falls in this block
                                    const int cs = base + a.nbs;
                                    if (act && (unsigned)cs < (unsigned)BK)
                                        put1<DT>(ahi + rbase, alo + rbase, rx, cs, silu_f(cur[k]) * sx);
                                }
                                float u = fmaf(cur[k], a.inv_h, u0);
                                // outside the extended knots, NaN, inf: no stores
                                const bool ok = act && u >= u_lo && u < u_hi;
                                u = ok ? u : 0.0f;
                                int sidx;
                                float f;
                                floor_split(u, sidx, f);
                                // basis indices whose columns lie in this block
                                const int mlo = ok ? max(0, -base) : 0;
                                const int mhi = ok ? min(a.nbs, BK - base) : 0;
                                if constexpr (KD == 3) {
                                    float w[4];
                                    weights_fma(u - f, w);
                                    scatter_win<DT, 4>(ahi + rbase, alo + rbase, rx, base, sidx, mlo, mhi, w, 3);
                                } else {
                                    float w[KAN_MAX_NW], dd[KAN_MAX_NW];
                                    weights_k<false>(u - f, a.k, 0.0f, w, dd);
                                    scatter_win<DT, KAN_MAX_NW>(ahi + rbase, alo + rbase, rx, base, sidx, mlo, mhi, w,
                                                                a.k);
                                }
                            }
                            }
                        }
                    } else {
                        // SiLU columns: BK consecutive inputs, dense (bf16 only: the fp32
                        // path carries silu(x) as one more column per input; in * 2 % 16 == 0
                        // with the base branch)
                        if constexpr (!F32) {
                            const int i0 = (kb - a.nkb_main) * BK;
#pragma unroll
                            for (int c = 0; c < 8; ++c) {
                                float v[8];
                                const int ic = i0 + c * 8;
                                if (row_ok && ic + 8 <= a.in) {
                                    const uint4 q4 = *reinterpret_cast<const uint4*>(xrow + ic);
                                    const uint32_t wd[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
                                    for (int e = 0; e < 8; ++e)
                                        v[e] = silu_f(__uint_as_float((e & 1) ? (wd[e / 2] & 0xFFFF0000u) : (wd[e / 2] << 16)));
                                } else {
#pragma unroll
                                    for (int e = 0; e < 8; ++e) v[e] = 0.0f;
                                }
                                put_a_chunk<DT>(ahi, alo, row, (uint32_t)c, v);
                            }
                        } else {
                            record_status(a.status, KAN_ERR_DEVICE_CHECK);   // never planned for fp32
                        }
                    }
                    fence_async_smem();
                    if (PAIR && !leader) mbar_arrive_cluster(mapa_shared(afull(s), 0));
                    else mbar_arrive(afull(s));
                    // the group's next window, issued only now: a release arrival waits for
                    // every earlier load of the thread, so loads in flight would delay it
                    if (it + NG < nk) fetch(kb + NG);
                }
                (void)uses;
            } else if constexpr (MODE == DCA) {
                // A tile, MN-major: batch rows b0..b0+BK-1 (K) by 128 columns (M) in
                // two 128-byte atoms of EPB = 64 columns, BK*128 bytes apart, 128-byte
                // swizzle (fp32: hi and lo tiles).  The columns are spline columns kt0.. (or, for a SiLU
                // tile, inputs i0..).  Groups of 128 threads take k-blocks in turn; a
                // thread fills one atom row: (batch row rb, atom).
                constexpr int NATOM = kBM / EPB;
                const int grp = p >> 7;                    // warp-uniform
                const int rb = p % BK;
                const int atom = (p / BK) % NATOM;         // warp-uniform
                const int mt = tile_m;
                // (the padding tile of a pair grid: all spline columns past Kt, so zero)
                const bool silu_tile = mt >= a.n_kt_tiles && mt < a.m_tiles;
                const int c_lo = (silu_tile ? (mt - a.n_kt_tiles) * kBM : mt * kBM) + atom * EPB;
                const int c_end = silu_tile ? min(c_lo + EPB, (int)a.in) : min(c_lo + EPB, a.Kt);
                const int i_first = (int)__umulhi((uint32_t)c_lo, a.nb_magic);
                const int n_inp = (!silu_tile && c_lo < c_end)
                                      ? (int)__umulhi((uint32_t)(c_end - 1), a.nb_magic) - i_first + 1 : 0;
                const float u0 = -a.lo * a.inv_h;
                const float u_lo = -(float)a.k, u_hi = (float)(a.G + a.k);
                XWindow<T, MAXI> nxw;   // (see the forward producer)
                nxw.o = -1;
#pragma unroll
                for (int j = 0; j < XWindow<T, MAXI>::NR; ++j) nxw.raw[j] = 0u;
                auto fetch = [&](int kb) {
                    const int64_t b = (int64_t)kb * BK + rb;
                    if (silu_tile || b >= a.batch) return;
                    if constexpr (TWOD) nxw.issue(X + b * a.x_ld, 2 * i_first, 2 * n_inp, (int)a.x_ld, a.x_vec != 0);
                    else nxw.issue(X + b * a.in, i_first, n_inp, (int)a.in, a.x_vec != 0);
                };
                // byte offset of column c (0..EPB-1) inside this thread's atom row
                auto col_off = [&](int c) -> uint32_t {
                    return sw128_byte((uint32_t)rb, (uint32_t)c * 2u) - (uint32_t)rb * 128u;
                };
                const int NG = min(Warps<MODE>::kGroups + (F32 ? 0 : 1), sa_n);   // see the forward producer
                if (grp < NG && grp < nk) fetch(kb_begin + grp);
                for (int it = grp; grp < NG && it < nk; it += NG) {
                    float cur[MAXI];
                    const XWindow<T, MAXI> cur_raw = nxw;   // this k-block's window (the next one is fetched below)
                    const int kb = kb_begin + it;
                    const int s = it % sa_n;
                    const uint32_t ph = (it / sa_n) & 1;
                    if (!acquire(s, ph)) break;
                    const int64_t b = (int64_t)kb * BK + rb;
                    const bool row_ok = b < a.batch;
                    const uint32_t roff = (uint32_t)atom * BK * 128u + (uint32_t)rb * 128u;
                    const uint32_t rb_hi = A_hi(s) + roff, rb_lo = A_lo(s) + roff;
                    // G + 3 = 8: each input of the atom row owns one whole 16-byte chunk (see
                    // the forward producer)
                    bool chunked = false;
                    if constexpr (MAXI == 9 && KD == 3) chunked = !silu_tile && a.nb == 8 && !a.ext && a.x_vec;
                    if (chunked) {
                        float xv[8];
                        aligned8(cur_raw, xv);
                        const int n8 = row_ok ? n_inp : 0;
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            const uint32_t off = (((uint32_t)c ^ ((uint32_t)rb & 7u)) << 4);
                            if constexpr (F32) {
                                int sidx;
                                uint64_t Ph, Pl;
                                input_chunk<DT>(xv[c], c < n8, a.inv_h, u0, u_hi, sidx, Ph, Pl);
                                const uint4 vh = chunk8(Ph, sidx), vl = chunk8(Pl, sidx);
                                st_shared_v4(rb_hi + off, vh.x, vh.y, vh.z, vh.w);
                                st_shared_v4(rb_lo + off, vl.x, vl.y, vl.z, vl.w);
                            } else {
                                uint32_t t, p0, p1;
                                input_prmt(xv[c], c < n8, a.inv_h, u0, u_hi, t, p0, p1);
                                const uint4 sel = sel_tab[t];
                                st_shared_v4(rb_hi + off, prmt(p0, p1, sel.x), prmt(p0, p1, sel.y),
                                             prmt(p0, p1, sel.z), prmt(p0, p1, sel.w));
                            }
                        }
                    } else if (!silu_tile) {
                        cur_raw.values(cur);
                        // this thread's atom row starts from zeros (rows past the batch stay zero)
                        zero_row<DT>(rb_hi, rb_lo, (uint32_t)rb & 7u);
                        if (row_ok && TWOD) {
                            const int cbase = i_first * a.nb - c_lo;
                            // surfaces: MAXI / 2 pair slots, 16 products each, in four runs of four columns
#pragma unroll
                            for (int k = 0; k < MAXI / 2; ++k) {
                                const int base = cbase + k * a.nb;
                                float uu = fmaf(cur[2 * k], a.inv_h, u0), uv = fmaf(cur[2 * k + 1], a.inv_h, u0);
                                const bool ok = k < n_inp && uu >= u_lo && uu < u_hi && uv >= u_lo && uv < u_hi;
                                uu = ok ? uu : 0.0f;
                                uv = ok ? uv : 0.0f;
                                int s1, s2;
                                float f1, f2, w1[4], w2[4];
                                floor_split(uu, s1, f1);
                                floor_split(uv, s2, f2);
                                weights_fma(uu - f1, w1);
                                weights_fma(uv - f2, w2);
#pragma unroll
                                for (int r1 = 0; r1 < 4; ++r1) {
                                    const int m1 = s1 + r1;
                                    const bool v = ok && m1 >= 0 && m1 < a.nb1;
                                    const int b1 = base + m1 * a.nb1;
                                    const int mlo = v ? max(0, -b1) : 0;
                                    const uint32_t width = v ? (uint32_t)(max(mlo, min(a.nb1, EPB - b1)) - mlo) : 0u;
#pragma unroll
                                    for (int q = 0; q < 4; ++q) {
                                        if ((uint32_t)(s2 + q - mlo) < width) {
                                            const uint32_t off = col_off(b1 + s2 + q);
                                            const float wv = w1[r1] * w2[q];
                                            if constexpr (F32) {
                                                uint16_t h, l;
                                                split_f16(wv, h, l);
                                                st_shared_u16(rb_hi + off, h);
                                                st_shared_u16(rb_lo + off, l);
                                            } else {
                                                st_shared_u16(rb_hi + off, __bfloat16_as_ushort(__float2bfloat16_rn(wv)));
                                            }
                                        }
                                    }
                                }
                            }
                        } else if (row_ok) {
                            const int cbase = i_first * a.nb - c_lo;
                            // straight-line over the MAXI input slots (see the forward producer)
#pragma unroll
                            for (int k = 0; k < MAXI; ++k) {
                                const bool act = k < n_inp;
                                if (F32 && a.ext) {   // input i_first+k's SiLU column, when it falls in this atom
                                    const int cs = cbase + k * a.nb + a.nbs;
                                    if (act && (unsigned)cs < (unsigned)EPB) {
                                        const float v = silu_f(cur[k]) * sx;
                                        const uint32_t off = col_off(cs);
                                        if constexpr (F32) {
                                            uint16_t h, l;
                                            split_f16(v, h, l);
                                            st_shared_u16(rb_hi + off, h);
                                            st_shared_u16(rb_lo + off, l);
                                        } else {
                                            st_shared_u16(rb_hi + off, __bfloat16_as_ushort(__float2bfloat16_rn(v)));
                                        }
                                    }
                                }
                                float u = fmaf(cur[k], a.inv_h, u0);
                                const bool ok = act && u >= u_lo && u < u_hi;   // NaN, inf fail
                                u = ok ? u : 0.0f;
                                int sidx;
                                float f;
                                floor_split(u, sidx, f);
                                constexpr int NW = KD == 3 ? 4 : KAN_MAX_NW;
                                float w[NW];
                                if constexpr (KD == 3) {
                                    weights_fma(u - f, w);
                                } else {
                                    float dd[KAN_MAX_NW];
                                    weights_k<false>(u - f, a.k, 0.0f, w, dd);
                                }
                                const int kq = KD == 3 ? 3 : a.k;
                                const int base = cbase + k * a.nb;
                                // basis indices whose columns lie in this atom (empty when !ok)
                                const int mlo = ok ? max(0, -base) : 0;
                                const uint32_t width = ok ? (uint32_t)(min(a.nbs, EPB - base) - mlo) : 0u;
                                const int col0 = base + sidx;
#pragma unroll
                                for (int q = 0; q < NW; ++q) {
                                    if (q <= kq && (uint32_t)(sidx + q - mlo) < width) {
                                        const uint32_t off = col_off(col0 + q);
                                        if constexpr (F32) {
                                            uint16_t h, l;
                                            split_f16(w[q], h, l);
                                            st_shared_u16(rb_hi + off, h);
                                            st_shared_u16(rb_lo + off, l);
                                        } else {
                                            st_shared_u16(rb_hi + off, __bfloat16_as_ushort(__float2bfloat16_rn(w[q])));
                                        }
                                    }
                                }
                            }
                        }
                    } else {
                        // SiLU columns: inputs c_lo..c_lo+EPB-1 of batch row b, dense
                        // (bf16 only: the fp32 path carries silu(x) as one more
                        // column per input; in * 2 % 16 == 0 with the base branch)
                        if constexpr (!F32) {
                            const T* xr = X + (row_ok ? b : 0) * a.in;
#pragma unroll
                            for (int c = 0; c < 8; ++c) {
                                float v[8];
                                const int ic = c_lo + c * 8;
                                if (row_ok && ic + 8 <= a.in) {
                                    const uint4 q4 = *reinterpret_cast<const uint4*>(xr + ic);
                                    const uint32_t wd[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
                                    for (int e = 0; e < 8; ++e)
                                        v[e] = silu_f(__uint_as_float((e & 1) ? (wd[e / 2] & 0xFFFF0000u) : (wd[e / 2] << 16)));
                                } else {
#pragma unroll
                                    for (int e = 0; e < 8; ++e) v[e] = 0.0f;
                                }
                                st_shared_v4(rb_hi + col_off(c * 8), pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]),
                                             pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
                            }
                        } else {
                            record_status(a.status, KAN_ERR_DEVICE_CHECK);   // never planned for fp32
                        }
                    }
                    fence_async_smem();
                    if (PAIR && !leader) mbar_arrive_cluster(mapa_shared(afull(s), 0));
                    else mbar_arrive(afull(s));
                    // the group's next window, issued only now: a release arrival waits for
                    // every earlier load of the thread, so loads in flight would delay it
                    if (it + NG < nk) fetch(kb + NG);
                }
            } else if constexpr (MODE == DCB) {
                // B tile, MN-major: batch rows b0..b0+BK-1 (K) by this CTA's bn_cta spline
                // columns (N) in atoms of EPB = 64 columns, BK*128 bytes apart; a pair's CTA
                // holds tile columns 128*rank + [0, 128) and 256 + h2*rank + [0, BN/2 - 128)
                // (the halves of each N = 256 MMA).  Groups of 128 threads take k-blocks in
                // turn; a thread fills the rows of batch row rb in atoms a0 and a0 + 2.
                const int NAT = (PAIR ? BN / 2 : BN) / EPB;
                const int grp = p >> 7;                    // warp-uniform
                const int rb = p % BK;
                const int a0 = (p / BK) & 1;               // warp-uniform
                const int h2 = (BN - 256) / 2;
                const float u0 = -a.lo * a.inv_h;
                const float u_lo = -3.0f, u_hi = (float)(a.G + 3);
                int c_lo[2], n_inp[2], i_first[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int at = a0 + 2 * e;
                    const int lc = at * EPB;
                    c_lo[e] = n0 + (lc < 128 ? 128 * (int)rank + lc : 256 + h2 * (int)rank + lc - 128);
                    const int c_end = min(c_lo[e] + EPB, a.Kt);
                    i_first[e] = (int)__umulhi((uint32_t)c_lo[e], a.nb_magic);
                    n_inp[e] = (at < NAT && c_lo[e] < c_end)
                                   ? (int)__umulhi((uint32_t)(c_end - 1), a.nb_magic) - i_first[e] + 1 : 0;
                }
                XWindow<T, MAXI> nxw[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    nxw[e].o = -1;
#pragma unroll
                    for (int j = 0; j < XWindow<T, MAXI>::NR; ++j) nxw[e].raw[j] = 0u;
                }
                auto fetch = [&](int kb) {
                    const int64_t b = (int64_t)kb * BK + rb;
                    if (b >= a.batch) return;
#pragma unroll
                    for (int e = 0; e < 2; ++e)
                        if (n_inp[e] > 0) nxw[e].issue(X + b * a.in, i_first[e], n_inp[e], (int)a.in, a.x_vec != 0);
                };
                const bool chunked = MAXI == 9 && a.nb == 8 && a.x_vec;
                const int NG = min(Warps<MODE>::kGroups + (F32 ? 0 : 1), sa_n);   // see the forward producer
                if (grp < NG && grp < nk) fetch(kb_begin + grp);
                for (int it = grp; grp < NG && it < nk; it += NG) {
                    const XWindow<T, MAXI> cur_raw[2] = {nxw[0], nxw[1]};
                    const int kb = kb_begin + it;
                    const int s = it % sa_n;
                    const uint32_t ph = (it / sa_n) & 1;
                    if (!acquire(s, ph)) break;
                    const int64_t b = (int64_t)kb * BK + rb;
                    const bool row_ok = b < a.batch;
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int at = a0 + 2 * e;
                        if (at >= NAT) continue;
                        const uint32_t rbase = A_hi(s) + (uint32_t)at * BK * 128u + (uint32_t)rb * 128u;
                        const int n8 = row_ok ? n_inp[e] : 0;
                        if (chunked) {
                            float xv[8];
                            aligned8(cur_raw[e], xv);
#pragma unroll
                            for (int c = 0; c < 8; ++c) {
                                uint32_t t, p0, p1;
                                input_prmt(xv[c], c < n8, a.inv_h, u0, u_hi, t, p0, p1);
                                const uint4 sel = sel_tab[t];
                                st_shared_v4(rbase + (((uint32_t)c ^ ((uint32_t)rb & 7u)) << 4), prmt(p0, p1, sel.x),
                                             prmt(p0, p1, sel.y), prmt(p0, p1, sel.z), prmt(p0, p1, sel.w));
                            }
                        } else {
                            float cur[MAXI];
                            cur_raw[e].values(cur);
                            zero_row<DT>(rbase, rbase, (uint32_t)rb & 7u);
                            const int cbase = i_first[e] * a.nb - c_lo[e];
#pragma unroll
                            for (int k = 0; k < MAXI; ++k) {
                                float u = fmaf(cur[k], a.inv_h, u0);
                                const bool ok = k < n8 && u >= u_lo && u < u_hi;   // NaN, inf fail
                                u = ok ? u : 0.0f;
                                int sidx;
                                float f, w[4];
                                floor_split(u, sidx, f);
                                weights_fma(u - f, w);
                                const int base = cbase + k * a.nb;
                                const int mlo = ok ? max(0, -base) : 0;
                                const uint32_t width = ok ? (uint32_t)(min(a.nbs, EPB - base) - mlo) : 0u;
#pragma unroll
                                for (int q = 0; q < 4; ++q)
                                    if ((uint32_t)(sidx + q - mlo) < width)
                                        st_shared_u16(rbase + (uint32_t)(sw128_byte((uint32_t)rb, (uint32_t)(base + sidx + q) * 2u) -
                                                                         (uint32_t)rb * 128u),
                                                      __bfloat16_as_ushort(__float2bfloat16_rn(w[q])));
                            }
                        }
                    }
                    fence_async_smem();
                    if (PAIR && !leader) mbar_arrive_cluster(mapa_shared(afull(s), 0));
                    else mbar_arrive(afull(s));
                    // the group's next window, issued only now: a release arrival waits for
                    // every earlier load of the thread, so loads in flight would delay it
                    if (it + NG < nk) fetch(kb + NG);
                }
            }
        }
        if (!producer_warp) {
        // ---------------- epilogue: the last 4 warps ----------------
        const int q = warp & 3;                       // TMEM lane quarter
        const uint32_t lane_off = (uint32_t)(32 * q) << 16;
        const uint32_t r = 32 * q + lane;             // tile row of this thread
        // DX: the x values (and dY.w_base terms) of the tile's inputs do not
        // depend on the MMA; fetch them in chunks of XC, the first one now.
        constexpr int XC = 16;
        uint32_t xa[XC], ga[XC];
        const int64_t dx_b = m0 + r;
        const int dx_i0 = MODE == DX ? blockIdx.x * a.n_in_tile : 0;
        const int dx_i1 = MODE == DX ? min((int)a.in, dx_i0 + a.n_in_tile) : 0;
        auto xfetch = [&](int i_start, uint32_t (&xv)[XC], uint32_t (&gv)[XC]) {
#pragma unroll
            for (int k = 0; k < XC; ++k) {
                const int i = i_start + k;
                const bool ok = dx_b < a.batch && i < dx_i1;
                xv[k] = ok ? __float_as_uint(to_f(reinterpret_cast<const T*>(a.x)[dx_b * a.in + i])) : 0u;
                gv[k] = (ok && a.has_base && !a.ext) ? __float_as_uint(a.out2[dx_b * a.in + i]) : 0u;
            }
        };
        if constexpr (MODE == DX) xfetch(dx_i0, xa, ga);
        bool go = nk > 0;
        if (F32 && go) {
            // promotion: total (+)= main[g & 1] for every segment
            for (int g = 0; g < nseg && go; ++g) {
                go = __all_sync(0xffffffffu, mbar_wait(seg_full(g & 1), (g >> 1) & 1, a.status));
                if (!go) break;
                tc_fence_after();
                const uint32_t tm = ((g & 1) ? t_main1 : t_main0) + lane_off;
                for (int c0 = 0; c0 < BN; c0 += 16) {
                    uint32_t v[16], w[16], t[16];
                    tmem_ld16(tm + c0, v);
                    if (merged) tmem_ld16(tm + BN + c0, w);   // the segment's hi*lo half
                    if (g > 0) tmem_ld16(t_total + lane_off + c0, t);
                    tmem_ld_wait();
                    if (merged) {   // (the hi*lo half carries the lo parts' 2^11)
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            v[e] = __float_as_uint(fmaf(__uint_as_float(w[e]), kLoInv, __uint_as_float(v[e])));
                    }
                    if (g > 0) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) + __uint_as_float(t[e]));
                    }
                    tmem_st16(t_total + lane_off + c0, v);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(seg_empty(g & 1));
            }
        }
        if (go) go = __all_sync(0xffffffffu, mbar_wait(accum_bar, 0, a.status));
        if (go) {
            tc_fence_after();
            // value of accumulator column c0..c0+15 of this thread's row (fp32:
            // total + corr * 2^-11, times `mul`, the inverse of the operand scales)
            // (columns c0..c0+31: both halves' loads in flight together; BN % 32 == 0)
            auto load32 = [&](int c0, float (&out)[32], float mul) {
                uint32_t v[2][16];
                if constexpr (F32) {
                    uint32_t w[2][16];
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        tmem_ld16(t_total + lane_off + c0 + 16 * j, v[j]);
                        tmem_ld16(t_corr + lane_off + c0 + 16 * j, w[j]);
                    }
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 2; ++j)
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            out[16 * j + e] = fmaf(__uint_as_float(w[j][e]), kLoInv, __uint_as_float(v[j][e])) * mul;
                } else {
                    (void)mul;
#pragma unroll
                    for (int j = 0; j < 2; ++j) tmem_ld16(t_main0 + lane_off + c0 + 16 * j, v[j]);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 2; ++j)
#pragma unroll
                        for (int e = 0; e < 16; ++e) out[16 * j + e] = __uint_as_float(v[j][e]);
                }
            };

            // The output tile through shared memory and TMA stores: boxes of 128 rows x
            // 128 bytes (32 fp32 or 64 bf16 columns) in a ring of 8 slots at the start of
            // the pipeline buffers (idle once the accumulator is complete), written in
            // the 128-byte swizzle (conflict-free), stored by one thread; whole lines
            // leave the SM instead of one 16-byte piece per row and store.
            auto store_tile = [&](bool bf16_out, float mul) {
                const int cpb = bf16_out ? 64 : 32;
                const bool issuer = warp == Warps<MODE>::kEpi0 && lane == 0;
                const int nslot = min(8, (int)((sa_n * a_stage + stages * b_stage) >> 14));   // 16 KB slots
                int box = 0;
                for (int c1 = 0; c1 < BN; c1 += cpb, ++box) {
                    const uint32_t slot = sbase + (uint32_t)(box % nslot) * 16384u;
                    if (box >= nslot) {   // the store that used this slot has read it
                        if (issuer) {
                            if (nslot == 8) bulk_wait_read<7>();
                            else bulk_wait_read<0>();
                        }
                        named_bar_sync(1, kEpi);
                    }
                    uint32_t wv[32];
                    if (bf16_out) {
                        float va[32], vb[32];
                        load32(c1, va, mul);
                        load32(c1 + 32, vb, mul);
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            wv[e] = pack_bf16(va[2 * e], va[2 * e + 1]);
                            wv[16 + e] = pack_bf16(vb[2 * e], vb[2 * e + 1]);
                        }
                    } else {
                        float v[32];
                        load32(c1, v, mul);
#pragma unroll
                        for (int e = 0; e < 32; ++e) wv[e] = __float_as_uint(v[e]);
                    }
                    const uint32_t rowp = slot + r * 128u;
#pragma unroll
                    for (uint32_t c = 0; c < 8; ++c)
                        st_shared_v4(rowp + ((c ^ (r & 7u)) << 4), wv[4 * c], wv[4 * c + 1], wv[4 * c + 2], wv[4 * c + 3]);
                    fence_async_smem();
                    named_bar_sync(1, kEpi);
                    if (issuer) {
                        // (a box wholly past the last row or column, e.g. a pair grid's padding
                        // tile, is not stored; its group stays empty)
                        if (m0 < (MODE == DCB ? a.out_f : a.batch) && n0 + c1 < (MODE == DCB ? (int64_t)a.Kt : a.out_f))
                            tma_store_2d(&tA_hi, slot, n0 + c1, (int)m0);
                        bulk_commit();
                    }
                }
                if (issuer) bulk_wait_read<0>();   // the boxes are read before the CTA may exit
            };

            if (MODE == FWD && a.store_tma && !a.partial) {
                store_tile(!F32, F32 ? 1.0f / scales_of(a.amax).c : 1.0f);
            } else if constexpr (MODE == FWD || MODE == GEMM) {
                const int64_t bo = m0 + r;
                const int64_t ncols = MODE == FWD ? a.out_f : a.in;
                const float mul = F32 ? 1.0f / scales_of(a.amax).c : 1.0f;   // y = acc / s_c
                for (int c1 = 0; c1 < BN; c1 += 32) {
                  float v32[32];
                  load32(c1, v32, mul);
#pragma unroll
                  for (int jh = 0; jh < 2; ++jh) {
                    const int c0 = c1 + 16 * jh;
                    float v[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[e] = v32[16 * jh + e];
                    if (bo >= a.batch) continue;
                    const int64_t j0 = n0 + c0;
                    if (MODE == GEMM || a.partial) {
                        float* dst = reinterpret_cast<float*>(a.out) +
                                     ((MODE == FWD ? (int64_t)blockIdx.z * a.batch : 0) + bo) * ncols + j0;
                        if (j0 + 16 <= ncols && (ncols & 3) == 0) {
#pragma unroll
                            for (int e = 0; e < 16; e += 4)
                                *reinterpret_cast<float4*>(dst + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                        } else {
#pragma unroll
                            for (int e = 0; e < 16; ++e)
                                if (j0 + e < ncols) dst[e] = v[e];
                        }
                    } else {
                        T* dst = reinterpret_cast<T*>(a.out) + bo * ncols + j0;
                        if constexpr (!F32) {
                            if (j0 + 16 <= ncols) {
                                uint32_t pk[8];
#pragma unroll
                                for (int e = 0; e < 8; ++e) pk[e] = pack_bf16(v[2 * e], v[2 * e + 1]);
                                *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                                *reinterpret_cast<uint4*>(dst + 8) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                            } else {
#pragma unroll
                                for (int e = 0; e < 16; ++e)
                                    if (j0 + e < ncols) dst[e] = __float2bfloat16_rn(v[e]);
                            }
                        } else {
                            if (j0 + 16 <= ncols && (ncols & 3) == 0) {
#pragma unroll
                                for (int e = 0; e < 16; e += 4)
                                    *reinterpret_cast<float4*>(dst + e) =
                                        make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                            } else {
    #pragma unroll
                            for (int e = 0; e < 16; ++e)
                                if (j0 + e < ncols) dst[e] = v[e];
                            }
                        }
                    }
                }
                }
            } else if constexpr (MODE == DCB) {
                // rows are outputs j, columns spline columns kt: dcoef[j, n0 + c]
                if (a.store_tma) {
                    store_tile(false, 1.0f);
                } else {
                    const int64_t j = m0 + r;
                    float* dst = reinterpret_cast<float*>(a.out) + (j < a.out_f ? j : 0) * a.Kt;
                    const bool vec = (a.Kt & 3) == 0;
                    for (int c1 = 0; c1 < BN; c1 += 32) {
                        float v32[32];
                        load32(c1, v32, 1.0f);
                        if (j >= a.out_f || !a.out) continue;
                        const int64_t k0 = n0 + c1;
                        if (vec && k0 + 32 <= a.Kt) {
#pragma unroll
                            for (int e = 0; e < 32; e += 4)
                                *reinterpret_cast<float4*>(dst + k0 + e) =
                                    make_float4(v32[e], v32[e + 1], v32[e + 2], v32[e + 3]);
                        } else {
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                if (k0 + e < a.Kt) dst[k0 + e] = v32[e];
                        }
                    }
                }
            } else if constexpr (MODE == DCA) {
                // rows are spline columns kt (or inputs of a SiLU tile); columns are outputs j
                const int mt = tile_m;
                const bool base_tile = mt >= a.n_kt_tiles;
                const int64_t rowg = base_tile ? (int64_t)(mt - a.n_kt_tiles) * kBM + r : (int64_t)mt * kBM + r;
                const bool row_ok = mt < a.m_tiles && (base_tile ? rowg < a.in : rowg < a.Kt);
                float* dst;
                int64_t ld;
                if (a.partial) {
                    dst = reinterpret_cast<float*>(a.out) + (int64_t)blockIdx.z * a.out_f * a.part_ld +
                          (base_tile ? a.Kt + rowg : rowg);
                    ld = a.part_ld;
                } else if (F32 && a.ext) {
                    // interleaved layout: column rowg is function m of input ii
                    const int ii = row_ok ? (int)__umulhi((uint32_t)rowg, a.nb_magic) : 0;
                    const int m = (int)rowg - ii * a.nb;
                    if (m < a.nbs) {
                        dst = a.out ? reinterpret_cast<float*>(a.out) + (int64_t)ii * a.nbs + m : nullptr;
                        ld = a.in * a.nbs;
                    } else {
                        dst = a.out2 ? a.out2 + ii : nullptr;
                        ld = a.in;
                    }
                } else {
                    float* basep = base_tile ? a.out2 : reinterpret_cast<float*>(a.out);
                    dst = basep ? basep + rowg : nullptr;   // an output the caller skipped
                    ld = base_tile ? a.in : a.Kt;
                }
                // fp32: dcoef = acc / s_d, dw_base (the SiLU rows) = acc / (s_d s_x)
                float mul = 1.0f;
                if constexpr (F32) {
                    const Scales sc = scales_of(a.amax);
                    mul = 1.0f / sc.d;
                    if (a.ext && row_ok) {
                        const int ii = (int)__umulhi((uint32_t)rowg, a.nb_magic);
                        if ((int)rowg - ii * a.nb >= a.nbs) mul /= sc.x;
                    }
                }
                for (int c1 = 0; c1 < BN; c1 += 32) {
                    float v32[32];
                    load32(c1, v32, mul);
                    if (!row_ok || !dst) continue;
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int64_t j = n0 + c1 + e;
                        if (j < a.out_f) dst[j * ld] = v32[e];
                    }
                }
            } else {
                // DX: Gm row -> shared staging (the pipeline buffers are free now),
                // then each input's 4 columns times B' (+ silu' * Gb).
                const int ldst = BN + 1;
                float* stage = reinterpret_cast<float*>(smem) + (size_t)(warp - Warps<MODE>::kEpi0) * 32 * ldst +
                               (size_t)lane * ldst;
                for (int c0 = 0; c0 < BN; c0 += 32) {
                    float v[32];
                    load32(c0, v, 1.0f);
#pragma unroll
                    for (int e = 0; e < 32; ++e) stage[c0 + e] = v[e];
                }
                // fp32: the staged columns are scaled by s_d s_c (spline) and s_d s_c / s_x (SiLU)
                float inv_dc = 1.0f, ext_mul = 1.0f;
                if constexpr (F32) {
                    const Scales sc = scales_of(a.amax);
                    inv_dc = 1.0f / (sc.d * sc.c);
                    ext_mul = inv_dc * sc.x;
                }
                if (dx_b < a.batch) {
                    const int kt_al = B_MN ? (dx_i0 * a.nb) / (16 / C::ESZ) * (16 / C::ESZ) : dx_i0 * a.nb;
                    T* dxr = reinterpret_cast<T*>(a.out) + dx_b * a.in;
                    for (int ic = dx_i0; ic < dx_i1; ic += XC) {
                        uint32_t xc[XC], gc[XC];
#pragma unroll
                        for (int k = 0; k < XC; ++k) {
                            xc[k] = xa[k];
                            gc[k] = ga[k];
                        }
                        if (ic + XC < dx_i1) xfetch(ic + XC, xa, ga);
#pragma unroll
                        for (int k = 0; k < XC; ++k) {
                            const int i = ic + k;
                            if (i >= dx_i1) break;
                            const float xv = __uint_as_float(xc[k]);
                            const Span sp = span_of(xv, a.lo, a.inv_h, a.G, a.k);
                            float acc = 0.0f;
                            if (sp.valid) {
                                constexpr int NW = KD == 3 ? 4 : KAN_MAX_NW;
                                float d[NW];
                                if constexpr (KD == 3) {
                                    dweights(sp.t, a.inv_h, d);
                                } else {
                                    float ww[KAN_MAX_NW];
                                    weights_k<true>(sp.t, a.k, a.inv_h, ww, d);
                                }
                                const int cb = i * a.nb - kt_al;
#pragma unroll
                                for (int qq = 0; qq < NW; ++qq) {
                                    const int m = sp.s + qq;
                                    if (qq <= a.k && m >= 0 && m < a.nbs) acc += stage[cb + m] * d[qq];
                                }
                            }
                            acc *= inv_dc;
                            if (F32 && a.ext) acc += dsilu_f(xv) * stage[i * a.nb - kt_al + a.nbs] * ext_mul;   // dY.w_base
                            else if (a.has_base) acc += dsilu_f(xv) * __uint_as_float(gc[k]);
                            dxr[i] = from_f<T>(acc);
                        }
                    }
                }
            }
        }
        }
    }

    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) cluster_sync();   // neither CTA leaves while the pair's MMAs or arrivals may touch it
    if (warp == 1) {
        tc_fence_after();
        if constexpr (PAIR) tmem_dealloc_pair(tmem, tmem_cols);
        else tmem_dealloc(tmem, tmem_cols);
    }
}

// ---------------------------------------------------------------------------
// dx, persistent: one CTA per SM walks the (batch tile, input group) tiles.
// Gm = dY . coef for a tile goes to one of two TMEM accumulators while the
// epilogue warps turn the previous tile's accumulator into dx, so the B'
// gather overlaps the next tile's MMA.  Warps: 0 TMA, 1 MMA issue + TMEM,
// 2-9 epilogue (two per TMEM lane quarter).  fp32 keeps the fp16 correction
// products in a second accumulator per buffer; the contraction over `out`
// is short enough (at most 32 k-blocks) that no promotion is needed.
// PAIR (bf16): clusters of two CTAs walk the same tiles of 256 batch rows; the
// leader issues cta_group::2 MMAs (M = 256) over both CTAs' dY rows and the two
// halves of the B columns, one held by each CTA, so each SM streams half of B;
// commits reach both CTAs and both CTAs' epilogues release the leader's
// accumulator buffers.
// ---------------------------------------------------------------------------
constexpr int kDxThreads = 320;   // warps: 0 TMA, 1 MMA, 2-9 epilogue

struct DxArgs {
    const void* x;
    void* dx;
    const float* gb;          // dY . w_base (fp32 [batch, in]) or null (none, or ext)
    unsigned int* status;
    int64_t batch, in, out;
    int G, nb;                // nb: columns per input of B (G+k, or G+k+1 with the SiLU column)
    int nbs;                  // spline functions per input (G+k)
    int k;                    // spline degree
    int nb1;                  // univariate basis functions (G+k); 2-D: nb = nbs = nb1^2
    int64_t x_ld;             // row length of x and dx
    int ext;                  // 1: column nbs of each input group is its dY.w_base column
    float lo, inv_h;
    int BN, stages, nkb;      // nkb: k-blocks over out
    int n_in_tile, n_tiles_n, n_tiles;
    int ld_stage;             // staging row stride in elements
    const unsigned int* amax; // fp32: absolute maxima of the operands (scales_of)
    int a_res;                // 1: short contraction (nkb k-blocks of dY fit beside the B ring): each
                              // CTA walks a contiguous run of tiles and keeps the dY rows resident
    int pair;                 // (informational) tiles of 2 x 128 batch rows run by CTA pairs
};

template <int DT, bool PAIR, int KD = 3>
__global__ void __launch_bounds__(kDxThreads, 1)
    dx_persistent_kernel(const __grid_constant__ CUtensorMap tA_hi, const __grid_constant__ CUtensorMap tA_lo,
                         const __grid_constant__ CUtensorMap tB_hi, const __grid_constant__ CUtensorMap tB_lo,
                         const DxArgs a)
{
    using C = Cfg<DT>;
    using T = typename C::T;
    constexpr int BK = C::BK;
    constexpr int EPB = 128 / C::ESZ;
    constexpr bool F32 = DT == KAN_F32;
    constexpr bool TWOD = KD == 32;      // units are input pairs with nb1^2 columns (cubic surfaces)
    constexpr bool B_MN = true;          // coef (its fp16 hi/lo copies for fp32) MN-major
    static_assert(!PAIR || DT == KAN_BF16, "CTA pairs: bf16 only");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    // the walk's units: clusters (PAIR) or CTAs
    const int unit = PAIR ? (int)blockIdx.x >> 1 : (int)blockIdx.x;
    const int n_units = PAIR ? (int)gridDim.x >> 1 : (int)gridDim.x;

    const int BN = a.BN, stages = a.stages;
    const bool ares = a.a_res != 0;
    // (a pair's CTA holds half of the B columns: BN / 2, whole 64-column atoms)
    const uint32_t a_bytes = kBM * 128, b_bytes = (uint32_t)(PAIR ? BN / 2 : BN) * 128;
    const uint32_t a_stage = a_bytes * C::SPLIT, b_stage = b_bytes * C::SPLIT;
    const uint32_t stage_bytes = a_stage + b_stage;
    const uint32_t sbase = smem_addr(smem);
    // Slots: a ring of `stages` (A, B) pairs; or, with the dY rows resident,
    // nkb A blocks followed by a ring of `stages` B slots.
    const uint32_t ring_bytes = ares ? a.nkb * a_stage + stages * b_stage : stages * stage_bytes;
    // staging of the accumulator rows: fp32 for fp32 operands, bf16 for bf16
    // operands (the dx it feeds is rounded to bf16 anyway)
    using ST = typename std::conditional<F32, float, __nv_bfloat16>::type;
    ST* staging = reinterpret_cast<ST*>(smem + ring_bytes);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + ring_bytes + 4 * 32 * a.ld_stage * (int)sizeof(ST));
    // full[S] empty[S] acc_full[2] acc_empty[2] a_full a_empty
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * stages + 6);
    volatile int* pair_ok = reinterpret_cast<volatile int*>(tmem_slot + 1);   // [4 quarters][2 warps]
    auto full = [&](int s) { return smem_addr(&bars[s]); };
    auto empty = [&](int s) { return smem_addr(&bars[stages + s]); };
    auto acc_full = [&](int b) { return smem_addr(&bars[2 * stages + b]); };
    auto acc_empty = [&](int b) { return smem_addr(&bars[2 * stages + 2 + b]); };
    const uint32_t a_full = smem_addr(&bars[2 * stages + 4]), a_empty = smem_addr(&bars[2 * stages + 5]);
    // A of ring slot s (or, resident, of k-block s)
    auto A_hi = [&](int s) { return sbase + s * (ares ? a_stage : stage_bytes); };
    auto A_lo = [&](int s) { return A_hi(s) + a_bytes; };
    auto B_hi = [&](int s) { return ares ? sbase + a.nkb * a_stage + s * b_stage : sbase + s * stage_bytes + a_stage; };
    auto B_lo = [&](int s) { return B_hi(s) + b_bytes; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t acc_cols = F32 ? 2u * BN : (uint32_t)BN;   // one buffer: [main | corr] or [acc]
    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        mbar_init(acc_full(0), 1);
        mbar_init(acc_full(1), 1);
        mbar_init(acc_empty(0), PAIR ? 16 : 8);   // every epilogue warp (of both CTAs)
        mbar_init(acc_empty(1), PAIR ? 16 : 8);
        mbar_init(a_full, 1);           // resident dY rows landed (TMA bytes)
        mbar_init(a_empty, 1);          // the MMA is done with them (commit)
        fence_barrier_init();
    }
    if (warp == 1) {
        if constexpr (PAIR) {
            tmem_alloc_pair(smem_addr(tmem_slot), 512);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_addr(tmem_slot), 512);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) cluster_sync();   // both CTAs' barriers exist before any remote arrival
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // tiles of this unit: t = unit + k * n_units, or (resident dY) the contiguous
    // run [t_begin, t_end); (batch tile, input group) = (t / n_tiles_n, t % n_tiles_n),
    // a batch tile being 128 rows, or 256 for a pair (rows 128 * rank.. of it here)
    const int t_begin = (int)((int64_t)a.n_tiles * unit / n_units);
    const int t_end = (int)((int64_t)a.n_tiles * (unit + 1) / n_units);
    const int my_tiles = ares ? t_end - t_begin : (a.n_tiles > unit ? (a.n_tiles - 1 - unit) / n_units + 1 : 0);
    auto tile_of = [&](int lt) { return ares ? t_begin + lt : unit + lt * n_units; };
    auto tile_coords = [&](int lt, int64_t& m0, int& i0) {
        const int t = tile_of(lt);
        m0 = (int64_t)(t / a.n_tiles_n) * (PAIR ? 2 * kBM : kBM) + (int64_t)kBM * rank;
        i0 = (t % a.n_tiles_n) * a.n_in_tile;
    };
    auto kt_start = [&](int i0) {
        return B_MN ? (i0 * a.nb) / (16 / C::ESZ) * (16 / C::ESZ) : i0 * a.nb;
    };

    if (warp == 0) {
        if (lane == 0 && my_tiles > 0) {
            prefetch_tmap(&tA_hi);
            prefetch_tmap(&tB_hi);
            int g = 0;   // k-block counter over all tiles
            int s = 0;   // its stage ring position and phase
            uint32_t ph = 0;
            bool ok = true;
            int a_loads = 0;          // resident dY loads issued
            int64_t a_m = -1;         // their batch tile
            for (int lt = 0; lt < my_tiles && ok; ++lt) {
                int64_t m0;
                int i0;
                tile_coords(lt, m0, i0);
                const int kt0 = kt_start(i0);
                if (ares && m0 != a_m) {
                    // new batch tile: once the MMA is done with the previous rows, load these
                    if (a_loads > 0 && !mbar_wait(a_empty, (a_loads - 1) & 1, a.status)) { ok = false; break; }
                    if constexpr (PAIR) {
                        // both CTAs' rows complete on the leader's barrier
                        const uint32_t af = mapa_shared(a_full, 0);
                        if (leader) mbar_arrive_expect_tx(a_full, 2u * a.nkb * a_stage);
                        for (int kb = 0; kb < a.nkb; ++kb) tma_load_2d_pair(A_hi(kb), &tA_hi, af, kb * BK, (int)m0);
                    } else {
                        mbar_arrive_expect_tx(a_full, a.nkb * a_stage);
                        for (int kb = 0; kb < a.nkb; ++kb) {
                            tma_load_2d(A_hi(kb), &tA_hi, a_full, kb * BK, (int)m0);
                            if (F32) tma_load_2d(A_lo(kb), &tA_lo, a_full, kb * BK, (int)m0);
                        }
                    }
                    ++a_loads;
                    a_m = m0;
                }
                for (int kb = 0; kb < a.nkb; ++kb, ++g, s = (s + 1 == stages) ? 0 : s + 1, ph ^= (s == 0)) {
                    if (!mbar_wait(empty(s), ph ^ 1, a.status)) { ok = false; break; }
                    if constexpr (PAIR) {
                        // this CTA's rows of dY and its half of the B columns (BN / 2 * rank..),
                        // landing on the leader's full barrier, which expects both CTAs' bytes
                        const uint32_t fl = mapa_shared(full(s), 0);
                        if (leader) mbar_arrive_expect_tx(full(s), 2u * (ares ? b_stage : stage_bytes));
                        if (!ares) tma_load_2d_pair(A_hi(s), &tA_hi, fl, kb * BK, (int)m0);
                        for (int c = 0; c < BN / 2 / EPB; ++c)
                            tma_load_2d_pair(B_hi(s) + (uint32_t)c * BK * 128, &tB_hi, fl,
                                             kt0 + BN / 2 * (int)rank + c * EPB, kb * BK);
                        continue;
                    }
                    mbar_arrive_expect_tx(full(s), ares ? b_stage : stage_bytes);
                    if (!ares) {
                        tma_load_2d(A_hi(s), &tA_hi, full(s), kb * BK, (int)m0);
                        if (F32) tma_load_2d(A_lo(s), &tA_lo, full(s), kb * BK, (int)m0);
                    }
                    if (B_MN) {
                        for (int c = 0; c < BN / EPB; ++c) {
                            tma_load_2d(B_hi(s) + (uint32_t)c * BK * 128, &tB_hi, full(s), kt0 + c * EPB, kb * BK);
                            if (F32)
                                tma_load_2d(B_lo(s) + (uint32_t)c * BK * 128, &tB_lo, full(s), kt0 + c * EPB, kb * BK);
                        }
                    } else {
                        tma_load_2d(B_hi(s), &tB_hi, full(s), kb * BK, kt0);
                        tma_load_2d(B_lo(s), &tB_lo, full(s), kb * BK, kt0);
                    }
                }
            }
            // every load issued lands before the CTA can exit (a pair's follower sees
            // that through the MMA's releases of its slots and of its resident rows)
            if (PAIR && !leader) {
                for (int q = max(0, g - stages); q < g; ++q) mbar_wait(empty(q % stages), (q / stages) & 1, a.status);
                if (a_loads > 0) mbar_wait(a_empty, (a_loads - 1) & 1, a.status);
            } else {
                for (int q = max(0, g - stages); q < g; ++q) mbar_wait(full(q % stages), (q / stages) & 1, a.status);
                if (a_loads > 0) mbar_wait(a_full, (a_loads - 1) & 1, a.status);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && my_tiles > 0 && leader) {
            const uint32_t idesc = instr_desc(C::FMT, 0, B_MN ? 1u : 0u, PAIR ? 2 * kBM : kBM, BN);
            // (a pair's waits see the other CTA's bytes and arrivals: cluster scope)
            auto wait = [&](uint32_t bar, uint32_t parity) {
                return PAIR ? mbar_wait_cluster(bar, parity, a.status) : mbar_wait(bar, parity, a.status);
            };
            auto commit = [&](uint32_t bar) {
                if constexpr (PAIR) mma_commit_pair(bar);
                else mma_commit(bar);
            };
            const uint32_t b_lbo = B_MN ? (uint32_t)BK * 128u : 16u;
            const uint32_t b_step = B_MN ? (uint32_t)C::UMMA_K * 128u : 32u;
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            int a_uses = 0;           // resident dY loads consumed
            int64_t a_m = -1;
            for (int lt = 0; lt < my_tiles && ok; ++lt) {
                const int buf = lt & 1;
                int64_t m0;
                int i0;
                tile_coords(lt, m0, i0);
                if (ares && m0 != a_m) {
                    if (!wait(a_full, a_uses & 1)) break;
                    ++a_uses;
                    a_m = m0;
                }
                if (lt >= 2 && !wait(acc_empty(buf), ((lt >> 1) - 1) & 1)) break;
                tc_fence_after();
                const uint32_t d_main = tmem + buf * acc_cols, d_corr = d_main + BN;
                for (int kb = 0; kb < a.nkb; ++kb, s = (s + 1 == stages) ? 0 : s + 1, ph ^= (s == 0)) {
                    if (!wait(full(s), ph)) { ok = false; break; }
                    tc_fence_after();
                    // k-steps advance the descriptors' start address field (no carry below 2^18)
                    const int sa = ares ? kb : s;
                    const uint64_t ad0 = smem_desc_sw128(A_hi(sa), 16, 1024);
                    const uint64_t bd0 = smem_desc_sw128(B_hi(s), b_lbo, 1024);
                    const uint64_t adl0 = F32 ? smem_desc_sw128(A_lo(sa), 16, 1024) : 0;
                    const uint64_t bdl0 = F32 ? smem_desc_sw128(B_lo(s), b_lbo, 1024) : 0;
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint64_t ad = ad0 + (uint64_t)(ks * 2);
                        const uint64_t bd = bd0 + (uint64_t)((ks * b_step) >> 4);
                        const uint32_t acc = (kb > 0 || ks > 0) ? 1u : 0u;
                        if constexpr (PAIR) {
                            mma_f16_ss_pair(d_main, ad, bd, idesc, acc);
                        } else if constexpr (!F32) {
                            mma_bf16_ss(d_main, ad, bd, idesc, acc);
                        } else {
                            const uint64_t adl = adl0 + (uint64_t)(ks * 2);
                            const uint64_t bdl = bdl0 + (uint64_t)((ks * b_step) >> 4);
                            mma_bf16_ss(d_corr, adl, bd, idesc, acc);
                            mma_bf16_ss(d_corr, ad, bdl, idesc, 1u);
                            mma_bf16_ss(d_main, ad, bd, idesc, acc);
                        }
                    }
                    commit(empty(s));
                }
                if (!ok) break;
                commit(acc_full(buf));
                // the last tile of this batch tile's run: release the resident rows
                // (a pair: after the last run too, which the follower waits for before it exits)
                if (ares) {
                    int64_t mn = -1;
                    int in_;
                    if (lt + 1 < my_tiles) tile_coords(lt + 1, mn, in_);
                    if (lt + 1 < my_tiles ? mn != m0 : PAIR) commit(a_empty);
                }
            }
        }
    } else {
        // ---------------- epilogue: warps 2-9 ----------------
        // Two warps per TMEM lane quarter (q = warp & 3; h = which of the two):
        // each stages half of the accumulator row's columns into the quarter's
        // shared staging rows, the pair meets at a named barrier, and then each
        // turns half of the tile's inputs into dx.
        const int q = warp & 3;
        const int h = (warp - 2) >> 2;
        const uint32_t lane_off = (uint32_t)(32 * q) << 16;
        const int r = 32 * q + lane;
        ST* srow = staging + (size_t)q * 32 * a.ld_stage + (size_t)lane * a.ld_stage;
        const int half_cols = BN / 2;                 // a multiple of 16
        constexpr int XC = 16;
        const bool x_vec = (a.in * (int64_t)sizeof(T)) % 16 == 0;
        const bool g_vec = (a.in * 4) % 16 == 0;
        // fp32: the staged columns carry s_d s_c (spline) and s_d s_c / s_x (SiLU)
        float inv_dc = 1.0f, ext_mul = 1.0f;
        if constexpr (F32) {
            const Scales sc = scales_of(a.amax);
            inv_dc = 1.0f / (sc.d * sc.c);
            ext_mul = inv_dc * sc.x;
        }
        // this lane's row and this warp's half of a tile's inputs
        auto tile_part = [&](int lt, int64_t& m0, int& i0, int64_t& b, int& ia, int& ib) {
            tile_coords(lt, m0, i0);
            b = m0 + r;
            const int i1 = min((int)a.in, i0 + a.n_in_tile);
            const int im = i0 + (i1 - i0 + 1) / 2;
            ia = h ? im : i0;
            ib = h ? i1 : im;
        };
        // x (and dY.w_base) windows: their loads are issued a chunk (across tiles,
        // a tile) ahead and shifted into place when the chunk starts
        XWindow<T, XC> xw;
        XWindow<float, XC> gw;
        xw.o = gw.o = -1;
#pragma unroll
        for (int j = 0; j < XWindow<T, XC>::NR; ++j) xw.raw[j] = 0u;
#pragma unroll
        for (int j = 0; j < XWindow<float, XC>::NR; ++j) gw.raw[j] = 0u;
        auto xfetch = [&](int64_t bq, int i_start, int i_end) {
            const int n = min(XC, i_end - i_start);
            if (bq < a.batch && n > 0) {
                xw.issue(reinterpret_cast<const T*>(a.x) + bq * a.in, i_start, n, (int)a.in, x_vec);
                if (a.gb) gw.issue(a.gb + bq * a.in, i_start, n, (int)a.in, g_vec);
            }
        };
        if (!TWOD && my_tiles > 0) {
            int64_t m0, b;
            int i0, ia, ib;
            tile_part(0, m0, i0, b, ia, ib);
            xfetch(b, ia, ib);
        }
        for (int lt = 0; lt < my_tiles; ++lt) {
            int64_t m0, b;
            int i0, ia, ib;
            tile_part(lt, m0, i0, b, ia, ib);
            const bool b_ok = b < a.batch;
            const int kt_al = kt_start(i0);
            // the next tile's first window, issued when this tile's last chunk starts
            // (exactly once per tile, also when this warp has no inputs in it)
            bool prefetched = false;
            auto prefetch_next = [&]() {
                prefetched = true;
                if (lt + 1 >= my_tiles) return;
                int64_t m0n, bn;
                int i0n, ian, ibn;
                tile_part(lt + 1, m0n, i0n, bn, ian, ibn);
                xfetch(bn, ian, ibn);
            };
            const int buf = lt & 1;
            // The pair agrees on the bounded wait's outcome (so that both leave the
            // loop together, never one of them waiting at a named barrier for the
            // other); the barrier also tells each that its partner has finished
            // reading the previous tile's staged row.
            const bool got = __all_sync(0xffffffffu, mbar_wait(acc_full(buf), (lt >> 1) & 1, a.status));
            if (lane == 0) pair_ok[2 * q + h] = got ? 1 : 0;
            named_bar_sync(1 + q, 64);
            if (!(pair_ok[2 * q] && pair_ok[2 * q + 1])) break;
            tc_fence_after();
            // stage this warp's half of the row: TMEM -> registers -> shared (16-byte
            // stores; the row stride is 16 bytes mod 128, so a warp's stores are conflict-free)
            const uint32_t t_main = tmem + buf * acc_cols + lane_off;
            // 64 columns per round: all of the round's TMEM loads are in flight
            // together and one wait covers them
            for (int c1 = h * half_cols; c1 < (h + 1) * half_cols; c1 += 64) {
                uint32_t v[4][16];
#pragma unroll
                for (int j = 0; j < 4; ++j) tmem_ld16(t_main + c1 + 16 * j, v[j]);
                if constexpr (F32) {   // main + corr * 2^-11
                    uint32_t w[4][16];
#pragma unroll
                    for (int j = 0; j < 4; ++j) tmem_ld16(t_main + BN + c1 + 16 * j, w[j]);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 4; ++j)
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            v[j][e] = __float_as_uint(fmaf(__uint_as_float(w[j][e]), kLoInv, __uint_as_float(v[j][e])));
                } else {
                    tmem_ld_wait();
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int c0 = c1 + 16 * j;
                    if constexpr (F32) {
#pragma unroll
                        for (int e = 0; e < 16; e += 4)
                            *reinterpret_cast<uint4*>(srow + c0 + e) =
                                make_uint4(v[j][e], v[j][e + 1], v[j][e + 2], v[j][e + 3]);
                    } else {
                        uint32_t pk[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            pk[e] = pack_bf16(__uint_as_float(v[j][2 * e]), __uint_as_float(v[j][2 * e + 1]));
                        *reinterpret_cast<uint4*>(srow + c0) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        *reinterpret_cast<uint4*>(srow + c0 + 8) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                    }
                }
            }
            // the accumulator buffer is free for the tile after next (one arrival per
            // warp, on the leader's barrier for a pair; relaxed: it publishes no data, and
            // a release would first wait for this warp's previous dx stores)
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (PAIR && !leader) mbar_arrive_cluster_relaxed(mapa_shared(acc_empty(buf), 0));
                else mbar_arrive_relaxed(acc_empty(buf));
            }
            // both halves of the row are staged
            named_bar_sync(1 + q, 64);
            if constexpr (TWOD) {
                // surfaces: for each pair (u, v) of this warp's units, the 16 staged columns
                // times B'(u) B(v) and B(u) B'(v); the pair's two dx values go out together
                if (b_ok) {
                    const T* xr = reinterpret_cast<const T*>(a.x) + b * a.x_ld;
                    T* dxr2 = reinterpret_cast<T*>(a.dx) + b * a.x_ld;
                    for (int i = ia; i < ib; ++i) {
                        const float xu = to_f(xr[2 * i]), xv = to_f(xr[2 * i + 1]);
                        const Span su = span_of(xu, a.lo, a.inv_h, a.G, 3), sv = span_of(xv, a.lo, a.inv_h, a.G, 3);
                        float du = 0.0f, dv = 0.0f;
                        if (su.valid && sv.valid) {
                            float wu[4], wv[4], gu[4], gv[4];
                            weights(su.t, wu);
                            weights(sv.t, wv);
                            dweights(su.t, a.inv_h, gu);
                            dweights(sv.t, a.inv_h, gv);
                            const int cb = i * a.nb - kt_al;
#pragma unroll
                            for (int r1 = 0; r1 < 4; ++r1) {
                                const int m1 = su.s + r1;
                                if (m1 < 0 || m1 >= a.nb1) continue;
#pragma unroll
                                for (int r2 = 0; r2 < 4; ++r2) {
                                    const int m2 = sv.s + r2;
                                    if (m2 < 0 || m2 >= a.nb1) continue;
                                    const float g = to_f(srow[cb + m1 * a.nb1 + m2]);
                                    du = fmaf(g, gu[r1] * wv[r2], du);
                                    dv = fmaf(g, wu[r1] * gv[r2], dv);
                                }
                            }
                            du *= inv_dc;
                            dv *= inv_dc;
                        }
                        if constexpr (F32) {
                            *reinterpret_cast<float2*>(dxr2 + 2 * i) = make_float2(du, dv);
                        } else {
                            *reinterpret_cast<uint32_t*>(dxr2 + 2 * i) = pack_bf16(du, dv);
                        }
                    }
                }
                __syncwarp();
                continue;
            }
            // dx of this warp's inputs [ia, ib): each lane computes its row's values
            // and parks them in slots slot_base + 0.. of its own staging row, which
            // lie below every column still to be read (input ia + k reads columns at
            // or above (ia + k) * nb - kt_al > slot_base + k - 1) and inside this
            // warp's own column range; the warp then writes its 32 x n block with
            // contiguous row segments instead of 32 scattered rows per store.
            const int slot_base = ia * a.nb - kt_al;
            const int n_mine = ib - ia;
            // Whole aligned chunks of XC inputs go out directly as 16-byte vectors (a
            // lane writes 32 or 64 contiguous bytes); otherwise bf16 values take the
            // block write below (2-byte scattered stores would cost an L2 sector
            // each), fp32 values are stored directly.
            const bool vec_out = n_mine % XC == 0 && (ia * (int)sizeof(T)) % 16 == 0 && (a.in * (int64_t)sizeof(T)) % 16 == 0;
            const bool block_out = !vec_out && !F32;
            T* dxr = reinterpret_cast<T*>(a.dx) + (b_ok ? b : 0) * a.in;
            if (b_ok) {
                for (int ic = ia; ic < ib; ic += XC) {
                    float xc[XC], gc[XC];
                    xw.values(xc);
                    gw.values(gc);
                    if (ic + XC < ib) xfetch(b, ic + XC, ib);
                    else prefetch_next();
                    const int nkc = min(XC, ib - ic);     // inputs in this chunk
                    auto dx_of = [&](int k) -> float {
                        const int i = ic + k;
                        const float xv = xc[k];
                        const Span sp = span_of(xv, a.lo, a.inv_h, a.G, a.k);
                        float acc = 0.0f;
                        if (sp.valid) {
                            constexpr int NW = KD == 3 ? 4 : KAN_MAX_NW;
                            float d[NW];
                            if constexpr (KD == 3) {
                                dweights(sp.t, a.inv_h, d);
                            } else {
                                float ww[KAN_MAX_NW];
                                weights_k<true>(sp.t, a.k, a.inv_h, ww, d);
                            }
                            const int cb = i * a.nb - kt_al;
#pragma unroll
                            for (int qq = 0; qq < NW; ++qq) {
                                const int m = sp.s + qq;
                                if (qq <= a.k && m >= 0 && m < a.nbs) acc += to_f(srow[cb + m]) * d[qq];
                            }
                        }
                        acc *= inv_dc;
                        if (F32 && a.ext) acc += dsilu_f(xv) * to_f(srow[i * a.nb - kt_al + a.nbs]) * ext_mul;   // dY.w_base, staged
                        else if (a.gb) acc += dsilu_f(xv) * gc[k];
                        return acc;
                    };
                    if (vec_out) {
                        float res[XC];
#pragma unroll
                        for (int k = 0; k < XC; ++k) res[k] = dx_of(k);
                        constexpr int VE = 16 / (int)sizeof(T);
#pragma unroll
                        for (int v0 = 0; v0 < XC; v0 += VE) {
                            if constexpr (F32) {
                                *reinterpret_cast<float4*>(dxr + ic + v0) =
                                    make_float4(res[v0], res[v0 + 1], res[v0 + 2], res[v0 + 3]);
                            } else {
                                *reinterpret_cast<uint4*>(dxr + ic + v0) =
                                    make_uint4(pack_bf16(res[v0], res[v0 + 1]), pack_bf16(res[v0 + 2], res[v0 + 3]),
                                               pack_bf16(res[v0 + 4], res[v0 + 5]), pack_bf16(res[v0 + 6], res[v0 + 7]));
                            }
                        }
                    } else {
#pragma unroll
                        for (int k = 0; k < XC; ++k) {
                            if (k >= nkc) break;
                            const float r = dx_of(k);
                            if (block_out) srow[slot_base + (ic - ia) + k] = from_f<ST>(r);
                            else dxr[ic + k] = from_f<T>(r);
                        }
                    }
                }
            }
            if (!prefetched) prefetch_next();
            __syncwarp();
            if (block_out && n_mine > 0) {
                // element e of the warp's block is (row e / n_mine, input e % n_mine); a
                // store instruction covers 32 consecutive elements
                const ST* sq = staging + (size_t)q * 32 * a.ld_stage;
                T* dxq = reinterpret_cast<T*>(a.dx) + (m0 + 32 * q) * a.in + ia;
                const int q32 = 32 / n_mine, r32 = 32 - q32 * n_mine;
                int rr = lane / n_mine, cc = lane - (lane / n_mine) * n_mine;
                for (int e = lane; e < 32 * n_mine; e += 32) {
                    if (m0 + 32 * q + rr < a.batch) dxq[(int64_t)rr * a.in + cc] = sq[(size_t)rr * a.ld_stage + slot_base + cc];
                    rr += q32;
                    cc += r32;
                    if (cc >= n_mine) {
                        cc -= n_mine;
                        ++rr;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) cluster_sync();   // neither CTA leaves while the pair's MMAs or arrivals may touch it
    if (warp == 1) {
        tc_fence_after();
        if constexpr (PAIR) tmem_dealloc_pair(tmem, 512);
        else tmem_dealloc(tmem, 512);
    }
}

// y[e] = sum over splits z (ascending) of part[z][e].
template <typename T>
__global__ void reduce_splits_kernel(const float* __restrict__ part, T* __restrict__ y, int64_t n, int splits)
{
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
        float acc = 0.f;
        for (int z = 0; z < splits; ++z) acc += part[(int64_t)z * n + e];
        y[e] = from_f<T>(acc);
    }
}

// dcoef[j, kt] and dw_base[j, i] from partials [splits][out][ld], split order.
// Columns: Kt spline columns then `in` SiLU columns, or (ext) input groups of
// nbx columns, the last of which is the input's SiLU column.  Rows j step
// by gridDim.y; column c / nbx through a multiply-high (nbx_magic = ceil(2^32 / nbx)).
__global__ void reduce_dcoef_kernel(const float* __restrict__ part, float* __restrict__ dcoef,
                                    float* __restrict__ dw_base, int64_t out, int64_t Kt, int64_t in, int64_t ld,
                                    int splits, int nbs, int nbx, int ext, uint32_t nbx_magic)
{
    const int64_t n = out * ld;
    for (int64_t j = blockIdx.y; j < out; j += gridDim.y)
    for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < (int)ld; c += gridDim.x * blockDim.x) {
        const int64_t e = j * ld + c;
        float acc = 0.f;
        for (int z = 0; z < splits; ++z) acc += part[(int64_t)z * n + e];
        if (ext) {
            const int i = (int)__umulhi((uint32_t)c, nbx_magic);
            const int m = c - i * nbx;
            if (m < nbs) {
                if (dcoef) dcoef[j * Kt + (int64_t)i * nbs + m] = acc;
            } else if (dw_base) {
                dw_base[j * in + i] = acc;
            }
        } else if (c < Kt) {
            if (dcoef) dcoef[j * Kt + c] = acc;
        } else if (dw_base) {
            dw_base[j * in + (c - Kt)] = acc;
        }
    }
}

// Absolute maxima of up to four fp32 arrays (amax[k] over src[k][0..n[k]),
// NaN ignored) as the bit patterns of non-negative floats, combined with
// atomicMax: the maximum does not depend on the order, so the result is
// deterministic.  amax must start at 0.  Arrays are 16-byte aligned and read
// as float4 (a scalar tail when n is not a multiple of 4).
struct AmaxArgs {
    const float* src[4];
    int64_t n[4];
};
__global__ void absmax_kernel(AmaxArgs a, unsigned int* __restrict__ amax)
{
    __shared__ unsigned int red[4];
    if (threadIdx.x < 4) red[threadIdx.x] = 0u;
    __syncthreads();
    const int64_t tid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x, nth = (int64_t)gridDim.x * blockDim.x;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        if (!a.src[k]) continue;
        float m = 0.0f;
        const int64_t n = a.n[k], n4 = n / 4;
        const float4* __restrict__ v4 = reinterpret_cast<const float4*>(a.src[k]);
        // four independent 16-byte loads in flight per thread and step
        for (int64_t e = tid; e < n4; e += 4 * nth) {
            float4 q[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) q[u] = e + u * nth < n4 ? v4[e + u * nth] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int u = 0; u < 4; ++u)
                m = fmaxf(m, fmaxf(fmaxf(fabsf(q[u].x), fabsf(q[u].y)), fmaxf(fabsf(q[u].z), fabsf(q[u].w))));
        }
        for (int64_t e = 4 * n4 + tid; e < n; e += nth) m = fmaxf(m, fabsf(a.src[k][e]));
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if ((threadIdx.x & 31) == 0) atomicMax(&red[k], __float_as_uint(m));
    }
    __syncthreads();
    if (threadIdx.x < 4 && a.src[threadIdx.x]) atomicMax(&amax[threadIdx.x], red[threadIdx.x]);
}

// fp16 hi/lo split of an fp32 array, times the dY scale (amax slot 3); four
// values per thread step (n % 4 == 0: n is batch * out with out % 8 == 0).
__global__ void split_f16_kernel(const float* __restrict__ src, uint16_t* __restrict__ hi, uint16_t* __restrict__ lo,
                                 int64_t n, const unsigned int* __restrict__ amax)
{
    const float sc = scales_of(amax).d;
    const int64_t n4 = n / 4;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n4; e += (int64_t)gridDim.x * blockDim.x) {
        const float4 q = reinterpret_cast<const float4*>(src)[e];
        uint16_t h[4], l[4];
        split_f16(q.x * sc, h[0], l[0]);
        split_f16(q.y * sc, h[1], l[1]);
        split_f16(q.z * sc, h[2], l[2]);
        split_f16(q.w * sc, h[3], l[3]);
        reinterpret_cast<uint2*>(hi)[e] = make_uint2(h[0] | ((uint32_t)h[1] << 16), h[2] | ((uint32_t)h[3] << 16));
        reinterpret_cast<uint2*>(lo)[e] = make_uint2(l[0] | ((uint32_t)l[1] << 16), l[2] | ((uint32_t)l[3] << 16));
    }
}

// The same split for a [rows, cols] matrix whose copy has rows of ld >= cols
// elements (ld % 8 == 0, so that the copy's rows are 16-byte aligned for TMA);
// the padding columns are written as 0.  One element per thread step.
__global__ void split_f16_rows_kernel(const float* __restrict__ src, uint16_t* __restrict__ hi,
                                      uint16_t* __restrict__ lo, int64_t rows, int64_t cols, int64_t ld,
                                      const unsigned int* __restrict__ amax)
{
    const float sc = scales_of(amax).d;
    const int64_t n = rows * ld;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = e / ld, c = e - r * ld;
        uint16_t h = 0, l = 0;
        if (c < cols) split_f16(src[r * cols + c] * sc, h, l);
        hi[e] = h;
        lo[e] = l;
    }
}

// fp16 hi/lo split of the coefficient matrix, row-major [out][in*nbx]:
// column i*nbx + m is coef[j, i, m] * s_c for m < nbs, and (with the SiLU
// branch, nbx = nbs + 1) w_base[j, i] * s_c / s_x for m == nbs.  Rows j step
// by gridDim.y, four consecutive columns per thread (8-byte writes; Kx % 4 == 0;
// the reads are consecutive apart from the SiLU columns); c / nbx through a
// multiply-high.
__global__ void split_coef_f16_kernel(const float* __restrict__ coef, const float* __restrict__ w_base, int64_t out,
                                      int64_t in, int nbs, int nbx, uint16_t* __restrict__ hi, uint16_t* __restrict__ lo,
                                      const unsigned int* __restrict__ amax, uint32_t nbx_magic)
{
    const Scales sc = scales_of(amax);
    const float sw = sc.c / sc.x;
    const int Kx = (int)(in * nbx);
    for (int64_t j = blockIdx.y; j < out; j += gridDim.y)
    for (int c4 = 4 * (blockIdx.x * blockDim.x + threadIdx.x); c4 < Kx; c4 += 4 * gridDim.x * blockDim.x) {
        const float* __restrict__ crow = coef + j * in * nbs;
        uint16_t h[4], l[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int c = c4 + e;
            const int i = (int)__umulhi((uint32_t)c, nbx_magic);
            const int m = c - i * nbx;
            const float v = m < nbs ? crow[i * nbs + m] * sc.c : w_base[j * in + i] * sw;
            split_f16(v, h[e], l[e]);
        }
        *reinterpret_cast<uint2*>(hi + j * Kx + c4) = make_uint2(h[0] | ((uint32_t)h[1] << 16), h[2] | ((uint32_t)h[3] << 16));
        *reinterpret_cast<uint2*>(lo + j * Kx + c4) = make_uint2(l[0] | ((uint32_t)l[1] << 16), l[2] | ((uint32_t)l[3] << 16));
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

// 2-D tiled map over a row-major [rows, cols] matrix of 2-byte operand
// elements (bf16, or the fp16 split copies of the fp32 path); box =
// [box_rows, box_cols] with box_cols * 2 = 128 bytes, 128-byte swizzle, zero
// fill out of bounds.
bool make_map_2d(CUtensorMap* m, const void* base, bool f16, int64_t rows, int64_t cols, int box_rows, int box_cols,
                 const char** detail, int64_t ld = -1)
{
    auto enc = get_encoder();
    if (!enc) {
        *detail = "cuTensorMapEncodeTiled is not available from the driver";
        return false;
    }
    const int esz = 2;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)((ld > 0 ? ld : cols) * esz)};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                     const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        *detail = "cuTensorMapEncodeTiled rejected a tensor map";
        return false;
    }
    return true;
}

inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t al256(size_t v) { return (v + 255) & ~(size_t)255; }

// Tensor map for the TMA-store epilogue: an output matrix [rows, cols] (fp32, or
// bf16 for y) in boxes of 128 rows x 128 bytes, 128-byte swizzle.  False (and
// the caller stores directly) when TMA cannot address it: a row length that is
// not a multiple of 16 bytes or a base that is not 16-byte aligned.
bool make_store_map(CUtensorMap* m, void* base, bool f32, int64_t rows, int64_t cols)
{
    const int esz = f32 ? 4 : 2;
    if (!base || (cols * esz) % 16 != 0 || (reinterpret_cast<uintptr_t>(base) & 15) != 0) return false;
    auto enc = get_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(cols * esz)};
    cuuint32_t box[2] = {(cuuint32_t)(128 / esz), (cuuint32_t)kBM};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Split-K count s (1..cap) minimising the estimated time
//   waves(s) / s * t_tile  +  waves(s) * t_wave  +  (s > 1 ? 2 (s + 1) t_part : 0),
// waves(s) = ceil(tiles * s / sms); t_tile: one whole output tile's contraction
// on one SM; t_wave: the fixed cost of a wave of CTAs (set-up, pipeline fill,
// epilogue); t_part: writing one set of fp32 partials for every tile (the
// reduction reads them back and launches once more, hence the factor 2).
// Splitting evens out a ragged last wave; it is taken only when the estimate
// improves on the unsplit one by at least 10%.
int pick_splits(int64_t tiles, int sms, int cap, double t_tile, double t_part)
{
    constexpr double t_wave = 4.0e-6;
    auto cost = [&](int s) {
        const double waves = (double)cdiv(tiles * s, sms);
        return waves / s * t_tile + waves * t_wave + (s > 1 ? 2.0 * (s + 1) * t_part : 0.0);
    };
    const double c1 = cost(1);
    int best = 1;
    double best_cost = c1;
    for (int s = 2; s <= std::max(1, cap); ++s) {
        const double c = cost(s);
        if (c < best_cost * (1.0 - 1e-9) && c < 0.9 * c1) {
            best_cost = c;
            best = s;
        }
    }
    return best;
}

// Seconds for one tile of BN output columns over K contraction elements on one
// SM (dense tensor rate; fp32 runs 3 fp16 products), and for writing one set of
// fp32 partials of `tiles` such tiles at HBM rate.
double tile_seconds(int BN, int64_t K, bool f32) { return 2.0 * kBM * BN * (double)K * (f32 ? 3 : 1) / 9.0e12; }
double partial_seconds(int64_t tiles, int BN) { return (double)tiles * kBM * BN * 4.0 / 5.0e12; }

// Tensor-core cycles per SM of one k-block (four K = 16 steps) of a CTA-pair tile
// BN columns wide, issued as instructions of N <= 256: about 161 cycles for
// N = 256 and about 97 for any N <= 128 (in between by interpolation).
double kblock_cycles(int BN)
{
    double c = 0.0;
    for (int n = BN; n > 0; n -= 256) {
        const int m = std::min(n, 256);
        c += m > 128 ? 97.0 + (m - 128) * 0.5 : 97.0;
    }
    return 4.0 * c;
}

// Tile width over n output columns.  An MN-major bf16 B operand is loaded in
// 64-column (128-byte) boxes, so its tile is at least one box wide.
int bn_for(int64_t n, bool f32, bool mn_major = false)
{
    const int cap = f32 ? 128 : 256;
    int bn = mn_major ? 64 : 32;
    while (bn < n && bn < cap) bn *= 2;
    return bn;
}

// bf16 tile width over `out` columns for the kernels whose basis operand is
// produced on chip: wider tiles reuse each produced A tile for more MMA
// work.  Among 256, 384 and 512 the one with the least padding wins, ties
// going to the wider; small `out` keeps the power-of-two width.
int wide_bn(int64_t out)
{
    if (out <= 256) return bn_for(out, false);
    int best = 256;
    int64_t best_pad = cdiv(out, 256) * 256;
    for (int bn : {384, 512}) {
        const int64_t pad = cdiv(out, bn) * bn;
        if (pad <= best_pad) {
            best_pad = pad;
            best = bn;
        }
    }
    return best;
}

int stages_for(int BN, bool f32)
{
    const int stage_bytes = (kBM * 128 + BN * 128) * (f32 ? 2 : 1);
    return std::min(8, (kSmemBudget - 1024 - 512) / stage_bytes);
}

// Kernels with a produced A tile: as many B slots as fit (at most 4) while
// the A ring keeps at least 4 slots (3 for fp32), then the rest of the shared
// memory to the A ring (at most 8 slots).  A wide B tile (64 KiB for 512
// bf16 columns) leaves room for only 2 B slots.
void stages_ab(int BN, bool f32, int& sb, int& sa)
{
    const int a_stage = kBM * 128 * (f32 ? 2 : 1), b_stage = BN * 128 * (f32 ? 2 : 1);
    const int avail = kSmemBudget - 1024 - 512;
    const int sa_min = f32 ? 3 : 4;
    sb = 4;
    while (sb > 2 && (avail - sb * b_stage) / a_stage < sa_min) --sb;
    sa = std::min(8, (avail - sb * b_stage) / a_stage);
}

// pipeline slots + 1024 alignment slack + 512 for the barrier block (2*stages + 2*stages_a + 5 mbarriers) and the TMEM slot
int smem_bytes(int BN, int stages, int stages_a, bool f32)
{
    return (stages * BN * 128 + stages_a * kBM * 128) * (f32 ? 2 : 1) + 1024 + 512;
}

// DCB (bf16 pairs): `stages` TMA slots of kBM dY^T rows and `stages_a` produced
// slots of bn_cta basis columns (64-column atoms of BK batch rows)
int smem_bytes_dcb(int bn_cta, int stages, int stages_a)
{
    return stages * kBM * 128 + stages_a * bn_cta * 128 + 1024 + 512;
}


// Workspace layout, shared by the size query and the launches.
struct Layout {
    size_t amax = 0;                             // fp32: 4 absolute maxima (the operand scales)
    size_t coef_hl = 0, dy_hl = 0;               // fp32: fp16 hi/lo copies of coef (w_base interleaved), dY
    size_t fwd_part = 0, dc_part = 0, gb = 0;   // split partials and dY.w_base
    size_t total = 0;
};

struct Plan {
    // row length of the fp16 copies of dY (fp32: out rounded up to 8, so that TMA can address them)
    int64_t ldo;
    // fp32 with the SiLU branch: interleaved coefficient copies (nbx = G+4
    // columns per input, Kx = in * nbx); otherwise nbx = G+k and Kx = Kt
    bool ext;
    int nbx;
    int64_t Kx;
    // forward
    int f_BN, f_stages, f_stages_a, f_n, f_m, f_splits, f_kps, f_nkb_main, f_nkb_total;
    bool f_pair, d_pair;   // bf16 tiles of 256, 384 or 512 columns: CTA pairs (f_my / d_my M tiles, even, along x)
    int f_my, d_my;
    // dcoef
    int d_BN, d_stages, d_stages_a, d_n, d_m, d_nkt, d_splits, d_kps, d_nkb;
    int64_t d_ld;
    // dcoef as DCB (outputs on M, spline columns on N), when that runs fewer tensor-core cycles
    bool dcb;
    int b_BN, b_stages, b_stages_a, b_m, b_my, b_n;
    // dx
    int x_BN, x_stages, x_n, x_m, x_nin, x_nkb;
    // dx, persistent kernel (used when p_ok)
    bool p_ok, p_ares, p_pair;
    int p_BN, p_stages, p_nin, p_ntn, p_tiles, p_ld, p_grid, p_smem;
    // dY . w_base
    int g_BN, g_stages, g_n, g_m;
    Layout fwd, bwd;
};

Plan make_plan(const Problem& p, int sms)
{
    Plan P{};
    const bool f32 = p.dtype == KAN_F32;
    const int BK = 64;   // K elements per 128-byte operand row (2-byte operands, both dtypes)
    P.ext = f32 && p.base;
    P.ldo = f32 ? (p.out + 7) / 8 * 8 : p.out;
    P.nbx = p.nb + (P.ext ? 1 : 0);
    P.Kx = p.in * P.nbx;
    const bool sep_silu = p.base && !P.ext;   // separate SiLU k-blocks / tiles / GEMM
    // forward: M = batch, N = out, K = spline (+ SiLU) columns
    P.f_BN = f32 ? bn_for(p.out, true) : wide_bn(p.out);
    P.f_pair = !f32 && P.f_BN >= 256;
    stages_ab(P.f_pair ? P.f_BN / 2 : P.f_BN, f32, P.f_stages, P.f_stages_a);
    P.f_n = (int)cdiv(p.out, P.f_BN);
    P.f_m = (int)cdiv(p.batch, kBM);
    P.f_my = P.f_pair ? (P.f_m + 1) / 2 * 2 : P.f_m;
    P.f_nkb_main = (int)cdiv(P.Kx, BK);
    P.f_nkb_total = P.f_nkb_main + (sep_silu ? (int)cdiv(p.in, BK) : 0);
    {
        const int64_t tiles = (int64_t)P.f_n * P.f_m;
        P.f_splits = pick_splits(tiles, sms, std::min(16, std::max(1, P.f_nkb_total / 8)),
                                 tile_seconds(P.f_BN, (int64_t)P.f_nkb_total * BK, f32), partial_seconds(tiles, P.f_BN));
    }
    P.f_kps = (int)cdiv(P.f_nkb_total, P.f_splits);
    P.f_splits = (int)cdiv(P.f_nkb_total, P.f_kps);
    // dcoef: M = spline columns (+ SiLU rows), N = out, K = batch
    P.d_BN = f32 ? bn_for(p.out, true, true) : std::max(64, wide_bn(p.out));
    P.d_pair = !f32 && P.d_BN >= 256;
    P.d_n = (int)cdiv(p.out, P.d_BN);
    P.d_nkt = (int)cdiv(P.Kx, kBM);
    P.d_m = P.d_nkt + (sep_silu ? (int)cdiv(p.in, kBM) : 0);
    P.d_my = P.d_pair ? (P.d_m + 1) / 2 * 2 : P.d_m;
    stages_ab(P.d_pair ? P.d_BN / 2 : P.d_BN, f32, P.d_stages, P.d_stages_a);
    P.d_nkb = (int)cdiv(p.batch, BK);
    {
        const int64_t tiles = (int64_t)P.d_n * P.d_m;
        P.d_splits = pick_splits(tiles, sms, std::min(16, std::max(1, P.d_nkb / 8)),
                                 tile_seconds(P.d_BN, (int64_t)P.d_nkb * BK, f32), partial_seconds(tiles, P.d_BN));
    }
    P.d_kps = (int)cdiv(std::max(1, P.d_nkb), P.d_splits);
    P.d_splits = (int)cdiv(std::max(1, P.d_nkb), P.d_kps);
    P.d_ld = P.ext ? P.Kx : p.Kt + (p.base ? p.in : 0);
    // DCB (bf16 cubic 1-D without the SiLU branch, G >= 5): M = outputs, N = spline columns in
    // 512-column pair tiles, K = batch, no split; taken when its waves of pair tiles
    // times the tile's k-block cycles undercut the DCA plan's by 5% (an `out` that
    // 512-column tiles would pad, e.g. 768 as two 384-column tiles)
    P.dcb = false;
    if (!f32 && !p.base && p.k == 3 && p.dims == 1 && P.nbx >= 8) {
        const int64_t slots = std::max(1, sms / 2);
        const int bBN = 512;
        const int b_m = (int)cdiv(p.out, kBM);
        const int b_my = (b_m + 1) / 2 * 2;
        const int b_n = (int)cdiv(p.Kt, bBN);
        const int64_t dca_ctas = (P.d_pair ? (int64_t)P.d_my : (int64_t)P.d_m) * P.d_n * P.d_splits;
        const double c_dca = (double)cdiv(P.d_pair ? dca_ctas / 2 : dca_ctas, P.d_pair ? slots : 2 * slots) *
                             (double)P.d_kps * kblock_cycles(P.d_BN);
        const double c_dcb = (double)cdiv((int64_t)b_my / 2 * b_n, slots) * (double)P.d_nkb * kblock_cycles(bBN);
        if (c_dcb < 0.95 * c_dca) {
            P.dcb = true;
            P.b_BN = bBN;
            P.b_m = b_m;
            P.b_my = b_my;
            P.b_n = b_n;
            P.b_stages = 3;
            P.b_stages_a = std::min(8, (kSmemBudget - 1024 - 512 - P.b_stages * kBM * 128) / (bBN / 2 * 128));
        }
    }
    // dx: M = batch, N = whole inputs' columns, K = out; coef (or its fp16
    // copies) is read MN-major and a tile's first column is rounded down to 16 bytes
    P.x_BN = f32 ? 128 : 256;
    P.x_stages = stages_for(P.x_BN, f32);
    const int maxoff = (P.nbx % 8 == 0) ? 0 : 7;
    P.x_nin = std::max(1, (P.x_BN - maxoff) / P.nbx);
    P.x_n = (int)cdiv(p.in, P.x_nin);
    P.x_m = (int)cdiv(p.batch, kBM);
    P.x_nkb = (int)cdiv(p.out, BK);
    // dx, persistent: BN 256 (bf16) / 128 (fp32), double-buffered TMEM, staged epilogue;
    // fp32 accumulates over `out` without promotion, so at most 1024 terms
    {
        P.p_BN = f32 ? 128 : 256;
        // bf16 with at least 4 batch tiles: CTA pairs over 256-row tiles, each CTA
        // holding half of the B columns
        P.p_pair = !f32 && P.x_m >= 4;
        P.p_nin = (P.p_BN - maxoff) / P.nbx;
        P.p_ld = f32 ? P.p_BN + 4 : P.p_BN + 8;          // row stride = 16 bytes mod 128
        const int staging = 4 * 32 * P.p_ld * (f32 ? 4 : 2);
        const int a_stage = kBM * 128 * (f32 ? 2 : 1), b_stage = (P.p_pair ? P.p_BN / 2 : P.p_BN) * 128 * (f32 ? 2 : 1);
        const int stage_bytes = a_stage + b_stage;
        const int avail = 232448 - 1024 - 256 - staging;
        P.p_stages = std::min(6, avail / stage_bytes);
        // A short contraction (at most 2 k-blocks over `out`): keep the dY rows
        // resident per batch tile when that leaves more B slots than the (A, B) ring
        P.p_ares = false;
        if (P.x_nkb <= 2) {
            const int sb = std::min(6, (avail - P.x_nkb * a_stage) / b_stage);
            if (sb >= 3 && sb > P.p_stages) {
                P.p_ares = true;
                P.p_stages = sb;
            }
        }
        P.p_ok = P.p_nin >= 1 && P.p_stages >= 2 && (!f32 || p.out <= 1024);
        if (P.p_ok) {
            P.p_ntn = (int)cdiv(p.in, P.p_nin);
            P.p_tiles = P.p_ntn * (P.p_pair ? (P.x_m + 1) / 2 : P.x_m);
            P.p_grid = P.p_pair ? std::max(2, std::min(2 * P.p_tiles, sms) / 2 * 2) : std::max(1, std::min(P.p_tiles, sms));
            P.p_smem = (P.p_ares ? P.x_nkb * a_stage + P.p_stages * b_stage : P.p_stages * stage_bytes) + staging +
                       1024 + 256;
        }
    }
    // dY . w_base (bf16 with the SiLU branch): M = batch, N = in, K = out
    P.g_BN = bn_for(p.in, f32, true);
    P.g_stages = stages_for(P.g_BN, f32);
    P.g_n = (int)cdiv(p.in, P.g_BN);
    P.g_m = P.x_m;

    // workspace, forward (fp32: maxima, fp16 hi/lo copy of coef with w_base interleaved)
    size_t o = 0;
    if (f32) {
        P.fwd.amax = o;
        o += 256;
        P.fwd.coef_hl = o;
        o += 2 * al256((size_t)p.out * P.Kx * 2);
    }
    if (P.f_splits > 1) {
        P.fwd.fwd_part = o;
        o += al256((size_t)P.f_splits * p.batch * p.out * 4);
    }
    P.fwd.total = o;
    // workspace, backward (fp32: maxima, fp16 hi/lo copies of dY and of coef)
    o = 0;
    if (f32) {
        P.bwd.amax = o;
        o += 256;
        P.bwd.coef_hl = o;
        o += 2 * al256((size_t)p.out * P.Kx * 2);
        P.bwd.dy_hl = o;
        o += 2 * al256((size_t)p.batch * P.ldo * 2);
    }
    if (P.d_splits > 1 && !P.dcb) {
        P.bwd.dc_part = o;
        o += al256((size_t)P.d_splits * p.out * P.d_ld * 4);
    }
    if (sep_silu) {
        P.bwd.gb = o;
        o += al256((size_t)p.batch * p.in * 4);
    }
    P.bwd.total = o;
    return P;
}

inline int grid_for(int64_t n) { return (int)std::min<int64_t>(std::max<int64_t>(1, (n + 255) / 256), 148 * 8); }

template <int MODE, int DT, int MAXI, bool PAIR, int KD>
cudaError_t launch(dim3 grid, int BN, int stages, const CUtensorMap* maps, const TcArgs& args, cudaStream_t st)
{
    constexpr bool produce = MODE == FWD || MODE == DCA || MODE == DCB;
    const int stages_a = produce ? args.stages_a : stages;
    // the MN-major bf16 B operand arrives in whole 128-byte boxes: BN must be a multiple of 64
    if (MODE != FWD && BN % 64 != 0) return cudaErrorInvalidConfiguration;
    if (BN % 16 != 0 || BN < 16 || BN > (produce ? 512 : 256) || (BN > 256 && BN % 128 != 0) ||
        (DT == KAN_F32 && BN > 128) || stages < 2 || stages_a < 2 || stages + stages_a > 24 ||
        (!produce && stages_a != stages))
        return cudaErrorInvalidConfiguration;
    // a pair's CTAs hold half of each N = 256 MMA's B rows; the grid is (M tiles, N tiles, splits)
    if (PAIR && (BN < 256 || BN % 128 != 0 || (MODE == FWD && args.fbox != (BN == 384 ? 64 : 128)) ||
                 grid.x % 2 != 0))
        return cudaErrorInvalidConfiguration;
    // (DCB: the TMA ring holds kBM-row dY^T tiles and the produced ring the B columns)
    const int smem = MODE == DCB ? smem_bytes_dcb(BN / 2, stages, stages_a)
                                 : smem_bytes(PAIR ? BN / 2 : BN, stages, stages_a, DT == KAN_F32);
    if (smem > kSmemBudget) return cudaErrorInvalidConfiguration;
    static int configured = 0;   // per instantiation; the attribute is per function
    if (configured < smem) {
        cudaError_t e = cudaFuncSetAttribute(tc_kernel<MODE, DT, MAXI, PAIR, KD>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget);
        if (e != cudaSuccess) return e;
        configured = kSmemBudget;
    }
    if constexpr (PAIR) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = grid;
        cfg.blockDim = dim3(Warps<MODE>::kThreads, 1, 1);
        cfg.dynamicSmemBytes = (size_t)smem;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaError_t e = cudaLaunchKernelEx(&cfg, tc_kernel<MODE, DT, MAXI, true, KD>, maps[0], maps[1], maps[2],
                                           maps[3], maps[4], maps[5], args);
        count_launch();
        if (e != cudaSuccess) return e;
    } else {
        tc_kernel<MODE, DT, MAXI, false, KD><<<grid, Warps<MODE>::kThreads, smem, st>>>(maps[0], maps[1], maps[2],
                                                                                        maps[3], maps[4], maps[5], args);
        count_launch();
    }
    return cudaGetLastError();
}

// x values a row of one produced k-block can touch: (BK - 1) / nb + 2 units,
// one x value each (two for the input pairs of 2-D surfaces).
int fwd_maxi_needed(int nb, bool twod) { return ((64 - 1) / nb + 2) * (twod ? 2 : 1); }

template <int MODE, int MAXI, int KD>
cudaError_t launch_m(bool f32, dim3 grid, int BN, int stages, const CUtensorMap* maps, const TcArgs& args,
                     cudaStream_t st)
{
    if constexpr (MODE == DCB) {   // bf16 CTA pairs only
        if (f32 || !args.pair) return cudaErrorInvalidConfiguration;
        return launch<DCB, KAN_BF16, MAXI, true, KD>(grid, BN, stages, maps, args, st);
    } else {
        if (f32) return launch<MODE, KAN_F32, MAXI, false, KD>(grid, BN, stages, maps, args, st);
        if constexpr (MODE == FWD || MODE == DCA) {
            if (args.pair) return launch<MODE, KAN_BF16, MAXI, true, KD>(grid, BN, stages, maps, args, st);
        }
        return launch<MODE, KAN_BF16, MAXI, false, KD>(grid, BN, stages, maps, args, st);
    }
}

template <int MODE, int KD>
cudaError_t launch_k(bool f32, dim3 grid, int BN, int stages, const CUtensorMap* maps, const TcArgs& args,
                     cudaStream_t st)
{
    if constexpr (MODE == FWD || MODE == DCA || MODE == DCB) {
        const int need = fwd_maxi_needed(args.nb, KD == 32);
        if (need <= 4) return launch_m<MODE, 4, KD>(f32, grid, BN, stages, maps, args, st);
        if (need <= 7) return launch_m<MODE, 7, KD>(f32, grid, BN, stages, maps, args, st);
        if (need <= 9) return launch_m<MODE, 9, KD>(f32, grid, BN, stages, maps, args, st);
        // (DCB keeps two x windows per thread: planned for nb >= 8 only)
        if constexpr (MODE != DCB)
            if (need <= 17) return launch_m<MODE, 17, KD>(f32, grid, BN, stages, maps, args, st);
        return cudaErrorInvalidConfiguration;   // nb >= 4 keeps need <= 17
    } else {
        return launch_m<MODE, 1, KD>(f32, grid, BN, stages, maps, args, st);
    }
}

// cubic splines run the closed-form instantiation; other degrees the general
// one (the GEMM of dY . w_base involves no basis)
template <int MODE>
cudaError_t launch_dt(bool f32, dim3 grid, int BN, int stages, const CUtensorMap* maps, const TcArgs& args,
                      cudaStream_t st)
{
    if constexpr (MODE == DCB) {   // cubic 1-D only
        if (args.twod || args.k != 3) return cudaErrorInvalidConfiguration;
        return launch_k<DCB, 3>(f32, grid, BN, stages, maps, args, st);
    } else {
        if (args.twod) {   // 2-D surfaces: produced-A kernels only (dx runs persistent)
            if constexpr (MODE == FWD || MODE == DCA) return launch_k<MODE, 32>(f32, grid, BN, stages, maps, args, st);
            return cudaErrorInvalidConfiguration;
        }
        if (MODE == GEMM || args.k == 3) return launch_k<MODE, 3>(f32, grid, BN, stages, maps, args, st);
        if constexpr (MODE != GEMM) return launch_k<MODE, 0>(f32, grid, BN, stages, maps, args, st);
        return cudaErrorInvalidConfiguration;
    }
}

template <int DT, bool PAIR, int KD>
cudaError_t launch_dx_persistent(const Plan& P, const CUtensorMap* maps, const DxArgs& d, cudaStream_t st)
{
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(dx_persistent_kernel<DT, PAIR, KD>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    if (P.p_smem > 232448 || d.BN % 16 != 0 || d.stages < 2) return cudaErrorInvalidConfiguration;
    // a pair's CTA loads BN / 2 columns of B in 64-column atoms; the grid is whole clusters
    if (PAIR && (d.BN % 128 != 0 || P.p_grid % 2 != 0)) return cudaErrorInvalidConfiguration;
    if constexpr (PAIR) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(P.p_grid, 1, 1);
        cfg.blockDim = dim3(kDxThreads, 1, 1);
        cfg.dynamicSmemBytes = (size_t)P.p_smem;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaError_t e =
            cudaLaunchKernelEx(&cfg, dx_persistent_kernel<DT, true, KD>, maps[0], maps[1], maps[2], maps[3], d);
        count_launch();
        if (e != cudaSuccess) return e;
    } else {
        dx_persistent_kernel<DT, false, KD><<<P.p_grid, kDxThreads, P.p_smem, st>>>(maps[0], maps[1], maps[2],
                                                                                     maps[3], d);
        count_launch();
    }
    return cudaGetLastError();
}

TcArgs base_args(const Problem& p, const Plan& P)
{
    TcArgs a{};
    a.status = device_status_ptr();
    a.batch = p.batch;
    a.in = p.in;
    a.out_f = p.out;
    a.G = p.G;
    a.k = p.k;
    a.nb1 = p.nb1;
    a.x_ld = p.x_ld;
    a.twod = p.dims == 2;
    a.nb = P.nbx;
    a.nbs = p.nb;
    a.ext = P.ext;
    a.lo = p.lo;
    a.inv_h = p.inv_h;
    a.Kt = (int)P.Kx;
    a.has_base = p.base;
    a.x_vec = (p.x_ld * (p.dtype == KAN_F32 ? 4 : 2)) % 16 == 0;
    a.nb_magic = (uint32_t)((((uint64_t)1 << 32) + (uint64_t)P.nbx - 1) / (uint64_t)P.nbx);
    return a;
}

// fp32 path: the absolute maxima of coef, w_base, x (with the SiLU branch) and
// dY (any may be null) into amax[0..3], the source of the operand scales.
cudaError_t amax_into(const Problem& p, const void* coef, const void* w_base, const void* x, const void* dY,
                      unsigned int* amax, cudaStream_t st)
{
    cudaError_t e = cudaMemsetAsync(amax, 0, 4 * sizeof(unsigned int), st);
    if (e != cudaSuccess) return e;
    AmaxArgs a{};
    a.src[0] = (const float*)coef;
    a.n[0] = p.out * p.Kt;
    a.src[1] = p.base ? (const float*)w_base : nullptr;
    a.n[1] = p.out * p.in;
    a.src[2] = p.base ? (const float*)x : nullptr;
    a.n[2] = p.batch * p.in;
    a.src[3] = (const float*)dY;
    a.n[3] = p.batch * p.out;
    int64_t nmax = 0;
    for (int k = 0; k < 4; ++k)
        if (a.src[k]) nmax = std::max(nmax, a.n[k]);
    absmax_kernel<<<std::min(grid_for(nmax / 4), 148 * 4), 256, 0, st>>>(a, amax);
    count_launch();
    return cudaGetLastError();
}

// fp16 hi/lo copies of coef (w_base interleaved), [out][Kx]; returns the (hi, lo) pointers.
cudaError_t split_coef_into(const Problem& p, const Plan& P, const void* coef, const void* w_base, uint8_t* dst,
                            const unsigned int* amax, const void** hi, const void** lo, cudaStream_t st)
{
    uint16_t* h = reinterpret_cast<uint16_t*>(dst);
    uint16_t* l = reinterpret_cast<uint16_t*>(dst + al256((size_t)p.out * P.Kx * 2));
    const dim3 grid((unsigned)std::min<int64_t>(cdiv(P.Kx, 4 * 256), 64), (unsigned)std::min<int64_t>(p.out, 65535));
    const uint32_t magic = (uint32_t)((((uint64_t)1 << 32) + (uint64_t)P.nbx - 1) / (uint64_t)P.nbx);
    split_coef_f16_kernel<<<grid, 256, 0, st>>>((const float*)coef, (const float*)w_base, p.out, p.in, p.nb, P.nbx, h,
                                                l, amax, magic);
    count_launch();
    *hi = h;
    *lo = l;
    return cudaGetLastError();
}

// fp16 hi/lo copies of dY, [batch][ldo] (ldo = out rounded up to 8); returns the (hi, lo) pointers.
cudaError_t split_dy_into(const Problem& p, int64_t ldo, const void* dY, uint8_t* dst, const unsigned int* amax,
                          const void** hi, const void** lo, cudaStream_t st)
{
    const int64_t n = p.batch * ldo;
    uint16_t* h = reinterpret_cast<uint16_t*>(dst);
    uint16_t* l = reinterpret_cast<uint16_t*>(dst + al256((size_t)n * 2));
    if (ldo == p.out)
        split_f16_kernel<<<grid_for(n / 4), 256, 0, st>>>((const float*)dY, h, l, n, amax);
    else
        split_f16_rows_kernel<<<grid_for(n), 256, 0, st>>>((const float*)dY, h, l, p.batch, p.out, ldo, amax);
    count_launch();
    *hi = h;
    *lo = l;
    return cudaGetLastError();
}

}  // namespace

bool tc_supported(const Problem& p, bool backward, const char** why)
{
    // Every tensor-core operand is 2 bytes wide: bf16 data as it is, or the fp16
    // hi/lo copies of fp32 data (coef with w_base interleaved: G+4 columns per input).
    const bool f32 = p.dtype == KAN_F32;
    const int64_t nbx = p.nb + ((f32 && p.base) ? 1 : 0);
    if ((p.in * nbx * 2) % 16 != 0) {
        *why = f32 ? "in*(G+k) (in*(G+k+1) with the SiLU branch) is not a multiple of 8 (TMA row stride of the "
                     "coefficient operand)"
                   : "in*(G+k)*2 is not a multiple of 16 bytes (TMA row stride of coef)";
        return false;
    }
    if (!f32 && p.base && (p.in * 2) % 16 != 0) {
        *why = "in*2 is not a multiple of 16 bytes (TMA row stride of w_base)";
        return false;
    }
    if (!f32 && (p.out * 2) % 16 != 0) {
        // (fp32 reads dY through its fp16 copies, whose rows are padded to 8 elements)
        *why = "bf16 with out not a multiple of 8 (TMA row stride of dY)";
        return false;
    }
    if (p.nb < 4) {
        *why = "fewer than 4 basis functions per input (G + degree < 4): too many inputs per k-block row";
        return false;
    }
    if (p.dims == 2 && f32 && p.out > 1024) {
        *why = "2-D surfaces in fp32 with more than 1024 outputs (the persistent dx kernel's limit)";
        return false;
    }

    if (nbx > 121 && (f32 || nbx > 249)) {
        *why = "G too large for one dx tile (the input's columns must fit the tile with its alignment offset)";
        return false;
    }
    if (p.Kt + p.in > ((int64_t)1 << 30) || p.in * nbx >= (((int64_t)1 << 32) / nbx) ||
        p.batch > ((int64_t)1 << 31) - 256 ||
        p.out > ((int64_t)1 << 30)) {
        *why = "problem too large for 32-bit tile coordinates";
        return false;
    }
    (void)backward;
    return true;
}

size_t tc_workspace_forward(const Problem& p, int num_sms) { return make_plan(p, num_sms).fwd.total; }
size_t tc_workspace_backward(const Problem& p, int num_sms) { return make_plan(p, num_sms).bwd.total; }

cudaError_t tc_forward(const Problem& p, const void* x, const void* coef, const void* w_base, void* y, void* ws,
                       int num_sms, cudaStream_t st, const char** detail)
{
    if (p.batch == 0) return cudaSuccess;
    const bool f32 = p.dtype == KAN_F32;
    const int BK = 64;
    const Plan P = make_plan(p, num_sms);
    uint8_t* w = reinterpret_cast<uint8_t*>(ws);
    const void *c_hi = coef, *c_lo = coef, *wb_hi = w_base, *wb_lo = w_base;
    unsigned int* amax = f32 ? reinterpret_cast<unsigned int*>(w + P.fwd.amax) : nullptr;
    cudaError_t e;
    if (f32) {
        // operand scales, then the fp16 hi/lo copy of coef (w_base interleaved)
        if ((e = amax_into(p, coef, w_base, x, nullptr, amax, st)) != cudaSuccess) return e;
        if ((e = split_coef_into(p, P, coef, w_base, w + P.fwd.coef_hl, amax, &c_hi, &c_lo, st)) != cudaSuccess)
            return e;
    }
    if ((e = record_mark(timing_marks().after_prep, st)) != cudaSuccess) return e;
    CUtensorMap maps[6];
    // (a pair's CTA loads 128 + (BN - 256) / 2 rows of each B tile: boxes of 64 rows for BN = 384)
    const int fbox = P.f_pair && P.f_BN == 384 ? 64 : std::min(P.f_BN, 128);
    if (!make_map_2d(&maps[2], c_hi, f32, p.out, P.Kx, fbox, BK, detail) ||
        !make_map_2d(&maps[3], c_lo, f32, p.out, P.Kx, fbox, BK, detail))
        return cudaErrorInvalidValue;
    if (p.base && !P.ext) {
        if (!make_map_2d(&maps[4], wb_hi, f32, p.out, p.in, fbox, BK, detail) ||
            !make_map_2d(&maps[5], wb_lo, f32, p.out, p.in, fbox, BK, detail))
            return cudaErrorInvalidValue;
    } else {
        maps[4] = maps[2];
        maps[5] = maps[3];
    }
    maps[0] = maps[2];
    maps[1] = maps[3];
    TcArgs a = base_args(p, P);
    a.x = x;
    a.amax = amax;
    a.out = P.f_splits > 1 ? (void*)(w + P.fwd.fwd_part) : y;
    a.BN = P.f_BN;
    a.stages = P.f_stages;
    a.stages_a = P.f_stages_a;
    a.fbox = fbox;
    a.nkb_main = P.f_nkb_main;
    a.nkb_total = P.f_nkb_total;
    a.kb_per_split = P.f_kps;
    a.partial = P.f_splits > 1;
    a.pair = P.f_pair ? 1 : 0;
    a.m_tiles = P.f_m;
    // unsplit: y leaves through TMA stores when the tile is whole boxes wide and TMA can address y
    a.store_tma = !a.partial && P.f_BN % (f32 ? 32 : 64) == 0 && make_store_map(&maps[0], y, f32, p.batch, p.out);
    const dim3 fgrid = P.f_pair ? dim3(P.f_my, P.f_n, P.f_splits) : dim3(P.f_n, P.f_m, P.f_splits);
    e = launch_dt<FWD>(f32, fgrid, P.f_BN, P.f_stages, maps, a, st);
    if (e != cudaSuccess) return e;
    if (P.f_splits > 1) {
        const int64_t n = p.batch * p.out;
        const float* part = reinterpret_cast<const float*>(w + P.fwd.fwd_part);
        if (f32) {
            reduce_splits_kernel<float><<<grid_for(n), 256, 0, st>>>(part, (float*)y, n, P.f_splits);
            count_launch();
        } else {
            reduce_splits_kernel<__nv_bfloat16><<<grid_for(n), 256, 0, st>>>(part, (__nv_bfloat16*)y, n, P.f_splits);
            count_launch();
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t tc_backward(const Problem& p, const void* x, const void* coef, const void* w_base, const void* dY,
                        void* dx, float* dcoef, float* dw_base, void* ws, int num_sms, cudaStream_t st,
                        const char** detail)
{
    const bool f32 = p.dtype == KAN_F32;
    const int BK = 64, EPB = 64;
    const Plan P = make_plan(p, num_sms);
    uint8_t* w = reinterpret_cast<uint8_t*>(ws);
    cudaError_t e;
    if (p.batch == 0) {
        if (dcoef && (e = zero_f32(dcoef, p.out * p.Kt, st)) != cudaSuccess) return e;
        if (dw_base && (e = zero_f32(dw_base, p.out * p.in, st)) != cudaSuccess) return e;
        return cudaSuccess;
    }
    unsigned int* amax = f32 ? reinterpret_cast<unsigned int*>(w + P.bwd.amax) : nullptr;
    const void *dy_hi = dY, *dy_lo = dY, *c_hi = coef, *c_lo = coef;
    if (f32) {
        // operand scales (coef and w_base for dx's coefficient copy, x for the
        // SiLU values, dY), then dY's fp16 hi/lo copy, shared by dcoef and dx,
        // and (for dx) the coefficients' copy
        if ((e = amax_into(p, dx ? coef : nullptr, dx ? w_base : nullptr, x, dY, amax, st)) != cudaSuccess) return e;
        if ((e = split_dy_into(p, P.ldo, dY, w + P.bwd.dy_hl, amax, &dy_hi, &dy_lo, st)) != cudaSuccess) return e;
        if (dx && (e = split_coef_into(p, P, coef, w_base, w + P.bwd.coef_hl, amax, &c_hi, &c_lo, st)) != cudaSuccess)
            return e;
    }
    if ((e = record_mark(timing_marks().after_prep, st)) != cudaSuccess) return e;
    // ---- dcoef / dw_base: A = basis^T (producers), B = dY MN-major (BK-batch x 64-output boxes) ----
    if (dcoef || dw_base) {
        CUtensorMap maps[6];
        if (!make_map_2d(&maps[2], dy_hi, f32, p.batch, p.out, BK, EPB, detail, P.ldo)) return cudaErrorInvalidValue;
        if (f32) {
            if (!make_map_2d(&maps[3], dy_lo, true, p.batch, p.out, BK, EPB, detail, P.ldo))
                return cudaErrorInvalidValue;
        } else {
            maps[3] = maps[2];
        }
        maps[0] = maps[4] = maps[2];
        maps[1] = maps[5] = maps[3];
        TcArgs a = base_args(p, P);
        a.x = x;
        a.amax = amax;
        float* partbuf = reinterpret_cast<float*>(w + P.bwd.dc_part);
        a.BN = P.d_BN;
        a.stages = P.d_stages;
        a.stages_a = P.d_stages_a;
        a.nkb_main = a.nkb_total = P.d_nkb;
        a.kb_per_split = P.d_kps;
        a.n_kt_tiles = P.d_nkt;
        a.part_ld = P.d_ld;
        a.partial = P.d_splits > 1;
        a.out = a.partial ? (void*)partbuf : (void*)dcoef;   // a skipped output is simply not stored
        a.out2 = dw_base;
        a.pair = P.d_pair ? 1 : 0;
        a.m_tiles = P.d_m;
        if (P.dcb) {
            // outputs on M (dY^T by TMA through the same boxes), spline columns on N
            a.BN = P.b_BN;
            a.stages = P.b_stages;
            a.stages_a = P.b_stages_a;
            a.kb_per_split = P.d_nkb;
            a.partial = 0;
            a.out = dcoef;
            a.pair = 1;
            a.m_tiles = P.b_m;
            a.store_tma = make_store_map(&maps[0], dcoef, true, p.out, p.Kt);
            e = launch_dt<DCB>(false, dim3(P.b_my, P.b_n, 1), P.b_BN, P.b_stages, maps, a, st);
        } else {
            const dim3 grid = P.d_pair ? dim3(P.d_my, P.d_n, P.d_splits) : dim3(P.d_n, P.d_m, P.d_splits);
            e = launch_dt<DCA>(f32, grid, P.d_BN, P.d_stages, maps, a, st);
        }
        if (e != cudaSuccess) return e;
        if (a.partial && !P.dcb) {
            const dim3 rgrid((unsigned)std::min<int64_t>(cdiv(P.d_ld, 256), 64),
                             (unsigned)std::min<int64_t>(p.out, 65535));
            reduce_dcoef_kernel<<<rgrid, 256, 0, st>>>(partbuf, dcoef, dw_base, p.out, p.Kt, p.in, P.d_ld, P.d_splits,
                                                       p.nb, P.nbx, P.ext ? 1 : 0, a.nb_magic);
            count_launch();
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
    }
    if ((e = record_mark(timing_marks().after_dcoef, st)) != cudaSuccess) return e;
    // ---- dx: A = dY K-major, B = coef MN-major (fp32: their fp16 hi/lo copies) ----
    if (dx) {
        float* gb = nullptr;
        if (p.base && !P.ext) {
            // bf16: Gb = dY . w_base (fp32 [batch, in]) for the SiLU term of dx
            gb = reinterpret_cast<float*>(w + P.bwd.gb);
            CUtensorMap maps[6];
            if (!make_map_2d(&maps[0], dY, false, p.batch, p.out, kBM, BK, detail) ||
                !make_map_2d(&maps[2], w_base, false, p.out, p.in, BK, EPB, detail))
                return cudaErrorInvalidValue;
            maps[1] = maps[0];
            maps[3] = maps[4] = maps[5] = maps[2];
            TcArgs a = base_args(p, P);
            a.out = gb;
            a.BN = P.g_BN;
            a.stages = P.g_stages;
            a.nkb_main = a.nkb_total = P.x_nkb;
            a.kb_per_split = P.x_nkb;
            e = launch_dt<GEMM>(f32, dim3(P.g_n, P.g_m, 1), P.g_BN, P.g_stages, maps, a, st);
            if (e != cudaSuccess) return e;
        }
        CUtensorMap maps[6];
        if (!make_map_2d(&maps[0], dy_hi, f32, p.batch, p.out, kBM, BK, detail, P.ldo)) return cudaErrorInvalidValue;
        if (f32) {
            if (!make_map_2d(&maps[1], dy_lo, true, p.batch, p.out, kBM, BK, detail, P.ldo))
                return cudaErrorInvalidValue;
            if (!make_map_2d(&maps[2], c_hi, true, p.out, P.Kx, BK, EPB, detail) ||
                !make_map_2d(&maps[3], c_lo, true, p.out, P.Kx, BK, EPB, detail))
                return cudaErrorInvalidValue;
        } else {
            maps[1] = maps[0];
            if (!make_map_2d(&maps[2], coef, false, p.out, p.Kt, BK, EPB, detail)) return cudaErrorInvalidValue;
            maps[3] = maps[2];
        }
        maps[4] = maps[2];
        maps[5] = maps[3];
        if (P.p_ok) {
            DxArgs d{};
            d.x = x;
            d.dx = dx;
            d.gb = gb;
            d.status = device_status_ptr();
            d.amax = amax;
            d.batch = p.batch;
            d.in = p.in;
            d.out = p.out;
            d.G = p.G;
            d.k = p.k;
            d.nb1 = p.nb1;
            d.x_ld = p.x_ld;
            d.nb = P.nbx;
            d.nbs = p.nb;
            d.ext = P.ext ? 1 : 0;
            d.lo = p.lo;
            d.inv_h = p.inv_h;
            d.BN = P.p_BN;
            d.stages = P.p_stages;
            d.nkb = P.x_nkb;
            d.n_in_tile = P.p_nin;
            d.n_tiles_n = P.p_ntn;
            d.n_tiles = P.p_tiles;
            d.ld_stage = P.p_ld;
            d.a_res = P.p_ares ? 1 : 0;
            d.pair = P.p_pair ? 1 : 0;
            if (p.dims == 2)
                e = f32 ? launch_dx_persistent<KAN_F32, false, 32>(P, maps, d, st)
                        : (P.p_pair ? launch_dx_persistent<KAN_BF16, true, 32>(P, maps, d, st)
                                    : launch_dx_persistent<KAN_BF16, false, 32>(P, maps, d, st));
            else if (p.k == 3)
                e = f32 ? launch_dx_persistent<KAN_F32, false, 3>(P, maps, d, st)
                        : (P.p_pair ? launch_dx_persistent<KAN_BF16, true, 3>(P, maps, d, st)
                                    : launch_dx_persistent<KAN_BF16, false, 3>(P, maps, d, st));
            else
                e = f32 ? launch_dx_persistent<KAN_F32, false, 0>(P, maps, d, st)
                        : (P.p_pair ? launch_dx_persistent<KAN_BF16, true, 0>(P, maps, d, st)
                                    : launch_dx_persistent<KAN_BF16, false, 0>(P, maps, d, st));
            if (e != cudaSuccess) return e;
        } else {
            if (p.dims == 2) return cudaErrorInvalidConfiguration;   // (tc_supported rules it out)
            TcArgs a = base_args(p, P);
            a.x = x;
            a.amax = amax;
            a.out = dx;
            a.out2 = gb;
            a.BN = P.x_BN;
            a.stages = P.x_stages;
            a.nkb_main = a.nkb_total = P.x_nkb;
            a.kb_per_split = P.x_nkb;
            a.n_in_tile = P.x_nin;
            e = launch_dt<DX>(f32, dim3(P.x_n, P.x_m, 1), P.x_BN, P.x_stages, maps, a, st);
            if (e != cudaSuccess) return e;
        }
    }
    return cudaSuccess;
}

}  // namespace kan
