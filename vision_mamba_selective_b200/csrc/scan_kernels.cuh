// scan_kernels.cuh -- sm_100a kernels of the bidirectional selective scan (S6).
//
// The work unit is a "pair": two S6 directions that visit the same L positions in
// opposite orders.  The Vim block (page "Vision Mamba Guide: Efficient Bidirectional
// SSM & VMamba", section "2. The Bidirectional Mamba Block") is one pair over the
// token order; the VMamba cross-scan (sections "1. Cross-Scan Traversal" to "3.
// Cross-Merge Reversal") is two pairs, one over the row-major order and one over the
// column-major order of the grid.
//
// A sequence of L tokens is cut into G chunks of up to `chunk` tokens.  One CTA owns
// one chunk of 64 channels of one batch item and runs both directions of the pair
// over it: warps 0-1 the forward direction (ascending), warps 2-3 the backward
// direction (descending), one thread per (channel, direction) with all d_state
// states of h in fp32 registers.  The chunk's inputs stream through shared memory in
// tiles of 16 tokens (cp.async for u and delta, register prefetch + fp32 conversion
// for B/C), double buffered.  The forward direction visits tile j at step j and the
// backward one at step nT-1-j: the first visitor leaves its partial output in a
// per-chunk fp32 buffer, the second adds its own; after the step's barrier all
// threads finish the completed tiles (z prefetched into registers, silu(z) gate,
// 16-byte stores), so every output is written once and no separate output pass is
// needed.
//
// Variants (template flags): CONV, the pathways' kernel-3 convolution + SiLU formed
// from staged x; ZOH, the exact zero-order-hold Bbar; DT, delta from the x_proj step
// input and the dt_proj weights; PIN, the cross-scan's second pair adding the first
// pair's fp32 partial.
//
// For G > 1 the state entering each chunk comes from two small kernels: `pair_carry`
// reduces every chunk to its end state from h = 0 plus its total Delta, and
// `pair_combine` folds those summaries along each direction.
//
// State form (structured A, first-order Bbar; VIMSCAN_GF): the main kernel runs the
// scaled state g = h / du, du = Delta u, instead of h (see main_tile): the decay chain
// absorbs du_(t-1) / du_t and the drive is B itself, which removes one multiply per
// state and token.  Units (bf16 I/O, first-order Bbar; VIMSCAN_L2U): Delta is kept as
// L = Delta / ln 2, so softplus is log2(1 + 2^(x log2 e)) with no rescaling, the decay
// base is 2^(A_0 L), and B is staged multiplied by ln 2; the chunk summaries leave
// their Delta sums in natural units.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace vimscan {

constexpr int kDC = 64;              // channels per CTA
constexpr int kThreads = 2 * kDC;    // one thread per (channel, direction)
constexpr int kTile = 16;            // tokens per staged tile
#ifndef VIMSCAN_KSUB
#define VIMSCAN_KSUB 4
#endif
#ifndef VIMSCAN_MIN_BLOCKS
#define VIMSCAN_MIN_BLOCKS 4
#endif
#ifndef VIMSCAN_CARRY_KSUB
#define VIMSCAN_CARRY_KSUB 8
#endif
#ifndef VIMSCAN_CARRY_DT_MIN_BLOCKS
#define VIMSCAN_CARRY_DT_MIN_BLOCKS 5   // the step-input carry spills at the register budget of 6
#endif
#ifndef VIMSCAN_CARRY_MIN_BLOCKS
#define VIMSCAN_CARRY_MIN_BLOCKS 6
#endif
#ifndef VIMSCAN_CARRY_ZOH_KSUB
#define VIMSCAN_CARRY_ZOH_KSUB 8
#endif
#ifndef VIMSCAN_CARRY_ZOH_MIN_BLOCKS
#define VIMSCAN_CARRY_ZOH_MIN_BLOCKS 4
#endif
constexpr int kSub = VIMSCAN_KSUB;   // tokens whose independent work is formed ahead of the recurrence
constexpr int kMinBlocks = VIMSCAN_MIN_BLOCKS;   // resident CTAs per SM the register budget targets
constexpr int kCarrySub = VIMSCAN_CARRY_KSUB;          // the same for the chunk-summary kernel
constexpr int kCarryMinBlocks = VIMSCAN_CARRY_MIN_BLOCKS;
constexpr int kCarryDtMinBlocks = VIMSCAN_CARRY_DT_MIN_BLOCKS;
constexpr int kCarryZohSub = VIMSCAN_CARRY_ZOH_KSUB;   // the same two with the exact hold
constexpr int kCarryZohMinBlocks = VIMSCAN_CARRY_ZOH_MIN_BLOCKS;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.69314718055994531f;
#ifndef VIMSCAN_GF
#define VIMSCAN_GF 1
#endif
#ifndef VIMSCAN_L2U
#define VIMSCAN_L2U 1
#endif
#ifndef VIMSCAN_COMBINE_AHEAD
#define VIMSCAN_COMBINE_AHEAD 16   // chunk summaries pair_combine loads before it folds them
#endif
// bf16 first-order kernels may keep Delta in log2 units (L = Delta / ln 2)
template <typename T, bool ZOH>
__host__ __device__ constexpr bool lu_mode() { return VIMSCAN_L2U && sizeof(T) == 2 && !ZOH; }

// ----------------------------------------------------------------------------
// element types
// ----------------------------------------------------------------------------
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> struct Vec;           // 16-byte vector of T
template <> struct Vec<float> { static constexpr int n = 4; };
template <> struct Vec<__nv_bfloat16> { static constexpr int n = 8; };

// 16 bytes of T -> 8 or 4 floats
__device__ __forceinline__ void unpack16(const uint4 &v, float (&f)[4]) {
    f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
}
__device__ __forceinline__ void unpack16(const uint4 &v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ uint4 pack16(const float (&f)[4]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
}
__device__ __forceinline__ uint4 pack16(const float (&f)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 p = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t *>(&p);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// 16 bytes of T, every element equal to x
template <typename T>
__device__ __forceinline__ uint4 pad16(float x) {
    float f[Vec<T>::n];
#pragma unroll
    for (int i = 0; i < Vec<T>::n; ++i) f[i] = x;
    return pack16(f);
}

// ----------------------------------------------------------------------------
// math
// ----------------------------------------------------------------------------
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// softplus(x) = max(x, 0) + log1p(exp(-|x|)), and x itself above 20.  log1p(e) for
// e in (0, 1] is evaluated as 2 atanh(s) with s = e / (2 + e) in (0, 1/3], through
// the Taylor series of atanh up to s^13 (truncation error below 2e-8 relative).
__device__ __forceinline__ float softplus(float x) {
    const float e = ex2(-fabsf(x) * kLog2e);
    const float s = e * rcp(2.0f + e);
    const float s2 = s * s;
    float p = fmaf(s2, 2.0f / 13.0f, 2.0f / 11.0f);
    p = fmaf(s2, p, 2.0f / 9.0f);
    p = fmaf(s2, p, 2.0f / 7.0f);
    p = fmaf(s2, p, 2.0f / 5.0f);
    p = fmaf(s2, p, 2.0f / 3.0f);
    p = fmaf(s2, p, 2.0f);
    const float r = fmaf(s, p, fmaxf(x, 0.0f));
    return x > 20.0f ? x : r;
}

// softplus from the MUFU exp2/log2 approximations: log2(1 + 2^(x log2 e)) ln 2, and x
// above 20.  Its absolute error is about 1e-7 (the log2 approximation near 1), far
// below the resolution of bf16 inputs; the fp32-I/O kernels use softplus() instead.
__device__ __forceinline__ float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float softplus_fast(float x) {
    const float r = lg2(1.0f + ex2(x * kLog2e)) * 0.69314718055994531f;
    return x > 20.0f ? x : r;
}

template <typename T>
__device__ __forceinline__ float softplus_io(float x) {
    if constexpr (sizeof(T) == 4) return softplus(x);
    else return softplus_fast(x);
}

// expm1(x) = exp(x) - 1 without the cancellation of exp(x) - 1 near 0: for |x| < 1/2
// the Taylor series x + x^2/2! + ... + x^8/8! (Horner), whose first omitted term is
// below 1.1e-8 of the result; elsewhere e - 1 with e = exp(x) given (from ex2), where
// |result| > 0.39 keeps the relative error of the difference within a few 1e-7.
__device__ __forceinline__ float expm1_acc(float x, float e) {
    float p = fmaf(x, 1.0f / 40320.0f, 1.0f / 5040.0f);
    p = fmaf(x, p, 1.0f / 720.0f);
    p = fmaf(x, p, 1.0f / 120.0f);
    p = fmaf(x, p, 1.0f / 24.0f);
    p = fmaf(x, p, 1.0f / 6.0f);
    p = fmaf(x, p, 0.5f);
    p = fmaf(x, p, 1.0f);
    return fabsf(x) < 0.5f ? x * p : e - 1.0f;
}
__device__ __forceinline__ float expm1_acc(float x) { return expm1_acc(x, ex2(x * kLog2e)); }

// Bbar_n / B_n of the exact zero-order hold for one state, (exp(Delta A_n) - 1) / A_n,
// and its limit Delta at A_n = 0
__device__ __forceinline__ float zoh_gain(float dt, float An) {
    return An != 0.0f ? expm1_acc(dt * An) / An : dt;
}

// silu(z) = z / (1 + exp(-z))
__device__ __forceinline__ float silu(float z) { return z * rcp(1.0f + ex2(-z * kLog2e)); }

// softplus in log2 units: log2(1 + 2^xl) for xl = x log2 e, and xl itself for x > 20
__device__ __forceinline__ float softplus_l2(float xl) {
    const float r = lg2(1.0f + ex2(xl));
    return xl > 20.0f * kLog2e ? xl : r;
}

// |du| kept at or above 1e-20 for the scaled state g = h / du (see main_tile)
__device__ __forceinline__ float clamp_du(float v) { return fabsf(v) < 1.0e-20f ? 1.0e-20f : v; }

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// Reads of the fp32 B/C rows staged in shared memory, as pairs of states.
template <int NP>
__device__ __forceinline__ void load_row(const float *row, float2 (&v)[NP]) {
    if constexpr (NP >= 2) {
        const float4 *r4 = reinterpret_cast<const float4 *>(row);
#pragma unroll
        for (int k = 0; k < NP / 2; ++k) {
            const float4 t = r4[k];
            v[2 * k] = f2(t.x, t.y);
            v[2 * k + 1] = f2(t.z, t.w);
        }
    } else {
        v[0] = *reinterpret_cast<const float2 *>(row);
    }
}

// ----------------------------------------------------------------------------
// division by the grid height H, which the column-major order needs for every row it
// stages: the method of Granlund and Montgomery, "Division by Invariant Integers using
// Multiplication" (PLDI 1994), Figure 4.1, for 32-bit unsigned n and 1 <= d < 2^32:
//   l = ceil(log2 d),  m = floor(2^32 (2^l - d) / d) + 1,  s1 = min(l, 1),  s2 = max(l - 1, 0),
//   t = high 32 bits of m n,  n / d = (t + ((n - t) >> s1)) >> s2.
// The host forms (m, s1, s2) once per call; the kernels then divide in four instructions
// instead of a full integer division per row.
// ----------------------------------------------------------------------------
struct DivInv {
    unsigned m;
    int s1, s2;
};
inline DivInv div_inv(unsigned d) {
    int l = 0;
    while (l < 32 && (1ull << l) < d) ++l;   // ceil(log2 d)
    DivInv v;
    v.m = (unsigned)((((1ull << l) - d) << 32) / d + 1);
    v.s1 = l < 1 ? l : 1;
    v.s2 = l > 1 ? l - 1 : 0;
    return v;
}
__host__ __device__ __forceinline__ unsigned div_by(unsigned n, const DivInv &v) {
#ifdef __CUDA_ARCH__
    const unsigned t = __umulhi(v.m, n);
#else
    const unsigned t = (unsigned)(((unsigned long long)v.m * n) >> 32);
#endif
    return (t + ((n - t) >> v.s1)) >> v.s2;
}

// ----------------------------------------------------------------------------
// arguments
// ----------------------------------------------------------------------------
struct PairArgs {
    const void *u, *delta, *z;      // [batch, L, Di] by position
    int64_t u_dir_stride;           // elements from the forward direction's u to the backward
                                    // one's (0: both read the same u)
    const void *B[2], *C[2];        // per direction of the pair: [batch, L, N] by position
    const float *A;                 // [2][Di][N]: forward, backward
    const float *D;                 // [2][Di]
    const float *bias;              // [2][Di]
    const float *conv_w;            // [2][Di][3] convolution front of the pathways, or null
    const float *conv_b;            // [2][Di]
    void *y;                        // final output [batch, L, Di] (element type), or null
    float *partial_out;             // fp32 [batch, L, Di] (ungated pair sum), or null
    const float *partial_in;        // fp32 [batch, L, Di] added before the gate, or null
    float *hloc;                    // [batch][G][2][Di][N] chunk summaries / carries
    float *ssum;                    // [batch][G][2][Di]    chunk Delta sums
    int batch, L, Di, H, W;
    int order;                      // 0: position = step; 1: column-major on H x W
    DivInv hdiv;                    // division by H (order 1)
    int chunk, G;                   // tokens per chunk (multiple of kTile), chunks
    const float *dt_in;             // [2][batch*L] step input per direction and position, or null
    const float *dt_w;              // [2][Di] its dt_proj weights: delta_raw = dt_in * dt_w
    int zoh;                        // exact zero-order-hold Bbar instead of Delta B
    int fold_reverse;               // pair_combine folds each direction against its order
    int carry_span;                 // consecutive chunks per pair_carry CTA (0 or 1: one)
    float *hck;                     // or null: the state entering every kCkTokens-token segment,
                                    // [batch][ceil(L/kCkTokens)][2][N][Di] fp32, in each direction's
                                    // visiting order (the Vim scan, with or without its front, and
                                    // each pair of the cross-scan, over the pair's steps)
};
constexpr int kCkTokens = 32;       // tokens per checkpoint segment (the derivative's chunk)

// position visited at step t of the forward direction
__device__ __forceinline__ int position(const PairArgs &p, int t) {
    if (p.order == 0) return t;
    const int w = (int)div_by((unsigned)t, p.hdiv), h = t - w * p.H;
    return h * p.W + w;
}

// Everything below is internal to each translation unit that includes this file:
// the kernel variants are split over several units, which compile in parallel, and
// each unit launches only the kernels it instantiates itself.
namespace {

// ----------------------------------------------------------------------------
// shared-memory staging of one step: the forward tile and the backward tile
// ----------------------------------------------------------------------------
// One slot: per direction [u rows][kDC] T then [delta rows][kDC] T, then
// [dir][B|C][kTile][N] fp32.  With the convolution front (CONV) the u area holds the
// raw input x with one halo row on each side: row rr is token row rr - 1.
template <typename T, int N, bool CONV = false>
struct Stage {
    static constexpr int kURows = CONV ? kTile + 2 : kTile;
    static constexpr int kDirUV = (kURows + kTile) * kDC;   // elements per direction
    static constexpr int kBC = kTile * N;                    // elements per B or C tile
    static constexpr int kUVBytes = 2 * kDirUV * (int)sizeof(T);
    static constexpr int kBCBytes = 2 * 2 * kBC * 4;
    static constexpr int kSlotBytes = kUVBytes + kBCBytes;

    __device__ static T *uv(char *slot, int dir, int which) {
        return reinterpret_cast<T *>(slot) + dir * kDirUV + (which ? kURows * kDC : 0);
    }
    __device__ static float *bc(char *slot, int dir, int which) {
        return reinterpret_cast<float *>(slot + kUVBytes) + (dir * 2 + which) * kBC;
    }
};

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, bool valid) {
    const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    const int n = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::); }

// B and C rows can be moved as 16-byte vectors when a row is a whole number of them
template <typename T, int N>
constexpr bool bc_vectorizable() { return (N * sizeof(T)) % 16 == 0; }

// Loads of one step (tile jf of the forward direction, jb of the backward one):
// u/delta by cp.async straight into the slot, B/C into registers first and then,
// converted to fp32, into the slot.
// Rows past the end of the chunk and channels past d_inner are zero-filled, so that
// they act as no-op tokens.
template <typename T, int N, bool VEC_BC, bool CONV = false, bool ZOH = false, bool DT = false, int NTHR = kThreads>
struct Stager {
    using S = Stage<T, N, CONV>;
    static constexpr int V = Vec<T>::n;                 // elements per 16-byte piece
    static constexpr int kRowPieces = kDC / V;          // pieces per u/delta row
    static constexpr int kUVRep = kTile * kRowPieces / NTHR;   // pieces per thread per tensor
    static constexpr int kBCRow = VEC_BC ? (int)(N * sizeof(T) / 16) : N;   // units per B/C row
    static constexpr int kBCUnits = 4 * kTile * kBCRow;
    static constexpr int kBCPer = (kBCUnits + NTHR - 1) / NTHR;
    static_assert(kTile * kRowPieces % NTHR == 0, "u/delta pieces must split evenly");
    static_assert(NTHR >= kTile, "one thread per row of the step input");

    const PairArgs &p;
    const int b, t0, tc, d0;
    const int tid;   // this thread's index among the NTHR staging threads
    uint4 pre_v[VEC_BC ? kBCPer : 1];
    float pre_s[VEC_BC ? 1 : kBCPer];

    __device__ Stager(const PairArgs &pa, int b_, int t0_, int tc_, int d0_, int tid_)
        : p(pa), b(b_), t0(t0_), tc(tc_), d0(d0_), tid(tid_) {}

    __device__ int rows_of(int j) const { return min(kTile, tc - j * kTile); }

    // element offset of row r of tile j, channel ch (valid rows only)
    __device__ size_t row_off(int j, int r, int ch) const {
        return ((size_t)b * p.L + position(p, t0 + j * kTile + r)) * p.Di + ch;
    }

    // u and delta of both tiles (with CONV: x and its halo rows instead of u)
    __device__ void issue(char *slot, int jf, int jb) const {
        const T *gd = static_cast<const T *>(p.delta);
#pragma unroll
        for (int dir = 0; dir < 2; ++dir) {
            const T *gu = static_cast<const T *>(p.u) + (dir ? p.u_dir_stride : 0);
            const int j = dir ? jb : jf;
            const int rows = rows_of(j);
#pragma unroll
            for (int m = 0; m < kUVRep; ++m) {
                const int li = tid + m * NTHR;
                const int v = li % kRowPieces, r = li / kRowPieces;
                const int ch = d0 + v * V;
                const bool ok = r < rows && ch < p.Di;
                const int so = r * kDC + v * V;
                if (ok) {
                    const size_t off = row_off(j, r, ch);
                    if (!CONV) cp_async16(S::uv(slot, dir, 0) + so, gu + off, true);
                    if (!DT) cp_async16(S::uv(slot, dir, 1) + so, gd + off, true);
                } else {
                    // outside the data: u = 0 and delta_raw = -1e4, so that Delta =
                    // softplus(-1e4 + bias) = 0 exactly (Abar = 1, Bbar u = 0): a no-op token
                    if (!CONV) *reinterpret_cast<uint4 *>(S::uv(slot, dir, 0) + so) = make_uint4(0, 0, 0, 0);
                    if (!DT) *reinterpret_cast<uint4 *>(S::uv(slot, dir, 1) + so) = pad16<T>(-1.0e4f);
                }
            }
            if constexpr (DT) {
                // the step input of each row (one value per token; the delta area holds
                // them as floats), NaN past the data: delta_at turns it into Delta = 0
                if (tid < kTile) {
                    const int r = tid;
                    float v = __int_as_float(0x7fc00000);
                    if (r < rows) v = p.dt_in[(size_t)dir * p.batch * p.L + (size_t)b * p.L + position(p, t0 + j * kTile + r)];
                    reinterpret_cast<float *>(S::uv(slot, dir, 1))[r] = v;
                }
            }
            if constexpr (CONV) {
                // x rows -1 .. kTile of the tile (the convolution's neighbours), zero
                // outside the sequence (the convolution's zero padding)
                for (int li = tid; li < S::kURows * kRowPieces; li += NTHR) {
                    const int v = li % kRowPieces, rr = li / kRowPieces;
                    const int ch = d0 + v * V;
                    const int t = t0 + j * kTile + rr - 1;
                    T *dst = S::uv(slot, dir, 0) + rr * kDC + v * V;
                    if (t >= 0 && t < p.L && ch < p.Di)
                        cp_async16(dst, gu + ((size_t)b * p.L + t) * p.Di + ch, true);
                    else
                        *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
                }
            }
        }
        cp_async_commit();
    }

    __device__ void load_bc(int jf, int jb) {
#pragma unroll
        for (int k = 0; k < kBCPer; ++k) {
            const int i = tid + k * NTHR;
            const int part = i % kBCRow;
            const int r = (i / kBCRow) % kTile;
            const int which = (i / (kBCRow * kTile)) % 2;
            const int dir = i / (kBCRow * kTile * 2);
            const int j = dir ? jb : jf;
            const bool ok = i < kBCUnits && r < rows_of(j);
            const void *base = dir ? (which ? p.C[1] : p.B[1]) : (which ? p.C[0] : p.B[0]);
            size_t row = 0;
            if (ok) row = ((size_t)b * p.L + position(p, t0 + j * kTile + r)) * N;
            if constexpr (VEC_BC) {
                pre_v[k] = ok ? *reinterpret_cast<const uint4 *>(static_cast<const T *>(base) + row +
                                                                 part * V)
                              : make_uint4(0, 0, 0, 0);
            } else {
                pre_s[k] = ok ? to_f32(static_cast<const T *>(base)[row + part]) : 0.0f;
            }
        }
    }

    // With the exact zero-order hold, B is staged as B_n / (n + 1) (the kernels' form
    // of Bbar divides by A_n = (n + 1) A_0; see main_tile); in log2 units as ln 2 B_n,
    // so that (L u)(ln 2 B) = Delta u B.
    __device__ void store_bc(char *slot) const {
        constexpr bool LU = lu_mode<T, ZOH>();
#pragma unroll
        for (int k = 0; k < kBCPer; ++k) {
            const int i = tid + k * NTHR;
            if (i >= kBCUnits) continue;
            const int part = i % kBCRow;
            const int r = (i / kBCRow) % kTile;
            const int which = (i / (kBCRow * kTile)) % 2;
            const int dir = i / (kBCRow * kTile * 2);
            float *dst = S::bc(slot, dir, which) + r * N;
            if constexpr (VEC_BC) {
                float f[V];
                unpack16(pre_v[k], f);
                if (ZOH && which == 0) {
#pragma unroll
                    for (int e = 0; e < V; ++e) f[e] *= __frcp_rn((float)(part * V + e + 1));
                }
                if (LU && which == 0) {
#pragma unroll
                    for (int e = 0; e < V; ++e) f[e] *= kLn2;
                }
                float4 *d4 = reinterpret_cast<float4 *>(dst + part * V);
#pragma unroll
                for (int q = 0; q < V / 4; ++q)
                    d4[q] = make_float4(f[4 * q], f[4 * q + 1], f[4 * q + 2], f[4 * q + 3]);
            } else {
                dst[part] = (ZOH && which == 0) ? pre_s[k] * __frcp_rn((float)(part + 1))
                            : (LU && which == 0) ? pre_s[k] * kLn2 : pre_s[k];
            }
        }
    }
};

// ----------------------------------------------------------------------------
// per-thread parameters of one (channel, direction)
// ----------------------------------------------------------------------------
template <int N>
struct ChannelParams {
    const float *A;     // A[dir][d][:] (general-A path)
    float A0;           // A[d][0] times log2(e) (natural units) or 1 (log2 units)
    float emul;         // the same factor for the general-A path
    float a0, inv_a0;   // A[d][0] and its reciprocal (0 when A[d][0] = 0)
    float D, bias;
    float cw_prev, cw_cur, cw_next, cbias;   // convolution front: taps on x[t-1], x[t], x[t+1]
    float dtw;          // dt_proj weight of the channel (step input mode)
    bool structured;    // A[d][n] == (n+1) A[d][0] for every n
    bool valid;

    // LU: Delta in log2 units; the bias and dt_proj weight are then scaled by log2 e
    template <bool LU = false>
    __device__ void load(const PairArgs &p, int dir, int d) {
        valid = d < p.Di;
        structured = true;
        emul = LU ? 1.0f : kLog2e;
        A0 = D = bias = a0 = inv_a0 = 0.0f;
        cw_prev = cw_cur = cw_next = cbias = dtw = 0.0f;
        A = p.A;
        if (!valid) return;
        if (p.conv_w) {
            // forward: w[0] x[t-1] + w[1] x[t] + w[2] x[t+1]; the backward pathway
            // convolves the reversed sequence: w[0] x[t+1] + w[1] x[t] + w[2] x[t-1]
            const float *w = p.conv_w + ((size_t)dir * p.Di + d) * 3;
            cw_prev = dir ? w[2] : w[0];
            cw_cur = w[1];
            cw_next = dir ? w[0] : w[2];
            cbias = p.conv_b[(size_t)dir * p.Di + d];
        }
        if (p.dt_w) dtw = p.dt_w[(size_t)dir * p.Di + d] * (LU ? kLog2e : 1.0f);
        A = p.A + ((size_t)dir * p.Di + d) * N;
        a0 = A[0];
#pragma unroll
        for (int n = 0; n < N; ++n) structured = structured && (A[n] == (float)(n + 1) * a0);
        A0 = a0 * emul;
        inv_a0 = a0 != 0.0f ? 1.0f / a0 : 0.0f;
        D = p.D[(size_t)dir * p.Di + d];
        bias = p.bias[(size_t)dir * p.Di + d] * (LU ? kLog2e : 1.0f);
    }
};

// row of the tile that step i of a walk over it visits (ascending or descending)
template <bool DESC>
__device__ __forceinline__ int walk_row(int i) { return DESC ? kTile - 1 - i : i; }

// u of one staged row: the input itself, or, with the convolution front, silu of the
// kernel-3 convolution of the staged x rows around it (section "2. The Bidirectional
// Mamba Block": "1D Conv -> SiLU" on each pathway)
template <typename T, int N, bool CONV>
__device__ __forceinline__ float u_of(const T *su, int r, int dl, const ChannelParams<N> &prm) {
    if constexpr (!CONV) {
        return to_f32(su[r * kDC + dl]);
    } else {
        const float v = fmaf(prm.cw_prev, to_f32(su[r * kDC + dl]),
                             fmaf(prm.cw_cur, to_f32(su[(r + 1) * kDC + dl]),
                                  fmaf(prm.cw_next, to_f32(su[(r + 2) * kDC + dl]), prm.cbias)));
        return silu(v);
    }
}

// Delta of one staged row (rows past the tile end hold delta_raw = -1e4: Delta = 0).
// In the step-input mode (DT) the row holds the token's x_proj step input s, and
// delta_raw = s * dt_w[d] (dt_proj); rows past the data hold NaN and give Delta = 0.
// With LU the result is in log2 units (bias and dtw prescaled by log2 e).
template <typename T, bool DT, bool LU = false>
__device__ __forceinline__ float delta_at(const void *sd, int r, int dl, float bias, float dtw) {
    if constexpr (DT) {
        const float s = static_cast<const float *>(sd)[r];
        if constexpr (LU) return s == s ? softplus_l2(fmaf(s, dtw, bias)) : 0.0f;
        else return s == s ? softplus_io<T>(fmaf(s, dtw, bias)) : 0.0f;
    } else if constexpr (LU) {
        return softplus_l2(fmaf(to_f32(static_cast<const T *>(sd)[r * kDC + dl]), kLog2e, bias));
    } else {
        return softplus_io<T>(to_f32(static_cast<const T *>(sd)[r * kDC + dl]) + bias);
    }
}

// ----------------------------------------------------------------------------
// kernel 1: chunk summaries (end state from h = 0, and the total Delta)
// ----------------------------------------------------------------------------
// Each direction walks its chunk in the reverse of its own visiting order and
// accumulates H_n = sum_s exp(A_n * S_s) * Delta_s * u_s * B_sn, where S_s is the
// Delta summed over the tokens the direction visits after s inside the chunk.  With
// A_n = (n+1) A_0 the weights are powers of w = exp(A_0 S_s), built by one multiply
// per state.
// The h-independent values of sub-batch `sub` of a summary walk (see carry_tile); S
// enters as the Delta walked before the sub-batch, and the Delta after it is returned.
template <typename T, int N, bool FAST, bool DESC, bool CONV, bool ZOH, bool DT, int KS>
__device__ __forceinline__ float carry_form(int sub, float S, float (&Sv)[KS], float (&duv)[KS],
                                            float (&qv)[ZOH ? KS : 1], const ChannelParams<N> &prm, int dl,
                                            const T *su, const void *sd) {
    constexpr int kCarrySub = KS;
    constexpr bool LU = lu_mode<T, ZOH>();
    // duv: Delta u (first-order Bbar); with the exact hold, the structured path
    // keeps kappa u with kappa = expm1(Delta A_0) / A_0 and q = exp(Delta A_0), the
    // general path u and Delta
#pragma unroll
    for (int k = 0; k < kCarrySub; ++k) {
        const int r = walk_row<DESC>(sub * kCarrySub + k);
        const float dt = delta_at<T, DT, LU>(sd, r, dl, prm.bias, prm.dtw);
        const float u = u_of<T, N, CONV>(su, r, dl, prm);
        if constexpr (!ZOH) {
            duv[k] = dt * u;
        } else if constexpr (FAST) {
            const float q = ex2(dt * prm.A0);
            const float em1 = expm1_acc(dt * prm.a0, q);
            duv[k] = u * (prm.a0 != 0.0f ? em1 * prm.inv_a0 : dt);
            qv[k] = q;
        } else {
            duv[k] = u;
            qv[k] = dt;
        }
        Sv[k] = S;             // Delta of the tokens walked before this one
        S += dt;
    }
    return S;
}

// The summary terms of the tokens of sub-batch `sub`, from their formed values.
template <typename T, int N, bool FAST, bool DESC, bool CONV, bool ZOH, bool DT, int KS>
__device__ __forceinline__ void carry_acc(int sub, const float (&Sv)[KS], const float (&duv)[KS],
                                          const float (&qv)[ZOH ? KS : 1], float2 (&H)[N / 2],
                                          const ChannelParams<N> &prm, const float *sB) {
    constexpr int NP = N / 2;
    constexpr int kCarrySub = KS;
#pragma unroll
    for (int k = 0; k < kCarrySub; ++k) {
        const int r = walk_row<DESC>(sub * kCarrySub + k);
        float2 Bv[NP];
        load_row<NP>(sB + r * N, Bv);
        if constexpr (FAST && !ZOH) {
            const float w = ex2(prm.A0 * Sv[k]);
            const float x0 = w * duv[k];
            float2 x = f2(x0, x0 * w);
            const float2 w2 = f2(w * w, w * w);
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                H[q] = fma2(x, Bv[q], H[q]);
                x = mul2(x, w2);
            }
        } else if constexpr (FAST) {
            // exact hold: state n gets w^(n+1) kappa u S_n B_n / (n+1) (B is staged
            // divided by n+1), S_n = 1 + q + ... + q^n.  W_n = w^(n+1) kappa u S_n
            // runs two states at a time: W_(n+2) = w^2 W_n + Q_n with
            // Q_n = w^2 kappa u (1+q) (wq)^(n+1).
            const float w = ex2(prm.A0 * Sv[k]);
            const float q = qv[k], ku = duv[k];
            const float c = ku * (1.0f + q);
            const float ww = w * w, wq = w * q, wqwq = wq * wq;
            float2 Wn = f2(ku * w, c * ww);
            float2 Q = f2(ww * c * wq, ww * c * wqwq);
            const float2 w2 = f2(ww, ww), wq2 = f2(wqwq, wqwq);
#pragma unroll
            for (int j = 0; j < NP; ++j) {
                H[j] = fma2(Wn, Bv[j], H[j]);
                Wn = fma2(w2, Wn, Q);
                Q = mul2(Q, wq2);
            }
        } else {
            const float2 du2 = f2(duv[k], duv[k]);
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                const float A0n = __ldg(prm.A + 2 * q), A1n = __ldg(prm.A + 2 * q + 1);
                float2 wq = f2(ex2(A0n * prm.emul * Sv[k]), ex2(A1n * prm.emul * Sv[k]));
                if constexpr (ZOH)   // gain per state, times n+1 against the staged B / (n+1)
                    wq = mul2(wq, f2(zoh_gain(qv[k], A0n) * (float)(2 * q + 1),
                                     zoh_gain(qv[k], A1n) * (float)(2 * q + 2)));
                H[q] = fma2(mul2(wq, du2), Bv[q], H[q]);
            }
        }
    }
}

template <typename T, int N, bool FAST, bool DESC, bool CONV, bool ZOH, bool DT>
__device__ __forceinline__ void carry_tile(float2 (&H)[N / 2], float &Ssum, const ChannelParams<N> &prm,
                                           int dl, const T *su, const void *sd, const float *sB) {
    constexpr int KS = ZOH ? kCarryZohSub : vimscan::kCarrySub;
    constexpr int kNSub = kTile / KS;
#pragma unroll 1
    for (int sub = 0; sub < kNSub; ++sub) {
        float Sv[KS], duv[KS], qv[ZOH ? KS : 1];
        Ssum = carry_form<T, N, FAST, DESC, CONV, ZOH, DT, KS>(sub, Ssum, Sv, duv, qv, prm, dl, su, sd);
        carry_acc<T, N, FAST, DESC, CONV, ZOH, DT, KS>(sub, Sv, duv, qv, H, prm, sB);
    }
}

// (the exact hold needs more registers per thread, so fewer CTAs per SM)
template <typename T, int N, bool VEC_BC, bool CONV, bool ZOH, bool DT = false, bool SPAN = false>
__global__ void __launch_bounds__(kThreads, ZOH ? kCarryZohMinBlocks : DT ? kCarryDtMinBlocks : kCarryMinBlocks)
    pair_carry(PairArgs p) {
    using S = Stage<T, N, CONV>;
    constexpr int NP = N / 2;
    constexpr int kSlot = S::kSlotBytes;
    extern __shared__ __align__(16) char smem[];

    // With SPAN the CTA walks p.carry_span consecutive chunks (short chunks amortise the
    // staging prologue this way) and writes each one's summary when its walk leaves it;
    // without, one chunk
    const int span = SPAN ? max(1, p.carry_span) : 1;
    const int b = blockIdx.z, c0 = blockIdx.y * span, d0 = blockIdx.x * kDC;
    const int dir = threadIdx.x / kDC, dl = threadIdx.x % kDC, d = d0 + dl;
    const int t0 = c0 * p.chunk, tc = min(span * p.chunk, p.L - t0);
    const int nT = (tc + kTile - 1) / kTile;
    const int tpc = p.chunk / kTile;   // tiles per chunk
    // the forward summary of the last chunk and the backward one of the first are unused
    auto is_active = [&](int cs) { return (dir == 0 ? (cs < p.G - 1) : (cs > 0)) && d < p.Di; };
    bool active = is_active(c0);
    constexpr bool LU = lu_mode<T, ZOH>();

    ChannelParams<N> prm;
    prm.template load<LU>(p, dir, d);
    const bool fast = __all_sync(0xffffffffu, prm.structured);

    // the forward direction walks tiles nT-1 .. 0, the backward one 0 .. nT-1
    Stager<T, N, VEC_BC, CONV, ZOH, DT> st(p, b, t0, tc, d0, threadIdx.x);
    st.issue(smem, nT - 1, 0);
    st.load_bc(nT - 1, 0);
    st.store_bc(smem);
    cp_async_wait_all();
    __syncthreads();

    float2 H[NP];
#pragma unroll
    for (int k = 0; k < NP; ++k) H[k] = f2(0.f, 0.f);
    float Ssum = 0.0f;
    auto write = [&](int cs) {
        const size_t base = (((size_t)b * p.G + cs) * 2 + dir) * p.Di + d;
        float2 *out = reinterpret_cast<float2 *>(p.hloc + base * N);
#pragma unroll
        for (int k = 0; k < NP; ++k) out[k] = H[k];
        p.ssum[base] = LU ? Ssum * kLn2 : Ssum;   // natural units
    };

    for (int s = 0; s < nT; ++s) {
        char *cur = smem + (s & 1) * kSlot;
        char *nxt = smem + ((s + 1) & 1) * kSlot;
        if (s + 1 < nT) {
            st.issue(nxt, nT - 2 - s, s + 1);
            st.load_bc(nT - 2 - s, s + 1);
        }
        const int j = dir == 0 ? nT - 1 - s : s;   // the tile this step walks
        const int cs = c0 + j / tpc;               // and its chunk
        if constexpr (SPAN) active = is_active(cs);
        if (active) {
            const T *su = S::uv(cur, dir, 0), *sd = S::uv(cur, dir, 1);
            const float *sB = S::bc(cur, dir, 0);
            if (dir == 0) {
                if (fast) carry_tile<T, N, true, true, CONV, ZOH, DT>(H, Ssum, prm, dl, su, sd, sB);
                else carry_tile<T, N, false, true, CONV, ZOH, DT>(H, Ssum, prm, dl, su, sd, sB);
            } else {
                if (fast) carry_tile<T, N, true, false, CONV, ZOH, DT>(H, Ssum, prm, dl, su, sd, sB);
                else carry_tile<T, N, false, false, CONV, ZOH, DT>(H, Ssum, prm, dl, su, sd, sB);
            }
        }
        if constexpr (SPAN) {
            // the walk leaves chunk cs after this tile: its summary, then the next from zero
            if (s < nT - 1 && (dir == 0 ? j - 1 : j + 1) / tpc != j / tpc) {
                if (active) write(cs);
#pragma unroll
                for (int k = 0; k < NP; ++k) H[k] = f2(0.f, 0.f);
                Ssum = 0.0f;
            }
        }
        if (s + 1 < nT) {
            st.store_bc(nxt);
            cp_async_wait_all();
        }
        __syncthreads();
    }
    // the chunk the walk ends in (with SPAN: the first chunk forward, the last backward)
    if constexpr (SPAN) active = is_active(dir == 0 ? c0 : c0 + (nT - 1) / tpc);
    if (active) write(dir == 0 ? c0 : c0 + (nT - 1) / tpc);
}

// ----------------------------------------------------------------------------
// kernel 2: fold the chunk summaries along each direction
// ----------------------------------------------------------------------------
// One thread per (batch, direction, channel, state).  hloc[b][c][dir][d][n] is
// replaced by the state entering chunk c in that direction's visiting order:
// H_in(next) = exp(A_n * Ssum(c)) * H_in(c) + H_loc(c).  Loads run 16 chunks ahead.
// The last chunk's summary in each direction was never formed and is not read (the
// state after the last chunk is not needed).  With fold_reverse
// each direction is folded from its last chunk to its first (the adjoint of the
// scan, whose summaries come from adj_carry).
template <int N>
__global__ void __launch_bounds__(256) pair_combine(PairArgs p) {
    constexpr int kAhead = VIMSCAN_COMBINE_AHEAD;
    // launched as a programmatic dependent of pair_carry: wait for its summaries
    cudaGridDependencySynchronize();
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;   // (b, dir, d, n), n fastest
    const int per_b = 2 * p.Di * N;
    if (idx >= p.batch * per_b) return;
    const int b = idx / per_b, rem = idx % per_b;            // rem = (dir * Di + d) * N + n
    const int dir = rem / (p.Di * N);
    const float A2n = p.A[rem] * kLog2e;                     // A is [2][Di][N]: same index
    // hloc[b][c][dir][d][n] and ssum[b][c][dir][d]: chunk c+1 lies per_b (per_b / N) further
    const bool desc = (dir != 0) != (p.fold_reverse != 0);
    const int c0 = desc ? p.G - 1 : 0;
    float *hl = p.hloc + ((size_t)b * p.G + c0) * per_b + rem;
    const float *ss = p.ssum + ((size_t)b * p.G + c0) * (per_b / N) + rem / N;
    const int hs = desc ? -per_b : per_b, sstep = desc ? -(per_b / N) : per_b / N;
    float h = 0.0f;
    for (int i0 = 0; i0 < p.G; i0 += kAhead) {
        const int cnt = min(kAhead, p.G - i0);
        float loc[kAhead], P[kAhead];
#pragma unroll
        for (int k = 0; k < kAhead; ++k) {
            loc[k] = P[k] = 0.0f;
            if (k < cnt && i0 + k < p.G - 1) {
                loc[k] = hl[k * hs];
                P[k] = ss[k * sstep];
            }
        }
#pragma unroll
        for (int k = 0; k < kAhead; ++k) P[k] = ex2(A2n * P[k]);   // exp(A_n * Ssum(c))
#pragma unroll
        for (int k = 0; k < kAhead; ++k) {
            if (k < cnt) {
                hl[k * hs] = h;                 // the state entering this chunk
                h = fmaf(P[k], h, loc[k]);      // (zero after the last chunk, unused)
            }
        }
        hl += kAhead * hs;
        ss += kAhead * sstep;
    }
}

// acc (+)= V consecutive floats (16-byte aligned), V a multiple of 4
template <int V, bool ADD>
__device__ __forceinline__ void add_f32(float (&acc)[V], const float *src) {
    const float4 *s4 = reinterpret_cast<const float4 *>(src);
#pragma unroll
    for (int q = 0; q < V / 4; ++q) {
        const float4 a = s4[q];
        if (ADD) {
            acc[4 * q] += a.x; acc[4 * q + 1] += a.y; acc[4 * q + 2] += a.z; acc[4 * q + 3] += a.w;
        } else {
            acc[4 * q] = a.x; acc[4 * q + 1] = a.y; acc[4 * q + 2] = a.z; acc[4 * q + 3] = a.w;
        }
    }
}

// ----------------------------------------------------------------------------
// kernel 3: both directions over one chunk, merge, gate, store
// ----------------------------------------------------------------------------
// One direction's pass over one staged tile: the softplus, Delta*u and decay base of
// kSub tokens are formed first (independent of h), then the recurrence runs through
// them.  Rows past the tile's end are no-op tokens.  The output of each token goes
// to the chunk's fp32 partial buffer: stored on the tile's first visit, added on the
// second (rows past the end only touch unread rows of the buffer).
//
// With structured A and the first-order Bbar, the scaled state g = h / du (du = Delta
// u, |du| kept at or above 1e-20) can be run instead of h (VIMSCAN_GF):
//     g_t = (Abar_t r_t) g_(t-1) + B_t,  r_t = du_(t-1) / du_t,  y_t = du_t C_t.g_t + D u_t,
// which drops the drive multiply du B_n of every state; dprev carries du_(t-1).
// The h-independent values of kSub tokens of sub-batch `sub` (softplus Delta, the decay
// base, Delta u), formed ahead of the recurrence that uses them.
template <typename T, int N, bool FAST, bool DESC, bool CONV, bool ZOH, bool DT>
__device__ __forceinline__ void main_form(int sub, float (&qv)[kSub], float (&duv)[kSub], float (&uv)[kSub],
                                          const ChannelParams<N> &prm, int dl, const T *su, const void *sd) {
    constexpr bool LU = lu_mode<T, ZOH>();
#pragma unroll
    for (int k = 0; k < kSub; ++k) {
        const int r = walk_row<DESC>(sub * kSub + k);
        const float dt = delta_at<T, DT, LU>(sd, r, dl, prm.bias, prm.dtw);
        uv[k] = u_of<T, N, CONV>(su, r, dl, prm);
        qv[k] = FAST ? ex2(dt * prm.A0) : dt;
        if constexpr (ZOH && FAST)
            duv[k] = uv[k] * (prm.a0 != 0.0f ? expm1_acc(dt * prm.a0, qv[k]) * prm.inv_a0 : dt);
        else
            duv[k] = dt * uv[k];
    }
}

// The recurrence over the kSub tokens of sub-batch `sub`, from their formed values.
template <typename T, int N, bool FAST, bool DESC, bool CONV, bool ZOH, bool DT>
__device__ __forceinline__ void main_recur(int sub, const float (&qv)[kSub], const float (&duv)[kSub],
                                           const float (&uv)[kSub], bool second, float2 (&h)[N / 2], float &dprev,
                                           const ChannelParams<N> &prm, const float *sB, const float *sC,
                                           float *ypart) {
    constexpr int NP = N / 2;
    constexpr bool GF = VIMSCAN_GF && FAST && !ZOH;
#pragma unroll
    for (int k = 0; k < kSub; ++k) {
        const int r = walk_row<DESC>(sub * kSub + k);
        const float4 *B4 = reinterpret_cast<const float4 *>(sB + r * N);
        const float4 *C4 = reinterpret_cast<const float4 *>(sC + r * N);
        const float2 du2 = f2(duv[k], duv[k]);
        float2 y0 = f2(0.f, 0.f), y1 = f2(0.f, 0.f);
        // decays a = (Abar_2q, Abar_2q+1): with A_n = (n+1) A_0 they are the powers
        // q^(2q+1), q^(2q+2) of q = exp(Delta A_0), one multiply per state
        const float q = qv[k];
        float2 a = FAST ? f2(q, q * q) : f2(0.f, 0.f);
        const float2 step = FAST ? f2(a.y, a.y) : f2(0.f, 0.f);
        float ysc = 1.0f;
        if constexpr (GF) {
            const float dv = clamp_du(duv[k]);
            const float rr = dprev * rcp(dv);
            dprev = dv;
            a = mul2(a, f2(rr, rr));
            ysc = dv;
        }
        // exact hold, structured A: Bbar_n u = kappa u S_n B_n / (n+1) with
        // S_n = 1 + q + ... + q^n and B staged divided by n+1; KS = kappa u S for two
        // states at a time, KS_(n+2) = KS_n + kappa u (1+q) q^(n+1)
        const float cz = (ZOH && FAST) ? duv[k] * (1.0f + q) : 0.0f;
        float2 KS = f2(duv[k], cz);
        const float2 cz2 = f2(cz, cz);
#pragma unroll
        for (int qq = 0; qq < NP; qq += 2) {
            float2 Bp[2], Cp[2];
            if constexpr (NP >= 2) {
                const float4 b4 = B4[qq / 2], c4 = C4[qq / 2];
                Bp[0] = f2(b4.x, b4.y); Bp[1] = f2(b4.z, b4.w);
                Cp[0] = f2(c4.x, c4.y); Cp[1] = f2(c4.z, c4.w);
            } else {
                Bp[0] = *reinterpret_cast<const float2 *>(sB + r * N);
                Cp[0] = *reinterpret_cast<const float2 *>(sC + r * N);
            }
#pragma unroll
            for (int e = 0; e < 2 && qq + e < NP; ++e) {
                const int qi = qq + e;
                float2 aq, drive;
                if constexpr (GF) {
                    aq = a;
                    a = mul2(a, step);
                    drive = Bp[e];
                } else if constexpr (FAST) {
                    aq = a;
                    a = mul2(a, step);
                    if constexpr (ZOH) {
                        drive = mul2(KS, Bp[e]);
                        KS = fma2(aq, cz2, KS);
                    } else {
                        drive = mul2(du2, Bp[e]);
                    }
                } else {
                    const float A0n = __ldg(prm.A + 2 * qi), A1n = __ldg(prm.A + 2 * qi + 1);
                    aq = f2(ex2(q * A0n * prm.emul), ex2(q * A1n * prm.emul));
                    if constexpr (ZOH)   // gain per state, times n+1 against the staged B / (n+1)
                        drive = mul2(mul2(f2(zoh_gain(q, A0n) * (float)(2 * qi + 1),
                                             zoh_gain(q, A1n) * (float)(2 * qi + 2)),
                                          f2(uv[k], uv[k])),
                                     Bp[e]);
                    else
                        drive = mul2(du2, Bp[e]);
                }
                h[qi] = fma2(aq, h[qi], drive);
                if (qi & 1) y1 = fma2(Cp[e], h[qi], y1);
                else y0 = fma2(Cp[e], h[qi], y0);
            }
        }
        const float2 ys = __fadd2_rn(y0, y1);
        const float yv = fmaf(ysc, ys.x + ys.y, prm.D * uv[k]);
        float *py = ypart + r * kDC;
        *py = second ? *py + yv : yv;
    }
}

template <typename T, int N, bool FAST, bool DESC, bool CONV, bool ZOH, bool DT>
__device__ __forceinline__ void main_tile(bool second, float2 (&h)[N / 2], float &dprev,
                                          const ChannelParams<N> &prm, int dl, const T *su, const void *sd,
                                          const float *sB, const float *sC, float *ypart) {
    constexpr int kNSub = kTile / kSub;
#pragma unroll 1
    for (int sub = 0; sub < kNSub; ++sub) {
        float qv[kSub], duv[kSub], uv[kSub];
        main_form<T, N, FAST, DESC, CONV, ZOH, DT>(sub, qv, duv, uv, prm, dl, su, sd);
        main_recur<T, N, FAST, DESC, CONV, ZOH, DT>(sub, qv, duv, uv, second, h, dprev, prm, sB, sC, ypart);
    }
}

// Completion of the tiles a step finishes.  A tile is complete once both directions
// have visited it; its sums sit in the chunk buffer (the middle tile of an odd tile
// count keeps the backward half in ymid).  Each thread finishes one 8-channel vector
// of one row per completed tile: it adds partial_in (the first pair's sum, for the
// second pair of the cross-scan), applies silu(z) and stores 16 or 32 bytes; the first
// pair of the cross-scan stores its ungated fp32 sum instead.  z and partial_in are
// loaded into registers at the start of the step, so their latency hides behind it.
template <typename T, bool PIN, int NTHR = kThreads>
struct Finisher {
    static constexpr int kG = 8;                                    // channels per vector
    static constexpr int kZ = kG * (int)sizeof(T) / 16;             // uint4 of z per vector
    static constexpr int kItems = kTile * (kDC / kG);               // vectors per tile
    static constexpr int kIPT = kItems / NTHR;                      // vectors per thread per tile
    static_assert(kItems % NTHR == 0, "a tile's vectors split evenly over the finishing threads");
    uint4 z[2][kIPT][kZ];
    float4 pin[2][kIPT][PIN ? 2 : 1];
    int ntiles, tile[2];
    int tid;   // this thread's index among the NTHR finishing threads

    __device__ explicit Finisher(int tid_) : ntiles(0), tid(tid_) {}
    __device__ int row(int m) const { return (tid + m * NTHR) / (kDC / kG); }
    __device__ int group(int m) const { return (tid + m * NTHR) % (kDC / kG); }

    // the tiles completed by step s (none before the middle of the chunk)
    __device__ void plan(int s, int nT) {
        ntiles = 0;
        if (2 * s < nT - 1) return;
        tile[0] = s;
        tile[1] = nT - 1 - s;
        ntiles = tile[0] == tile[1] ? 1 : 2;
    }

    template <class ST>
    __device__ void prefetch(const ST &st, const PairArgs &p) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            if (i >= ntiles) break;
            const int j = tile[i];
#pragma unroll
            for (int m = 0; m < kIPT; ++m) {
                const int r = row(m), ch = st.d0 + group(m) * kG;
                if (r >= st.rows_of(j) || ch >= p.Di) continue;
                const size_t off = st.row_off(j, r, ch);
                if (p.z) {
                    const uint4 *zs = reinterpret_cast<const uint4 *>(static_cast<const T *>(p.z) + off);
#pragma unroll
                    for (int q = 0; q < kZ; ++q)
                        if (sizeof(T) == 2 || ch + 4 * q < p.Di) z[i][m][q] = zs[q];
                }
                if constexpr (PIN) {
                    const float4 *ps = reinterpret_cast<const float4 *>(p.partial_in + off);
                    pin[i][m][0] = ps[0];
                    if (ch + 4 < p.Di) pin[i][m][1] = ps[1];
                }
            }
        }
    }

    template <class ST>
    __device__ void finish(const ST &st, const PairArgs &p, const float *ybuf,
                           const float *ymid) const {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            if (i >= ntiles) break;
            const int j = tile[i];
#pragma unroll
            for (int m = 0; m < kIPT; ++m) {
                const int r = row(m), cl = group(m) * kG, ch = st.d0 + cl;
                if (r >= st.rows_of(j) || ch >= p.Di) continue;
                float acc[kG];
                add_f32<kG, false>(acc, ybuf + (size_t)(j * kTile + r) * kDC + cl);
                if (ntiles == 1) add_f32<kG, true>(acc, ymid + r * kDC + cl);
                if constexpr (PIN) {
                    const float4 a = pin[i][m][0], b = pin[i][m][PIN ? 1 : 0];
                    acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
                    acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
                }
                const size_t off = st.row_off(j, r, ch);
                const bool whole = ch + kG <= p.Di;   // fp32 channel counts may end half-way
                if (p.partial_out) {
                    float4 *po = reinterpret_cast<float4 *>(p.partial_out + off);
                    po[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
                    if (whole) po[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
                    continue;
                }
                if (p.z) {
                    float zf[kG];
                    if constexpr (sizeof(T) == 2) {
                        unpack16(z[i][m][0], zf);
                    } else {
                        float a4[4], b4[4];
                        unpack16(z[i][m][0], a4);
                        unpack16(z[i][m][kZ - 1], b4);
#pragma unroll
                        for (int e = 0; e < 4; ++e) { zf[e] = a4[e]; zf[4 + e] = b4[e]; }
                    }
#pragma unroll
                    for (int e = 0; e < kG; ++e) acc[e] *= silu(zf[e]);
                }
                uint4 *yo = reinterpret_cast<uint4 *>(static_cast<T *>(p.y) + off);
                if constexpr (sizeof(T) == 2) {
                    yo[0] = pack16(acc);
                } else {
                    float a4[4] = {acc[0], acc[1], acc[2], acc[3]}, b4[4] = {acc[4], acc[5], acc[6], acc[7]};
                    yo[0] = pack16(a4);
                    if (whole) yo[1] = pack16(b4);
                }
            }
        }
    }
};

template <typename T, int N, bool VEC_BC, bool PIN, bool CONV, bool ZOH, bool DT = false>
__global__ void __launch_bounds__(kThreads, kMinBlocks) pair_main(PairArgs p) {
    using S = Stage<T, N, CONV>;
    constexpr int NP = N / 2;
    constexpr int kSlot = S::kSlotBytes;
    extern __shared__ __align__(16) char smem[];
    float *ybuf = reinterpret_cast<float *>(smem + 2 * kSlot);   // [chunk][kDC]
    float *ymid = ybuf + (size_t)p.chunk * kDC;                   // [kTile][kDC]

    const int b = blockIdx.z, c = blockIdx.y, d0 = blockIdx.x * kDC;
    const int dir = threadIdx.x / kDC, dl = threadIdx.x % kDC, d = d0 + dl;
    const int t0 = c * p.chunk, tc = min(p.chunk, p.L - t0);
    const int nT = (tc + kTile - 1) / kTile;

    ChannelParams<N> prm;
    prm.template load<lu_mode<T, ZOH>()>(p, dir, d);
    const bool fast = __all_sync(0xffffffffu, prm.structured);

    Stager<T, N, VEC_BC, CONV, ZOH, DT> st(p, b, t0, tc, d0, threadIdx.x);
    st.issue(smem, 0, nT - 1);
    st.load_bc(0, nT - 1);

    // state entering this chunk.  With several chunks this kernel is launched as a
    // programmatic dependent of pair_combine (whose own predecessor, pair_carry, was an
    // ordinary launch, so the inputs were complete before the chain began): everything
    // above only reads the inputs; the carries are read after the wait.
    float2 h[NP];
#pragma unroll
    for (int k = 0; k < NP; ++k) h[k] = f2(0.f, 0.f);
    float dprev = 1.0f;   // du before the chunk's first token (scaled state: g = h_in)
    if (p.G > 1) cudaGridDependencySynchronize();
    if (p.G > 1 && (dir == 0 ? c > 0 : c < p.G - 1) && prm.valid) {
        const size_t base = (((size_t)b * p.G + c) * 2 + dir) * p.Di + d;
        const float2 *hin = reinterpret_cast<const float2 *>(p.hloc + base * N);
#pragma unroll
        for (int k = 0; k < NP; ++k) h[k] = hin[k];
    }

    st.store_bc(smem);
    cp_async_wait_all();
    __syncthreads();

    Finisher<T, PIN> fin(threadIdx.x);
    // one step of the recurrence warps: tile j = s (forward) or nT-1-s (backward) from
    // the slot `cur`; the first visitor of a tile stores its partial, the second adds to
    // it; when both come in the same step (the middle tile) the backward one writes to
    // ymid instead
    auto recur = [&](int s, char *cur) {
        const int j = dir ? nT - 1 - s : s;
        const int twice = 2 * s - (nT - 1);
        float *ypart = (twice == 0 && dir == 1) ? ymid + dl : ybuf + (size_t)j * kTile * kDC + dl;
        if (!prm.valid) return;
        if constexpr (!DT) {
            // the state entering a checkpoint segment: chunks start at multiples of
            // kCkTokens, so a segment is two tiles; the forward direction enters it at its
            // even tile, the backward one at its odd tile (or the chunk's last tile).  In
            // the scaled form the state is dprev g.
            static_assert(kCkTokens == 2 * kTile, "a checkpoint segment is two tiles");
            if (p.hck && (dir == 0 ? (j & 1) == 0 : ((j & 1) == 1 || j == nT - 1))) {
                // state-major rows: a warp's 32 channels of one state are 128 contiguous bytes
                const int seg = (t0 + j * kTile) / kCkTokens, nseg = (p.L + kCkTokens - 1) / kCkTokens;
                float *o = p.hck + (((size_t)b * nseg + seg) * 2 + dir) * N * p.Di + d;
#pragma unroll
                for (int k = 0; k < NP; ++k) {
                    o[(size_t)(2 * k) * p.Di] = h[k].x * dprev;
                    o[(size_t)(2 * k + 1) * p.Di] = h[k].y * dprev;
                }
            }
        }
        const T *su = S::uv(cur, dir, 0), *sd = S::uv(cur, dir, 1);
        const float *sB = S::bc(cur, dir, 0), *sC = S::bc(cur, dir, 1);
        const bool second = twice > 0;
        if (dir == 0) {
            if (fast) main_tile<T, N, true, false, CONV, ZOH, DT>(second, h, dprev, prm, dl, su, sd, sB, sC, ypart);
            else main_tile<T, N, false, false, CONV, ZOH, DT>(second, h, dprev, prm, dl, su, sd, sB, sC, ypart);
        } else {
            if (fast) main_tile<T, N, true, true, CONV, ZOH, DT>(second, h, dprev, prm, dl, su, sd, sB, sC, ypart);
            else main_tile<T, N, false, true, CONV, ZOH, DT>(second, h, dprev, prm, dl, su, sd, sB, sC, ypart);
        }
    };
    for (int s = 0; s < nT; ++s) {
        char *cur = smem + (s & 1) * kSlot;
        char *nxt = smem + ((s + 1) & 1) * kSlot;
        if (s + 1 < nT) {
            st.issue(nxt, s + 1, nT - 2 - s);
            st.load_bc(s + 1, nT - 2 - s);
        }
        fin.plan(s, nT);
        fin.prefetch(st, p);
        recur(s, cur);
        if (s + 1 < nT) {
            st.store_bc(nxt);
            cp_async_wait_all();
        }
        __syncthreads();
        // the tiles this step completed are read by no later step of this chunk, so
        // they can be finished while the next step runs without another barrier
        fin.finish(st, p, ybuf, ymid);
    }
}

// ----------------------------------------------------------------------------
// CS-Merge alone
// ----------------------------------------------------------------------------
struct MergeArgs {
    const void *ys;   // [4][batch][L][C] in scan order
    const void *z;    // [batch][L][C] or null
    void *y;          // [batch][L][C]
    int batch, H, W, C;
};

// scan step at which direction k visits grid position pos
__device__ __forceinline__ int merge_step(int k, int pos, int H, int W) {
    const int L = H * W;
    if (k < 2) return k == 0 ? pos : L - 1 - pos;
    const int h = pos / W, w = pos % W;
    const int t = w * H + h;
    return k == 2 ? t : L - 1 - t;
}

template <typename T>
__global__ void __launch_bounds__(256) merge4(MergeArgs a) {
    constexpr int V = Vec<T>::n;
    const int per_row = a.C / V;
    const int L = a.H * a.W;
    const int64_t items = (int64_t)a.batch * L * per_row;
    const T *ys = static_cast<const T *>(a.ys);
    const size_t dir_stride = (size_t)a.batch * L * a.C;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < items;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int v = (int)(i % per_row);
        const int64_t bp = i / per_row;
        const int pos = (int)(bp % L);
        const int b = (int)(bp / L);
        float acc[V];
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] = 0.0f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int t = merge_step(k, pos, a.H, a.W);
            float f[V];
            unpack16(*reinterpret_cast<const uint4 *>(ys + k * dir_stride + ((size_t)b * L + t) * a.C + v * V), f);
#pragma unroll
            for (int e = 0; e < V; ++e) acc[e] += f[e];
        }
        const size_t off = ((size_t)b * L + pos) * a.C + v * V;
        if (a.z) {
            float zf[V];
            unpack16(*reinterpret_cast<const uint4 *>(static_cast<const T *>(a.z) + off), zf);
#pragma unroll
            for (int e = 0; e < V; ++e) acc[e] *= silu(zf[e]);
        }
        *reinterpret_cast<uint4 *>(static_cast<T *>(a.y) + off) = pack16(acc);
    }
}

}  // namespace
}  // namespace vimscan
