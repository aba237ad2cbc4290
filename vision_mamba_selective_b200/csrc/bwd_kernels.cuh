// bwd_kernels.cuh -- sm_100a kernels of the derivative of the Vim two-direction scan.
//
// The loss's derivative dout with respect to y = (y^f + y^b) * silu(z) is carried back
// through the scan (first-order Bbar = Delta B, or with ZOH the exact hold), for every
// input: u, the raw delta, z, B, C, A, D and the delta bias.  Per direction, with g_t the adjoint of h_t
// (g_t = C_t dy_t + Abar_(t+1) g_(t+1), dy = dout * silu(z)):
//   dC_t += dy_t h_t                        dB_t += g_t Delta_t u_t
//   du_t += D dy_t + Delta_t (g_t . B_t)    dD   += dy_t u_t
//   dDelta_t = sum_n g_tn Abar_tn A_n h_(t-1)n + u_t (g_t . B_t)
//   dA_n += Delta_t g_tn Abar_tn h_(t-1)n   d delta_raw = dDelta * sigmoid(delta_raw + bias)
// and dz = dout * (y^f + y^b) * silu'(z).
//
// The sequence is cut into chunks of kBwdChunk tokens.  The state h entering each
// chunk comes from the forward scan's own summary kernels (pair_carry, pair_combine);
// the adjoint g entering each chunk from the later side comes from adj_carry plus
// pair_combine folding against the direction.  bwd_main then runs one chunk of 16
// or 32 channels, both directions: a forward sweep that keeps h every kBwdSeg tokens (in
// shared memory) and forms y (for dz) and the dC terms, then segment by segment in
// reverse a re-run of h over the segment followed by the adjoint sweep.  A thread
// holds NT (4, or 8 when built so) states of one (channel, direction), as pairs for
// the f32x2 arithmetic, so the segment's h and decays fit in registers (the
// checkpoints go to shared memory); Q = N / NT threads share a channel.  Each warp
// serves one direction, whose code is compiled separately so that its token addresses
// are constants.
// Sums over channels (dB, dC) are reduced across the warp by shuffles, a segment's
// tokens at a time (one reduce-scatter, so the shuffles are independent), then across
// the CTA's warps and directions in shared memory, and written per CTA; sums over
// tokens (dA, dD, dbias) are written per chunk.  Small reduction kernels finish both.
// Every sum is taken in a fixed order (no floating-point atomics), so results repeat
// bit for bit.
#pragma once

#include <cooperative_groups.h>

#include "scan_kernels.cuh"

namespace vimscan {

constexpr int kBwdChunk = 32;                 // tokens per chunk
constexpr int kBwdSeg = 4;                    // tokens between checkpoints of h
constexpr int kBwdNSeg = kBwdChunk / kBwdSeg;
constexpr int kAdjCh = 64;                    // channels per adj_carry CTA
#ifndef VIMSCAN_BWD_CARRY_SPAN
#define VIMSCAN_BWD_CARRY_SPAN 3
#endif
constexpr int kBwdCarrySpan = VIMSCAN_BWD_CARRY_SPAN;   // chunks per CTA of the forward summaries
constexpr int kReduceParts = 32;              // row groups of the first parameter-reduction pass
#ifndef VIMSCAN_BWD_NT
#define VIMSCAN_BWD_NT 4                         // states per thread of bwd_main (4 or 8)
#endif
#ifndef VIMSCAN_BWD_BATCH
#define VIMSCAN_BWD_BATCH 1                      // reductions batched over each segment's tokens
#endif
#ifndef VIMSCAN_BWD_RTDIR
#define VIMSCAN_BWD_RTDIR 1                      // one copy of the sweeps for both directions (bit 0:
#endif                                           // exact hold, bit 1: first order)
#ifndef VIMSCAN_BWD_MIN_WARPS
#define VIMSCAN_BWD_MIN_WARPS 16                 // resident warps per SM the register budget targets
#endif
#ifndef VIMSCAN_BWD_CHAIN
#define VIMSCAN_BWD_CHAIN 1                      // structured A: decays as powers of exp(Delta A_0)
#endif                                           // (bit 0: exact hold, bit 1: first order)

struct BwdArgs {
    const void *u, *delta, *z, *dout;   // [batch, L, Di]
    const void *B[2], *C[2];            // per direction [batch, L, N]
    const float *A, *D, *bias;          // [2][Di][N], [2][Di], [2][Di]
    void *du, *ddelta, *dz;             // [batch, L, Di] (dz null when z is)
    float *dB_part[2], *dC_part[2];     // [batch][L][ncol][N] per B/C set ([1] = [0] when shared)
    float *par;                         // per-chunk sums over tokens, one row per (batch, chunk):
                                        // [dA: 2*Di*N | dD: 2*Di | d delta_bias: 2*Di]
    const float *hin;                   // [batch][G][2][Di][N] h entering each chunk (direction order)
    float *gloc;                        // [batch][G][2][Di][N] adjoint summaries, then adjoint entering
    float *gsum;                        // [batch][G][2][Di] chunk Delta sums
    int batch, L, Di, G, nblk;
    int cl;                             // CTAs per thread-block cluster along the channel blocks (1: none)
    int ncol;                           // columns of the dB/dC partials: nblk / cl
    int separate_bc;
    int vec_io;                         // u, delta, dout, z, du, d delta_raw, dz allow vector access
    int vec_bc;                         // B and C rows move as 16-byte vectors
    int order, H, W;                    // visiting order of the pair (0: position = step;
                                        // 1: column-major on H x W, the cross-scan's second pair)
    DivInv hdiv;                        // division by H (order 1)
    int stage;                          // 0: one pair (Vim), final outputs; 1: first pair of the
                                        // cross-scan, fp32 partials to acc_*; 2: second pair, adds them
    float *acc_y, *acc_du, *acc_dd;     // [batch, L, Di] fp32 by position (stages 1 and 2)
    int64_t u_dir_stride;               // with per-direction inputs (bwd_main's U2; u is then fp32):
                                        // elements from the forward direction's u to the backward one's
    float *du2;                         // with U2: [2][batch, L, Di] fp32 dl/du_k per direction
    const float *dt_in;                 // with DT: [2][batch*L] step input per direction and position;
    const float *dt_w;                  // [2][Di] dt_proj weights: delta_raw_k = dt_in_k * dt_w_k
    float *dd2;                         // with DT: [2][batch, L, Di] fp32 dl/ddelta_raw_k per direction
    int hin_given;                      // hin holds the forward pass's checkpoints, state-major
                                        // [batch][G][2][N][Di]: no forward summaries
};

namespace {

// grid position visited at step t of the pair's forward direction
__device__ __forceinline__ int bpos(const BwdArgs &p, int t) {
    if (p.order == 0) return t;
    const int w = (int)div_by((unsigned)t, p.hdiv), h = t - w * p.H;
    return h * p.W + w;
}

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

template <typename T>
__device__ __forceinline__ float ld(const void *p, size_t i) { return to_f32(static_cast<const T *>(p)[i]); }

// four consecutive channels of an [.., Di] tensor of T (16-byte vector loads for fp32,
// 8-byte for bf16; the channel index is a multiple of 4)
template <typename T>
__device__ __forceinline__ void load4(const void *base, size_t i, bool vec, float (&f)[4]) {
    const T *s = static_cast<const T *>(base) + i;
    if (vec) {
        if constexpr (sizeof(T) == 4) {
            const float4 v = *reinterpret_cast<const float4 *>(s);
            f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
        } else {
            const uint2 v = *reinterpret_cast<const uint2 *>(s);
            f[0] = __uint_as_float(v.x << 16); f[1] = __uint_as_float(v.x & 0xffff0000u);
            f[2] = __uint_as_float(v.y << 16); f[3] = __uint_as_float(v.y & 0xffff0000u);
        }
    } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) f[e] = to_f32(s[e]);
    }
}
template <typename T>
__device__ __forceinline__ void store4(void *base, size_t i, bool vec, const float (&f)[4]) {
    T *d = static_cast<T *>(base) + i;
    if (vec) {
        if constexpr (sizeof(T) == 4) {
            *reinterpret_cast<float4 *>(d) = make_float4(f[0], f[1], f[2], f[3]);
        } else {
            __nv_bfloat162 a = __floats2bfloat162_rn(f[0], f[1]), c = __floats2bfloat162_rn(f[2], f[3]);
            *reinterpret_cast<uint2 *>(d) =
                make_uint2(*reinterpret_cast<uint32_t *>(&a), *reinterpret_cast<uint32_t *>(&c));
        }
    } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) d[e] = from_f32<T>(f[e]);
    }
}

// d softplus / dx = 1 / (1 + e^-x), and 1 above the cut at 20
__device__ __forceinline__ float softplus_grad(float x) {
    return x > 20.0f ? 1.0f : rcp(1.0f + ex2(-x * kLog2e));
}
// d silu / dz = s (1 + z (1 - s)), s = 1 / (1 + e^-z)
__device__ __forceinline__ float silu_grad(float z) {
    const float s = rcp(1.0f + ex2(-z * kLog2e));
    return s * fmaf(z, 1.0f - s, 1.0f);
}

// ----------------------------------------------------------------------------
// adjoint summaries: per chunk and direction, the adjoint a chunk passes to the one
// its direction visits before it, from zero entering the chunk:
//   G_n = sum_s exp(A_n S_s) C_sn dy_s,  S_s = Delta summed over the chunk's tokens
// visited up to and including s.  One thread per (channel, direction), all N states;
// with A_n = (n+1) A_0 (checked per warp) the weights are powers of one exp.
// ----------------------------------------------------------------------------
// DT: delta_raw of direction k is dt_in_k[t] * dt_w_k[d] (the projections' step input)
template <typename T, int N, bool DT = false>
__global__ void __launch_bounds__(2 * kAdjCh) adj_carry(BwdArgs p) {
    __shared__ __align__(16) float sDr[DT ? 1 : kBwdChunk][kAdjCh], sDy[kBwdChunk][kAdjCh];
    __shared__ __align__(16) float sC[2][kBwdChunk][N];
    __shared__ float sS[2][DT ? kBwdChunk : 1];
    const int b = blockIdx.z, c = blockIdx.y, d0 = blockIdx.x * kAdjCh;
    const int t0 = c * kBwdChunk, tc = min(kBwdChunk, p.L - t0);
    // four channels per item (d_inner is a multiple of 4)
    for (int li = threadIdx.x; li < kBwdChunk * (kAdjCh / 4); li += 2 * kAdjCh) {
        const int r = li / (kAdjCh / 4), c0 = (li % (kAdjCh / 4)) * 4, ch = d0 + c0;
        float dr[4] = {0.0f, 0.0f, 0.0f, 0.0f}, e[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        if (r < tc && ch < p.Di) {
            const size_t i = ((size_t)b * p.L + bpos(p, t0 + r)) * p.Di + ch;
            if constexpr (!DT) load4<T>(p.delta, i, p.vec_io, dr);
            load4<T>(p.dout, i, p.vec_io, e);
            if (p.z) {
                float zz[4];
                load4<T>(p.z, i, p.vec_io, zz);
#pragma unroll
                for (int k = 0; k < 4; ++k) e[k] *= silu(zz[k]);
            }
        }
        if constexpr (!DT) *reinterpret_cast<float4 *>(&sDr[r][c0]) = make_float4(dr[0], dr[1], dr[2], dr[3]);
        *reinterpret_cast<float4 *>(&sDy[r][c0]) = make_float4(e[0], e[1], e[2], e[3]);
    }
    if constexpr (DT) {
        for (int li = threadIdx.x; li < 2 * kBwdChunk; li += 2 * kAdjCh) {
            const int k = li / kBwdChunk, r = li % kBwdChunk;
            sS[k][r] = r < tc ? p.dt_in[(size_t)k * p.batch * p.L + (size_t)b * p.L + bpos(p, t0 + r)] : 0.0f;
        }
    }
    bool c_done = false;
    if constexpr ((N * sizeof(T)) % 16 == 0) {
        if (p.vec_bc) {
            constexpr int VB = 16 / (int)sizeof(T), RV = N / VB;   // states per vector, vectors per row
            for (int li = threadIdx.x; li < 2 * kBwdChunk * RV; li += 2 * kAdjCh) {
                const int k = li / (kBwdChunk * RV), r = (li / RV) % kBwdChunk, v = li % RV;
                float f[VB];
                if (r < tc) {
                    unpack16(*reinterpret_cast<const uint4 *>(static_cast<const T *>(p.C[k]) +
                                                              ((size_t)b * p.L + bpos(p, t0 + r)) * N + v * VB),
                             f);
                } else {
#pragma unroll
                    for (int e2 = 0; e2 < VB; ++e2) f[e2] = 0.0f;
                }
                float4 *dst = reinterpret_cast<float4 *>(&sC[k][r][v * VB]);
#pragma unroll
                for (int e2 = 0; e2 < VB / 4; ++e2)
                    dst[e2] = make_float4(f[4 * e2], f[4 * e2 + 1], f[4 * e2 + 2], f[4 * e2 + 3]);
            }
            c_done = true;
        }
    }
    for (int li = threadIdx.x; !c_done && li < 2 * kBwdChunk * N; li += 2 * kAdjCh) {
        const int k = li / (kBwdChunk * N), r = (li / N) % kBwdChunk, n = li % N;
        sC[k][r][n] = r < tc ? ld<T>(p.C[k], ((size_t)b * p.L + bpos(p, t0 + r)) * N + n) : 0.0f;
    }
    __syncthreads();

    const int dir = threadIdx.x / kAdjCh, dl = threadIdx.x % kAdjCh, d = d0 + dl;
    const bool valid = d < p.Di;
    constexpr int NP = N / 2;
    const float *Ad = p.A + ((size_t)dir * p.Di + (valid ? d : 0)) * N;
    bool structured = true;
#pragma unroll
    for (int n = 0; n < N; ++n) structured = structured && (Ad[n] == (float)(n + 1) * Ad[0]);
    const bool fast = __all_sync(0xffffffffu, structured);
    if (!valid) return;
    const float A0 = Ad[0] * kLog2e;
    const float bias = p.bias[(size_t)dir * p.Di + d];
    const float wdt = DT ? p.dt_w[(size_t)dir * p.Di + d] : 0.0f;
    float2 G[NP];
#pragma unroll
    for (int k = 0; k < NP; ++k) G[k] = f2(0.f, 0.f);
    float S = 0.0f;
    // a fixed trip count (tokens past the chunk add Delta = 0 and dy = 0) lets the
    // compiler overlap the independent softplus of later tokens with the chain
#pragma unroll 4
    for (int i = 0; i < kBwdChunk; ++i) {
        const bool ok = i < tc;
        const int r = ok ? (dir ? tc - 1 - i : i) : 0;
        S += ok ? softplus_io<T>((DT ? sS[dir][r] * wdt : sDr[DT ? 0 : r][dl]) + bias) : 0.0f;
        const float e = ok ? sDy[r][dl] : 0.0f;
        float2 Cv[NP];
        load_row<NP>(&sC[dir][r][0], Cv);
        if (fast) {
            // weights exp(A_n S) = w^(n+1), w = exp(A_0 S), two states at a time
            const float w = ex2(A0 * S);
            float2 x = f2(w * e, w * w * e);
            const float2 w2 = f2(w * w, w * w);
#pragma unroll
            for (int k = 0; k < NP; ++k) {
                G[k] = fma2(x, Cv[k], G[k]);
                x = mul2(x, w2);
            }
        } else {
#pragma unroll
            for (int k = 0; k < NP; ++k)
                G[k] = fma2(f2(ex2(Ad[2 * k] * kLog2e * S) * e, ex2(Ad[2 * k + 1] * kLog2e * S) * e), Cv[k], G[k]);
        }
    }
    const size_t base = (((size_t)b * p.G + c) * 2 + dir) * p.Di + d;
    float2 *out = reinterpret_cast<float2 *>(p.gloc + base * N);
#pragma unroll
    for (int k = 0; k < NP; ++k) out[k] = G[k];
    p.gsum[base] = S;
}

// Sum over the channels of one warp (one direction) of v[0..NT) for every state:
// lanes are (channel, quarter) with quarter fastest, Q quarters per channel.  The
// values are halved at each step while more than one remains (each lane keeps the
// half its lane bit selects), then summed.  On return v[0] is the sum for state
// q*NT + *off over the warp's channels, valid where *writer.
template <int NT, int Q, int CW>
__device__ __forceinline__ void reduce_channels(float (&v)[NT], int lane, int *off, bool *writer) {
    int k = NT, o = 0;
    bool w = true;
#pragma unroll
    for (int s = Q; s < Q * CW; s <<= 1) {
        const bool hi = (lane & s) != 0;
        if (k > 1) {
            const int half = k / 2;
#pragma unroll
            for (int i = 0; i < NT / 2; ++i) {
                if (i < half) {
                    const float send = hi ? v[i] : v[i + half];
                    const float keep = hi ? v[i + half] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
                }
            }
            o += hi ? half : 0;
            k = half;
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], s);
            w = w && !hi;
        }
    }
    *off = o;
    *writer = w && k == 1;
}

// Reduce-scatter of V values over the lanes whose index bits are S0, 2 S0, .. below S1:
// at each bit the lane keeps the half of its values that the bit selects and adds
// its partner's copy of that half.  On return v[0 ..) hold the sums of the values
// that had indices off, off + 1, .. (off returned).
template <int V, int S0, int S1>
__device__ __forceinline__ int reduce_scatter(float (&v)[V], int lane) {
    int k = V, off = 0;
#pragma unroll
    for (int s = S0; s < S1; s <<= 1) {
        const bool hi = (lane & s) != 0;
        const int half = k / 2;
#pragma unroll
        for (int i = 0; i < V / 2; ++i) {
            if (i < half) {
                const float send = hi ? v[i] : v[i + half];
                const float keep = hi ? v[i + half] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
            }
        }
        off += hi ? half : 0;
        k = half;
    }
    return off;
}

// ----------------------------------------------------------------------------
// the derivative over one chunk of CH channels, both directions
// ----------------------------------------------------------------------------
template <int N> struct BwdShape {
    static constexpr int NT = N < VIMSCAN_BWD_NT ? N : VIMSCAN_BWD_NT;   // states per thread
    static constexpr int NP = NT / 2;                        // state pairs per thread (f32x2 arithmetic)
    static constexpr int CKW = (NT + 3) / 4;                 // float4 per checkpoint per thread
    static constexpr int Q = N / NT;                         // threads per (channel, direction)
    static constexpr int CH = 32 / Q > 16 ? 32 / Q : 16;     // channels per CTA (whole warps per direction)
    static constexpr int kThr = 2 * CH * Q;
    static constexpr int WPD = CH * Q / 32;                  // warps per direction
    static constexpr int CW = 32 / Q;                        // channels per warp
    static constexpr int kMinBlocks = VIMSCAN_BWD_MIN_WARPS * 32 / kThr;
    static constexpr int TC = kBwdChunk;
    // with 4 lanes of 4 states per channel the shuffle reductions of a segment's tokens
    // are taken together (reduce-scatter: independent shuffles, one store per lane)
    static constexpr bool BATCH = Q == 4 && NT == 4 && VIMSCAN_BWD_BATCH;
    // shared memory, in floats (every row of the chunk):
    //   tok [TC][CH] float2 {u, dy}
    //   dsg [2][TC][CH] float2 {Delta^k, sigmoid(delta_raw + bias^k)}
    //   yb  [2][TC][CH]  y^k in the forward sweep, then du^k in the adjoint sweep
    //   dd  [2][TC][CH]  d delta_raw from direction k
    //   dzf [TC][CH]     dout silu'(z), dz's factor of y
    //   B, C [2][TC][N]
    //   red [2][WPD][TC][N]  per direction and warp: the dC terms, then the dB terms
    //   ck  [kBwdNSeg][CKW][kThr] float4  h at every kBwdSeg-th token, per thread
    static constexpr int oTok = 0;
    static constexpr int oSig = oTok + TC * CH * 2;
    static constexpr int oYb = oSig + 2 * TC * CH * 2;
    static constexpr int oDd = oYb + 2 * TC * CH;
    static constexpr int oDz = oDd + 2 * TC * CH;
    static constexpr int oB = oDz + TC * CH;
    static constexpr int oC = oB + 2 * TC * N;
    static constexpr int oRed = oC + 2 * TC * N;
    static constexpr int oCk = oRed + 2 * WPD * TC * N;
    static constexpr int kFloats = oCk + kBwdNSeg * CKW * kThr * 4;
    static constexpr size_t kSmemBytes = (size_t)kFloats * 4;
    static_assert(oCk % 4 == 0 && oB % 4 == 0 && oC % 4 == 0 && oRed % 4 == 0 && oYb % 4 == 0 && oDd % 4 == 0 &&
                      oDz % 4 == 0 && CH % 4 == 0,
                  "float4 areas must be 16-byte aligned");
    static_assert(oSig % 2 == 0, "float2 areas must be 8-byte aligned");
    static_assert(NT % 2 == 0, "states per thread come in pairs");
};

template <int N>
struct BwdSmem {
    using SH = BwdShape<N>;
    float2 *tok, *dsg;
    float *yb, *dd, *dzf, *B, *C, *red;
    float4 *ck;
    __device__ explicit BwdSmem(float *base)
        : tok(reinterpret_cast<float2 *>(base + SH::oTok)), dsg(reinterpret_cast<float2 *>(base + SH::oSig)),
          yb(base + SH::oYb), dd(base + SH::oDd), dzf(base + SH::oDz), B(base + SH::oB), C(base + SH::oC), red(base + SH::oRed),
          ck(reinterpret_cast<float4 *>(base + SH::oCk)) {}
};

// per-thread identity and parameters of one (channel, direction, state group)
template <int N>
struct BwdThread {
    using SH = BwdShape<N>;
    int tid, lane, q, cl, dir, wid, j0, d;
    bool valid;
    float2 A2[SH::NP], Araw[SH::NP];   // A of the thread's states, times log2(e) and as given
    float2 invA[SH::NP];               // 1 / A_n (0 where A_n = 0), for the exact hold
    float2 w1[SH::NP];                 // 1 / ((n + 1) A_0) of the thread's states (0 when A_0 = 0)
    float a0;                          // A_0 of the channel
    bool structured;                   // A_n = (n + 1) A_0 for every state of the channel
    float Dk;
    size_t cbase;   // [b][c][dir][d]
};

// The exact hold's gain of one state, e = Bbar_n / B_n = (exp(z) - 1) / A_n with
// z = Delta A_n, and its A-derivative, from z and Abar_n = exp(z) already formed:
//   e       = Delta sum_{k>=0} z^k / (k+1)!            (Delta at A_n = 0)
//   de/dA_n = (Delta Abar_n - e) / A_n = Delta^2 sum_{k>=1} k z^(k-1) / (k+1)!
// (de/dDelta = Abar_n).  For |z| < 1/2 the series to z^7 (first omitted term below
// 2e-8 of the sum), elsewhere the closed forms, which lose at most a few units of
// rounding there.
__device__ __forceinline__ float hold_gain(float dl, float z, float abar, float inv_a) {
    if (fabsf(z) < 0.5f) {
        float q = fmaf(z, 1.0f / 40320.0f, 1.0f / 5040.0f);
        q = fmaf(z, q, 1.0f / 720.0f);
        q = fmaf(z, q, 1.0f / 120.0f);
        q = fmaf(z, q, 1.0f / 24.0f);
        q = fmaf(z, q, 1.0f / 6.0f);
        q = fmaf(z, q, 0.5f);
        q = fmaf(z, q, 1.0f);
        return dl * q;
    }
    return (abar - 1.0f) * inv_a;
}
__device__ __forceinline__ float hold_gain_dA(float dl, float z, float abar, float inv_a, float e) {
    if (fabsf(z) < 0.5f) {
        float q = fmaf(z, 1.0f / 45360.0f, 1.0f / 5760.0f);
        q = fmaf(z, q, 1.0f / 840.0f);
        q = fmaf(z, q, 1.0f / 144.0f);
        q = fmaf(z, q, 1.0f / 30.0f);
        q = fmaf(z, q, 1.0f / 8.0f);
        q = fmaf(z, q, 1.0f / 3.0f);
        q = fmaf(z, q, 0.5f);
        return dl * dl * q;
    }
    return fmaf(dl, abar, -e) * inv_a;
}
__device__ __forceinline__ float2 hold_gain2(float dl, float2 z, float2 abar, float2 inv_a) {
    return f2(hold_gain(dl, z.x, abar.x, inv_a.x), hold_gain(dl, z.y, abar.y, inv_a.y));
}

// The exact hold's gains (and with DA their A-derivatives) of the thread's states when
// A_n = (n + 1) A_0, from one evaluation per token instead of one per state.  With
// z = Delta A_0, q = exp(z), z_n = (n + 1) z, E_n = expm1(z_n) and F_n = z_n exp(z_n) - E_n:
//   e_n = E_n / ((n + 1) A_0),   de_n/dA_n = F_n / ((n + 1) A_0)^2,
//   E_(n+1) = q E_n + E_0,       F_(n+1) = q F_n + z (E_(n+1) - z chi(z)),
// (E_0 = expm1(z), the gain recurrence's constant term)
// chi(z) = (phi(z) - 1) / z, phi(z) = expm1(z) / z.  Every step adds terms of one sign
// (no cancellation).  E and F of the thread's first state come from series (|z| < 1/2)
// or closed forms; at A_0 = 0 the limits Delta and Delta^2 / 2.
//
// q, E_0 and z chi(z) are the same for the Q lanes that share a channel.  hold_seg forms
// them once per segment, token m by lane m mod Q of the channel, and hold_states takes
// token m's by a shuffle from that lane (every lane of the warp takes part).
template <int N, bool DA>
struct HoldSeg {
    static constexpr int K = kBwdSeg / BwdShape<N>::Q;   // tokens of the segment per lane
    float q[K], e0[K], zc[DA ? K : 1];
};
template <int N, bool DA>
__device__ __forceinline__ HoldSeg<N, DA> hold_seg(const BwdSmem<N> &sm, const BwdThread<N> &th, int DIR, int sg) {
    using SH = BwdShape<N>;
    static_assert(kBwdSeg % SH::Q == 0, "a segment's tokens split evenly over a channel's lanes");
    HoldSeg<N, DA> s;
#pragma unroll
    for (int k = 0; k < HoldSeg<N, DA>::K; ++k) {
        const int i = sg * kBwdSeg + th.q + k * SH::Q, r = DIR ? SH::TC - 1 - i : i;
        const float dl = reinterpret_cast<const float *>(sm.dsg)[2 * ((DIR * SH::TC + r) * SH::CH + th.cl)];
        const float z = dl * th.a0;
        s.q[k] = ex2(z * kLog2e);
        s.e0[k] = expm1_acc(z, s.q[k]);
        if constexpr (DA) {
            // z chi(z) = phi(z) - 1 = sum_(k>=1) z^k / (k+1)!, or expm1(z) / z - 1
            float ch = fmaf(z, 1.0f / 362880.0f, 1.0f / 40320.0f);
            ch = fmaf(z, ch, 1.0f / 5040.0f);
            ch = fmaf(z, ch, 1.0f / 720.0f);
            ch = fmaf(z, ch, 1.0f / 120.0f);
            ch = fmaf(z, ch, 1.0f / 24.0f);
            ch = fmaf(z, ch, 1.0f / 6.0f);
            ch = fmaf(z, ch, 0.5f);
            s.zc[k] = fabsf(z) < 0.5f ? z * ch : s.e0[k] / z - 1.0f;
        }
    }
    return s;
}
template <int N>
__device__ __forceinline__ float hold_take(const BwdThread<N> &th, const float (&v)[HoldSeg<N, false>::K], int m) {
    constexpr int Q = BwdShape<N>::Q;
    if constexpr (Q == 1) return v[m];
    else return __shfl_sync(0xffffffffu, v[m / Q], (th.lane & ~(Q - 1)) | (m % Q));
}

template <int N, bool DA, bool SDA>
__device__ __forceinline__ void hold_states(const BwdThread<N> &th, float dl, float q,
                                            const float2 (&ab)[BwdShape<N>::NP], const HoldSeg<N, SDA> &hs, int m,
                                            float2 (&gn)[BwdShape<N>::NP], float2 (&dg)[BwdShape<N>::NP]) {
    using SH = BwdShape<N>;
    constexpr int NP = SH::NP, NT = SH::NT;
    static_assert(SDA || !DA, "the A-derivative needs the segment's z chi(z)");
    const float e0 = hold_take<N>(th, hs.e0, m);
    float zc = 0.0f;
    if constexpr (DA) zc = hold_take<N>(th, hs.zc, m);
    if (th.a0 == 0.0f) {
#pragma unroll
        for (int k = 0; k < NP; ++k) {
            gn[k] = f2(dl, dl);
            if constexpr (DA) dg[k] = f2(0.5f * dl * dl, 0.5f * dl * dl);
        }
        return;
    }
    const float z = dl * th.a0;
    const float zj = (float)(th.j0 + 1) * z;   // the thread's first state; exp(zj) = ab[0].x
    float E = expm1_acc(zj, ab[0].x);
    float F = 0.0f;
    if constexpr (DA) {
        // F at zj: zj^2 psi(zj), psi(x) = sum_k k x^(k-1) / (k+1)!, or zj exp(zj) - E
        float ps = fmaf(zj, 1.0f / 45360.0f, 1.0f / 5760.0f);
        ps = fmaf(zj, ps, 1.0f / 840.0f);
        ps = fmaf(zj, ps, 1.0f / 144.0f);
        ps = fmaf(zj, ps, 1.0f / 30.0f);
        ps = fmaf(zj, ps, 1.0f / 8.0f);
        ps = fmaf(zj, ps, 1.0f / 3.0f);
        ps = fmaf(zj, ps, 0.5f);
        F = fabsf(zj) < 0.5f ? zj * zj * ps : fmaf(zj, ab[0].x, -E);
    }
    float ev[NT], fv[NT];
#pragma unroll
    for (int i = 0; i < NT; ++i) {
        ev[i] = E;
        if constexpr (DA) fv[i] = F;
        if (i + 1 < NT) {
            const float En = fmaf(q, E, e0);
            if constexpr (DA) F = fmaf(q, F, z * (En - zc));
            E = En;
        }
    }
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        const float2 w = th.w1[k];
        gn[k] = mul2(f2(ev[2 * k], ev[2 * k + 1]), w);
        if constexpr (DA) dg[k] = mul2(mul2(f2(fv[2 * k], fv[2 * k + 1]), w), w);
    }
}

// q = exp(Delta A_0) of a segment's tokens for the first-order structured-A decays,
// formed as hold_seg forms it: token m by lane m mod Q of the channel, taken by the
// others with hold_take.
template <int N>
struct QSeg {
    float q[HoldSeg<N, false>::K];
};
template <int N>
__device__ __forceinline__ QSeg<N> q_seg(const BwdSmem<N> &sm, const BwdThread<N> &th, int DIR, int sg) {
    using SH = BwdShape<N>;
    QSeg<N> s;
#pragma unroll
    for (int k = 0; k < HoldSeg<N, false>::K; ++k) {
        const int i = sg * kBwdSeg + th.q + k * SH::Q, r = DIR ? SH::TC - 1 - i : i;
        const float dl = reinterpret_cast<const float *>(sm.dsg)[2 * ((DIR * SH::TC + r) * SH::CH + th.cl)];
        s.q[k] = ex2(dl * th.a0 * kLog2e);
    }
    return s;
}

// Abar_n = exp(Delta A_n) of the thread's states at one token.  With structured A
// (A_n = (n + 1) A_0 for the channel, CHAIN) the first state's exp(Delta A_j0) and then
// powers of q = exp(Delta A_0): one exp2 and one multiply per state pair instead of one
// exp2 per state.  Otherwise one exp2 per state.
template <int N, bool CHAIN>
__device__ __forceinline__ void state_decays(const BwdThread<N> &th, float dl, float q,
                                             float2 (&ab)[BwdShape<N>::NP]) {
    constexpr int NP = BwdShape<N>::NP;
    if constexpr (CHAIN) {
        const float b0 = ex2(dl * th.A2[0].x);
        ab[0] = f2(b0, b0 * q);
        const float q2 = q * q;
#pragma unroll
        for (int k = 1; k < NP; ++k) ab[k] = mul2(ab[k - 1], f2(q2, q2));
    } else {
        const float2 dl2 = f2(dl, dl);
#pragma unroll
        for (int k = 0; k < NP; ++k) {
            const float2 e = mul2(dl2, th.A2[k]);
            ab[k] = f2(ex2(e.x), ex2(e.y));
        }
    }
}

// h (or g) of the thread's states, from an fp32 row in global memory
template <int NP>
__device__ __forceinline__ void load_pairs(const float *row, float2 (&v)[NP]) {
    const float2 *r2 = reinterpret_cast<const float2 *>(row);
#pragma unroll
    for (int k = 0; k < NP; ++k) v[k] = r2[k];
}

// checkpoint of h for segment sg (float4 slots, unused lanes of the last slot zero)
template <int N>
__device__ __forceinline__ void store_ck(const BwdSmem<N> &sm, int tid, int sg, const float2 (&h)[BwdShape<N>::NP]) {
    using SH = BwdShape<N>;
#pragma unroll
    for (int w = 0; w < SH::CKW; ++w) {
        const float2 lo = h[2 * w], hi = 2 * w + 1 < SH::NP ? h[2 * w + 1 < SH::NP ? 2 * w + 1 : 0] : f2(0.f, 0.f);
        sm.ck[(sg * SH::CKW + w) * SH::kThr + tid] = make_float4(lo.x, lo.y, hi.x, hi.y);
    }
}
template <int N>
__device__ __forceinline__ void load_ck(const BwdSmem<N> &sm, int tid, int sg, float2 (&h)[BwdShape<N>::NP]) {
    using SH = BwdShape<N>;
#pragma unroll
    for (int w = 0; w < SH::CKW; ++w) {
        const float4 c4 = sm.ck[(sg * SH::CKW + w) * SH::kThr + tid];
        h[2 * w] = f2(c4.x, c4.y);
        if (2 * w + 1 < SH::NP) h[2 * w + 1 < SH::NP ? 2 * w + 1 : 0] = f2(c4.z, c4.w);
    }
}

// One token's dB (or dC) terms of this thread's states, summed over the warp's channels
// by shuffles into red_w[r][n] (red_w: this direction's and warp's slots)
template <int N>
__device__ __forceinline__ void channel_sum(const BwdThread<N> &th, float *red_w, const float2 (&v)[BwdShape<N>::NP],
                                            int r) {
    using SH = BwdShape<N>;
    float w[SH::NT];
#pragma unroll
    for (int k = 0; k < SH::NP; ++k) { w[2 * k] = v[k].x; w[2 * k + 1] = v[k].y; }
    int off;
    bool wr;
    reduce_channels<SH::NT, SH::Q, SH::CW>(w, th.lane, &off, &wr);
    if (wr) red_w[r * N + th.j0 + off] = w[0];
}

// forward sweep of direction DIR: checkpoints, y^DIR (ungated) and the dC terms
// (ZOH: the exact hold's Bbar in the state update; FAST: structured A, the decays from
// state_decays' power chain and the exact hold's gains from hold_states)
// u of token row r for direction DIR: the shared u, or with U2 the backward
// direction's own (staged in the dz-factor area, which U2 does not use)
template <int N, bool U2>
__device__ __forceinline__ float u_of_dir(const BwdSmem<N> &sm, int DIR, int r, int cl, float shared_u) {
    if constexpr (U2) return DIR ? sm.dzf[r * BwdShape<N>::CH + cl] : shared_u;
    else return shared_u;
}

template <int N, int DIRT, bool ZOH, bool FAST, bool U2>
__device__ __forceinline__ void bwd_forward(const BwdArgs &p, const BwdSmem<N> &sm, const BwdThread<N> &th) {
    using SH = BwdShape<N>;
    constexpr int NP = SH::NP, Q = SH::Q, CH = SH::CH, TC = SH::TC;
    const int DIR = DIRT < 0 ? th.dir : DIRT;   // DIRT < 0: the direction at run time
    float *red_w = sm.red + (DIR * SH::WPD + th.wid) * TC * N;
    constexpr bool fast = ZOH && FAST;
    constexpr bool chain = FAST && ((VIMSCAN_BWD_CHAIN >> (ZOH ? 0 : 1)) & 1);
    float2 h[NP];
#pragma unroll
    for (int k = 0; k < NP; ++k) h[k] = f2(0.f, 0.f);
    if (p.G > 1 && th.valid) {
        if (p.hin_given) {   // the forward pass's checkpoints: [unit][N][Di], unit = cbase / Di
            const float *row = p.hin + (th.cbase / p.Di) * N * p.Di + th.d;
#pragma unroll
            for (int k = 0; k < NP; ++k)
                h[k] = f2(row[(size_t)(th.j0 + 2 * k) * p.Di], row[(size_t)(th.j0 + 2 * k + 1) * p.Di]);
        } else {
            load_pairs<NP>(p.hin + th.cbase * N + th.j0, h);
        }
    }
#pragma unroll 1
    for (int sg = 0; sg < kBwdNSeg; ++sg) {
        store_ck<N>(sm, th.tid, sg, h);
        [[maybe_unused]] HoldSeg<N, false> hs;
        [[maybe_unused]] QSeg<N> qs;
        if constexpr (fast) hs = hold_seg<N, false>(sm, th, DIR, sg);
        else if constexpr (chain) qs = q_seg<N>(sm, th, DIR, sg);
        float yv[kBwdSeg], vc[SH::BATCH ? kBwdSeg * SH::NT : 1];   // batched: y partials, dC terms
#pragma unroll
        for (int m = 0; m < kBwdSeg; ++m) {
            const int i = sg * kBwdSeg + m, r = DIR ? TC - 1 - i : i;
            const float2 tk0 = sm.tok[r * CH + th.cl];   // u, dy
            const float2 tk = f2(u_of_dir<N, U2>(sm, DIR, r, th.cl, tk0.x), tk0.y);
            const float dl = reinterpret_cast<const float *>(sm.dsg)[2 * ((DIR * TC + r) * CH + th.cl)];
            const float du = dl * tk.x;
            float2 Bp[NP], Cp[NP], v[NP];
            load_row<NP>(sm.B + (DIR * TC + r) * N + th.j0, Bp);
            load_row<NP>(sm.C + (DIR * TC + r) * N + th.j0, Cp);
            const float2 dl2 = f2(dl, dl), du2 = f2(du, du), dy2 = f2(tk.y, tk.y);
            float2 yp = f2(th.q == 0 ? th.Dk * tk.x : 0.0f, 0.0f);
            float2 abk[NP], gnk[NP];
            float qm = 0.0f;
            if constexpr (fast) qm = hold_take<N>(th, hs.q, m);
            else if constexpr (chain) qm = hold_take<N>(th, qs.q, m);
            state_decays<N, chain>(th, dl, qm, abk);
            if constexpr (ZOH) {
                if constexpr (fast) {
                    float2 unused[NP];
                    hold_states<N, false>(th, dl, qm, abk, hs, m, gnk, unused);
                } else {
#pragma unroll
                    for (int k = 0; k < NP; ++k) gnk[k] = hold_gain2(dl, mul2(dl2, th.Araw[k]), abk[k], th.invA[k]);
                }
            }
#pragma unroll
            for (int k = 0; k < NP; ++k) {
                const float2 ab = abk[k];
                float2 drive;
                if constexpr (ZOH) {
                    drive = mul2(mul2(gnk[k], Bp[k]), f2(tk.x, tk.x));
                } else {
                    drive = mul2(du2, Bp[k]);
                }
                h[k] = fma2(ab, h[k], drive);
                yp = fma2(Cp[k], h[k], yp);
                v[k] = mul2(dy2, h[k]);
            }
            if constexpr (SH::BATCH) {
                yv[m] = yp.x + yp.y;
#pragma unroll
                for (int k = 0; k < NP; ++k) { vc[m * SH::NT + 2 * k] = v[k].x; vc[m * SH::NT + 2 * k + 1] = v[k].y; }
            } else {
                float y = yp.x + yp.y;
#pragma unroll
                for (int s = 1; s < Q; s <<= 1) y += __shfl_xor_sync(0xffffffffu, y, s);
                if (th.q == 0) sm.yb[(DIR * TC + r) * CH + th.cl] = y;
                channel_sum<N>(th, red_w, v, r);
            }
        }
        if constexpr (SH::BATCH) {
            // y: one token of the segment per lane of the channel; dC: two terms per lane
            const int oy = reduce_scatter<kBwdSeg, 1, Q>(yv, th.lane);
            const int iy = sg * kBwdSeg + oy;
            sm.yb[(DIR * TC + (DIR ? TC - 1 - iy : iy)) * CH + th.cl] = yv[0];
            const int oc = reduce_scatter<kBwdSeg * SH::NT, Q, 32>(vc, th.lane);
            const int ic = sg * kBwdSeg + oc / SH::NT;
            *reinterpret_cast<float2 *>(red_w + (DIR ? TC - 1 - ic : ic) * N + th.j0 + oc % SH::NT) = f2(vc[0], vc[1]);
        }
    }
}

// adjoint sweep of direction DIR, segment by segment from the last: h re-run over
// the segment from its checkpoint (keeping h and the decays), then g backwards
template <int N, int DIRT, bool ZOH, bool FAST, bool U2>
__device__ __forceinline__ void bwd_adjoint(const BwdArgs &p, const BwdSmem<N> &sm, const BwdThread<N> &th) {
    using SH = BwdShape<N>;
    constexpr int NP = SH::NP, Q = SH::Q, CH = SH::CH, TC = SH::TC;
    const int DIR = DIRT < 0 ? th.dir : DIRT;   // DIRT < 0: the direction at run time
    // with Q > 1 lane q = 0 gathers du and lane q = 1 d delta_raw of the channel
    constexpr int kDdLane = Q > 1 ? 1 : 0;
    float *red_w = sm.red + (DIR * SH::WPD + th.wid) * TC * N;
    constexpr bool fast = ZOH && FAST;
    constexpr bool chain = FAST && ((VIMSCAN_BWD_CHAIN >> (ZOH ? 0 : 1)) & 1);
    float2 g[NP], dA[NP];
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        g[k] = f2(0.f, 0.f);
        dA[k] = f2(0.f, 0.f);
    }
    if (p.G > 1 && th.valid) load_pairs<NP>(p.gloc + th.cbase * N + th.j0, g);
    float dD = 0.0f, dbias = 0.0f;
#pragma unroll 1
    for (int sg = kBwdNSeg - 1; sg >= 0; --sg) {
        float2 h0[NP];
        load_ck<N>(sm, th.tid, sg, h0);
        [[maybe_unused]] HoldSeg<N, true> hs;
        [[maybe_unused]] QSeg<N> qs;
        if constexpr (fast) hs = hold_seg<N, true>(sm, th, DIR, sg);
        else if constexpr (chain) qs = q_seg<N>(sm, th, DIR, sg);
        float2 hh[kBwdSeg][NP], aa[kBwdSeg][NP];
        [[maybe_unused]] float qv[kBwdSeg];   // the exact hold's q of each token, for its second use
        // batched: [slot][du, d delta_raw] partials and [slot][state] dB terms, slot = 3 - m
        float xq[SH::BATCH ? 2 * kBwdSeg : 1], vb[SH::BATCH ? kBwdSeg * SH::NT : 1];
#pragma unroll
        for (int m = 0; m < kBwdSeg; ++m) {
            const int i = sg * kBwdSeg + m, r = DIR ? TC - 1 - i : i;
            const float u = u_of_dir<N, U2>(sm, DIR, r, th.cl, reinterpret_cast<const float *>(sm.tok)[2 * (r * CH + th.cl)]);
            const float dl = reinterpret_cast<const float *>(sm.dsg)[2 * ((DIR * TC + r) * CH + th.cl)];
            const float du = dl * u;
            float2 Bp[NP];
            load_row<NP>(sm.B + (DIR * TC + r) * N + th.j0, Bp);
            const float2 dl2 = f2(dl, dl), du2 = f2(du, du);
            float qm = 0.0f;
            if constexpr (fast) qm = hold_take<N>(th, hs.q, m);
            else if constexpr (chain) qm = hold_take<N>(th, qs.q, m);
            if constexpr (fast) qv[m] = qm;
            state_decays<N, chain>(th, dl, qm, aa[m]);
            float2 gnk[NP];
            if constexpr (ZOH) {
                if constexpr (fast) {
                    float2 unused[NP];
                    hold_states<N, false>(th, dl, qm, aa[m], hs, m, gnk, unused);
                } else {
#pragma unroll
                    for (int k = 0; k < NP; ++k) gnk[k] = hold_gain2(dl, mul2(dl2, th.Araw[k]), aa[m][k], th.invA[k]);
                }
            }
#pragma unroll
            for (int k = 0; k < NP; ++k) {
                float2 drive;
                if constexpr (ZOH) {
                    drive = mul2(mul2(gnk[k], Bp[k]), f2(u, u));
                } else {
                    drive = mul2(du2, Bp[k]);
                }
                hh[m][k] = fma2(aa[m][k], m > 0 ? hh[m > 0 ? m - 1 : 0][k] : h0[k], drive);
            }
        }
#pragma unroll
        for (int m = kBwdSeg - 1; m >= 0; --m) {
            const int i = sg * kBwdSeg + m, r = DIR ? TC - 1 - i : i;
            const float2 tk0 = sm.tok[r * CH + th.cl];                  // u, dy
            const float2 tk = f2(u_of_dir<N, U2>(sm, DIR, r, th.cl, tk0.x), tk0.y);
            const float2 ds = sm.dsg[(DIR * TC + r) * CH + th.cl];      // Delta, sigmoid
            const float dl = ds.x, sgm = ds.y, du = dl * tk.x;
            float2 Bp[NP], Cp[NP], v[NP];
            load_row<NP>(sm.B + (DIR * TC + r) * N + th.j0, Bp);
            load_row<NP>(sm.C + (DIR * TC + r) * N + th.j0, Cp);
            const float2 dl2 = f2(dl, dl), du2 = f2(du, du), dy2 = f2(tk.y, tk.y);
            float2 sA = f2(0.f, 0.f), sB = f2(0.f, 0.f), sBa = f2(0.f, 0.f);
            float2 gnk[NP], dgk[NP];
            if constexpr (ZOH) {
                if constexpr (fast) {
                    hold_states<N, true>(th, dl, qv[m], aa[m], hs, m, gnk, dgk);
                } else {
#pragma unroll
                    for (int k = 0; k < NP; ++k) {
                        const float2 zz = mul2(dl2, th.Araw[k]);
                        gnk[k] = hold_gain2(dl, zz, aa[m][k], th.invA[k]);
                        dgk[k] = f2(hold_gain_dA(dl, zz.x, aa[m][k].x, th.invA[k].x, gnk[k].x),
                                    hold_gain_dA(dl, zz.y, aa[m][k].y, th.invA[k].y, gnk[k].y));
                    }
                }
            }
#pragma unroll
            for (int k = 0; k < NP; ++k) {
                g[k] = fma2(Cp[k], dy2, g[k]);                               // dl/dh_t
                const float2 hp = m > 0 ? hh[m > 0 ? m - 1 : 0][k] : h0[k];  // h_(t-1)
                const float2 ga = mul2(aa[m][k], g[k]);
                const float2 w = mul2(ga, hp);
                dA[k] = fma2(dl2, w, dA[k]);
                sA = fma2(th.Araw[k], w, sA);
                if constexpr (ZOH) {
                    // Bbar_n = e_n B_n: du and dB take e_n for Delta, the Delta term
                    // de_n/dDelta = Abar_n, and dA_n gains g B_n u de_n/dA_n
                    const float2 gn = gnk[k], dg = dgk[k];
                    const float2 gB = mul2(g[k], Bp[k]), uu = f2(tk.x, tk.x);
                    sB = fma2(gB, gn, sB);
                    sBa = fma2(gB, aa[m][k], sBa);
                    dA[k] = fma2(mul2(gB, uu), dg, dA[k]);
                    v[k] = mul2(mul2(g[k], gn), uu);
                } else {
                    sB = fma2(g[k], Bp[k], sB);
                    v[k] = mul2(g[k], du2);
                }
                g[k] = ga;                                                   // dl/dh_(t-1) part
            }
            const float sAs = sA.x + sA.y, sBg = sB.x + sB.y;
            // this thread's share of du and d delta_raw, gathered over the Q lanes of
            // the channel: lane q = 0 ends with du, lane q = 1 with d delta_raw
            float x0, x1;
            if constexpr (ZOH) {
                x0 = sBg;
                x1 = fmaf(tk.x, sBa.x + sBa.y, sAs) * sgm;
            } else {
                x0 = dl * sBg;
                x1 = fmaf(tk.x, sBg, sAs) * sgm;
            }
            if constexpr (SH::BATCH) {
                const int sl = kBwdSeg - 1 - m;
                xq[2 * sl] = x0;
                xq[2 * sl + 1] = x1;
#pragma unroll
                for (int k = 0; k < NP; ++k) { vb[sl * SH::NT + 2 * k] = v[k].x; vb[sl * SH::NT + 2 * k + 1] = v[k].y; }
                continue;
            }
            if constexpr (Q > 1) {
                const bool odd = (th.q & 1) != 0;
                const float send = odd ? x0 : x1;
                float keep = odd ? x1 : x0;
                keep += __shfl_xor_sync(0xffffffffu, send, 1);
#pragma unroll
                for (int s = 2; s < Q; s <<= 1) keep += __shfl_xor_sync(0xffffffffu, keep, s);
                x0 = keep;
                x1 = keep;
            }
            if (th.q == 0) {
                sm.yb[(DIR * TC + r) * CH + th.cl] = fmaf(th.Dk, tk.y, x0);
                dD = fmaf(tk.y, tk.x, dD);
            }
            if (th.q == kDdLane) {
                sm.dd[(DIR * TC + r) * CH + th.cl] = x1;
                dbias += x1;
            }
            channel_sum<N>(th, red_w, v, r);
        }
        if constexpr (SH::BATCH) {
            // du and d delta_raw of one token of the segment per lane of the channel
            const int ox = reduce_scatter<2 * kBwdSeg, 1, Q>(xq, th.lane);
            const int ix = sg * kBwdSeg + kBwdSeg - 1 - ox / 2, rx = DIR ? TC - 1 - ix : ix;
            const float2 tk0 = sm.tok[rx * CH + th.cl];   // u, dy
            const float2 tk = f2(u_of_dir<N, U2>(sm, DIR, rx, th.cl, tk0.x), tk0.y);
            sm.yb[(DIR * TC + rx) * CH + th.cl] = fmaf(th.Dk, tk.y, xq[0]);
            sm.dd[(DIR * TC + rx) * CH + th.cl] = xq[1];
            dD = fmaf(tk.y, tk.x, dD);
            dbias += xq[1];
            const int ob = reduce_scatter<kBwdSeg * SH::NT, Q, 32>(vb, th.lane);
            const int ib = sg * kBwdSeg + kBwdSeg - 1 - ob / SH::NT;
            *reinterpret_cast<float2 *>(red_w + (DIR ? TC - 1 - ib : ib) * N + th.j0 + ob % SH::NT) = f2(vb[0], vb[1]);
        }
    }
    if constexpr (SH::BATCH) {
        // every lane of the channel summed its own tokens
#pragma unroll
        for (int s = 1; s < Q; s <<= 1) {
            dD += __shfl_xor_sync(0xffffffffu, dD, s);
            dbias += __shfl_xor_sync(0xffffffffu, dbias, s);
        }
    }
    if (th.valid) {
        // row (b, c) of par; cbase = (row * 2 + dir) * Di + d
        const size_t row = th.cbase / ((size_t)2 * p.Di), col = th.cbase % ((size_t)2 * p.Di);
        float *pr = p.par + row * ((size_t)2 * p.Di * (N + 2));
        float2 *pa = reinterpret_cast<float2 *>(pr + col * N + th.j0);
#pragma unroll
        for (int k = 0; k < NP; ++k) pa[k] = dA[k];
        if (th.q == 0) pr[(size_t)2 * p.Di * N + col] = dD;
        if (th.q == kDdLane) pr[(size_t)2 * p.Di * (N + 1) + col] = dbias;
    }
}

// one sweep of the thread's direction: forward (ADJ false) or adjoint
template <int N, bool ZOH, bool FAST, bool ADJ, bool U2>
__device__ __forceinline__ void bwd_sweep(const BwdArgs &p, const BwdSmem<N> &sm, const BwdThread<N> &th) {
    if constexpr ((VIMSCAN_BWD_RTDIR >> (ZOH ? 0 : 1)) & 1) {
        if constexpr (ADJ) bwd_adjoint<N, -1, ZOH, FAST, U2>(p, sm, th);
        else bwd_forward<N, -1, ZOH, FAST, U2>(p, sm, th);
    } else if constexpr (ADJ) {
        if (th.dir == 0) bwd_adjoint<N, 0, ZOH, FAST, U2>(p, sm, th);
        else bwd_adjoint<N, 1, ZOH, FAST, U2>(p, sm, th);
    } else {
        if (th.dir == 0) bwd_forward<N, 0, ZOH, FAST, U2>(p, sm, th);
        else bwd_forward<N, 1, ZOH, FAST, U2>(p, sm, th);
    }
}

// The CTA's per-token sums over its channels of the dB (or dC) terms, from the
// per-direction, per-warp slots, into part[set][b][t][col][n]: the two directions
// add into one set when B and C are shared.  Four states at a time.  In a cluster of
// p.cl CTAs (consecutive channel blocks), the CTAs first wait for one another; then
// CTA rank r sums rows r*TC/cl .. of every CTA's slots (read through distributed
// shared memory, in rank order) into column blk / cl, and the CTAs wait again before
// any of them reuses or leaves its slots.  The order of every sum is fixed.
template <int N>
__device__ __forceinline__ void store_bc_part(const BwdArgs &p, const float *red, float *const (&part)[2], int b,
                                              int t0, int tc, int blk) {
    using SH = BwdShape<N>;
    constexpr int TC = SH::TC, V = N % 4 == 0 ? 4 : 2;
    const int nsets = p.separate_bc ? 2 : 1;
    if (p.cl > 1) {
        namespace cg = cooperative_groups;
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();
        const int rank = (int)cluster.block_rank(), rows = TC / p.cl, r0 = rank * rows;
        for (int li = threadIdx.x; li < nsets * rows * (N / V); li += SH::kThr) {
            const int k = li / (rows * (N / V)), r = r0 + (li / (N / V)) % rows, n = (li % (N / V)) * V;
            if (r >= tc) continue;
            float acc[V];
#pragma unroll
            for (int e = 0; e < V; ++e) acc[e] = 0.0f;
            for (int pr = 0; pr < p.cl; ++pr) {
                const float *peer = cluster.map_shared_rank(red, pr);
#pragma unroll
                for (int dir = 0; dir < 2; ++dir) {
                    if (p.separate_bc && dir != k) continue;
#pragma unroll
                    for (int w = 0; w < SH::WPD; ++w) {
                        const float *src = peer + ((dir * SH::WPD + w) * TC + r) * N + n;
                        if constexpr (V == 4) {
                            const float4 v4 = *reinterpret_cast<const float4 *>(src);
                            acc[0] += v4.x; acc[1] += v4.y; acc[2] += v4.z; acc[3] += v4.w;
                        } else {
                            const float2 v2 = *reinterpret_cast<const float2 *>(src);
                            acc[0] += v2.x; acc[1] += v2.y;
                        }
                    }
                }
            }
            float *dst = part[k] + (((size_t)b * p.L + bpos(p, t0 + r)) * p.ncol + blk / p.cl) * N + n;
            if constexpr (V == 4) *reinterpret_cast<float4 *>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
            else *reinterpret_cast<float2 *>(dst) = f2(acc[0], acc[1]);
        }
        cluster.sync();
        return;
    }
    for (int li = threadIdx.x; li < nsets * TC * (N / V); li += SH::kThr) {
        const int k = li / (TC * (N / V)), r = (li / (N / V)) % TC, n = (li % (N / V)) * V;
        if (r >= tc) continue;
        float acc[V];
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] = 0.0f;
#pragma unroll
        for (int dir = 0; dir < 2; ++dir) {
            if (p.separate_bc && dir != k) continue;
#pragma unroll
            for (int w = 0; w < SH::WPD; ++w) {
                const float *src = red + ((dir * SH::WPD + w) * TC + r) * N + n;
#pragma unroll
                for (int e = 0; e < V; ++e) acc[e] += src[e];
            }
        }
        float *dst = part[k] + (((size_t)b * p.L + bpos(p, t0 + r)) * p.ncol + blk) * N + n;
        if constexpr (V == 4) *reinterpret_cast<float4 *>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        else *reinterpret_cast<float2 *>(dst) = f2(acc[0], acc[1]);
    }
}

// U2: each direction scans its own u, fp32 (the backward one's at p.u +
// p.u_dir_stride), and dl/du leaves per direction in p.du2 (fp32); the Vim pair only.
// DT: delta_raw of direction k is p.dt_in_k[t] * p.dt_w_k[d], and dl/ddelta_raw leaves
// per direction in p.dd2 (fp32) instead of summed into p.ddelta.
template <typename T, int N, bool ZOH, bool U2 = false, bool DT = false>
__global__ void __launch_bounds__(BwdShape<N>::kThr, BwdShape<N>::kMinBlocks) bwd_main(BwdArgs p) {
    using SH = BwdShape<N>;
    constexpr int NP = SH::NP, Q = SH::Q, CH = SH::CH, TC = SH::TC;
    constexpr int kG = 4;   // channels per staged or stored group (d_inner is a multiple of 4)
    extern __shared__ __align__(16) float smem_f[];
    const BwdSmem<N> sm(smem_f);

    const int b = blockIdx.z, c = blockIdx.y, blk = blockIdx.x, d0 = blk * CH;
    const int t0 = c * TC, tc = min(TC, p.L - t0);
    const bool vio = p.vec_io != 0;

    // ---- stage the chunk: {u, dy} and per direction {Delta, sigmoid} per (token,
    // channel), four channels per item; B and C rows ------------------------------------
    for (int li = threadIdx.x; li < TC * (CH / kG); li += SH::kThr) {
        const int r = li / (CH / kG), c0 = (li % (CH / kG)) * kG, ch = d0 + c0;
        const bool ok = r < tc && ch < p.Di;
        float u[kG], dr[kG], e[kG], zf[kG];
#pragma unroll
        for (int k = 0; k < kG; ++k) { u[k] = 0.0f; dr[k] = 0.0f; e[k] = 0.0f; zf[k] = 0.0f; }
        if (ok) {
            const size_t i = ((size_t)b * p.L + bpos(p, t0 + r)) * p.Di + ch;
            if constexpr (U2) load4<float>(p.u, i, true, u);   // fp32 pathway inputs
            else load4<T>(p.u, i, vio, u);
            if constexpr (!DT) load4<T>(p.delta, i, vio, dr);
            load4<T>(p.dout, i, vio, e);
            if (p.z) {
                float zz[kG];
                load4<T>(p.z, i, vio, zz);
#pragma unroll
                for (int k = 0; k < kG; ++k) {
                    zf[k] = e[k] * silu_grad(zz[k]);
                    e[k] *= silu(zz[k]);
                }
            }
            // U2: the dz-factor area holds the backward direction's u (dz re-reads its factor)
            if constexpr (U2) load4<float>(static_cast<const float *>(p.u) + p.u_dir_stride, i, true, zf);
        }
        float ds0[2 * kG], ds1[2 * kG];
        float sdt0 = 0.0f, sdt1 = 0.0f;   // DT: the two directions' step inputs of this token
        if constexpr (DT) {
            if (ok) {
                const size_t m = (size_t)b * p.L + bpos(p, t0 + r);
                sdt0 = p.dt_in[m];
                sdt1 = p.dt_in[(size_t)p.batch * p.L + m];
            }
        }
#pragma unroll
        for (int k = 0; k < kG; ++k) {
            float dl0 = 0.0f, dl1 = 0.0f, sg0 = 0.0f, sg1 = 0.0f;
            if (ok) {
                const float r0 = DT ? sdt0 * p.dt_w[ch + k] : dr[k], r1 = DT ? sdt1 * p.dt_w[p.Di + ch + k] : dr[k];
                const float x0 = r0 + p.bias[ch + k], x1 = r1 + p.bias[p.Di + ch + k];
                dl0 = softplus_io<T>(x0); sg0 = softplus_grad(x0);
                dl1 = softplus_io<T>(x1); sg1 = softplus_grad(x1);
            }
            ds0[2 * k] = dl0; ds0[2 * k + 1] = sg0;
            ds1[2 * k] = dl1; ds1[2 * k + 1] = sg1;
        }
        // 16-byte stores: two channels' pairs per float4
        float4 *t4 = reinterpret_cast<float4 *>(sm.tok + r * CH + c0);
        float4 *d4 = reinterpret_cast<float4 *>(sm.dsg + r * CH + c0);
        float4 *e4 = reinterpret_cast<float4 *>(sm.dsg + (TC + r) * CH + c0);
#pragma unroll
        for (int h = 0; h < kG / 2; ++h) {
            t4[h] = make_float4(u[2 * h], e[2 * h], u[2 * h + 1], e[2 * h + 1]);
            d4[h] = make_float4(ds0[4 * h], ds0[4 * h + 1], ds0[4 * h + 2], ds0[4 * h + 3]);
            e4[h] = make_float4(ds1[4 * h], ds1[4 * h + 1], ds1[4 * h + 2], ds1[4 * h + 3]);
        }
        *reinterpret_cast<float4 *>(sm.dzf + r * CH + c0) = make_float4(zf[0], zf[1], zf[2], zf[3]);
    }
    bool bc_done = false;
    if constexpr ((N * sizeof(T)) % 16 == 0) {
        if (p.vec_bc) {
            constexpr int VB = 16 / (int)sizeof(T);   // states per 16-byte vector
            constexpr int RV = N / VB;                 // vectors per row
            for (int li = threadIdx.x; li < 2 * 2 * TC * RV; li += SH::kThr) {
                const int which = li / (2 * TC * RV), k = (li / (TC * RV)) % 2, r = (li / RV) % TC, v = li % RV;
                float f[VB];
                if (r < tc) {
                    const T *src = static_cast<const T *>(which ? p.C[k] : p.B[k]) +
                                   ((size_t)b * p.L + bpos(p, t0 + r)) * N + v * VB;
                    unpack16(*reinterpret_cast<const uint4 *>(src), f);
                } else {
#pragma unroll
                    for (int e = 0; e < VB; ++e) f[e] = 0.0f;
                }
                float4 *dst = reinterpret_cast<float4 *>((which ? sm.C : sm.B) + (k * TC + r) * N + v * VB);
#pragma unroll
                for (int e = 0; e < VB / 4; ++e) dst[e] = make_float4(f[4 * e], f[4 * e + 1], f[4 * e + 2], f[4 * e + 3]);
            }
            bc_done = true;
        }
    }
    for (int li = threadIdx.x; !bc_done && li < 2 * TC * N; li += SH::kThr) {
        const int k = li / (TC * N), r = (li / N) % TC, n = li % N;
        const size_t i = ((size_t)b * p.L + (r < tc ? bpos(p, t0 + r) : 0)) * N + n;
        sm.B[li] = r < tc ? ld<T>(p.B[k], i) : 0.0f;
        sm.C[li] = r < tc ? ld<T>(p.C[k], i) : 0.0f;
    }

    BwdThread<N> th;
    th.tid = threadIdx.x;
    th.lane = th.tid & 31;
    th.q = th.tid % Q;
    th.cl = (th.tid / Q) % CH;
    th.dir = th.tid / (Q * CH);
    th.wid = (th.tid / 32) % SH::WPD;
    th.j0 = th.q * SH::NT;
    th.d = d0 + th.cl;
    th.valid = th.d < p.Di;
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        const float *Ar = p.A + ((size_t)th.dir * p.Di + (th.valid ? th.d : 0)) * N + th.j0 + 2 * k;
        const float2 a = th.valid ? f2(Ar[0], Ar[1]) : f2(0.f, 0.f);
        th.Araw[k] = a;
        th.A2[k] = f2(a.x * kLog2e, a.y * kLog2e);
        th.invA[k] = f2(a.x != 0.0f ? 1.0f / a.x : 0.0f, a.y != 0.0f ? 1.0f / a.y : 0.0f);
    }
    {
        const float *Ar = p.A + ((size_t)th.dir * p.Di + (th.valid ? th.d : 0)) * N;
        th.a0 = th.valid ? Ar[0] : 0.0f;
        const float inv_a0 = th.a0 != 0.0f ? 1.0f / th.a0 : 0.0f;
#pragma unroll
        for (int k = 0; k < NP; ++k) {
            const float2 in1 = f2(1.0f / (float)(th.j0 + 2 * k + 1), 1.0f / (float)(th.j0 + 2 * k + 2));
            th.w1[k] = mul2(in1, f2(inv_a0, inv_a0));
        }
        th.structured = true;
#pragma unroll
        for (int n = 0; n < N; ++n) th.structured = th.structured && (!th.valid || Ar[n] == (float)(n + 1) * th.a0);
    }
    th.Dk = th.valid ? p.D[(size_t)th.dir * p.Di + th.d] : 0.0f;
    th.cbase = (((size_t)b * p.G + c) * 2 + th.dir) * p.Di + th.d;
    __syncthreads();
    // with several chunks this kernel is launched as a programmatic dependent of the
    // adjoint fold (whose predecessors were ordinary launches, so the inputs were
    // complete before the chain began): everything above reads only the inputs; the
    // carries are read after the wait
    if (p.G > 1) cudaGridDependencySynchronize();

    // the path is chosen once per warp: the structured-A code (decays as powers of
    // exp(Delta A_0), and the exact hold's gains from hold_states) and the general code
    // are separate copies of the sweeps, with no branch between them per token, and a
    // warp fetches only the copy it runs
    constexpr bool kTwo = ZOH || ((VIMSCAN_BWD_CHAIN >> 1) & 1);   // a structured-A copy exists
    const bool fast = kTwo && __all_sync(0xffffffffu, th.structured);
    if (fast) bwd_sweep<N, ZOH, kTwo, false, U2>(p, sm, th);
    else bwd_sweep<N, ZOH, false, false, U2>(p, sm, th);
    __syncthreads();
    // dz = dout silu'(z) (sum of the directions' y), and the CTA's dC terms; the
    // cross-scan's first pair leaves its y for the second
    if (p.dz || p.stage == 1) {
        for (int li = threadIdx.x; li < TC * (CH / kG); li += SH::kThr) {
            const int r = li / (CH / kG), c0 = (li % (CH / kG)) * kG, ch = d0 + c0;
            if (r < tc && ch < p.Di) {
                const size_t i = ((size_t)b * p.L + bpos(p, t0 + r)) * p.Di + ch;
                const float4 y0 = *reinterpret_cast<const float4 *>(sm.yb + r * CH + c0);
                const float4 y1 = *reinterpret_cast<const float4 *>(sm.yb + (TC + r) * CH + c0);
                float y[kG] = {y0.x + y1.x, y0.y + y1.y, y0.z + y1.z, y0.w + y1.w};
                if (p.stage == 1) {
                    *reinterpret_cast<float4 *>(p.acc_y + i) = make_float4(y[0], y[1], y[2], y[3]);
                } else {
                    if (p.stage == 2) {
                        const float4 a = *reinterpret_cast<const float4 *>(p.acc_y + i);
                        y[0] += a.x; y[1] += a.y; y[2] += a.z; y[3] += a.w;
                    }
                    float4 f;
                    if constexpr (U2) {   // the factor dout silu'(z), formed again from its inputs
                        float e[kG], zz[kG];
                        load4<T>(p.dout, i, vio, e);
                        load4<T>(p.z, i, vio, zz);
                        f = make_float4(e[0] * silu_grad(zz[0]), e[1] * silu_grad(zz[1]), e[2] * silu_grad(zz[2]),
                                        e[3] * silu_grad(zz[3]));
                    } else {
                        f = *reinterpret_cast<const float4 *>(sm.dzf + r * CH + c0);
                    }
                    y[0] *= f.x; y[1] *= f.y; y[2] *= f.z; y[3] *= f.w;
                    store4<T>(p.dz, i, vio, y);
                }
            }
        }
    }
    store_bc_part<N>(p, sm.red, p.dC_part, b, t0, tc, blk);
    __syncthreads();

    if (fast) bwd_sweep<N, ZOH, kTwo, true, U2>(p, sm, th);
    else bwd_sweep<N, ZOH, false, true, U2>(p, sm, th);
    __syncthreads();
    for (int li = threadIdx.x; li < TC * (CH / kG); li += SH::kThr) {
        const int r = li / (CH / kG), c0 = (li % (CH / kG)) * kG, ch = d0 + c0;
        if (r < tc && ch < p.Di) {
            const size_t i = ((size_t)b * p.L + bpos(p, t0 + r)) * p.Di + ch;
            const float4 a0 = *reinterpret_cast<const float4 *>(sm.yb + r * CH + c0);
            const float4 a1 = *reinterpret_cast<const float4 *>(sm.yb + (TC + r) * CH + c0);
            const float4 b0 = *reinterpret_cast<const float4 *>(sm.dd + r * CH + c0);
            const float4 b1 = *reinterpret_cast<const float4 *>(sm.dd + (TC + r) * CH + c0);
            float du[kG] = {a0.x + a1.x, a0.y + a1.y, a0.z + a1.z, a0.w + a1.w};
            float dd[kG] = {b0.x + b1.x, b0.y + b1.y, b0.z + b1.z, b0.w + b1.w};
            if constexpr (U2 || DT) {   // per direction where the mode asks, else summed as usual
                const size_t plane = (size_t)p.batch * p.L * p.Di;
                if constexpr (U2) {
                    *reinterpret_cast<float4 *>(p.du2 + i) = a0;
                    *reinterpret_cast<float4 *>(p.du2 + plane + i) = a1;
                } else {
                    store4<T>(p.du, i, vio, du);
                }
                if constexpr (DT) {
                    *reinterpret_cast<float4 *>(p.dd2 + i) = b0;
                    *reinterpret_cast<float4 *>(p.dd2 + plane + i) = b1;
                } else {
                    store4<T>(p.ddelta, i, vio, dd);
                }
            } else if (p.stage == 1) {
                *reinterpret_cast<float4 *>(p.acc_du + i) = make_float4(du[0], du[1], du[2], du[3]);
                *reinterpret_cast<float4 *>(p.acc_dd + i) = make_float4(dd[0], dd[1], dd[2], dd[3]);
            } else {
                if (p.stage == 2) {
                    const float4 a = *reinterpret_cast<const float4 *>(p.acc_du + i);
                    const float4 e = *reinterpret_cast<const float4 *>(p.acc_dd + i);
                    du[0] += a.x; du[1] += a.y; du[2] += a.z; du[3] += a.w;
                    dd[0] += e.x; dd[1] += e.y; dd[2] += e.z; dd[3] += e.w;
                }
                store4<T>(p.du, i, vio, du);
                store4<T>(p.ddelta, i, vio, dd);
            }
        }
    }
    store_bc_part<N>(p, sm.red, p.dB_part, b, t0, tc, blk);
}

// ----------------------------------------------------------------------------
// the pathways' convolution fronts and their derivative (vim_scan_bidir_conv_bwd)
// ----------------------------------------------------------------------------
// pre_k[t] = cb_k + w_k[0] x[s_k0] + w_k[1] x[t] + w_k[2] x[s_k2], with the forward
// pathway's taps on x[t-1], x[t], x[t+1] and the backward one's on x[t+1], x[t], x[t-1]
// (x = 0 outside the sequence); u_k = silu(pre_k).
template <int K>
__device__ __forceinline__ float conv_pre(const float *w, float cb, float xm, float x0, float xp) {
    return K == 0 ? fmaf(w[0], xm, fmaf(w[1], x0, fmaf(w[2], xp, cb))) : fmaf(w[0], xp, fmaf(w[1], x0, fmaf(w[2], xm, cb)));
}

#ifndef VIMSCAN_FRONT_ROWS
#define VIMSCAN_FRONT_ROWS 64
#endif
// The front kernels work on tiles of kFrontRows tokens x kFrontCh channels of one batch
// item, one CTA of 256 threads each (grid x: batch item and run of tokens, grid y:
// channel tile).  The tile's x rows, with a halo, are staged in shared memory by
// coalesced vector loads; then every thread owns one channel and a set of rows.
constexpr int kFrontRows = VIMSCAN_FRONT_ROWS;   // tokens per tile (one row of partial sums each)
constexpr int kFrontCh = 32;                     // channels per tile
constexpr int kFrontThr = 256;
constexpr int kFrontGroups = kFrontThr / kFrontCh;   // row groups of a tile
static_assert(kFrontRows % kFrontGroups == 0, "a tile's rows split evenly over its row groups");

// x rows tfirst .. tfirst + nrows - 1 of channels c0 .. c0 + kFrontCh - 1 of batch item b
// into xs[nrows][kFrontCh] (fp32; 0 outside the sequence and past Di, a multiple of 4)
template <typename T>
__device__ __forceinline__ void front_stage(const T *x, float *xs, int nrows, int tfirst, int c0, int b, int L,
                                            int Di, int vec) {
    constexpr int V = kFrontCh / 4;
    for (int li = threadIdx.x; li < nrows * V; li += kFrontThr) {
        const int r = li / V, cg = (li % V) * 4, t = tfirst + r, ch = c0 + cg;
        float v[4] = {0.f, 0.f, 0.f, 0.f};
        if (t >= 0 && t < L && ch < Di) load4<T>(x, ((size_t)b * L + t) * Di + ch, vec != 0, v);
        *reinterpret_cast<float4 *>(xs + r * kFrontCh + cg) = make_float4(v[0], v[1], v[2], v[3]);
    }
}

// u2[k] = u_k for both pathways, [2][batch, L, Di] fp32.  Each thread walks kFrontRows /
// kFrontGroups consecutive rows of its channel with x[t-1], x[t], x[t+1] from the staged
// rows; a warp stores 32 consecutive channels of a row.
template <typename T>
__global__ void __launch_bounds__(kFrontThr) conv_front_fwd(const T *x, const float *conv_w, const float *conv_b,
                                                            float *u2, int batch, int L, int Di, int vec) {
    constexpr int TR = kFrontRows, CC = kFrontCh, RPT = TR / kFrontGroups;
    __shared__ __align__(16) float xs[(TR + 2) * CC];   // rows t0 - 1 .. t0 + TR
    const int runs = (L + TR - 1) / TR;
    const int b = blockIdx.x / runs, t0 = (blockIdx.x % runs) * TR, c0 = blockIdx.y * CC;
    front_stage<T>(x, xs, TR + 2, t0 - 1, c0, b, L, Di, vec);
    __syncthreads();
    const int c = threadIdx.x % CC, g = threadIdx.x / CC, d = c0 + c;
    if (d >= Di) return;   // no barrier follows
    float wf[3], wb[3];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        wf[j] = conv_w[(size_t)d * 3 + j];
        wb[j] = conv_w[((size_t)Di + d) * 3 + j];
    }
    const float bf = conv_b[d], bb = conv_b[Di + d];
    const int64_t plane = (int64_t)batch * L * Di;
    const int rb = g * RPT;   // first row of the thread; xs row s holds token t0 - 1 + s
    float xm = xs[rb * CC + c], x0 = xs[(rb + 1) * CC + c];
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
        const int t = t0 + rb + k;
        const float xp = xs[(rb + k + 2) * CC + c];
        if (t < L) {
            const size_t i = ((size_t)b * L + t) * Di + d;
            u2[i] = silu(conv_pre<0>(wf, bf, xm, x0, xp));
            u2[plane + i] = silu(conv_pre<1>(wb, bb, xm, x0, xp));
        }
        xm = x0;
        x0 = xp;
    }
}

// Derivative of the fronts from dl/du_k (du2, fp32): with dpre_k = dl/du_k silu'(pre_k),
//   dl/dx[t]  = w_f[0] dpre_f[t+1] + w_f[1] dpre_f[t] + w_f[2] dpre_f[t-1]
//             + w_b[0] dpre_b[t-1] + w_b[1] dpre_b[t] + w_b[2] dpre_b[t+1],
//   dl/dw_k[j] = sum_t dpre_k[t] x[s_kj(t)],   dl/dcb_k = sum_t dpre_k[t].
// Per tile: x rows with two halo rows each side staged; dpre of both pathways for the
// tile's rows and one either side, into shared memory (each thread a channel and every
// kFrontGroups-th row, so the du2 loads of a thread are independent); then per thread a
// channel and kFrontRows / kFrontGroups consecutive rows: dx and the eight tap and bias
// sums, summed over the row groups in order into the tile's slice of one row of partial
// sums part[b * runs + run][8 Di] = [dw: (k * Di + d) * 3 + j | dcb: 6 Di + k * Di + d].
template <typename T>
__global__ void __launch_bounds__(kFrontThr) conv_front_bwd(const T *x, const float *conv_w, const float *conv_b,
                                                            const float *du2, T *dx, float *part, int batch, int L,
                                                            int Di, int vec) {
    constexpr int TR = kFrontRows, CC = kFrontCh, G = kFrontGroups, RPT = TR / G;
    static_assert(G == 8, "one row group per partial sum in the final pass");
    __shared__ __align__(16) float xs[(TR + 4) * CC];      // x rows t0 - 2 .. t0 + TR + 1
    __shared__ __align__(16) float dp[2 * (TR + 2) * CC];  // dpre_k rows t0 - 1 .. t0 + TR
    const int runs = (L + TR - 1) / TR;
    const int b = blockIdx.x / runs, run = blockIdx.x % runs, t0 = run * TR, c0 = blockIdx.y * CC;
    front_stage<T>(x, xs, TR + 4, t0 - 2, c0, b, L, Di, vec);
    __syncthreads();
    const int c = threadIdx.x % CC, g = threadIdx.x / CC, d = c0 + c;
    const bool dv = d < Di;
    float w[2][3], cb[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        cb[k] = dv ? conv_b[k * Di + d] : 0.0f;
#pragma unroll
        for (int j = 0; j < 3; ++j) w[k][j] = dv ? conv_w[((size_t)k * Di + d) * 3 + j] : 0.0f;
    }
    const int64_t plane = (int64_t)batch * L * Di;
    // dpre row r <-> token t0 - 1 + r, whose x[t-1], x[t], x[t+1] are xs rows r, r+1, r+2
#pragma unroll
    for (int k = 0; k < (TR + 2 + G - 1) / G; ++k) {
        const int r = g + k * G, t = t0 - 1 + r;
        if (r >= TR + 2) break;
        float pf = 0.0f, pb = 0.0f;
        if (dv && t >= 0 && t < L) {
            const size_t i = ((size_t)b * L + t) * Di + d;
            const float xm = xs[r * CC + c], x0 = xs[(r + 1) * CC + c], xp = xs[(r + 2) * CC + c];
            pf = du2[i] * silu_grad(conv_pre<0>(w[0], cb[0], xm, x0, xp));
            pb = du2[plane + i] * silu_grad(conv_pre<1>(w[1], cb[1], xm, x0, xp));
        }
        dp[r * CC + c] = pf;
        dp[(TR + 2 + r) * CC + c] = pb;
    }
    __syncthreads();
    const float *df = dp, *db = dp + (TR + 2) * CC;
    float sum[8];   // dw_f[0..2], dw_b[0..2], dcb_f, dcb_b
#pragma unroll
    for (int e = 0; e < 8; ++e) sum[e] = 0.0f;
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
        const int r = g * RPT + k, t = t0 + r;   // dpre rows r, r+1, r+2 = t-1, t, t+1; xs rows r+1..r+3
        if (dv && t < L) {
            const float fm = df[r * CC + c], f0 = df[(r + 1) * CC + c], fp = df[(r + 2) * CC + c];
            const float bm = db[r * CC + c], b0 = db[(r + 1) * CC + c], bp = db[(r + 2) * CC + c];
            float gx = w[0][0] * fp;
            gx = fmaf(w[0][1], f0, gx);
            gx = fmaf(w[0][2], fm, gx);
            gx = fmaf(w[1][0], bm, gx);
            gx = fmaf(w[1][1], b0, gx);
            gx = fmaf(w[1][2], bp, gx);
            dx[((size_t)b * L + t) * Di + d] = from_f32<T>(gx);
            const float xa = xs[(r + 1) * CC + c], xb = xs[(r + 2) * CC + c], xc = xs[(r + 3) * CC + c];
            sum[0] = fmaf(f0, xa, sum[0]);   // forward taps: x[t-1], x[t], x[t+1]
            sum[1] = fmaf(f0, xb, sum[1]);
            sum[2] = fmaf(f0, xc, sum[2]);
            sum[3] = fmaf(b0, xc, sum[3]);   // backward taps: x[t+1], x[t], x[t-1]
            sum[4] = fmaf(b0, xb, sum[4]);
            sum[5] = fmaf(b0, xa, sum[5]);
            sum[6] += f0;
            sum[7] += b0;
        }
    }
    __syncthreads();   // dp is reused for the row groups' sums
    float *red = dp;   // [8 sums][G][CC]
#pragma unroll
    for (int e = 0; e < 8; ++e) red[(e * G + g) * CC + c] = sum[e];
    __syncthreads();
    if (dv) {
        const int e = g;   // this thread sums partial e of its channel over the row groups
        float acc = 0.0f;
#pragma unroll
        for (int q = 0; q < G; ++q) acc += red[(e * G + q) * CC + c];
        float *row = part + ((size_t)b * runs + run) * (8 * (size_t)Di);
        if (e < 6) row[((size_t)(e / 3) * Di + d) * 3 + e % 3] = acc;
        else row[6 * (size_t)Di + (size_t)(e - 6) * Di + d] = acc;
    }
}

// dB / dC: sum of the per-CTA (or per-cluster) partials, [batch][L][ncol][N] -> [batch][L][N]
template <int N>
__global__ void __launch_bounds__(256) bwd_reduce_bc(const float *part, float *out, int rows, int nblk) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;   // (row, n)
    if (i >= (int64_t)rows * N) return;
    const int64_t row = i / N;
    const int n = (int)(i % N);
    const float *src = part + row * nblk * N + n;
    float acc = 0.0f;
    for (int k = 0; k < nblk; ++k) acc += src[(int64_t)k * N];
    out[i] = acc;
}

// column sums of a [rows][cols] fp32 array in two passes: rows split into
// kReduceParts groups (first pass, into tmp[part][cols]), then the groups summed
__global__ void __launch_bounds__(256) bwd_reduce_cols1(const float *src, float *tmp, int rows, int cols) {
    const int col = blockIdx.x * blockDim.x + threadIdx.x, part = blockIdx.y;
    if (col >= cols) return;
    const int per = (rows + kReduceParts - 1) / kReduceParts;
    const int r0 = part * per, r1 = min(rows, r0 + per);
    float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
    int r = r0;
    for (; r + 4 <= r1; r += 4) {
        a0 += src[(int64_t)r * cols + col];
        a1 += src[(int64_t)(r + 1) * cols + col];
        a2 += src[(int64_t)(r + 2) * cols + col];
        a3 += src[(int64_t)(r + 3) * cols + col];
    }
    for (; r < r1; ++r) a0 += src[(int64_t)r * cols + col];
    tmp[(int64_t)part * cols + col] = (a0 + a1) + (a2 + a3);
}
// second pass; the columns are [dA: 2*Di*N | dD: 2*Di | d delta_bias: 2*Di]
__global__ void __launch_bounds__(256) bwd_reduce_cols2(const float *tmp, float *dA, float *dD, float *dbias,
                                                        int nA, int nD) {
    const int cols = nA + 2 * nD;
    const int col = blockIdx.x * blockDim.x + threadIdx.x;
    if (col >= cols) return;
    float acc = 0.0f;
    for (int part = 0; part < kReduceParts; ++part) acc += tmp[(int64_t)part * cols + col];
    if (col < nA) dA[col] = acc;
    else if (col < nA + nD) dD[col - nA] = acc;
    else dbias[col - nA - nD] = acc;
}

}  // namespace
}  // namespace vimscan
