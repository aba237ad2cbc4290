// bwd_kernels.cuh -- sm_100a kernels of the derivative of the Vim two-direction scan.
//
// The loss's derivative dout with respect to y = (y^f + y^b) * silu(z) is carried back
// through the scan (first-order Bbar = Delta B), for every input: u, the raw delta,
// z, B, C, A, D and the delta bias.  Per direction, with g_t the adjoint of h_t
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
// registers) and forms y (for dz) and the dC terms, then segment by segment in
// reverse a re-run of h over the segment followed by the adjoint sweep.  A thread
// holds NT (4, or 8 when built so) states of one (channel, direction), so the segment's h and decays fit
// in registers (the checkpoints go to shared memory); Q = N / NT threads share a
// channel.  Each warp serves one direction, whose code is compiled separately so that
// its token addresses are constants.
// Sums over channels (dB, dC) are reduced across the warp by shuffles, then across
// the CTA's warps and directions in shared memory, and written per CTA; sums over
// tokens (dA, dD, dbias) are written per chunk.  Small reduction kernels finish both.
// Every sum is taken in a fixed order (no floating-point atomics), so results repeat
// bit for bit.
#pragma once

#include "scan_kernels.cuh"

namespace vimscan {

constexpr int kBwdChunk = 32;                 // tokens per chunk
constexpr int kBwdSeg = 4;                    // tokens between checkpoints of h
constexpr int kBwdNSeg = kBwdChunk / kBwdSeg;
constexpr int kAdjCh = 64;                    // channels per adj_carry CTA
constexpr int kReduceParts = 32;              // row groups of the first parameter-reduction pass
#ifndef VIMSCAN_BWD_NT
#define VIMSCAN_BWD_NT 4                         // states per thread of bwd_main (4 or 8)
#endif
#ifndef VIMSCAN_BWD_MIN_WARPS
#define VIMSCAN_BWD_MIN_WARPS 16                 // resident warps per SM the register budget targets
#endif

struct BwdArgs {
    const void *u, *delta, *z, *dout;   // [batch, L, Di]
    const void *B[2], *C[2];            // per direction [batch, L, N]
    const float *A, *D, *bias;          // [2][Di][N], [2][Di], [2][Di]
    void *du, *ddelta, *dz;             // [batch, L, Di] (dz null when z is)
    float *dB_part[2], *dC_part[2];     // [batch][L][nblk][N] per B/C set ([1] = [0] when shared)
    float *par;                         // per-chunk sums over tokens, one row per (batch, chunk):
                                        // [dA: 2*Di*N | dD: 2*Di | d delta_bias: 2*Di]
    const float *hin;                   // [batch][G][2][Di][N] h entering each chunk (direction order)
    float *gloc;                        // [batch][G][2][Di][N] adjoint summaries, then adjoint entering
    float *gsum;                        // [batch][G][2][Di] chunk Delta sums
    int batch, L, Di, G, nblk;
    int separate_bc;
    int order, H, W;                    // visiting order of the pair (0: position = step;
                                        // 1: column-major on H x W, the cross-scan's second pair)
    int stage;                          // 0: one pair (Vim), final outputs; 1: first pair of the
                                        // cross-scan, fp32 partials to acc_*; 2: second pair, adds them
    float *acc_y, *acc_du, *acc_dd;     // [batch, L, Di] fp32 by position (stages 1 and 2)
};

namespace {

// grid position visited at step t of the pair's forward direction
__device__ __forceinline__ int bpos(const BwdArgs &p, int t) {
    if (p.order == 0) return t;
    const int h = t % p.H, w = t / p.H;
    return h * p.W + w;
}

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

template <typename T>
__device__ __forceinline__ float ld(const void *p, size_t i) { return to_f32(static_cast<const T *>(p)[i]); }

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
template <typename T, int N>
__global__ void __launch_bounds__(2 * kAdjCh) adj_carry(BwdArgs p) {
    __shared__ float sDr[kBwdChunk][kAdjCh], sDy[kBwdChunk][kAdjCh];
    __shared__ __align__(16) float sC[2][kBwdChunk][N];
    const int b = blockIdx.z, c = blockIdx.y, d0 = blockIdx.x * kAdjCh;
    const int t0 = c * kBwdChunk, tc = min(kBwdChunk, p.L - t0);
    for (int li = threadIdx.x; li < kBwdChunk * kAdjCh; li += 2 * kAdjCh) {
        const int r = li / kAdjCh, cl = li % kAdjCh, ch = d0 + cl;
        float dr = 0.0f, e = 0.0f;
        if (r < tc && ch < p.Di) {
            const size_t i = ((size_t)b * p.L + bpos(p, t0 + r)) * p.Di + ch;
            dr = ld<T>(p.delta, i);
            e = ld<T>(p.dout, i);
            if (p.z) e *= silu(ld<T>(p.z, i));
        }
        sDr[r][cl] = dr;
        sDy[r][cl] = e;
    }
    for (int li = threadIdx.x; li < 2 * kBwdChunk * N; li += 2 * kAdjCh) {
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
        S += ok ? softplus_io<T>(sDr[r][dl] + bias) : 0.0f;
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

// ----------------------------------------------------------------------------
// the derivative over one chunk of 16 channels, both directions
// ----------------------------------------------------------------------------
// ----------------------------------------------------------------------------
// the derivative over one chunk of CH channels, both directions
// ----------------------------------------------------------------------------
template <int N> struct BwdShape {
    static constexpr int NT = N < VIMSCAN_BWD_NT ? N : VIMSCAN_BWD_NT;   // states per thread
    static constexpr int CKW = (NT + 3) / 4;                 // float4 per checkpoint per thread
    static constexpr int Q = N / NT;                         // threads per (channel, direction)
    static constexpr int CH = 32 / Q > 16 ? 32 / Q : 16;     // channels per CTA (whole warps per direction)
    static constexpr int kThr = 2 * CH * Q;
    static constexpr int WPD = CH * Q / 32;                  // warps per direction
    static constexpr int CW = 32 / Q;                        // channels per warp
    static constexpr int kMinBlocks = VIMSCAN_BWD_MIN_WARPS * 32 / kThr;
    static constexpr int TC = kBwdChunk;
    // shared memory, in floats (every row of the chunk):
    //   tok[2][TC][CH] float4 {Delta, u, dy, sigmoid(delta_raw + bias)} per direction
    //   yb[2][TC][CH]  y^k in the forward sweep, then du^k in the adjoint sweep
    //   dd[2][TC][CH]  d delta_raw from direction k
    //   B[2][TC][N], C[2][TC][N]
    //   red[2][WPD][TC][N]  per direction and warp: the dC terms, then the dB terms
    //   ck[kBwdNSeg][CKW][kThr] float4  h at every kBwdSeg-th token, per thread
    static constexpr int oTok = 0;
    static constexpr int oYb = oTok + 2 * TC * CH * 4;
    static constexpr int oDd = oYb + 2 * TC * CH;
    static constexpr int oB = oDd + 2 * TC * CH;
    static constexpr int oC = oB + 2 * TC * N;
    static constexpr int oRed = oC + 2 * TC * N;
    static constexpr int oCk = oRed + 2 * WPD * TC * N;
    static constexpr int kFloats = oCk + kBwdNSeg * CKW * kThr * 4;
    static constexpr size_t kSmemBytes = (size_t)kFloats * 4;
    static_assert(oCk % 4 == 0 && oTok % 4 == 0, "float4 areas must be 16-byte aligned");
};

template <int N>
struct BwdSmem {
    using SH = BwdShape<N>;
    float4 *tok;
    float *yb, *dd, *B, *C, *red;
    float4 *ck;
    __device__ explicit BwdSmem(float *base)
        : tok(reinterpret_cast<float4 *>(base + SH::oTok)), yb(base + SH::oYb), dd(base + SH::oDd),
          B(base + SH::oB), C(base + SH::oC), red(base + SH::oRed), ck(reinterpret_cast<float4 *>(base + SH::oCk)) {}
};

// per-thread identity and parameters of one (channel, direction, state group)
template <int N>
struct BwdThread {
    using SH = BwdShape<N>;
    int tid, lane, q, cl, dir, wid, j0, d;
    bool valid;
    float A2[SH::NT], Araw[SH::NT];
    float Dk;
    size_t cbase;   // [b][c][dir][d]
};

template <int NT>
__device__ __forceinline__ void load_states(const float *row, float (&v)[NT]) {
    if constexpr (NT % 4 == 0) {
#pragma unroll
        for (int q = 0; q < NT / 4; ++q) {
            const float4 t = *reinterpret_cast<const float4 *>(row + 4 * q);
            v[4 * q] = t.x; v[4 * q + 1] = t.y; v[4 * q + 2] = t.z; v[4 * q + 3] = t.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < NT; ++j) v[j] = row[j];
    }
}

// forward sweep of direction DIR: checkpoints, y^DIR (ungated) and the dC terms
template <int N, int DIR>
__device__ __forceinline__ void bwd_forward(const BwdArgs &p, const BwdSmem<N> &sm, const BwdThread<N> &th) {
    using SH = BwdShape<N>;
    constexpr int NT = SH::NT, Q = SH::Q, CH = SH::CH, TC = SH::TC;
    float h[NT];
#pragma unroll
    for (int j = 0; j < NT; ++j) h[j] = (p.G > 1 && th.valid) ? p.hin[th.cbase * N + th.j0 + j] : 0.0f;
#pragma unroll 1
    for (int sg = 0; sg < kBwdNSeg; ++sg) {
#pragma unroll
        for (int w = 0; w < SH::CKW; ++w) {
            float q4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) q4[e] = 4 * w + e < NT ? h[4 * w + e < NT ? 4 * w + e : 0] : 0.0f;
            sm.ck[(sg * SH::CKW + w) * SH::kThr + th.tid] = make_float4(q4[0], q4[1], q4[2], q4[3]);
        }
#pragma unroll
        for (int m = 0; m < kBwdSeg; ++m) {
            const int i = sg * kBwdSeg + m, r = DIR ? TC - 1 - i : i;
            const float4 tk = sm.tok[(DIR * TC + r) * CH + th.cl];   // Delta, u, dy, sigmoid
            float Bv[NT], Cv[NT], v[NT];
            load_states<NT>(sm.B + (DIR * TC + r) * N + th.j0, Bv);
            load_states<NT>(sm.C + (DIR * TC + r) * N + th.j0, Cv);
            const float du = tk.x * tk.y;
            float yp = th.q == 0 ? th.Dk * tk.y : 0.0f;
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                h[j] = fmaf(ex2(tk.x * th.A2[j]), h[j], du * Bv[j]);
                yp = fmaf(Cv[j], h[j], yp);
                v[j] = tk.z * h[j];
            }
#pragma unroll
            for (int s = 1; s < Q; s <<= 1) yp += __shfl_xor_sync(0xffffffffu, yp, s);
            if (th.q == 0) sm.yb[(DIR * TC + r) * CH + th.cl] = yp;
            int off;
            bool wr;
            reduce_channels<NT, Q, SH::CW>(v, th.lane, &off, &wr);
            if (wr) sm.red[((DIR * SH::WPD + th.wid) * TC + r) * N + th.j0 + off] = v[0];
        }
    }
}

// adjoint sweep of direction DIR, segment by segment from the last: h re-run over
// the segment from its checkpoint (keeping h and the decays), then g backwards
template <int N, int DIR>
__device__ __forceinline__ void bwd_adjoint(const BwdArgs &p, const BwdSmem<N> &sm, const BwdThread<N> &th) {
    using SH = BwdShape<N>;
    constexpr int NT = SH::NT, Q = SH::Q, CH = SH::CH, TC = SH::TC;
    // with Q > 1 lane q = 0 gathers du and lane q = 1 d delta_raw of the channel
    constexpr int kDdLane = Q > 1 ? 1 : 0;
    float g[NT], dA[NT];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
        g[j] = (p.G > 1 && th.valid) ? p.gloc[th.cbase * N + th.j0 + j] : 0.0f;
        dA[j] = 0.0f;
    }
    float dD = 0.0f, dbias = 0.0f;
#pragma unroll 1
    for (int sg = kBwdNSeg - 1; sg >= 0; --sg) {
        float h0[4 * SH::CKW];
#pragma unroll
        for (int w = 0; w < SH::CKW; ++w) {
            const float4 c4 = sm.ck[(sg * SH::CKW + w) * SH::kThr + th.tid];
            h0[4 * w] = c4.x; h0[4 * w + 1] = c4.y; h0[4 * w + 2] = c4.z; h0[4 * w + 3] = c4.w;
        }
        float hh[kBwdSeg][NT], aa[kBwdSeg][NT];
#pragma unroll
        for (int m = 0; m < kBwdSeg; ++m) {
            const int i = sg * kBwdSeg + m, r = DIR ? TC - 1 - i : i;
            const float4 tk = sm.tok[(DIR * TC + r) * CH + th.cl];
            float Bv[NT];
            load_states<NT>(sm.B + (DIR * TC + r) * N + th.j0, Bv);
            const float du = tk.x * tk.y;
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                aa[m][j] = ex2(tk.x * th.A2[j]);
                hh[m][j] = fmaf(aa[m][j], m > 0 ? hh[m > 0 ? m - 1 : 0][j] : h0[j], du * Bv[j]);
            }
        }
#pragma unroll
        for (int m = kBwdSeg - 1; m >= 0; --m) {
            const int i = sg * kBwdSeg + m, r = DIR ? TC - 1 - i : i;
            const float4 tk = sm.tok[(DIR * TC + r) * CH + th.cl];   // Delta, u, dy, sigmoid
            float Bv[NT], Cv[NT], v[NT];
            load_states<NT>(sm.B + (DIR * TC + r) * N + th.j0, Bv);
            load_states<NT>(sm.C + (DIR * TC + r) * N + th.j0, Cv);
            const float du = tk.x * tk.y;
            float sA = 0.0f, sBg = 0.0f;
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                g[j] = fmaf(Cv[j], tk.z, g[j]);                           // dl/dh_t
                const float hp = m > 0 ? hh[m > 0 ? m - 1 : 0][j] : h0[j];  // h_(t-1)
                const float ga = aa[m][j] * g[j];
                const float w = ga * hp;
                dA[j] = fmaf(tk.x, w, dA[j]);
                sA = fmaf(th.Araw[j], w, sA);
                sBg = fmaf(g[j], Bv[j], sBg);
                v[j] = g[j] * du;
                g[j] = ga;                                                // dl/dh_(t-1) part
            }
            // this thread's share of du and d delta_raw, gathered over the Q lanes of
            // the channel: lane q = 0 ends with du, lane q = 1 with d delta_raw
            float x0 = tk.x * sBg, x1 = fmaf(tk.y, sBg, sA) * tk.w;
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
                sm.yb[(DIR * TC + r) * CH + th.cl] = fmaf(th.Dk, tk.z, x0);
                dD = fmaf(tk.z, tk.y, dD);
            }
            if (th.q == kDdLane) {
                sm.dd[(DIR * TC + r) * CH + th.cl] = x1;
                dbias += x1;
            }
            int off;
            bool wr;
            reduce_channels<NT, Q, SH::CW>(v, th.lane, &off, &wr);
            if (wr) sm.red[((DIR * SH::WPD + th.wid) * TC + r) * N + th.j0 + off] = v[0];
        }
    }
    if (th.valid) {
        // row (b, c) of par; cbase = (row * 2 + dir) * Di + d
        const size_t row = th.cbase / ((size_t)2 * p.Di), col = th.cbase % ((size_t)2 * p.Di);
        float *pr = p.par + row * ((size_t)2 * p.Di * (N + 2));
#pragma unroll
        for (int j = 0; j < NT; ++j) pr[col * N + th.j0 + j] = dA[j];
        if (th.q == 0) pr[(size_t)2 * p.Di * N + col] = dD;
        if (th.q == kDdLane) pr[(size_t)2 * p.Di * (N + 1) + col] = dbias;
    }
}

// The CTA's per-token sums over its channels of the dB (or dC) terms, from the
// per-direction, per-warp slots, into part[set][b][t][blk][n]: the two directions
// add into one set when B and C are shared.
template <int N>
__device__ __forceinline__ void store_bc_part(const BwdArgs &p, const float *red, float *const (&part)[2], int b,
                                              int t0, int tc, int blk) {
    using SH = BwdShape<N>;
    constexpr int TC = SH::TC;
    const int nsets = p.separate_bc ? 2 : 1;
    for (int li = threadIdx.x; li < nsets * TC * N; li += SH::kThr) {
        const int k = li / (TC * N), r = (li / N) % TC, n = li % N;
        if (r >= tc) continue;
        float acc = 0.0f;
#pragma unroll
        for (int dir = 0; dir < 2; ++dir) {
            if (p.separate_bc && dir != k) continue;
#pragma unroll
            for (int w = 0; w < SH::WPD; ++w) acc += red[((dir * SH::WPD + w) * TC + r) * N + n];
        }
        part[k][(((size_t)b * p.L + bpos(p, t0 + r)) * p.nblk + blk) * N + n] = acc;
    }
}

template <typename T, int N>
__global__ void __launch_bounds__(BwdShape<N>::kThr, BwdShape<N>::kMinBlocks) bwd_main(BwdArgs p) {
    using SH = BwdShape<N>;
    constexpr int NT = SH::NT, Q = SH::Q, CH = SH::CH, TC = SH::TC;
    extern __shared__ __align__(16) float smem_f[];
    const BwdSmem<N> sm(smem_f);

    const int b = blockIdx.z, c = blockIdx.y, blk = blockIdx.x, d0 = blk * CH;
    const int t0 = c * TC, tc = min(TC, p.L - t0);

    // ---- stage the chunk: {Delta, u, dy, sigmoid} per direction, B and C ------------
    for (int li = threadIdx.x; li < TC * CH; li += SH::kThr) {
        const int r = li / CH, cl = li % CH, ch = d0 + cl;
        float u = 0.0f, e = 0.0f, dl0 = 0.0f, dl1 = 0.0f, sg0 = 0.0f, sg1 = 0.0f;
        if (r < tc && ch < p.Di) {
            const size_t i = ((size_t)b * p.L + bpos(p, t0 + r)) * p.Di + ch;
            u = ld<T>(p.u, i);
            const float dr = ld<T>(p.delta, i);
            e = ld<T>(p.dout, i);
            if (p.z) e *= silu(ld<T>(p.z, i));
            const float x0 = dr + p.bias[ch], x1 = dr + p.bias[p.Di + ch];
            dl0 = softplus_io<T>(x0); sg0 = softplus_grad(x0);
            dl1 = softplus_io<T>(x1); sg1 = softplus_grad(x1);
        }
        sm.tok[r * CH + cl] = make_float4(dl0, u, e, sg0);
        sm.tok[(TC + r) * CH + cl] = make_float4(dl1, u, e, sg1);
    }
    for (int li = threadIdx.x; li < 2 * TC * N; li += SH::kThr) {
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
    th.j0 = th.q * NT;
    th.d = d0 + th.cl;
    th.valid = th.d < p.Di;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
        th.Araw[j] = th.valid ? p.A[((size_t)th.dir * p.Di + th.d) * N + th.j0 + j] : 0.0f;
        th.A2[j] = th.Araw[j] * kLog2e;
    }
    th.Dk = th.valid ? p.D[(size_t)th.dir * p.Di + th.d] : 0.0f;
    th.cbase = (((size_t)b * p.G + c) * 2 + th.dir) * p.Di + th.d;
    __syncthreads();

    if (th.dir == 0) bwd_forward<N, 0>(p, sm, th);
    else bwd_forward<N, 1>(p, sm, th);
    __syncthreads();
    // dz = dout silu'(z) (sum of the directions' y), and the CTA's dC terms; the
    // cross-scan's first pair leaves its y for the second
    if (p.dz || p.stage == 1) {
        for (int li = threadIdx.x; li < TC * CH; li += SH::kThr) {
            const int r = li / CH, c2 = li % CH, ch = d0 + c2;
            if (r < tc && ch < p.Di) {
                const size_t i = ((size_t)b * p.L + bpos(p, t0 + r)) * p.Di + ch;
                float y = sm.yb[r * CH + c2] + sm.yb[(TC + r) * CH + c2];
                if (p.stage == 1) {
                    p.acc_y[i] = y;
                } else {
                    if (p.stage == 2) y += p.acc_y[i];
                    static_cast<T *>(p.dz)[i] = from_f32<T>(ld<T>(p.dout, i) * silu_grad(ld<T>(p.z, i)) * y);
                }
            }
        }
    }
    store_bc_part<N>(p, sm.red, p.dC_part, b, t0, tc, blk);
    __syncthreads();

    if (th.dir == 0) bwd_adjoint<N, 0>(p, sm, th);
    else bwd_adjoint<N, 1>(p, sm, th);
    __syncthreads();
    for (int li = threadIdx.x; li < TC * CH; li += SH::kThr) {
        const int r = li / CH, c2 = li % CH, ch = d0 + c2;
        if (r < tc && ch < p.Di) {
            const size_t i = ((size_t)b * p.L + bpos(p, t0 + r)) * p.Di + ch;
            float du = sm.yb[r * CH + c2] + sm.yb[(TC + r) * CH + c2];
            float dd = sm.dd[r * CH + c2] + sm.dd[(TC + r) * CH + c2];
            if (p.stage == 1) {
                p.acc_du[i] = du;
                p.acc_dd[i] = dd;
            } else {
                if (p.stage == 2) {
                    du += p.acc_du[i];
                    dd += p.acc_dd[i];
                }
                static_cast<T *>(p.du)[i] = from_f32<T>(du);
                static_cast<T *>(p.ddelta)[i] = from_f32<T>(dd);
            }
        }
    }
    store_bc_part<N>(p, sm.red, p.dB_part, b, t0, tc, blk);
}

// dB / dC: sum of the per-CTA partials, [batch][L][nblk][N] -> [batch][L][N]
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
