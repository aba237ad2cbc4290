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
// channels, both directions: a forward sweep that keeps h every kBwdSeg tokens (in
// registers) and forms y (for dz) and the dC terms, then segment by segment in
// reverse a re-run of h over the segment followed by the adjoint sweep.  A thread
// holds NT <= 4 states of one (channel, direction), so the checkpoints and the
// segment's h fit in registers; Q = N / NT threads share a channel.
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
constexpr int kBwdCh = 16;                    // channels per bwd_main CTA
constexpr int kAdjCh = 64;                    // channels per adj_carry CTA
constexpr int kReduceParts = 32;              // row groups of the first parameter-reduction pass
#ifndef VIMSCAN_BWD_MIN_WARPS
#define VIMSCAN_BWD_MIN_WARPS 16                 // resident warps per SM the register budget targets
#endif

struct BwdArgs {
    const void *u, *delta, *z, *dout;   // [batch, L, Di]
    const void *B[2], *C[2];            // per direction [batch, L, N]
    const float *A, *D, *bias;          // [2][Di][N], [2][Di], [2][Di]
    void *du, *ddelta, *dz;             // [batch, L, Di] (dz null when z is)
    float *dB_part[2], *dC_part[2];     // [batch][L][nblk][N] per B/C set ([1] = [0] when shared)
    float *dA_part;                     // [batch][G][2][Di][N]
    float *dD_part, *dbias_part;        // [batch][G][2][Di]
    const float *hin;                   // [batch][G][2][Di][N] h entering each chunk (direction order)
    float *gloc;                        // [batch][G][2][Di][N] adjoint summaries, then adjoint entering
    float *gsum;                        // [batch][G][2][Di] chunk Delta sums
    int batch, L, Di, G, nblk;
    int separate_bc;
};

namespace {

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
// visited up to and including s.  One thread per (channel, direction), all N states.
// ----------------------------------------------------------------------------
template <typename T, int N>
__global__ void __launch_bounds__(2 * kAdjCh) adj_carry(BwdArgs p) {
    __shared__ float sDr[kBwdChunk][kAdjCh], sDy[kBwdChunk][kAdjCh];
    __shared__ float sC[2][kBwdChunk][N];
    const int b = blockIdx.z, c = blockIdx.y, d0 = blockIdx.x * kAdjCh;
    const int t0 = c * kBwdChunk, tc = min(kBwdChunk, p.L - t0);
    for (int li = threadIdx.x; li < kBwdChunk * kAdjCh; li += 2 * kAdjCh) {
        const int r = li / kAdjCh, cl = li % kAdjCh, ch = d0 + cl;
        float dr = 0.0f, e = 0.0f;
        if (r < tc && ch < p.Di) {
            const size_t i = ((size_t)b * p.L + t0 + r) * p.Di + ch;
            dr = ld<T>(p.delta, i);
            e = ld<T>(p.dout, i);
            if (p.z) e *= silu(ld<T>(p.z, i));
        }
        sDr[r][cl] = dr;
        sDy[r][cl] = e;
    }
    for (int li = threadIdx.x; li < 2 * kBwdChunk * N; li += 2 * kAdjCh) {
        const int k = li / (kBwdChunk * N), r = (li / N) % kBwdChunk, n = li % N;
        sC[k][r][n] = r < tc ? ld<T>(p.C[k], ((size_t)b * p.L + t0 + r) * N + n) : 0.0f;
    }
    __syncthreads();

    const int dir = threadIdx.x / kAdjCh, dl = threadIdx.x % kAdjCh, d = d0 + dl;
    if (d >= p.Di) return;
    float A2[N], G[N];
#pragma unroll
    for (int n = 0; n < N; ++n) {
        A2[n] = p.A[((size_t)dir * p.Di + d) * N + n] * kLog2e;
        G[n] = 0.0f;
    }
    const float bias = p.bias[(size_t)dir * p.Di + d];
    float S = 0.0f;
    for (int i = 0; i < tc; ++i) {
        const int r = dir ? tc - 1 - i : i;
        S += softplus(sDr[r][dl] + bias);
        const float e = sDy[r][dl];
#pragma unroll
        for (int n = 0; n < N; ++n) G[n] = fmaf(ex2(A2[n] * S) * sC[dir][r][n], e, G[n]);
    }
    const size_t base = (((size_t)b * p.G + c) * 2 + dir) * p.Di + d;
#pragma unroll
    for (int n = 0; n < N; ++n) p.gloc[base * N + n] = G[n];
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
// The CTA's per-token sums over its channels of the dB (or dC) terms, from the
// per-direction, per-warp slots, into part[set][b][t][blk][n]: the two directions
// add into one set when B and C are shared.
template <int N, int WPD>
__device__ __forceinline__ void store_bc_part(const BwdArgs &p, const float (&red)[2][WPD][kBwdChunk][N],
                                              float *const (&part)[2], int b, int t0, int tc, int blk) {
    const int nsets = p.separate_bc ? 2 : 1;
    for (int li = threadIdx.x; li < nsets * kBwdChunk * N; li += blockDim.x) {
        const int k = li / (kBwdChunk * N), r = (li / N) % kBwdChunk, n = li % N;
        if (r >= tc) continue;
        float acc = 0.0f;
#pragma unroll
        for (int dir = 0; dir < 2; ++dir) {
            if (p.separate_bc && dir != k) continue;
#pragma unroll
            for (int w = 0; w < WPD; ++w) acc += red[dir][w][r][n];
        }
        part[k][(((size_t)b * p.L + t0 + r) * p.nblk + blk) * N + n] = acc;
    }
}

template <int N> struct BwdShape {
    static constexpr int NT = N < 4 ? N : 4;           // states per thread
    static constexpr int Q = N / NT;                   // threads per (channel, direction)
    static constexpr int kThr = 2 * kBwdCh * Q;
    static constexpr int CW = (32 / Q < kBwdCh) ? 32 / Q : kBwdCh;   // channels per warp
    static constexpr int WPD = (kBwdCh * Q + 31) / 32;                // warps per direction
    static constexpr int kMinBlocks = VIMSCAN_BWD_MIN_WARPS * 32 / kThr;   // resident CTAs per SM aimed at
};

template <typename T, int N>
__global__ void __launch_bounds__(BwdShape<N>::kThr, BwdShape<N>::kMinBlocks) bwd_main(BwdArgs p) {
    using SH = BwdShape<N>;
    constexpr int NT = SH::NT, Q = SH::Q, CH = kBwdCh, TC = kBwdChunk;
    constexpr int WPD = SH::WPD;
    __shared__ float sU[TC][CH], sDy[TC][CH], sDzf[TC][CH];
    __shared__ float sY[2][TC][CH], sDu[2][TC][CH], sDd[2][TC][CH];   // per direction
    __shared__ float sDelta[2][TC][CH], sSig[2][TC][CH];
    __shared__ __align__(16) float sB[2][TC][N], sC[2][TC][N];
    __shared__ float sRed[2][WPD][TC][N];   // per direction and warp: dC terms, then dB terms

    const int b = blockIdx.z, c = blockIdx.y, blk = blockIdx.x, d0 = blk * CH;
    const int t0 = c * TC, tc = min(TC, p.L - t0);

    // ---- stage the chunk: u, dy = dout silu(z), dout silu'(z), Delta and
    // sigmoid(delta_raw + bias) per direction, B and C per direction ----------------
    for (int li = threadIdx.x; li < TC * CH; li += SH::kThr) {
        const int r = li / CH, cl = li % CH, ch = d0 + cl;
        float u = 0.0f, e = 0.0f, ezf = 0.0f, dl0 = 0.0f, dl1 = 0.0f, sg0 = 0.0f, sg1 = 0.0f;
        if (r < tc && ch < p.Di) {
            const size_t i = ((size_t)b * p.L + t0 + r) * p.Di + ch;
            u = ld<T>(p.u, i);
            const float dr = ld<T>(p.delta, i), o = ld<T>(p.dout, i);
            if (p.z) {
                const float z = ld<T>(p.z, i);
                e = o * silu(z);
                ezf = o * silu_grad(z);
            } else {
                e = o;
            }
            const float x0 = dr + p.bias[ch], x1 = dr + p.bias[p.Di + ch];
            dl0 = softplus(x0); sg0 = softplus_grad(x0);
            dl1 = softplus(x1); sg1 = softplus_grad(x1);
        }
        sU[r][cl] = u; sDy[r][cl] = e; sDzf[r][cl] = ezf;
        sDelta[0][r][cl] = dl0; sDelta[1][r][cl] = dl1;
        sSig[0][r][cl] = sg0; sSig[1][r][cl] = sg1;
    }
    for (int li = threadIdx.x; li < 2 * TC * N; li += SH::kThr) {
        const int k = li / (TC * N), r = (li / N) % TC, n = li % N;
        const size_t i = ((size_t)b * p.L + t0 + r) * N + n;
        sB[k][r][n] = r < tc ? ld<T>(p.B[k], i) : 0.0f;
        sC[k][r][n] = r < tc ? ld<T>(p.C[k], i) : 0.0f;
    }
    __syncthreads();

    const int tid = threadIdx.x, lane = tid & 31;
    const int q = tid % Q, cl = (tid / Q) % CH, dir = tid / (Q * CH), d = d0 + cl;
    const bool valid = d < p.Di;
    const int j0 = q * NT;                       // first state of this thread
    const int wid = (tid / 32) % WPD;            // warp within the direction
    float A2[NT], Araw[NT];
    float Dk = 0.0f;
#pragma unroll
    for (int j = 0; j < NT; ++j) Araw[j] = valid ? p.A[((size_t)dir * p.Di + d) * N + j0 + j] : 0.0f;
#pragma unroll
    for (int j = 0; j < NT; ++j) A2[j] = Araw[j] * kLog2e;
    if (valid) Dk = p.D[(size_t)dir * p.Di + d];
    const size_t cbase = (((size_t)b * p.G + c) * 2 + dir) * p.Di + d;   // [b][c][dir][d]

    // ---- forward sweep: checkpoints, y (ungated) and the dC terms -------------------
    float h[NT], ck[kBwdNSeg][NT];
#pragma unroll
    for (int j = 0; j < NT; ++j) h[j] = (p.G > 1 && valid) ? p.hin[cbase * N + j0 + j] : 0.0f;
#pragma unroll
    for (int i = 0; i < TC; ++i) {
        const int r = dir ? TC - 1 - i : i;
        if (i % kBwdSeg == 0) {
#pragma unroll
            for (int j = 0; j < NT; ++j) ck[i / kBwdSeg][j] = h[j];
        }
        const float dt = sDelta[dir][r][cl], x = sU[r][cl], e = sDy[r][cl];
        const float du = dt * x;
        float yp = q == 0 ? Dk * x : 0.0f;
        float v[NT];
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            h[j] = fmaf(ex2(dt * A2[j]), h[j], du * sB[dir][r][j0 + j]);
            yp = fmaf(sC[dir][r][j0 + j], h[j], yp);
            v[j] = e * h[j];
        }
#pragma unroll
        for (int s = 1; s < Q; s <<= 1) yp += __shfl_xor_sync(0xffffffffu, yp, s);
        if (q == 0) sY[dir][r][cl] = yp;
        int off;
        bool wr;
        reduce_channels<NT, Q, SH::CW>(v, lane, &off, &wr);
        if (wr) sRed[dir][wid][r][j0 + off] = v[0];
    }
    __syncthreads();
    // dz = dout silu'(z) (y^f + y^b), and the CTA's dC terms
    if (p.dz) {
        for (int li = threadIdx.x; li < TC * CH; li += SH::kThr) {
            const int r = li / CH, c2 = li % CH, ch = d0 + c2;
            if (r < tc && ch < p.Di)
                static_cast<T *>(p.dz)[((size_t)b * p.L + t0 + r) * p.Di + ch] =
                    from_f32<T>(sDzf[r][c2] * (sY[0][r][c2] + sY[1][r][c2]));
        }
    }
    store_bc_part<N, WPD>(p, sRed, p.dC_part, b, t0, tc, blk);
    __syncthreads();

    // ---- reverse: per segment, re-run h over it, then the adjoint sweep -------------
    float g[NT], dA[NT];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
        g[j] = (p.G > 1 && valid) ? p.gloc[cbase * N + j0 + j] : 0.0f;
        dA[j] = 0.0f;
    }
    float dD = 0.0f, dbias = 0.0f;
#pragma unroll
    for (int sg = kBwdNSeg - 1; sg >= 0; --sg) {
        float hist[kBwdSeg][NT];
#pragma unroll
        for (int j = 0; j < NT; ++j) h[j] = ck[sg][j];
#pragma unroll
        for (int m = 0; m < kBwdSeg; ++m) {
            const int i = sg * kBwdSeg + m, r = dir ? TC - 1 - i : i;
            const float dt = sDelta[dir][r][cl], du = dt * sU[r][cl];
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                h[j] = fmaf(ex2(dt * A2[j]), h[j], du * sB[dir][r][j0 + j]);
                hist[m][j] = h[j];
            }
        }
#pragma unroll
        for (int m = kBwdSeg - 1; m >= 0; --m) {
            const int i = sg * kBwdSeg + m, r = dir ? TC - 1 - i : i;
            const float dt = sDelta[dir][r][cl], x = sU[r][cl], e = sDy[r][cl];
            float sA = 0.0f, sBg = 0.0f, v[NT];
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                g[j] = fmaf(sC[dir][r][j0 + j], e, g[j]);                 // dl/dh_t
                const float hp = m > 0 ? hist[m - 1][j] : ck[sg][j];     // h_(t-1)
                const float ga = ex2(dt * A2[j]) * g[j];
                const float w = ga * hp;
                dA[j] = fmaf(dt, w, dA[j]);
                sA = fmaf(Araw[j], w, sA);
                sBg = fmaf(g[j], sB[dir][r][j0 + j], sBg);
                v[j] = g[j] * (dt * x);
                g[j] = ga;                                               // dl/dh_(t-1) part
            }
            float dup = dt * sBg;
            float ddp = fmaf(x, sBg, sA) * sSig[dir][r][cl];
#pragma unroll
            for (int s = 1; s < Q; s <<= 1) {
                dup += __shfl_xor_sync(0xffffffffu, dup, s);
                ddp += __shfl_xor_sync(0xffffffffu, ddp, s);
            }
            if (q == 0) {
                sDu[dir][r][cl] = fmaf(Dk, e, dup);
                sDd[dir][r][cl] = ddp;
                dD = fmaf(e, x, dD);
                dbias += ddp;
            }
            int off;
            bool wr;
            reduce_channels<NT, Q, SH::CW>(v, lane, &off, &wr);
            if (wr) sRed[dir][wid][r][j0 + off] = v[0];
        }
    }

    // ---- per-chunk sums over tokens ------------------------------------------------
    if (valid) {
#pragma unroll
        for (int j = 0; j < NT; ++j) p.dA_part[cbase * N + j0 + j] = dA[j];
        if (q == 0) {
            p.dD_part[cbase] = dD;
            p.dbias_part[cbase] = dbias;
        }
    }
    __syncthreads();
    for (int li = threadIdx.x; li < TC * CH; li += SH::kThr) {
        const int r = li / CH, c2 = li % CH, ch = d0 + c2;
        if (r < tc && ch < p.Di) {
            const size_t i = ((size_t)b * p.L + t0 + r) * p.Di + ch;
            static_cast<T *>(p.du)[i] = from_f32<T>(sDu[0][r][c2] + sDu[1][r][c2]);
            static_cast<T *>(p.ddelta)[i] = from_f32<T>(sDd[0][r][c2] + sDd[1][r][c2]);
        }
    }
    store_bc_part<N, WPD>(p, sRed, p.dB_part, b, t0, tc, blk);
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
__global__ void __launch_bounds__(256) bwd_reduce_cols2(const float *tmp, float *out, int cols) {
    const int col = blockIdx.x * blockDim.x + threadIdx.x;
    if (col >= cols) return;
    float acc = 0.0f;
    for (int part = 0; part < kReduceParts; ++part) acc += tmp[(int64_t)part * cols + col];
    out[col] = acc;
}

}  // namespace
}  // namespace vimscan
