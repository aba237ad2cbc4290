// proj_kernels.cuh -- sm_100a kernel of the S6 modules' input projection (x_proj).
//
// Each pathway k of the Vim block derives B, C and its one-column step input s from
// its own smoothed input u_k (page "Vision Mamba Guide", the SimpleSelectiveSSM
// module: a bias-free linear map to 2N + 1 columns, split as B | C | s; dt_proj then
// maps s back to every channel, which the scan does in registers):
//   P_k[m, :] = u_k[m, :] Wx[k],   u_k = silu(conv_k(x)) or x,
//   B_k = P_k[:, 0:N],  C_k = P_k[:, N:2N],  s_k = P_k[:, 2N]
// A CTA serves one pathway: it stages Wx[k] transposed once, then for each of its
// 128-token tiles (rows of the flattened [batch*L] sequence) forms u_k one 64-channel
// slice at a time in shared memory (bf16), stores it for the scan when asked, and
// multiplies on the tensor cores with mma.sync m16n8k16 (bf16 in, fp32 accumulate),
// one warp per 16 rows.  The
// product has only 2N + 1 <= 33 columns, so the kernel is bound by reading x, not by
// the tensor pipe.
#pragma once

#include <algorithm>
#include <atomic>
#include <type_traits>

#include "scan_kernels.cuh"

namespace vimscan {

struct ProjArgs {
    const void *x;                  // [M][Di] bf16
    const float *conv_w, *conv_b;   // [2][Di][3], [2][Di], or null: no convolution front
    const void *Wx;                 // [2][Di][2N+1] bf16
    void *Bo, *Co;                  // [2][M][N] bf16
    float *s;                       // [2][M] fp32
    void *uo;                       // [2][M][Di] bf16: each pathway's u as the scan reads it, or null
    int64_t M;
    int L, Di;
};

#ifndef VIMSCAN_PROJ_ROWS
#define VIMSCAN_PROJ_ROWS 128
#endif
constexpr int kProjRows = VIMSCAN_PROJ_ROWS;   // tokens per tile: 16 per warp
constexpr int kProjThreads = 2 * kProjRows;    // one warp per 16 rows
constexpr int kProjK = 64;          // channels per K slice
constexpr int kProjPad = 8;         // row padding (bf16 elements) of the shared tiles

namespace {

#ifndef VIMSCAN_PROJ_TANH
#define VIMSCAN_PROJ_TANH 1
#endif
__device__ __forceinline__ float tanh_approx(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int N> struct ProjShape {
    static constexpr int NO = 2 * N + 1;
    static constexpr int NT8 = (NO + 7) / 8;                 // n8 tiles of the output
    static constexpr int LDU = kProjK + kProjPad;            // row length (bf16) of sX and sU
    static constexpr int XROWS = kProjRows + 2;              // x rows of a tile with both neighbours
    // dynamic shared memory: sX [2][XROWS][LDU] (x slices, double buffered), sU
    // [kProjRows][LDU], then Wx[k]^T [NT8*8][Di + kProjPad]
    static size_t smem_bytes(int Di) {
        return ((size_t)2 * XROWS * LDU + (size_t)kProjRows * LDU + (size_t)NT8 * 8 * (Di + kProjPad)) * 2;
    }
};

// One CTA per pathway and group of kProjRows-token tiles.  Wx[k] is staged once, transposed
// ([output column][channel]).  The (tile, 64-channel slice) steps form one pipeline:
// cp.async brings the next step's x rows (the tile plus one neighbour row on each side)
// while the current step forms u -- thread (pair p, group q) takes channels 2p, 2p+1 of
// rows 16q .. 16q+15 -- and the warps run its tensor-core products.
template <int N, bool CONV>
__global__ void __launch_bounds__(kProjThreads) xproj_kernel(ProjArgs p) {
    using PS = ProjShape<N>;
    constexpr int NO = PS::NO, NT8 = PS::NT8, LDU = PS::LDU, XROWS = PS::XROWS;
    extern __shared__ __align__(16) __nv_bfloat16 psm[];
    __nv_bfloat16 *sX = psm;                                        // [2][XROWS][LDU]
    __nv_bfloat16(*sU)[LDU] = reinterpret_cast<__nv_bfloat16(*)[LDU]>(psm + 2 * XROWS * LDU);
    __nv_bfloat16 *sW = psm + 2 * XROWS * LDU + kProjRows * LDU;
    const int LDW = p.Di + kProjPad;

    const int dir = blockIdx.x;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32, g = lane / 4, tg = lane % 4;
    const __nv_bfloat16 *x = static_cast<const __nv_bfloat16 *>(p.x);
    const __nv_bfloat16 *W = static_cast<const __nv_bfloat16 *>(p.Wx) + (size_t)dir * p.Di * NO;
    const int M = (int)p.M;          // the entry point keeps batch * L * d_inner below 2^31
    const int nslice = (p.Di + kProjK - 1) / kProjK;
    const int ntiles = (M + kProjRows - 1) / kProjRows;
    const int mytiles = blockIdx.y < ntiles ? (ntiles - 1 - blockIdx.y) / gridDim.y + 1 : 0;
    const int nsteps = mytiles * nslice;

    // x rows m0-1 .. m0+kProjRows, channels kc .. kc+63 of step `st` into buffer `buf`; rows
    // outside 0..M-1 and channels past d_inner are zero-filled
    auto issue = [&](int st, int buf) {
        const int tile = blockIdx.y + (st / nslice) * gridDim.y, kc = (st % nslice) * kProjK;
        const int m0 = tile * kProjRows;
        __nv_bfloat16 *dst = sX + buf * XROWS * LDU;
        for (int li = tid; li < XROWS * (kProjK / 8); li += kProjThreads) {
            const int r = li / (kProjK / 8), c8 = (li % (kProjK / 8)) * 8;
            const int m = m0 - 1 + r, d = kc + c8;
            const bool ok = m >= 0 && m < M && d < p.Di;
            cp_async16(dst + r * LDU + c8, ok ? x + (size_t)m * p.Di + d : x, ok);
        }
        cp_async_commit();
    };

    if (nsteps > 0) issue(0, 0);
    // Wx[k] transposed: read in its own order (coalesced), eight loads in flight per thread
    const int nW = p.Di * NO;
#pragma unroll 8
    for (int li = tid; li < nW; li += kProjThreads) {
        const int d = li / NO, jcol = li % NO;
        sW[jcol * LDW + d] = W[li];
    }
    for (int li = tid; li < (NT8 * 8 - NO) * p.Di; li += kProjThreads)
        sW[(NO + li / p.Di) * LDW + li % p.Di] = __float2bfloat16_rn(0.0f);

    const int cp = lane, rg = warp;          // channel pair and row group of the u pass
    // the pair's taps on x[t-1], x[t], x[t+1] and bias for the slice of step `st`, as
    // (channel d, channel d+1); the backward pathway convolves the reversed sequence,
    // which swaps the outer taps.  Loaded one step ahead, beside that step's x rows.
    struct Taps { float2 wm, wc, wp, cb; };
    auto taps_of = [&](int st) {
        Taps tp{f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};
        const int d = (st % nslice) * kProjK + 2 * cp;
        if (CONV && d < p.Di) {
            const float *wa = p.conv_w + ((size_t)dir * p.Di + d) * 3;
            tp.wm = dir ? f2(wa[2], wa[5]) : f2(wa[0], wa[3]);
            tp.wc = f2(wa[1], wa[4]);
            tp.wp = dir ? f2(wa[0], wa[3]) : f2(wa[2], wa[5]);
            tp.cb = f2(p.conv_b[(size_t)dir * p.Di + d], p.conv_b[(size_t)dir * p.Di + d + 1]);
        }
        return tp;
    };
    Taps next_taps = taps_of(0);
    float acc[NT8][4];
    for (int st = 0; st < nsteps; ++st) {
        const Taps taps = next_taps;
        const int tile = blockIdx.y + (st / nslice) * gridDim.y, kc = (st % nslice) * kProjK;
        const int m0 = tile * kProjRows;
        if (kc == 0) {
#pragma unroll
            for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[nt][e] = 0.0f;
        }
        if (st + 1 < nsteps) {
            issue(st + 1, (st + 1) & 1);
            next_taps = taps_of(st + 1);
            asm volatile("cp.async.wait_group 1;\n" ::);
        } else {
            cp_async_wait_all();
        }
        __syncthreads();

        // u for channels kc + 2cp, +1 of rows r0 .. r0+15 (x row r of the tile is sX row r+1)
        const __nv_bfloat16 *xs = sX + (st & 1) * XROWS * LDU;
        const int d = kc + 2 * cp;
        const bool dvalid = d < p.Di;            // d_inner is a multiple of 8: pairs are whole
        const float2 wm = taps.wm, wc = taps.wc, wp = taps.wp, cbv = taps.cb;
        const int r0 = rg * 16;
        const int t = (m0 + r0) % p.L;            // position of row r0 in its sequence
        auto xrow = [&](int r) {                  // x of tile row r (-1 .. kProjRows), channels d, d+1
            return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(xs + (r + 1) * LDU + 2 * cp));
        };
        // sliding window over the rows, kept in registers (one shared-memory load per row).
        // MASK: the group reaches a sequence end (where the convolution's outer taps meet
        // its zero padding) or the data's end, or the pair lies past d_inner; the other
        // groups run without the per-row selects
        auto form_rows = [&](auto mask) {
            constexpr bool MASK = decltype(mask)::value;
            int tt = t;
            float2 xm = CONV ? xrow(r0 - 1) : f2(0.f, 0.f), x0 = xrow(r0);
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float2 u = x0;
                float2 xp = f2(0.f, 0.f);
                if (CONV) {
                    xp = xrow(r0 + r + 1);
                    float2 mm = wm, mp = wp;
                    if constexpr (MASK) {   // neighbours outside the sequence are the zero padding
                        if (tt == 0) mm = f2(0.f, 0.f);
                        if (tt == p.L - 1) mp = f2(0.f, 0.f);
                    }
                    const float2 v = fma2(mm, xm, fma2(wc, x0, fma2(mp, xp, cbv)));
#if VIMSCAN_PROJ_TANH
                    // silu(v) = v (1 + tanh(v/2)) / 2 with the MUFU tanh (relative error near
                    // 2^-11, below the bf16 rounding that u takes next)
                    const float2 hv = mul2(v, f2(0.5f, 0.5f));
                    u = fma2(hv, f2(tanh_approx(hv.x), tanh_approx(hv.y)), hv);
#else
                    const float2 e = mul2(v, f2(-kLog2e, -kLog2e));
                    const float2 den = f2(1.0f + ex2(e.x), 1.0f + ex2(e.y));
                    u = mul2(v, f2(rcp(den.x), rcp(den.y)));          // silu(v) = v / (1 + e^-v)
#endif
                }
                if constexpr (MASK) {
                    if (m0 + r0 + r >= M || !dvalid) u = f2(0.f, 0.f);
                    tt = tt + 1 == p.L ? 0 : tt + 1;
                }
                *reinterpret_cast<__nv_bfloat162 *>(&sU[r0 + r][2 * cp]) = __floats2bfloat162_rn(u.x, u.y);
                if (CONV) {
                    xm = x0;
                    x0 = xp;
                } else if (r + 1 < 16) {
                    x0 = xrow(r0 + r + 1);
                }
            }
        };
        // rows t .. t+15 of one sequence, none at its first or last position, all below M
        if (dvalid && t > 0 && t + 16 < p.L && m0 + r0 + 16 <= M) form_rows(std::false_type{});
        else form_rows(std::true_type{});
        __syncthreads();
        if (p.uo) {
            // the slice of u_k, 16 bytes at a time, for the scan (which then forms no front)
            __nv_bfloat16 *uo = static_cast<__nv_bfloat16 *>(p.uo) + (size_t)dir * p.M * p.Di;
            for (int li = tid; li < kProjRows * (kProjK / 8); li += kProjThreads) {
                const int r = li / (kProjK / 8), c8 = (li % (kProjK / 8)) * 8;
                const int m = m0 + r, dd = kc + c8;
                if (m < M && dd < p.Di)
                    *reinterpret_cast<uint4 *>(uo + (size_t)m * p.Di + dd) = *reinterpret_cast<const uint4 *>(&sU[r][c8]);
            }
        }
#pragma unroll
        for (int ks = 0; ks < kProjK / 16; ++ks) {
            const int ra = warp * 16 + g, k0 = ks * 16 + tg * 2;
            uint32_t a[4];
            a[0] = *reinterpret_cast<const uint32_t *>(&sU[ra][k0]);
            a[1] = *reinterpret_cast<const uint32_t *>(&sU[ra + 8][k0]);
            a[2] = *reinterpret_cast<const uint32_t *>(&sU[ra][k0 + 8]);
            a[3] = *reinterpret_cast<const uint32_t *>(&sU[ra + 8][k0 + 8]);
#pragma unroll
            for (int nt = 0; nt < NT8; ++nt) {
                const __nv_bfloat16 *wr = sW + (nt * 8 + g) * LDW + kc + k0;
                const uint32_t b0 = (kc + k0 < p.Di) ? *reinterpret_cast<const uint32_t *>(wr) : 0u;
                const uint32_t b1 = (kc + k0 + 8 < p.Di) ? *reinterpret_cast<const uint32_t *>(wr + 8) : 0u;
                mma_bf16_16816(acc[nt], a, b0, b1);
            }
        }

        if (kc + kProjK >= p.Di) {
            // epilogue of the tile: row g (and g + 8) of the warp's 16, columns nt*8 + 2*tg (+1)
            __nv_bfloat16 *Bo = static_cast<__nv_bfloat16 *>(p.Bo) + (size_t)dir * p.M * N;
            __nv_bfloat16 *Co = static_cast<__nv_bfloat16 *>(p.Co) + (size_t)dir * p.M * N;
            float *so = p.s + (size_t)dir * p.M;
#pragma unroll
            for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int m = m0 + warp * 16 + g + (e >= 2 ? 8 : 0);
                    const int col = nt * 8 + tg * 2 + (e & 1);
                    if (m >= M || col >= NO) continue;
                    if (col < N) Bo[(size_t)m * N + col] = __float2bfloat16_rn(acc[nt][e]);
                    else if (col < 2 * N) Co[(size_t)m * N + col - N] = __float2bfloat16_rn(acc[nt][e]);
                    else so[m] = acc[nt][e];
                }
        }
        // sU and this step's sX buffer are rewritten two steps on: the barrier at the
        // top of the next step orders the reads above before those writes
    }
}

// ----------------------------------------------------------------------------
// launch of the projection kernel (host side)
// ----------------------------------------------------------------------------
template <int N, bool CONV>
vim_status launch_proj_c(const ProjArgs &pa, cudaStream_t stream) {
    const size_t sm = ProjShape<N>::smem_bytes(pa.Di);
    auto kernel = xproj_kernel<N, CONV>;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) != cudaSuccess)
        return VIM_ERR_CUDA;
    // resident CTAs per SM for this variant and d_inner, looked up once (per device: the
    // first device's answer serves every B200 of a node)
    static std::atomic<int> cached_sms{0}, cached_per_sm{0}, cached_di{-1};
    int sms = cached_sms.load(), per_sm = cached_per_sm.load();
    if (sms == 0 || cached_di.load() != pa.Di) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kProjThreads, sm) != cudaSuccess)
            return VIM_ERR_CUDA;
        cached_sms.store(sms);
        cached_per_sm.store(per_sm);
        cached_di.store(pa.Di);
    }
    // each pathway's tiles spread over about half the resident CTAs; Wx is staged once per CTA
    const int64_t tiles = (pa.M + kProjRows - 1) / kProjRows;
    const int64_t ctas = std::max<int64_t>(1, std::min<int64_t>(tiles, (int64_t)sms * std::max(per_sm, 1) / 2));
    kernel<<<dim3(2, (unsigned)ctas), kProjThreads, sm, stream>>>(pa);
    return cudaGetLastError() == cudaSuccess ? VIM_OK : VIM_ERR_CUDA;
}

template <int N>
vim_status launch_proj(const ProjArgs &pa, bool conv, cudaStream_t stream) {
    return conv ? launch_proj_c<N, true>(pa, stream) : launch_proj_c<N, false>(pa, stream);
}

}  // namespace
}  // namespace vimscan
