// proj_bwd.cu -- host side and kernels of vim_block_scan_bwd: the derivative of the
// Vim block's two S6 modules with their input projections (x_proj, dt_proj) and the
// convolution fronts.  Declared in include/vimscan.h.
//
// The forward steps are formed again (the projection kernel for B, C and the step
// input s of both pathways; the fronts for u_k in fp32), the scan's derivative runs in
// its per-direction and step-input modes (each direction on its own u_k, B_k, C_k and
// delta_raw_k = s_k Wdt_k, leaving dl/du_k and dl/ddelta_raw_k per direction), and
// then the chain rule runs back through the projections:
//   dl/ds_k[m]  = sum_d dl/ddelta_raw_k[m, d] Wdt_k[d],   dl/dWdt_k[d] = sum_m dl/ddelta_raw_k[m, d] s_k[m],
//   dP_k[m, :]  = [dl/dB_k[m, :] | dl/dC_k[m, :] | dl/ds_k[m]],
//   dl/du_k    += dP_k Wx_k^T,                             dl/dWx_k = u_k^T dP_k,
// and through the fronts (or the identity) to x.
#include "vimscan.h"

#include <algorithm>
#include <cstdint>
#include <cstring>

#include "bwd_launch.cuh"
#include "proj_kernels.cuh"

namespace vimscan {
namespace {

constexpr int kPbRows = 128;   // tokens per CTA of proj_bwd_du_dwx
constexpr int kPbCh = 128;     // channels per CTA of proj_bwd_du_dwx (one per thread)

// u2[k] = x (fp32) for both pathways: the block without convolution fronts
__global__ void __launch_bounds__(256) block_u_copy(const __nv_bfloat16 *x, float *u2, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float v = __bfloat162float(x[i]);
        u2[i] = v;
        u2[n + i] = v;
    }
}

// Back through dt_proj, per pathway k and tile of kWdtRows tokens (one CTA of 256
// threads; warp w takes rows 8w .. 8w+7 of the tile, lane l channels l, l + 32, ...):
//   dl/ds_k[m] = sum_d dd2_k[m, d] Wdt_k[d]      (the row dP_k[m, :] = [dl/dB_k | dl/dC_k | dl/ds_k]),
//   part[tile][k * Di + d] = sum over the tile's rows of dd2_k[m, d] s_k[m]   (dl/dWdt partials).
// dd2 is read once, kDtSteps 32-channel steps of the warp's 8 rows in flight per lane (16
// loads); each warp's column sums go to its row of red[8][Di] in shared memory (dynamic,
// 32 Di bytes), which the CTA adds in warp order after one barrier; the column kernels sum
// the tiles.
constexpr int kWdtRows = 64;
#ifndef VIMSCAN_DT_STEPS
#define VIMSCAN_DT_STEPS 2
#endif
constexpr int kDtSteps = VIMSCAN_DT_STEPS;   // 32-channel steps of a lane's loads in flight
#ifndef VIMSCAN_DT_MINB
#define VIMSCAN_DT_MINB 3     // resident CTAs per SM the register budget targets
#endif
__global__ void __launch_bounds__(256, VIMSCAN_DT_MINB)
    proj_bwd_dt(const float *dd2, const float *Wdt, const float *s2, const float *dB2, const float *dC2, float *dP,
                float *tmp, int64_t M, int Di, int N) {
    constexpr int RW = kWdtRows / 8;   // rows per warp
    extern __shared__ float red[];     // [8][Di]
    const int k = blockIdx.y, warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t m0 = (int64_t)blockIdx.x * kWdtRows + warp * RW;   // the warp's first row
    const float *src = dd2 + ((size_t)k * M) * Di, *wdt = Wdt + (size_t)k * Di, *sk = s2 + (size_t)k * M;
    float sv[RW], rs[RW];
#pragma unroll
    for (int r = 0; r < RW; ++r) {
        sv[r] = m0 + r < M ? sk[m0 + r] : 0.0f;
        rs[r] = 0.0f;
    }
    for (int c0 = 0; c0 < Di; c0 += 32 * kDtSteps) {
        float v[kDtSteps][RW];
#pragma unroll
        for (int e = 0; e < kDtSteps; ++e)
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                const int d = c0 + 32 * e + lane;
                v[e][r] = (m0 + r < M && d < Di) ? src[(size_t)(m0 + r) * Di + d] : 0.0f;
            }
#pragma unroll
        for (int e = 0; e < kDtSteps; ++e) {
            const int d = c0 + 32 * e + lane;
            if (d < Di) {
                const float wd = wdt[d];
                float cs = 0.0f;
#pragma unroll
                for (int r = 0; r < RW; ++r) {
                    rs[r] = fmaf(v[e][r], wd, rs[r]);
                    cs = fmaf(v[e][r], sv[r], cs);
                }
                red[warp * Di + d] = cs;
            }
        }
    }
    __syncthreads();
    for (int d = threadIdx.x; d < Di; d += 256) {
        float a = 0.0f;
#pragma unroll
        for (int q = 0; q < 8; ++q) a += red[q * Di + d];
        tmp[(size_t)blockIdx.x * 2 * Di + (size_t)k * Di + d] = a;
    }
    const int NO = 2 * N + 1;
#pragma unroll
    for (int r = 0; r < RW; ++r) {
        float a = rs[r];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        const int64_t m = m0 + r;
        if (m < M) {
            const size_t row = (size_t)k * M + m;
            float *out = dP + row * NO;
            for (int j = lane; j < NO; j += 32) out[j] = j < N ? dB2[row * N + j] : j < 2 * N ? dC2[row * N + j - N] : a;
        }
    }
}

// dl/du_k += dP_k Wx_k^T, and dl/dWx_k partial sums over a tile of kPbRows tokens:
// part[tile][(k * Di + d) * NO + j] = sum_m u_k[m, d] dP_k[m, j].  One thread per channel
// d holds Wx_k[d, :] and its NO partial sums; the tile's dP rows are staged in shared
// memory.
template <int N>
__global__ void __launch_bounds__(kPbCh) proj_bwd_du_dwx(const float *dP, const __nv_bfloat16 *Wx, const float *u2,
                                                         float *du2, float *part, int64_t M, int Di) {
    constexpr int NO = 2 * N + 1;
    constexpr int NQ = (NO + 3) / 4;   // float4 per staged row (the row padded with zeros)
    __shared__ __align__(16) float4 sP[kPbRows][NQ];
    const int k = blockIdx.z, tile = blockIdx.y, d = blockIdx.x * kPbCh + threadIdx.x;
    const int64_t m0 = (int64_t)tile * kPbRows;
    const int rows = (int)(M - m0 < kPbRows ? M - m0 : kPbRows);
    const float *src = dP + ((size_t)k * M + m0) * NO;
    float *sp = reinterpret_cast<float *>(sP);
    for (int i = threadIdx.x; i < kPbRows * NQ * 4; i += kPbCh) {
        const int r = i / (NQ * 4), j = i % (NQ * 4);
        sp[i] = (r < rows && j < NO) ? src[(size_t)r * NO + j] : 0.0f;
    }
    __syncthreads();
    if (d >= Di) return;
    float2 w[2 * NQ], acc[2 * NQ];   // columns (2q, 2q+1), zero past NO
#pragma unroll
    for (int q = 0; q < 2 * NQ; ++q) {
        const int j0 = 2 * q, j1 = 2 * q + 1;
        const __nv_bfloat16 *wr = Wx + ((size_t)k * Di + d) * NO;
        w[q] = f2(j0 < NO ? __bfloat162float(wr[j0]) : 0.0f, j1 < NO ? __bfloat162float(wr[j1]) : 0.0f);
        acc[q] = f2(0.0f, 0.0f);
    }
    const size_t plane = (size_t)M * Di;
    const float *u = u2 + (size_t)k * plane + (size_t)m0 * Di + d;
    float *g = du2 + (size_t)k * plane + (size_t)m0 * Di + d;
    // kPbAhead tokens at a time: their u and dl/du loads are in flight together
    constexpr int kPbAhead = 8;
    for (int r0 = 0; r0 < rows; r0 += kPbAhead) {
        float uv[kPbAhead], gv[kPbAhead];
#pragma unroll
        for (int e = 0; e < kPbAhead; ++e) {
            const bool ok = r0 + e < rows;
            uv[e] = ok ? u[(size_t)(r0 + e) * Di] : 0.0f;
            gv[e] = ok ? g[(size_t)(r0 + e) * Di] : 0.0f;
        }
#pragma unroll
        for (int e = 0; e < kPbAhead; ++e) {
            const int r = r0 + e;
            if (r >= rows) break;
            const float2 ur2 = f2(uv[e], uv[e]);
            float2 s = f2(0.0f, 0.0f);
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
                const float4 p = sP[r][q];
                const float2 pa = f2(p.x, p.y), pb = f2(p.z, p.w);
                s = fma2(pa, w[2 * q], s);
                s = fma2(pb, w[2 * q + 1], s);
                acc[2 * q] = fma2(ur2, pa, acc[2 * q]);
                acc[2 * q + 1] = fma2(ur2, pb, acc[2 * q + 1]);
            }
            g[(size_t)r * Di] = gv[e] + (s.x + s.y);
        }
    }
    float *o = part + (size_t)tile * 2 * Di * NO + ((size_t)k * Di + d) * NO;
#pragma unroll
    for (int q = 0; q < 2 * NQ; ++q) {
        if (2 * q < NO) o[2 * q] = acc[q].x;
        if (2 * q + 1 < NO) o[2 * q + 1] = acc[q].y;
    }
}

// dx = dl/du_f + dl/du_b (the block without convolution fronts)
__global__ void __launch_bounds__(256) block_dx_sum(const float *du2, __nv_bfloat16 *dx, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        dx[i] = __float2bfloat16_rn(du2[i] + du2[n + i]);
}

struct BlockBwdPlan {
    BwdPlan pl;
    int runs, tiles;
    size_t off_B, off_C, off_s, off_u2, off_du2, off_dd2, off_dB, off_dC, off_dP, off_wtmp, off_xpart, off_xtmp,
        off_part, off_ptmp, total;
};

BlockBwdPlan block_bwd_plan(int batch, int L, int Di, int N) {
    BlockBwdPlan c;
    c.pl = bwd_plan(batch, L, Di, N, 1);
    const size_t M = (size_t)batch * L, NO = 2 * (size_t)N + 1, act = M * Di;
    size_t o = round_up(c.pl.total);
    auto take = [&](size_t bytes) { const size_t at = o; o += round_up(bytes); return at; };
    c.runs = (L + kFrontRows - 1) / kFrontRows;
    c.tiles = (int)((M + kPbRows - 1) / kPbRows);
    c.off_B = take(2 * M * N * 2);
    c.off_C = take(2 * M * N * 2);
    c.off_s = take(2 * M * 4);
    c.off_u2 = take(2 * act * 4);
    c.off_du2 = take(2 * act * 4);
    c.off_dd2 = take(2 * act * 4);
    c.off_dB = take(2 * M * N * 4);
    c.off_dC = take(2 * M * N * 4);
    c.off_dP = take(2 * M * NO * 4);
    c.off_wtmp = take(((M + 63) / 64 + kReduceParts) * 2 * Di * 4);   // the parts, then the column pass
    c.off_xpart = take((size_t)c.tiles * 2 * Di * NO * 4);
    c.off_xtmp = take((size_t)kReduceParts * 2 * Di * NO * 4);
    c.off_part = take((size_t)batch * c.runs * 8 * Di * 4);
    c.off_ptmp = take((size_t)kReduceParts * 8 * Di * 4);
    c.total = o;
    return c;
}

bool al4(const void *p) { return (reinterpret_cast<uintptr_t>(p) % 4) == 0; }

template <int N>
vim_status block_bwd_n(const void *x, const float *conv_w, const float *conv_b, const void *Wx, const float *Wdt,
                       const float *dt_bias, const float *A, const float *D, const void *z, const void *dout, void *dx,
                       float *dconv_w, float *dconv_b, float *dWx, float *dWdt, float *ddt_bias, float *dA, float *dD,
                       void *dz, int batch, int L, int Di, char *ws, const BlockBwdPlan &cp, cudaStream_t stream) {
    const BwdPlan &pl = cp.pl;
    const bool conv = conv_w != nullptr;
    const int64_t M = (int64_t)batch * L, act = M * Di;
    constexpr int NO = 2 * N + 1;
    const __nv_bfloat16 *xb = static_cast<const __nv_bfloat16 *>(x);
    float *s2 = reinterpret_cast<float *>(ws + cp.off_s), *u2 = reinterpret_cast<float *>(ws + cp.off_u2);
    float *du2 = reinterpret_cast<float *>(ws + cp.off_du2), *dd2 = reinterpret_cast<float *>(ws + cp.off_dd2);
    float *dB2 = reinterpret_cast<float *>(ws + cp.off_dB), *dC2 = reinterpret_cast<float *>(ws + cp.off_dC);
    float *dP = reinterpret_cast<float *>(ws + cp.off_dP);
    const unsigned grid_stride = 148 * 16;

    // ---- the forward steps: the projections (B, C, s) and both pathways' u in fp32 ----
    ProjArgs pa;
    std::memset(&pa, 0, sizeof(pa));
    pa.x = x; pa.conv_w = conv_w; pa.conv_b = conv_b; pa.Wx = Wx;
    pa.Bo = ws + cp.off_B; pa.Co = ws + cp.off_C; pa.s = s2; pa.uo = nullptr;
    pa.M = M; pa.L = L; pa.Di = Di;
    vim_status st = launch_proj<N>(pa, conv, stream);
    if (st != VIM_OK) return st;
    if (conv) {
        st = launch_front_fwd<__nv_bfloat16>(xb, conv_w, conv_b, u2, batch, L, Di, 1, stream);
        if (st != VIM_OK) return st;
    } else {
        block_u_copy<<<(unsigned)std::min<int64_t>((act + 255) / 256, grid_stride), 256, 0, stream>>>(xb, u2, act);
        if (cudaGetLastError() != cudaSuccess) return VIM_ERR_CUDA;
    }

    // ---- the scan's derivative, per direction ----------------------------------------
    const __nv_bfloat16 *Bw = reinterpret_cast<const __nv_bfloat16 *>(ws + cp.off_B);
    const __nv_bfloat16 *Cw = reinterpret_cast<const __nv_bfloat16 *>(ws + cp.off_C);
    BwdArgs a;
    std::memset(&a, 0, sizeof(a));
    a.u = u2; a.u_dir_stride = act; a.du2 = du2;
    a.dt_in = s2; a.dt_w = Wdt; a.dd2 = dd2;
    a.z = z; a.dout = dout; a.dz = dz;
    a.B[0] = Bw; a.B[1] = Bw + M * N; a.C[0] = Cw; a.C[1] = Cw + M * N;
    a.A = A; a.D = D; a.bias = dt_bias;
    const size_t set_elems = (size_t)M * pl.ncol * N;
    a.dB_part[0] = reinterpret_cast<float *>(ws + pl.off_dBp);
    a.dC_part[0] = reinterpret_cast<float *>(ws + pl.off_dCp);
    a.dB_part[1] = a.dB_part[0] + set_elems;
    a.dC_part[1] = a.dC_part[0] + set_elems;
    a.par = reinterpret_cast<float *>(ws + pl.off_par);
    a.hin = reinterpret_cast<const float *>(ws + pl.off_hloc);
    a.gloc = reinterpret_cast<float *>(ws + pl.off_gloc);
    a.gsum = reinterpret_cast<float *>(ws + pl.off_gsum);
    a.batch = batch; a.L = L; a.Di = Di; a.G = pl.G; a.nblk = pl.nblk; a.cl = pl.cl; a.ncol = pl.ncol;
    a.separate_bc = 1;
    a.vec_io = aligned_to(dout, 8) && (!z || aligned_to(z, 8)) && (!dz || aligned_to(dz, 8));
    a.vec_bc = (N * 2) % 16 == 0;   // the workspace's B and C rows are 256-byte aligned planes

    PairArgs f;
    std::memset(&f, 0, sizeof(f));
    f.u = x; f.conv_w = conv_w; f.conv_b = conv_b;
    f.B[0] = a.B[0]; f.B[1] = a.B[1]; f.C[0] = a.C[0]; f.C[1] = a.C[1];
    f.A = A; f.D = D; f.bias = dt_bias;
    f.dt_in = s2; f.dt_w = Wdt;
    f.hloc = reinterpret_cast<float *>(ws + pl.off_hloc);
    f.ssum = reinterpret_cast<float *>(ws + pl.off_ssum);
    f.batch = batch; f.L = L; f.Di = Di; f.H = 1; f.W = L; f.order = 0;
    f.chunk = kBwdChunk; f.G = pl.G;

    float *dBo[2] = {dB2, dB2 + M * N}, *dCo[2] = {dC2, dC2 + M * N};
    float *tmp = reinterpret_cast<float *>(ws + pl.off_tmp);
    st = conv ? launch_bwd<__nv_bfloat16, N, false, true, true, true>(a, f, dBo, dCo, dA, dD, ddt_bias, tmp, stream,
                                                                      nullptr)
              : launch_bwd<__nv_bfloat16, N, false, true, true, false>(a, f, dBo, dCo, dA, dD, ddt_bias, tmp, stream,
                                                                       nullptr);
    if (st != VIM_OK) return st;

    // ---- back through dt_proj and x_proj ------------------------------------------------
    float *wtmp = reinterpret_cast<float *>(ws + cp.off_wtmp);
    const int wparts = (int)((M + kWdtRows - 1) / kWdtRows);
    float *wtmp2 = wtmp + (size_t)wparts * 2 * Di;
    const size_t dt_smem = (size_t)8 * Di * sizeof(float);
    if (dt_smem > 48 * 1024 &&
        cudaFuncSetAttribute(proj_bwd_dt, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dt_smem) != cudaSuccess)
        return VIM_ERR_CUDA;
    proj_bwd_dt<<<dim3(wparts, 2), 256, dt_smem, stream>>>(dd2, Wdt, s2, dB2, dC2, dP, wtmp, M, Di, N);
    if (cudaGetLastError() != cudaSuccess) return VIM_ERR_CUDA;
    bwd_reduce_cols1<<<dim3((2 * Di + 255) / 256, kReduceParts), 256, 0, stream>>>(wtmp, wtmp2, wparts, 2 * Di);
    if (cudaGetLastError() != cudaSuccess) return VIM_ERR_CUDA;
    bwd_reduce_cols2<<<(2 * Di + 255) / 256, 256, 0, stream>>>(wtmp2, dWdt, nullptr, nullptr, 2 * Di, 0);
    if (cudaGetLastError() != cudaSuccess) return VIM_ERR_CUDA;
    float *xpart = reinterpret_cast<float *>(ws + cp.off_xpart), *xtmp = reinterpret_cast<float *>(ws + cp.off_xtmp);
    proj_bwd_du_dwx<N><<<dim3((Di + kPbCh - 1) / kPbCh, cp.tiles, 2), kPbCh, 0, stream>>>(
        dP, static_cast<const __nv_bfloat16 *>(Wx), u2, du2, xpart, M, Di);
    if (cudaGetLastError() != cudaSuccess) return VIM_ERR_CUDA;
    const int xcols = 2 * Di * NO;
    bwd_reduce_cols1<<<dim3((xcols + 255) / 256, kReduceParts), 256, 0, stream>>>(xpart, xtmp, cp.tiles, xcols);
    if (cudaGetLastError() != cudaSuccess) return VIM_ERR_CUDA;
    bwd_reduce_cols2<<<(xcols + 255) / 256, 256, 0, stream>>>(xtmp, dWx, nullptr, nullptr, xcols, 0);
    if (cudaGetLastError() != cudaSuccess) return VIM_ERR_CUDA;

    // ---- through the fronts (or the identity) to x --------------------------------------
    if (conv)
        return launch_fronts_bwd<__nv_bfloat16>(xb, conv_w, conv_b, du2, static_cast<__nv_bfloat16 *>(dx),
                                                reinterpret_cast<float *>(ws + cp.off_part),
                                                reinterpret_cast<float *>(ws + cp.off_ptmp), dconv_w, dconv_b, batch, L,
                                                Di, cp.runs, 1, stream);
    block_dx_sum<<<(unsigned)std::min<int64_t>((act + 255) / 256, grid_stride), 256, 0, stream>>>(
        du2, static_cast<__nv_bfloat16 *>(dx), act);
    return cudaGetLastError() == cudaSuccess ? VIM_OK : VIM_ERR_CUDA;
}

}  // namespace
}  // namespace vimscan

using namespace vimscan;

extern "C" {

size_t vim_block_bwd_workspace_bytes(int batch, int L, int d_inner, int d_state) {
    if (check_common(batch, L, d_inner, d_state, VIM_BF16) != VIM_OK) return 0;
    if (batch <= 0 || L <= 0 || d_inner <= 0) return 0;
    return block_bwd_plan(batch, L, d_inner, d_state).total;
}

vim_status vim_block_scan_bwd(const void *x, const float *conv_w, const float *conv_b, const void *Wx,
                              const float *Wdt, const float *dt_bias, const float *A, const float *D, const void *z,
                              const void *dout, void *dx, float *dconv_w, float *dconv_b, float *dWx, float *dWdt,
                              float *ddt_bias, float *dA, float *dD, void *dz, int batch, int L, int d_inner,
                              int d_state, vim_dtype dt, void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    vim_status st = check_common(batch, L, d_inner, d_state, dt);
    if (st != VIM_OK) return st;
    if (dt != VIM_BF16) return VIM_ERR_UNSUPPORTED;
    if (!conv_w != !conv_b || !conv_w != !dconv_w || !conv_w != !dconv_b) return VIM_ERR_INVALID_ARG;
    if ((z == nullptr) != (dz == nullptr)) return VIM_ERR_INVALID_ARG;
    if (ProjShape<16>::smem_bytes(d_inner) > (size_t)227 * 1024) return VIM_ERR_UNSUPPORTED;
    if (!Wx || !Wdt || !dt_bias || !A || !D || !dWx || !dWdt || !ddt_bias || !dA || !dD) return VIM_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(Wx) % 2) || !al4(Wdt) || !al4(dt_bias) || !al4(A) || !al4(D) || !al4(dWx) ||
        !al4(dWdt) || !al4(ddt_bias) || !al4(dA) || !al4(dD) || !al4(conv_w) || !al4(conv_b) || !al4(dconv_w) ||
        !al4(dconv_b))
        return VIM_ERR_INVALID_ARG;
    const int NO = 2 * d_state + 1;
    if (batch == 0 || L == 0 || d_inner == 0) {
        // no tokens: every parameter derivative is zero
        const size_t Di = (size_t)d_inner;
        if (cudaMemsetAsync(dWx, 0, sizeof(float) * 2 * Di * NO, stream) != cudaSuccess ||
            cudaMemsetAsync(dWdt, 0, sizeof(float) * 2 * Di, stream) != cudaSuccess ||
            cudaMemsetAsync(ddt_bias, 0, sizeof(float) * 2 * Di, stream) != cudaSuccess ||
            cudaMemsetAsync(dA, 0, sizeof(float) * 2 * Di * d_state, stream) != cudaSuccess ||
            cudaMemsetAsync(dD, 0, sizeof(float) * 2 * Di, stream) != cudaSuccess ||
            (dconv_w && cudaMemsetAsync(dconv_w, 0, sizeof(float) * 6 * Di, stream) != cudaSuccess) ||
            (dconv_b && cudaMemsetAsync(dconv_b, 0, sizeof(float) * 2 * Di, stream) != cudaSuccess))
            return VIM_ERR_CUDA;
        return VIM_OK;
    }
    if (!x || !dout || !dx) return VIM_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(dx) || (reinterpret_cast<uintptr_t>(dout) % 2) ||
        (z && reinterpret_cast<uintptr_t>(z) % 2) || (dz && reinterpret_cast<uintptr_t>(dz) % 2))
        return VIM_ERR_INVALID_ARG;
    const BlockBwdPlan cp = block_bwd_plan(batch, L, d_inner, d_state);
    if (!workspace || workspace_bytes < cp.total || !aligned_to(workspace, kAlign)) return VIM_ERR_WORKSPACE;
    char *ws = static_cast<char *>(workspace);
    switch (d_state) {
        case 2: return block_bwd_n<2>(x, conv_w, conv_b, Wx, Wdt, dt_bias, A, D, z, dout, dx, dconv_w, dconv_b, dWx,
                                      dWdt, ddt_bias, dA, dD, dz, batch, L, d_inner, ws, cp, stream);
        case 4: return block_bwd_n<4>(x, conv_w, conv_b, Wx, Wdt, dt_bias, A, D, z, dout, dx, dconv_w, dconv_b, dWx,
                                      dWdt, ddt_bias, dA, dD, dz, batch, L, d_inner, ws, cp, stream);
        case 8: return block_bwd_n<8>(x, conv_w, conv_b, Wx, Wdt, dt_bias, A, D, z, dout, dx, dconv_w, dconv_b, dWx,
                                      dWdt, ddt_bias, dA, dD, dz, batch, L, d_inner, ws, cp, stream);
        case 16: return block_bwd_n<16>(x, conv_w, conv_b, Wx, Wdt, dt_bias, A, D, z, dout, dx, dconv_w, dconv_b, dWx,
                                        dWdt, ddt_bias, dA, dD, dz, batch, L, d_inner, ws, cp, stream);
        default: return VIM_ERR_UNSUPPORTED;
    }
}

}  // extern "C"
