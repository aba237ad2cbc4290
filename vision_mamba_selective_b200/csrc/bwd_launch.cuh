// bwd_launch.cuh -- host-side planning and launch sequence of the derivative kernels,
// shared by the translation units of the derivative entry points (bwd.cu: the scan and
// the scan with its convolution front; proj_bwd.cu: the block scan with its
// projections).  Everything here is internal to each unit that includes it.
#pragma once

#include <algorithm>
#include <cstdint>
#include <cstring>

#include "bwd_kernels.cuh"
#include "launch.cuh"

#ifndef VIMSCAN_BWD_CLUSTER
#define VIMSCAN_BWD_CLUSTER 1
#endif

namespace vimscan {
namespace {

struct BwdPlan {
    int G, nblk, nsets;
    int cl, ncol;   // cluster size along the channel blocks, and the partials' columns
    size_t off_hloc, off_ssum, off_gloc, off_gsum, off_par, off_dBp, off_dCp, off_tmp, total;
};

BwdPlan bwd_plan(int batch, int L, int Di, int N, int separate_bc) {
    BwdPlan pl;
    pl.G = (L + kBwdChunk - 1) / kBwdChunk;
    const int ch = N >= 8 ? BwdShape<16>::CH : BwdShape<4>::CH;   // channels per bwd_main CTA
    pl.nblk = (Di + ch - 1) / ch;
    pl.nsets = separate_bc ? 2 : 1;
    // channel blocks reduce their dB/dC terms in clusters of up to 8 (whole clusters of
    // the grid; the chunk's 32 rows split evenly over the ranks)
    pl.cl = 1;
    for (int c = VIMSCAN_BWD_CLUSTER; c > 1; c /= 2)
        if (pl.nblk % c == 0 && kBwdChunk % c == 0) { pl.cl = c; break; }
    pl.ncol = pl.nblk / pl.cl;
    const size_t units = (size_t)batch * pl.G * 2 * Di;      // (b, chunk, dir, channel)
    const size_t cols = (size_t)2 * Di * (N + 2);        // [dA | dD | d delta_bias]
    size_t o = 0;
    auto take = [&](size_t bytes) { const size_t at = o; o += round_up(bytes); return at; };
    pl.off_hloc = take(units * N * 4);
    pl.off_ssum = take(units * 4);
    pl.off_gloc = take(units * N * 4);
    pl.off_gsum = take(units * 4);
    pl.off_par = take(units * (N + 2) * 4);
    pl.off_dBp = take((size_t)pl.nsets * batch * L * pl.ncol * N * 4);
    pl.off_dCp = take((size_t)pl.nsets * batch * L * pl.ncol * N * 4);
    pl.off_tmp = take((size_t)kReduceParts * cols * 4);
    pl.total = o;
    return pl;
}

// column sums of the per-chunk rows [dA | dD | d delta_bias] (two passes through tmp)
vim_status reduce_params(const float *par, float *tmp, float *dA, float *dD, float *dbias, int rows, int Di, int N,
                         cudaStream_t stream) {
    const int nA = 2 * Di * N, nD = 2 * Di, cols = nA + 2 * nD;
    const dim3 g1((cols + 255) / 256, kReduceParts);
    bwd_reduce_cols1<<<g1, 256, 0, stream>>>(par, tmp, rows, cols);
    if (cudaGetLastError() != cudaSuccess) return VIM_ERR_CUDA;
    bwd_reduce_cols2<<<(cols + 255) / 256, 256, 0, stream>>>(tmp, dA, dD, dbias, nA, nD);
    return cudaGetLastError() == cudaSuccess ? VIM_OK : VIM_ERR_CUDA;
}

// events: null, or 4 events recorded before the summaries, after them, after bwd_main
// and after the reductions
inline bool rec(cudaEvent_t *ev, int i, cudaStream_t stream) {
    return !ev || cudaEventRecord(ev[i], stream) == cudaSuccess;
}

// ZOH: the exact hold's derivative (its own forward summaries and main kernel; the
// adjoint summaries do not involve Bbar)
// U2: per-direction fp32 inputs u; FRONT: the forward summaries form them from x by the
// convolution fronts (else they read fwd.u); DT: delta_raw from the projections' step
// input (fwd.dt_in, dt_w)
template <typename T, int N, bool ZOH, bool U2 = false, bool DT = false, bool FRONT = U2>
vim_status launch_bwd(const BwdArgs &a, const PairArgs &fwd, float *dB_out[2], float *dC_out[2], float *dA,
                      float *dD, float *dbias, float *tmp, cudaStream_t stream, cudaEvent_t *ev) {
    if (!rec(ev, 0, stream)) return VIM_ERR_CUDA;
    if (a.G > 1 && !a.hin_given) {
        // h entering each chunk: the forward scan's own summary kernels, each CTA walking
        // kBwdCarrySpan consecutive chunks (skipped when the forward pass left them)
        PairArgs fc = fwd;
        fc.carry_span = kBwdCarrySpan;
        const dim3 gf((a.Di + kDC - 1) / kDC, (a.G + kBwdCarrySpan - 1) / kBwdCarrySpan, a.batch);
        // (U2: the pathways' inputs formed from x by the convolution fronts, as in the
        // scan with its front)
        const size_t sc = 2 * (size_t)Stage<T, N, FRONT>::kSlotBytes;
        auto carry = pair_carry<T, N, false, FRONT, ZOH, DT, true>;
        if constexpr (bc_vectorizable<T, N>()) {
            // B and C rows as 16-byte vectors when every base allows it
            if (aligned16(fwd.B[0]) && aligned16(fwd.B[1]) && aligned16(fwd.C[0]) && aligned16(fwd.C[1]))
                carry = pair_carry<T, N, true, FRONT, ZOH, DT, true>;
        }
        if (cudaFuncSetAttribute(carry, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sc) != cudaSuccess)
            return VIM_ERR_CUDA;
        carry<<<gf, kThreads, sc, stream>>>(fc);
        if (cudaGetLastError() != cudaSuccess) return VIM_ERR_CUDA;
        const int64_t units = (int64_t)a.batch * 2 * a.Di * N;
        const dim3 gc((unsigned)((units + 255) / 256));
        pair_combine<N><<<gc, 256, 0, stream>>>(fwd);
        if (cudaGetLastError() != cudaSuccess) return VIM_ERR_CUDA;
    }
    if (a.G > 1) {
        const int64_t units = (int64_t)a.batch * 2 * a.Di * N;
        const dim3 gc((unsigned)((units + 255) / 256));
        // adjoint entering each chunk from the side its direction visits later
        adj_carry<T, N, DT><<<dim3((a.Di + kAdjCh - 1) / kAdjCh, a.G, a.batch), 2 * kAdjCh, 0, stream>>>(a);
        if (cudaGetLastError() != cudaSuccess) return VIM_ERR_CUDA;
        PairArgs adj = fwd;
        adj.hloc = a.gloc;
        adj.ssum = a.gsum;
        adj.fold_reverse = 1;
        pair_combine<N><<<gc, 256, 0, stream>>>(adj);
        if (cudaGetLastError() != cudaSuccess) return VIM_ERR_CUDA;
    }
    if (!rec(ev, 1, stream)) return VIM_ERR_CUDA;
    constexpr size_t sm = BwdShape<N>::kSmemBytes;
    if (cudaFuncSetAttribute(bwd_main<T, N, ZOH, U2, DT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) !=
        cudaSuccess)
        return VIM_ERR_CUDA;
    const dim3 gm(a.nblk, a.G, a.batch);
    {
        // with several chunks, a programmatic dependent of the adjoint fold: its launch
        // and the staging of the first CTAs overlap the fold's end; it waits for the
        // fold before it reads the carries.  Clusters of a.cl CTAs along the channel
        // blocks reduce the dB/dC terms on chip.
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = gm;
        cfg.blockDim = dim3(BwdShape<N>::kThr);
        cfg.dynamicSmemBytes = sm;
        cfg.stream = stream;
        cudaLaunchAttribute attr[2];
        int na = 0;
        if (a.cl > 1) {
            attr[na].id = cudaLaunchAttributeClusterDimension;
            attr[na].val.clusterDim.x = (unsigned)a.cl;
            attr[na].val.clusterDim.y = 1;
            attr[na].val.clusterDim.z = 1;
            ++na;
        }
        if (a.G > 1 && VIMSCAN_PDL) {
            attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            attr[na].val.programmaticStreamSerializationAllowed = 1;
            ++na;
        }
        cfg.attrs = attr;
        cfg.numAttrs = na;
        if (cudaLaunchKernelEx(&cfg, bwd_main<T, N, ZOH, U2, DT>, a) != cudaSuccess) return VIM_ERR_CUDA;
    }
    if (cudaGetLastError() != cudaSuccess) return VIM_ERR_CUDA;
    if (!rec(ev, 2, stream)) return VIM_ERR_CUDA;
    const int sets = a.separate_bc ? 2 : 1;
    const int rows = a.batch * a.L;
    for (int k = 0; k < sets; ++k) {
        const unsigned blocks = (unsigned)(((int64_t)rows * N + 255) / 256);
        bwd_reduce_bc<N><<<blocks, 256, 0, stream>>>(a.dB_part[k], dB_out[k], rows, a.ncol);
        bwd_reduce_bc<N><<<blocks, 256, 0, stream>>>(a.dC_part[k], dC_out[k], rows, a.ncol);
        if (cudaGetLastError() != cudaSuccess) return VIM_ERR_CUDA;
    }
    const int prow = a.batch * a.G;
    if (reduce_params(a.par, tmp, dA, dD, dbias, prow, a.Di, N, stream) != VIM_OK) return VIM_ERR_CUDA;
    return rec(ev, 3, stream) ? VIM_OK : VIM_ERR_CUDA;
}

template <typename T, bool ZOH, bool U2 = false, bool DT = false, bool FRONT = U2>
vim_status launch_bwd_n(int N, const BwdArgs &a, const PairArgs &fwd, float *dB[2], float *dC[2], float *dA,
                        float *dD, float *dbias, float *tmp, cudaStream_t stream, cudaEvent_t *ev) {
    switch (N) {
        case 2: return launch_bwd<T, 2, ZOH, U2, DT, FRONT>(a, fwd, dB, dC, dA, dD, dbias, tmp, stream, ev);
        case 4: return launch_bwd<T, 4, ZOH, U2, DT, FRONT>(a, fwd, dB, dC, dA, dD, dbias, tmp, stream, ev);
        case 8: return launch_bwd<T, 8, ZOH, U2, DT, FRONT>(a, fwd, dB, dC, dA, dD, dbias, tmp, stream, ev);
        case 16: return launch_bwd<T, 16, ZOH, U2, DT, FRONT>(a, fwd, dB, dC, dA, dD, dbias, tmp, stream, ev);
        default: return VIM_ERR_UNSUPPORTED;
    }
}

bool aligned_to(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// vector access of four channels (8 bytes of bf16, 16 of fp32) to every [.., Di]
// tensor, and of whole 16-byte B/C vectors, when the pointers allow it
void set_vector_flags(BwdArgs &a, vim_dtype dt, int N) {
    const size_t va = dt == VIM_F32 ? 16 : 8;
    a.vec_io = aligned_to(a.u, va) && aligned_to(a.delta, va) && aligned_to(a.dout, va) &&
               (!a.z || aligned_to(a.z, va)) && aligned_to(a.du, va) && aligned_to(a.ddelta, va) &&
               (!a.dz || aligned_to(a.dz, va));
    a.vec_bc = (N * elem_size(dt)) % 16 == 0 && aligned16(a.B[0]) && aligned16(a.B[1]) && aligned16(a.C[0]) &&
               aligned16(a.C[1]);
}


// ---- the convolution fronts ------------------------------------------------------

// the derivative's own workspace, then both pathways' u (element type) and dl/du
// (fp32), and the fronts' partial sums with their reduction buffer
struct ConvBwdPlan {
    BwdPlan pl;
    int runs;
    size_t off_u2, off_du2, off_part, off_ptmp, total;
};

ConvBwdPlan conv_bwd_plan(int batch, int L, int Di, int N, vim_dtype dt, int separate_bc) {
    ConvBwdPlan c;
    c.pl = bwd_plan(batch, L, Di, N, separate_bc);
    size_t o = round_up(c.pl.total);
    auto take = [&](size_t bytes) { const size_t at = o; o += round_up(bytes); return at; };
    const size_t act = (size_t)batch * L * Di;
    c.runs = (L + kFrontRows - 1) / kFrontRows;
    c.off_u2 = take(2 * act * 4);
    c.off_du2 = take(2 * act * 4);
    c.off_part = take((size_t)batch * c.runs * 8 * Di * 4);
    c.off_ptmp = take((size_t)kReduceParts * 8 * Di * 4);
    c.total = o;
    return c;
}

// grid of the front kernels: (batch item, run of kFrontRows tokens) x channel tiles
inline dim3 front_grid(int batch, int L, int Di) {
    return dim3((unsigned)((int64_t)batch * ((L + kFrontRows - 1) / kFrontRows)),
                (unsigned)((Di + kFrontCh - 1) / kFrontCh));
}

// both pathways' smoothed inputs u_k = silu(conv_k(x)) into u2 [2][batch, L, Di] fp32
template <typename T>
vim_status launch_front_fwd(const T *x, const float *conv_w, const float *conv_b, float *u2, int batch, int L, int Di,
                            int vec, cudaStream_t stream) {
    conv_front_fwd<T><<<front_grid(batch, L, Di), kFrontThr, 0, stream>>>(x, conv_w, conv_b, u2, batch, L, Di, vec);
    return cudaGetLastError() == cudaSuccess ? VIM_OK : VIM_ERR_CUDA;
}

template <typename T>
vim_status launch_fronts_bwd(const T *x, const float *conv_w, const float *conv_b, const float *du2, T *dx,
                             float *part, float *ptmp, float *dconv_w, float *dconv_b, int batch, int L, int Di,
                             int runs, int vec, cudaStream_t stream) {
    conv_front_bwd<T><<<front_grid(batch, L, Di), kFrontThr, 0, stream>>>(x, conv_w, conv_b, du2, dx, part, batch, L,
                                                                           Di, vec);
    if (cudaGetLastError() != cudaSuccess) return VIM_ERR_CUDA;
    // rows of [dw: 6 Di | dcb: 2 Di] summed in a fixed order
    const int cols = 8 * Di;
    bwd_reduce_cols1<<<dim3((cols + 255) / 256, kReduceParts), 256, 0, stream>>>(part, ptmp, batch * runs, cols);
    if (cudaGetLastError() != cudaSuccess) return VIM_ERR_CUDA;
    bwd_reduce_cols2<<<(cols + 255) / 256, 256, 0, stream>>>(ptmp, dconv_w, dconv_b, dconv_b + Di, 6 * Di, Di);
    return cudaGetLastError() == cudaSuccess ? VIM_OK : VIM_ERR_CUDA;
}

}  // namespace
}  // namespace vimscan
