// proj.cu -- host side of vim_block_scan: the Vim block's two S6 modules from their
// common input, with the input projections (x_proj on the tensor cores, dt_proj folded
// into the scan) and optionally the convolution front.  Declared in include/vimscan.h.
#include "vimscan.h"

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>

#include "launch.cuh"
#include "proj_kernels.cuh"

namespace vimscan {
namespace {

struct BlockPlan {
    size_t off_B, off_C, off_s, off_u, off_sum, total;
};

// conv: the pathways' u (formed by the projection kernel) is kept for the scan
BlockPlan block_plan(int batch, int L, int Di, int N, bool conv) {
    BlockPlan pl;
    const size_t M = (size_t)batch * L;
    size_t o = 0;
    auto take = [&](size_t bytes) { const size_t at = o; o += round_up(bytes); return at; };
    pl.off_B = take(2 * M * N * 2);
    pl.off_C = take(2 * M * N * 2);
    pl.off_s = take(2 * M * 4);
    pl.off_u = take(conv ? 2 * M * Di * 2 : 0);
    pl.off_sum = take(summary_bytes(batch, L, Di, N));
    pl.total = o;
    return pl;
}

bool al(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace
}  // namespace vimscan

using namespace vimscan;

extern "C" {

size_t vim_block_workspace_bytes(int batch, int L, int d_inner, int d_state) {
    if (batch <= 0 || L <= 0 || d_inner <= 0 || d_state <= 0) return 0;
    return block_plan(batch, L, d_inner, d_state, true).total;
}

vim_status vim_block_scan(const void *x, const float *conv_w, const float *conv_b, const void *Wx,
                          const float *Wdt, const float *dt_bias, const float *A, const float *D, const void *z,
                          void *y, int batch, int L, int d_inner, int d_state, vim_dtype dt, void *workspace,
                          size_t workspace_bytes, cudaStream_t stream, cudaEvent_t *events) {
    vim_status st = check_common(batch, L, d_inner, d_state, dt);
    if (st != VIM_OK) return st;
    if (dt != VIM_BF16) return VIM_ERR_UNSUPPORTED;
    if (!conv_w != !conv_b) return VIM_ERR_INVALID_ARG;
    // the transposed Wx of one pathway must fit in one CTA's shared memory
    if (ProjShape<16>::smem_bytes(d_inner) > (size_t)227 * 1024) return VIM_ERR_UNSUPPORTED;
    if (batch == 0 || L == 0 || d_inner == 0) return VIM_OK;
    if (!x || !Wx || !Wdt || !dt_bias || !A || !D || !y) return VIM_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y) || (z && !aligned16(z)) || !al(Wx, 2) || !al(Wdt, 4) || !al(dt_bias, 4) ||
        !al(A, 4) || !al(D, 4) || !al(conv_w, 4) || !al(conv_b, 4))
        return VIM_ERR_INVALID_ARG;
    const bool conv = conv_w != nullptr;
    const BlockPlan pl = block_plan(batch, L, d_inner, d_state, conv);
    if (!workspace || workspace_bytes < pl.total || !al(workspace, kAlign)) return VIM_ERR_WORKSPACE;
    char *ws = static_cast<char *>(workspace);
    const int64_t M = (int64_t)batch * L;

    ProjArgs pa;
    std::memset(&pa, 0, sizeof(pa));
    pa.x = x; pa.conv_w = conv_w; pa.conv_b = conv_b; pa.Wx = Wx;
    pa.Bo = ws + pl.off_B; pa.Co = ws + pl.off_C; pa.s = reinterpret_cast<float *>(ws + pl.off_s);
    pa.uo = conv ? ws + pl.off_u : nullptr;
    pa.M = M; pa.L = L; pa.Di = d_inner;

    if (events && cudaEventRecord(events[0], stream) != cudaSuccess) return VIM_ERR_CUDA;
    switch (d_state) {
        case 2: st = launch_proj<2>(pa, conv, stream); break;
        case 4: st = launch_proj<4>(pa, conv, stream); break;
        case 8: st = launch_proj<8>(pa, conv, stream); break;
        case 16: st = launch_proj<16>(pa, conv, stream); break;
        default: return VIM_ERR_UNSUPPORTED;
    }
    if (st != VIM_OK) return st;
    if (events && cudaEventRecord(events[1], stream) != cudaSuccess) return VIM_ERR_CUDA;

    const Plan sp = plan_for(batch, L, d_inner);
    PairArgs a;
    std::memset(&a, 0, sizeof(a));
    // with the convolution front the scan reads each pathway's u as the projection
    // stored it; without it both directions read x
    a.u = conv ? static_cast<const void *>(ws + pl.off_u) : x;
    a.u_dir_stride = conv ? M * d_inner : 0;
    a.z = z;
    const __nv_bfloat16 *Bw = reinterpret_cast<const __nv_bfloat16 *>(ws + pl.off_B);
    const __nv_bfloat16 *Cw = reinterpret_cast<const __nv_bfloat16 *>(ws + pl.off_C);
    a.B[0] = Bw; a.B[1] = Bw + M * d_state;
    a.C[0] = Cw; a.C[1] = Cw + M * d_state;
    a.A = A; a.D = D; a.bias = dt_bias;
    a.dt_in = pa.s; a.dt_w = Wdt;
    a.y = y;
    a.batch = batch; a.L = L; a.Di = d_inner; a.H = 1; a.W = L; a.order = 0;
    a.chunk = sp.chunk; a.G = sp.G;
    if (sp.G > 1) {
        const size_t units = (size_t)batch * sp.G * 2 * d_inner;
        a.hloc = reinterpret_cast<float *>(ws + pl.off_sum);
        a.ssum = reinterpret_cast<float *>(ws + pl.off_sum + round_up(units * d_state * 4));
    }
    return launch_pair(a, d_state, dt, stream, events ? events + 2 : nullptr);
}

}  // extern "C"
