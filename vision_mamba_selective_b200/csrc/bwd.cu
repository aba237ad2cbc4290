// bwd.cu -- host side of the derivative of the Vim two-direction scan:
// vim_scan_bidir_bwd and its workspace query (declared in include/vimscan.h).
#include "vimscan.h"

#include <algorithm>
#include <cstdint>
#include <cstring>

#include "bwd_launch.cuh"


using namespace vimscan;

extern "C" {

size_t vim_scan_bwd_workspace_bytes(int batch, int L, int d_inner, int d_state, int separate_bc) {
    if (batch <= 0 || L <= 0 || d_inner <= 0 || d_state <= 0) return 0;
    return bwd_plan(batch, L, d_inner, d_state, separate_bc).total;
}

}  // extern "C"

namespace {

// the derivative of vim_scan_bidir; ckpt, or null: the forward pass's checkpoints
// (vim_scan_bidir_ckpt), which replace the derivative's own forward summaries
vim_status bidir_bwd_impl(const void *u, const void *delta, const void *z, const void *B, const void *C,
                          int64_t bc_dir_stride, const float *A, const float *D, const float *delta_bias,
                          const void *dout, void *du, void *ddelta, void *dz, float *dB, float *dC, float *dA,
                          float *dD, float *ddelta_bias, int batch, int L, int d_inner, int d_state, vim_dtype dt,
                          unsigned flags, void *workspace, size_t workspace_bytes, cudaStream_t stream,
                          cudaEvent_t *events, const float *ckpt) {
    if (flags & ~VIM_FLAG_ZOH_EXACT) return VIM_ERR_INVALID_ARG;
    const bool zoh = (flags & VIM_FLAG_ZOH_EXACT) != 0;
    vim_status st = check_common(batch, L, d_inner, d_state, dt);
    if (st != VIM_OK) return st;
    if (bc_dir_stride < 0) return VIM_ERR_INVALID_ARG;
    if ((z == nullptr) != (dz == nullptr)) return VIM_ERR_INVALID_ARG;
    if (!A || !D || !delta_bias || !dA || !dD || !ddelta_bias) return VIM_ERR_INVALID_ARG;
    if (!aligned_to(A, 4) || !aligned_to(D, 4) || !aligned_to(delta_bias, 4) || !aligned_to(dA, 4) ||
        !aligned_to(dD, 4) || !aligned_to(ddelta_bias, 4))
        return VIM_ERR_INVALID_ARG;
    const size_t es = elem_size(dt);
    if (batch == 0 || L == 0 || d_inner == 0) {
        // no tokens: the parameter derivatives are zero
        if (cudaMemsetAsync(dA, 0, sizeof(float) * 2 * (size_t)d_inner * d_state, stream) != cudaSuccess ||
            cudaMemsetAsync(dD, 0, sizeof(float) * 2 * (size_t)d_inner, stream) != cudaSuccess ||
            cudaMemsetAsync(ddelta_bias, 0, sizeof(float) * 2 * (size_t)d_inner, stream) != cudaSuccess)
            return VIM_ERR_CUDA;
        return VIM_OK;
    }
    if (!u || !delta || !B || !C || !dout || !du || !ddelta || !dB || !dC) return VIM_ERR_INVALID_ARG;
    if (!aligned16(u) || !aligned16(delta) || !aligned_to(B, es) || !aligned_to(C, es) || !aligned_to(dout, es) ||
        !aligned_to(du, es) || !aligned_to(ddelta, es) || (z && !aligned_to(z, es)) || (dz && !aligned_to(dz, es)) ||
        !aligned_to(dB, 4) || !aligned_to(dC, 4))
        return VIM_ERR_INVALID_ARG;
    const int separate = bc_dir_stride > 0 ? 1 : 0;
    const BwdPlan pl = bwd_plan(batch, L, d_inner, d_state, separate);
    if (!workspace || workspace_bytes < pl.total || !aligned_to(workspace, kAlign)) return VIM_ERR_WORKSPACE;
    char *ws = static_cast<char *>(workspace);

    BwdArgs a;
    std::memset(&a, 0, sizeof(a));
    a.u = u; a.delta = delta; a.z = z; a.dout = dout;
    a.B[0] = B; a.C[0] = C;
    a.B[1] = static_cast<const char *>(B) + bc_dir_stride * (int64_t)es;
    a.C[1] = static_cast<const char *>(C) + bc_dir_stride * (int64_t)es;
    a.A = A; a.D = D; a.bias = delta_bias;
    a.du = du; a.ddelta = ddelta; a.dz = dz;
    const size_t set_elems = (size_t)batch * L * pl.ncol * d_state;
    a.dB_part[0] = reinterpret_cast<float *>(ws + pl.off_dBp);
    a.dC_part[0] = reinterpret_cast<float *>(ws + pl.off_dCp);
    a.dB_part[1] = separate ? a.dB_part[0] + set_elems : a.dB_part[0];
    a.dC_part[1] = separate ? a.dC_part[0] + set_elems : a.dC_part[0];
    a.par = reinterpret_cast<float *>(ws + pl.off_par);
    a.hin = ckpt ? ckpt : reinterpret_cast<const float *>(ws + pl.off_hloc);
    a.hin_given = ckpt ? 1 : 0;
    a.gloc = reinterpret_cast<float *>(ws + pl.off_gloc);
    a.gsum = reinterpret_cast<float *>(ws + pl.off_gsum);
    a.batch = batch; a.L = L; a.Di = d_inner; a.G = pl.G; a.nblk = pl.nblk; a.cl = pl.cl; a.ncol = pl.ncol;
    a.separate_bc = separate;
    set_vector_flags(a, dt, d_state);
    static_assert(kCkTokens == kBwdChunk, "the forward pass's checkpoints are the derivative's chunk starts");

    PairArgs f;
    std::memset(&f, 0, sizeof(f));
    f.u = u; f.delta = delta;
    f.B[0] = a.B[0]; f.B[1] = a.B[1]; f.C[0] = a.C[0]; f.C[1] = a.C[1];
    f.A = A; f.D = D; f.bias = delta_bias;
    f.hloc = reinterpret_cast<float *>(ws + pl.off_hloc);
    f.ssum = reinterpret_cast<float *>(ws + pl.off_ssum);
    f.batch = batch; f.L = L; f.Di = d_inner; f.H = 1; f.W = L; f.order = 0;
    f.chunk = kBwdChunk; f.G = pl.G;

    float *dBo[2] = {dB, dB + bc_dir_stride}, *dCo[2] = {dC, dC + bc_dir_stride};
    float *tmp = reinterpret_cast<float *>(ws + pl.off_tmp);
    if (dt == VIM_F32)
        return zoh ? launch_bwd_n<float, true>(d_state, a, f, dBo, dCo, dA, dD, ddelta_bias, tmp, stream, events)
                   : launch_bwd_n<float, false>(d_state, a, f, dBo, dCo, dA, dD, ddelta_bias, tmp, stream, events);
    return zoh ? launch_bwd_n<__nv_bfloat16, true>(d_state, a, f, dBo, dCo, dA, dD, ddelta_bias, tmp, stream, events)
               : launch_bwd_n<__nv_bfloat16, false>(d_state, a, f, dBo, dCo, dA, dD, ddelta_bias, tmp, stream,
                                                    events);
}

}  // namespace

extern "C" {

vim_status vim_scan_bidir_bwd_ex(const void *u, const void *delta, const void *z, const void *B, const void *C,
                                 int64_t bc_dir_stride, const float *A, const float *D, const float *delta_bias,
                                 const void *dout, void *du, void *ddelta, void *dz, float *dB, float *dC,
                                 float *dA, float *dD, float *ddelta_bias, int batch, int L, int d_inner,
                                 int d_state, vim_dtype dt, unsigned flags, void *workspace, size_t workspace_bytes,
                                 cudaStream_t stream, cudaEvent_t *events) {
    return bidir_bwd_impl(u, delta, z, B, C, bc_dir_stride, A, D, delta_bias, dout, du, ddelta, dz, dB, dC, dA, dD,
                          ddelta_bias, batch, L, d_inner, d_state, dt, flags, workspace, workspace_bytes, stream,
                          events, nullptr);
}

vim_status vim_scan_bidir_bwd_ckpt(const void *u, const void *delta, const void *z, const void *B, const void *C,
                                   int64_t bc_dir_stride, const float *A, const float *D, const float *delta_bias,
                                   const float *ckpt, const void *dout, void *du, void *ddelta, void *dz, float *dB,
                                   float *dC, float *dA, float *dD, float *ddelta_bias, int batch, int L,
                                   int d_inner, int d_state, vim_dtype dt, unsigned flags, void *workspace,
                                   size_t workspace_bytes, cudaStream_t stream, cudaEvent_t *events) {
    if (batch > 0 && L > 0 && d_inner > 0 && (!ckpt || !aligned_to(ckpt, 8))) return VIM_ERR_INVALID_ARG;
    return bidir_bwd_impl(u, delta, z, B, C, bc_dir_stride, A, D, delta_bias, dout, du, ddelta, dz, dB, dC, dA, dD,
                          ddelta_bias, batch, L, d_inner, d_state, dt, flags, workspace, workspace_bytes, stream,
                          events, ckpt);
}

vim_status vim_scan_bidir_bwd_events(const void *u, const void *delta, const void *z, const void *B,
                                     const void *C, int64_t bc_dir_stride, const float *A, const float *D,
                                     const float *delta_bias, const void *dout, void *du, void *ddelta, void *dz,
                                     float *dB, float *dC, float *dA, float *dD, float *ddelta_bias, int batch,
                                     int L, int d_inner, int d_state, vim_dtype dt, void *workspace,
                                     size_t workspace_bytes, cudaStream_t stream, cudaEvent_t *events) {
    return vim_scan_bidir_bwd_ex(u, delta, z, B, C, bc_dir_stride, A, D, delta_bias, dout, du, ddelta, dz, dB, dC,
                                 dA, dD, ddelta_bias, batch, L, d_inner, d_state, dt, 0u, workspace, workspace_bytes,
                                 stream, events);
}

vim_status vim_scan_bidir_bwd(const void *u, const void *delta, const void *z, const void *B, const void *C,
                              int64_t bc_dir_stride, const float *A, const float *D, const float *delta_bias,
                              const void *dout, void *du, void *ddelta, void *dz, float *dB, float *dC,
                              float *dA, float *dD, float *ddelta_bias, int batch, int L, int d_inner,
                              int d_state, vim_dtype dt, void *workspace, size_t workspace_bytes,
                              cudaStream_t stream) {
    return vim_scan_bidir_bwd_events(u, delta, z, B, C, bc_dir_stride, A, D, delta_bias, dout, du, ddelta, dz,
                                     dB, dC, dA, dD, ddelta_bias, batch, L, d_inner, d_state, dt, workspace,
                                     workspace_bytes, stream, nullptr);
}

}  // extern "C"

// ----------------------------------------------------------------------------
// the derivative of the scan with its convolution front
// ----------------------------------------------------------------------------

extern "C" {

size_t vim_scan_conv_bwd_workspace_bytes(int batch, int L, int d_inner, int d_state, vim_dtype dt, int separate_bc) {
    if (check_common(batch, L, d_inner, d_state, dt) != VIM_OK) return 0;
    if (batch <= 0 || L <= 0 || d_inner <= 0) return 0;
    return conv_bwd_plan(batch, L, d_inner, d_state, dt, separate_bc).total;
}

}  // extern "C"

namespace {

// the derivative of vim_scan_bidir_conv; ckpt, or null: the forward pass's checkpoints
// (vim_scan_bidir_conv_ckpt), which replace the derivative's own forward summaries
vim_status conv_bwd_impl(const void *x, const float *conv_w, const float *conv_b, const void *delta, const void *z,
                         const void *B, const void *C, int64_t bc_dir_stride, const float *A, const float *D,
                         const float *delta_bias, const void *dout, void *dx, float *dconv_w, float *dconv_b,
                         void *ddelta, void *dz, float *dB, float *dC, float *dA, float *dD, float *ddelta_bias,
                         int batch, int L, int d_inner, int d_state, vim_dtype dt, unsigned flags, void *workspace,
                         size_t workspace_bytes, cudaStream_t stream, const float *ckpt) {
    if (flags & ~VIM_FLAG_ZOH_EXACT) return VIM_ERR_INVALID_ARG;
    const bool zoh = (flags & VIM_FLAG_ZOH_EXACT) != 0;
    vim_status st = check_common(batch, L, d_inner, d_state, dt);
    if (st != VIM_OK) return st;
    if (bc_dir_stride < 0) return VIM_ERR_INVALID_ARG;
    if ((z == nullptr) != (dz == nullptr)) return VIM_ERR_INVALID_ARG;
    if (!A || !D || !delta_bias || !dA || !dD || !ddelta_bias || !conv_w || !conv_b || !dconv_w || !dconv_b)
        return VIM_ERR_INVALID_ARG;
    if (!aligned_to(A, 4) || !aligned_to(D, 4) || !aligned_to(delta_bias, 4) || !aligned_to(dA, 4) ||
        !aligned_to(dD, 4) || !aligned_to(ddelta_bias, 4) || !aligned_to(conv_w, 4) || !aligned_to(conv_b, 4) ||
        !aligned_to(dconv_w, 4) || !aligned_to(dconv_b, 4))
        return VIM_ERR_INVALID_ARG;
    const size_t es = elem_size(dt);
    if (batch == 0 || L == 0 || d_inner == 0) {
        // no tokens: the parameter derivatives are zero
        if (cudaMemsetAsync(dA, 0, sizeof(float) * 2 * (size_t)d_inner * d_state, stream) != cudaSuccess ||
            cudaMemsetAsync(dD, 0, sizeof(float) * 2 * (size_t)d_inner, stream) != cudaSuccess ||
            cudaMemsetAsync(ddelta_bias, 0, sizeof(float) * 2 * (size_t)d_inner, stream) != cudaSuccess ||
            cudaMemsetAsync(dconv_w, 0, sizeof(float) * 6 * (size_t)d_inner, stream) != cudaSuccess ||
            cudaMemsetAsync(dconv_b, 0, sizeof(float) * 2 * (size_t)d_inner, stream) != cudaSuccess)
            return VIM_ERR_CUDA;
        return VIM_OK;
    }
    if (!x || !delta || !B || !C || !dout || !dx || !ddelta || !dB || !dC) return VIM_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(delta) || !aligned_to(B, es) || !aligned_to(C, es) || !aligned_to(dout, es) ||
        !aligned_to(dx, es) || !aligned_to(ddelta, es) || (z && !aligned_to(z, es)) || (dz && !aligned_to(dz, es)) ||
        !aligned_to(dB, 4) || !aligned_to(dC, 4))
        return VIM_ERR_INVALID_ARG;
    const int separate = bc_dir_stride > 0 ? 1 : 0;
    const ConvBwdPlan cp = conv_bwd_plan(batch, L, d_inner, d_state, dt, separate);
    const BwdPlan &pl = cp.pl;
    if (!workspace || workspace_bytes < cp.total || !aligned_to(workspace, kAlign)) return VIM_ERR_WORKSPACE;
    char *ws = static_cast<char *>(workspace);
    float *u2 = reinterpret_cast<float *>(ws + cp.off_u2);
    float *du2 = reinterpret_cast<float *>(ws + cp.off_du2);
    const int64_t act = (int64_t)batch * L * d_inner;
    const int vec = aligned_to(x, dt == VIM_F32 ? 16 : 8) && aligned_to(dx, dt == VIM_F32 ? 16 : 8) ? 1 : 0;

    // both pathways' smoothed inputs
    st = dt == VIM_F32 ? launch_front_fwd<float>(static_cast<const float *>(x), conv_w, conv_b, u2, batch, L,
                                                 d_inner, vec, stream)
                       : launch_front_fwd<__nv_bfloat16>(static_cast<const __nv_bfloat16 *>(x), conv_w, conv_b, u2,
                                                         batch, L, d_inner, vec, stream);
    if (st != VIM_OK) return st;

    BwdArgs a;
    std::memset(&a, 0, sizeof(a));
    a.u = u2; a.u_dir_stride = act; a.du2 = du2;
    a.delta = delta; a.z = z; a.dout = dout;
    a.B[0] = B; a.C[0] = C;
    a.B[1] = static_cast<const char *>(B) + bc_dir_stride * (int64_t)es;
    a.C[1] = static_cast<const char *>(C) + bc_dir_stride * (int64_t)es;
    a.A = A; a.D = D; a.bias = delta_bias;
    a.ddelta = ddelta; a.dz = dz;
    const size_t set_elems = (size_t)batch * L * pl.ncol * d_state;
    a.dB_part[0] = reinterpret_cast<float *>(ws + pl.off_dBp);
    a.dC_part[0] = reinterpret_cast<float *>(ws + pl.off_dCp);
    a.dB_part[1] = separate ? a.dB_part[0] + set_elems : a.dB_part[0];
    a.dC_part[1] = separate ? a.dC_part[0] + set_elems : a.dC_part[0];
    a.par = reinterpret_cast<float *>(ws + pl.off_par);
    a.hin = ckpt ? ckpt : reinterpret_cast<const float *>(ws + pl.off_hloc);
    a.hin_given = ckpt ? 1 : 0;
    a.gloc = reinterpret_cast<float *>(ws + pl.off_gloc);
    a.gsum = reinterpret_cast<float *>(ws + pl.off_gsum);
    a.batch = batch; a.L = L; a.Di = d_inner; a.G = pl.G; a.nblk = pl.nblk; a.cl = pl.cl; a.ncol = pl.ncol;
    a.separate_bc = separate;
    set_vector_flags(a, dt, d_state);

    PairArgs f;
    std::memset(&f, 0, sizeof(f));
    f.u = x; f.conv_w = conv_w; f.conv_b = conv_b; f.delta = delta;
    f.B[0] = a.B[0]; f.B[1] = a.B[1]; f.C[0] = a.C[0]; f.C[1] = a.C[1];
    f.A = A; f.D = D; f.bias = delta_bias;
    f.hloc = reinterpret_cast<float *>(ws + pl.off_hloc);
    f.ssum = reinterpret_cast<float *>(ws + pl.off_ssum);
    f.batch = batch; f.L = L; f.Di = d_inner; f.H = 1; f.W = L; f.order = 0;
    f.chunk = kBwdChunk; f.G = pl.G;

    float *dBo[2] = {dB, dB + bc_dir_stride}, *dCo[2] = {dC, dC + bc_dir_stride};
    float *tmp = reinterpret_cast<float *>(ws + pl.off_tmp);
    float *part = reinterpret_cast<float *>(ws + cp.off_part), *ptmp = reinterpret_cast<float *>(ws + cp.off_ptmp);
    if (dt == VIM_F32) {
        st = zoh ? launch_bwd_n<float, true, true>(d_state, a, f, dBo, dCo, dA, dD, ddelta_bias, tmp, stream, nullptr)
                 : launch_bwd_n<float, false, true>(d_state, a, f, dBo, dCo, dA, dD, ddelta_bias, tmp, stream, nullptr);
        if (st != VIM_OK) return st;
        return launch_fronts_bwd<float>(static_cast<const float *>(x), conv_w, conv_b, du2, static_cast<float *>(dx),
                                        part, ptmp, dconv_w, dconv_b, batch, L, d_inner, cp.runs, vec, stream);
    }
    st = zoh ? launch_bwd_n<__nv_bfloat16, true, true>(d_state, a, f, dBo, dCo, dA, dD, ddelta_bias, tmp, stream,
                                                       nullptr)
             : launch_bwd_n<__nv_bfloat16, false, true>(d_state, a, f, dBo, dCo, dA, dD, ddelta_bias, tmp, stream,
                                                        nullptr);
    if (st != VIM_OK) return st;
    return launch_fronts_bwd<__nv_bfloat16>(static_cast<const __nv_bfloat16 *>(x), conv_w, conv_b, du2,
                                            static_cast<__nv_bfloat16 *>(dx), part, ptmp, dconv_w, dconv_b, batch, L,
                                            d_inner, cp.runs, vec, stream);
}

}  // namespace

extern "C" {

vim_status vim_scan_bidir_conv_bwd_ex(const void *x, const float *conv_w, const float *conv_b, const void *delta,
                                      const void *z, const void *B, const void *C, int64_t bc_dir_stride,
                                      const float *A, const float *D, const float *delta_bias, const void *dout,
                                      void *dx, float *dconv_w, float *dconv_b, void *ddelta, void *dz, float *dB,
                                      float *dC, float *dA, float *dD, float *ddelta_bias, int batch, int L,
                                      int d_inner, int d_state, vim_dtype dt, unsigned flags, void *workspace,
                                      size_t workspace_bytes, cudaStream_t stream) {
    return conv_bwd_impl(x, conv_w, conv_b, delta, z, B, C, bc_dir_stride, A, D, delta_bias, dout, dx, dconv_w,
                         dconv_b, ddelta, dz, dB, dC, dA, dD, ddelta_bias, batch, L, d_inner, d_state, dt, flags,
                         workspace, workspace_bytes, stream, nullptr);
}

vim_status vim_scan_bidir_conv_bwd_ckpt(const void *x, const float *conv_w, const float *conv_b, const void *delta,
                                        const void *z, const void *B, const void *C, int64_t bc_dir_stride,
                                        const float *A, const float *D, const float *delta_bias, const float *ckpt,
                                        const void *dout, void *dx, float *dconv_w, float *dconv_b, void *ddelta,
                                        void *dz, float *dB, float *dC, float *dA, float *dD, float *ddelta_bias,
                                        int batch, int L, int d_inner, int d_state, vim_dtype dt, unsigned flags,
                                        void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (batch > 0 && L > 0 && d_inner > 0 && (!ckpt || !aligned_to(ckpt, 8))) return VIM_ERR_INVALID_ARG;
    return conv_bwd_impl(x, conv_w, conv_b, delta, z, B, C, bc_dir_stride, A, D, delta_bias, dout, dx, dconv_w,
                         dconv_b, ddelta, dz, dB, dC, dA, dD, ddelta_bias, batch, L, d_inner, d_state, dt, flags,
                         workspace, workspace_bytes, stream, ckpt);
}

vim_status vim_scan_bidir_conv_bwd(const void *x, const float *conv_w, const float *conv_b, const void *delta,
                                   const void *z, const void *B, const void *C, int64_t bc_dir_stride,
                                   const float *A, const float *D, const float *delta_bias, const void *dout,
                                   void *dx, float *dconv_w, float *dconv_b, void *ddelta, void *dz, float *dB,
                                   float *dC, float *dA, float *dD, float *ddelta_bias, int batch, int L,
                                   int d_inner, int d_state, vim_dtype dt, void *workspace, size_t workspace_bytes,
                                   cudaStream_t stream) {
    return vim_scan_bidir_conv_bwd_ex(x, conv_w, conv_b, delta, z, B, C, bc_dir_stride, A, D, delta_bias, dout, dx,
                                      dconv_w, dconv_b, ddelta, dz, dB, dC, dA, dD, ddelta_bias, batch, L, d_inner,
                                      d_state, dt, 0u, workspace, workspace_bytes, stream);
}

size_t vmamba_cross_scan4_bwd_workspace_bytes(int batch, int H, int W, int channels, int d_state) {
    if (batch <= 0 || H <= 0 || W <= 0 || channels <= 0 || d_state <= 0) return 0;
    const int L = H * W;
    return bwd_plan(batch, L, channels, d_state, 1).total + 3 * round_up((size_t)batch * L * channels * 4);
}

}  // extern "C"

namespace {

// the derivative of vmamba_cross_scan4; ckpt, or null: the forward pass's checkpoints
// (vmamba_cross_scan4_ckpt, [2 pairs][batch][ceil(L/32)][2][N][C]), which replace each
// pair's own forward summaries
vim_status cross_bwd_impl(const void *u, const void *delta, const void *z, const void *B, const void *C,
                          const float *A, const float *D, const float *delta_bias, const void *dout, void *du,
                          void *ddelta, void *dz, float *dB, float *dC, float *dA, float *dD, float *ddelta_bias,
                          int batch, int H, int W, int channels, int d_state, vim_dtype dt, unsigned flags,
                          void *workspace, size_t workspace_bytes, cudaStream_t stream, const float *ckpt) {
    if (flags & ~VIM_FLAG_ZOH_EXACT) return VIM_ERR_INVALID_ARG;
    const bool zoh = (flags & VIM_FLAG_ZOH_EXACT) != 0;
    if (H < 0 || W < 0) return VIM_ERR_INVALID_ARG;
    if ((int64_t)H * W > INT32_MAX) return VIM_ERR_UNSUPPORTED;
    const int L = H * W;
    vim_status st = check_common(batch, L, channels, d_state, dt);
    if (st != VIM_OK) return st;
    if ((z == nullptr) != (dz == nullptr)) return VIM_ERR_INVALID_ARG;
    if (!A || !D || !delta_bias || !dA || !dD || !ddelta_bias) return VIM_ERR_INVALID_ARG;
    if (!aligned_to(A, 4) || !aligned_to(D, 4) || !aligned_to(delta_bias, 4) || !aligned_to(dA, 4) ||
        !aligned_to(dD, 4) || !aligned_to(ddelta_bias, 4))
        return VIM_ERR_INVALID_ARG;
    const size_t es = elem_size(dt);
    if (batch == 0 || L == 0 || channels == 0) {
        if (cudaMemsetAsync(dA, 0, sizeof(float) * 4 * (size_t)channels * d_state, stream) != cudaSuccess ||
            cudaMemsetAsync(dD, 0, sizeof(float) * 4 * (size_t)channels, stream) != cudaSuccess ||
            cudaMemsetAsync(ddelta_bias, 0, sizeof(float) * 4 * (size_t)channels, stream) != cudaSuccess)
            return VIM_ERR_CUDA;
        return VIM_OK;
    }
    if (!u || !delta || !B || !C || !dout || !du || !ddelta || !dB || !dC) return VIM_ERR_INVALID_ARG;
    if (!aligned16(u) || !aligned16(delta) || !aligned_to(B, es) || !aligned_to(C, es) || !aligned_to(dout, es) ||
        !aligned_to(du, es) || !aligned_to(ddelta, es) || (z && !aligned_to(z, es)) || (dz && !aligned_to(dz, es)) ||
        !aligned_to(dB, 4) || !aligned_to(dC, 4))
        return VIM_ERR_INVALID_ARG;
    const BwdPlan pl = bwd_plan(batch, L, channels, d_state, 1);
    const size_t acc_bytes = round_up((size_t)batch * L * channels * 4);
    if (!workspace || workspace_bytes < pl.total + 3 * acc_bytes || !aligned_to(workspace, kAlign))
        return VIM_ERR_WORKSPACE;
    char *ws = static_cast<char *>(workspace);
    float *acc = reinterpret_cast<float *>(ws + pl.total);
    const size_t bc = (size_t)batch * L * d_state;               // elements per direction of B, C
    const size_t set_elems = (size_t)batch * L * pl.ncol * d_state;

    vim_status rc = VIM_OK;
    for (int pair = 0; pair < 2 && rc == VIM_OK; ++pair) {
        BwdArgs a;
        std::memset(&a, 0, sizeof(a));
        a.u = u; a.delta = delta; a.z = z; a.dout = dout;
        for (int k = 0; k < 2; ++k) {
            a.B[k] = static_cast<const char *>(B) + (2 * pair + k) * bc * es;
            a.C[k] = static_cast<const char *>(C) + (2 * pair + k) * bc * es;
        }
        a.A = A + (size_t)2 * pair * channels * d_state;
        a.D = D + (size_t)2 * pair * channels;
        a.bias = delta_bias + (size_t)2 * pair * channels;
        a.du = du; a.ddelta = ddelta; a.dz = dz;
        a.dB_part[0] = reinterpret_cast<float *>(ws + pl.off_dBp);
        a.dC_part[0] = reinterpret_cast<float *>(ws + pl.off_dCp);
        a.dB_part[1] = a.dB_part[0] + set_elems;
        a.dC_part[1] = a.dC_part[0] + set_elems;
        a.par = reinterpret_cast<float *>(ws + pl.off_par);
        a.hin = ckpt ? ckpt + (size_t)pair * batch * pl.G * 2 * d_state * channels
                     : reinterpret_cast<const float *>(ws + pl.off_hloc);
        a.hin_given = ckpt ? 1 : 0;
        a.gloc = reinterpret_cast<float *>(ws + pl.off_gloc);
        a.gsum = reinterpret_cast<float *>(ws + pl.off_gsum);
        a.batch = batch; a.L = L; a.Di = channels; a.G = pl.G; a.nblk = pl.nblk; a.cl = pl.cl; a.ncol = pl.ncol;
        a.separate_bc = 1;
        set_vector_flags(a, dt, d_state);
        a.order = pair; a.H = H; a.W = W; a.hdiv = div_inv((unsigned)H);
        a.stage = pair + 1;                  // the row pair leaves partials, the column pair finishes
        a.acc_y = acc;
        a.acc_du = reinterpret_cast<float *>(ws + pl.total + acc_bytes);
        a.acc_dd = reinterpret_cast<float *>(ws + pl.total + 2 * acc_bytes);

        PairArgs f;
        std::memset(&f, 0, sizeof(f));
        f.u = u; f.delta = delta;
        f.B[0] = a.B[0]; f.B[1] = a.B[1]; f.C[0] = a.C[0]; f.C[1] = a.C[1];
        f.A = a.A; f.D = a.D; f.bias = a.bias;
        f.hloc = reinterpret_cast<float *>(ws + pl.off_hloc);
        f.ssum = reinterpret_cast<float *>(ws + pl.off_ssum);
        f.batch = batch; f.L = L; f.Di = channels; f.H = H; f.W = W; f.order = pair; f.hdiv = div_inv((unsigned)H);
        f.chunk = kBwdChunk; f.G = pl.G;

        float *dBo[2] = {dB + (2 * pair) * bc, dB + (2 * pair + 1) * bc};
        float *dCo[2] = {dC + (2 * pair) * bc, dC + (2 * pair + 1) * bc};
        float *tmp = reinterpret_cast<float *>(ws + pl.off_tmp);
        float *dAp = dA + (size_t)2 * pair * channels * d_state;
        float *dDp = dD + (size_t)2 * pair * channels, *dbp = ddelta_bias + (size_t)2 * pair * channels;
        if (dt == VIM_F32)
            rc = zoh ? launch_bwd_n<float, true>(d_state, a, f, dBo, dCo, dAp, dDp, dbp, tmp, stream, nullptr)
                     : launch_bwd_n<float, false>(d_state, a, f, dBo, dCo, dAp, dDp, dbp, tmp, stream, nullptr);
        else
            rc = zoh ? launch_bwd_n<__nv_bfloat16, true>(d_state, a, f, dBo, dCo, dAp, dDp, dbp, tmp, stream, nullptr)
                     : launch_bwd_n<__nv_bfloat16, false>(d_state, a, f, dBo, dCo, dAp, dDp, dbp, tmp, stream,
                                                          nullptr);
    }
    return rc;
}

}  // namespace

extern "C" {

vim_status vmamba_cross_scan4_bwd_ex(const void *u, const void *delta, const void *z, const void *B, const void *C,
                                     const float *A, const float *D, const float *delta_bias, const void *dout,
                                     void *du, void *ddelta, void *dz, float *dB, float *dC, float *dA, float *dD,
                                     float *ddelta_bias, int batch, int H, int W, int channels, int d_state,
                                     vim_dtype dt, unsigned flags, void *workspace, size_t workspace_bytes,
                                     cudaStream_t stream) {
    return cross_bwd_impl(u, delta, z, B, C, A, D, delta_bias, dout, du, ddelta, dz, dB, dC, dA, dD, ddelta_bias,
                          batch, H, W, channels, d_state, dt, flags, workspace, workspace_bytes, stream, nullptr);
}

vim_status vmamba_cross_scan4_bwd_ckpt(const void *u, const void *delta, const void *z, const void *B,
                                       const void *C, const float *A, const float *D, const float *delta_bias,
                                       const float *ckpt, const void *dout, void *du, void *ddelta, void *dz,
                                       float *dB, float *dC, float *dA, float *dD, float *ddelta_bias, int batch,
                                       int H, int W, int channels, int d_state, vim_dtype dt, unsigned flags,
                                       void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (batch > 0 && H > 0 && W > 0 && channels > 0 && (!ckpt || !aligned_to(ckpt, 8))) return VIM_ERR_INVALID_ARG;
    return cross_bwd_impl(u, delta, z, B, C, A, D, delta_bias, dout, du, ddelta, dz, dB, dC, dA, dD, ddelta_bias,
                          batch, H, W, channels, d_state, dt, flags, workspace, workspace_bytes, stream, ckpt);
}

vim_status vmamba_cross_scan4_bwd(const void *u, const void *delta, const void *z, const void *B, const void *C,
                                  const float *A, const float *D, const float *delta_bias, const void *dout,
                                  void *du, void *ddelta, void *dz, float *dB, float *dC, float *dA, float *dD,
                                  float *ddelta_bias, int batch, int H, int W, int channels, int d_state,
                                  vim_dtype dt, void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    return vmamba_cross_scan4_bwd_ex(u, delta, z, B, C, A, D, delta_bias, dout, du, ddelta, dz, dB, dC, dA, dD,
                                     ddelta_bias, batch, H, W, channels, d_state, dt, 0u, workspace, workspace_bytes,
                                     stream);
}

}  // extern "C"
