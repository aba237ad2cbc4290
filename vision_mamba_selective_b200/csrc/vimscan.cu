// vimscan.cu -- host side of libvimscan.so: argument checks, planning, launches.
//
// Entry points are declared (with their contracts) in include/vimscan.h.  Every
// check runs on the host before the first launch; nothing here allocates memory or
// synchronises the stream.
#include "vimscan.h"

#include <cstdint>
#include <cstring>
#include <mutex>

#include "launch.cuh"


using namespace vimscan;

extern "C" {

const char *vim_status_string(vim_status s) {
    switch (s) {
        case VIM_OK: return "ok";
        case VIM_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, or negative size)";
        case VIM_ERR_UNSUPPORTED: return "unsupported size (d_state or channel count)";
        case VIM_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case VIM_ERR_CUDA: return "CUDA launch failed";
        case VIM_ERR_TIMEOUT: return "a bounded device-side wait ran out";
        default: return "unknown status";
    }
}

size_t vim_scan_workspace_bytes(int which, int batch, int L_or_H, int W, int channels, int d_state) {
    if (batch < 0 || L_or_H < 0 || channels < 0 || !supported_state(d_state)) return 0;
    if (which == 0) return summary_bytes(batch, L_or_H, channels, d_state);
    if (which == 1) {
        if (W < 0) return 0;
        const int L = L_or_H * W;
        const size_t partial = round_up((size_t)batch * L * channels * sizeof(float));
        return summary_bytes(batch, L, channels, d_state) + partial;
    }
    return 0;
}

}  // extern "C"

namespace {
constexpr unsigned kKnownFlags = VIM_FLAG_ZOH_EXACT;

// vim_scan_bidir with an optional convolution front (conv_w/conv_b non-null: u holds x)
vim_status bidir_impl(const void *u, const float *conv_w, const float *conv_b, const void *delta,
                      const void *z, const void *B, const void *C, int64_t bc_dir_stride, const float *A,
                      const float *D, const float *delta_bias, void *y, int batch, int L, int d_inner,
                      int d_state, vim_dtype dt, unsigned flags, void *workspace, size_t workspace_bytes,
                      cudaStream_t stream, cudaEvent_t *events) {
    vim_status st = check_common(batch, L, d_inner, d_state, dt);
    if (st != VIM_OK) return st;
    if (bc_dir_stride < 0 || (flags & ~kKnownFlags)) return VIM_ERR_INVALID_ARG;
    if (!conv_w != !conv_b) return VIM_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(conv_w) | reinterpret_cast<uintptr_t>(conv_b)) % 4)
        return VIM_ERR_INVALID_ARG;
    if (batch == 0 || L == 0 || d_inner == 0) return VIM_OK;
    if (!u || !delta || !B || !C || !A || !D || !delta_bias || !y) return VIM_ERR_INVALID_ARG;
    if (!aligned16(u) || !aligned16(delta) || !aligned16(y) || (z && !aligned16(z)))
        return VIM_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(B) | reinterpret_cast<uintptr_t>(C)) % elem_size(dt))
        return VIM_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(D) |
         reinterpret_cast<uintptr_t>(delta_bias)) % 4)
        return VIM_ERR_INVALID_ARG;
    const size_t need = summary_bytes(batch, L, d_inner, d_state);
    if (need > 0) {
        if (!workspace || workspace_bytes < need) return VIM_ERR_WORKSPACE;
        if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return VIM_ERR_WORKSPACE;
    }
    const Plan pl = plan_for(batch, L, d_inner);
    PairArgs a;
    std::memset(&a, 0, sizeof(a));
    a.u = u; a.delta = delta; a.z = z;
    const char *Bc = static_cast<const char *>(B), *Cc = static_cast<const char *>(C);
    a.B[0] = B; a.C[0] = C;
    a.B[1] = Bc + bc_dir_stride * (int64_t)elem_size(dt);
    a.C[1] = Cc + bc_dir_stride * (int64_t)elem_size(dt);
    a.A = A; a.D = D; a.bias = delta_bias;
    a.conv_w = conv_w; a.conv_b = conv_b;
    a.y = y;
    a.batch = batch; a.L = L; a.Di = d_inner; a.H = 1; a.W = L; a.order = 0;
    a.chunk = pl.chunk; a.G = pl.G;
    a.zoh = (flags & VIM_FLAG_ZOH_EXACT) ? 1 : 0;
    if (pl.G > 1) {
        const size_t units = (size_t)batch * pl.G * 2 * d_inner;
        a.hloc = static_cast<float *>(workspace);
        a.ssum = reinterpret_cast<float *>(static_cast<char *>(workspace) + round_up(units * d_state * 4));
    }
    if (mark(events, 0, stream) != VIM_OK) return VIM_ERR_CUDA;
    return launch_pair(a, d_state, dt, stream, events ? events + 1 : nullptr);
}

}  // namespace

extern "C" {

vim_status vim_scan_bidir_events(const void *u, const void *delta, const void *z, const void *B,
                                 const void *C, int64_t bc_dir_stride, const float *A,
                                 const float *D, const float *delta_bias, void *y, int batch, int L,
                                 int d_inner, int d_state, vim_dtype dt, void *workspace,
                                 size_t workspace_bytes, cudaStream_t stream, cudaEvent_t *events) {
    return bidir_impl(u, nullptr, nullptr, delta, z, B, C, bc_dir_stride, A, D, delta_bias, y, batch, L,
                      d_inner, d_state, dt, 0u, workspace, workspace_bytes, stream, events);
}

vim_status vim_scan_bidir_ex(const void *u, const float *conv_w, const float *conv_b, const void *delta,
                             const void *z, const void *B, const void *C, int64_t bc_dir_stride,
                             const float *A, const float *D, const float *delta_bias, void *y, int batch,
                             int L, int d_inner, int d_state, vim_dtype dt, unsigned flags, void *workspace,
                             size_t workspace_bytes, cudaStream_t stream, cudaEvent_t *events) {
    return bidir_impl(u, conv_w, conv_b, delta, z, B, C, bc_dir_stride, A, D, delta_bias, y, batch, L,
                      d_inner, d_state, dt, flags, workspace, workspace_bytes, stream, events);
}

vim_status vim_scan_bidir_conv_events(const void *x, const float *conv_w, const float *conv_b,
                                      const void *delta, const void *z, const void *B, const void *C,
                                      int64_t bc_dir_stride, const float *A, const float *D,
                                      const float *delta_bias, void *y, int batch, int L, int d_inner,
                                      int d_state, vim_dtype dt, void *workspace, size_t workspace_bytes,
                                      cudaStream_t stream, cudaEvent_t *events) {
    if (batch > 0 && L > 0 && d_inner > 0 && (!conv_w || !conv_b)) return VIM_ERR_INVALID_ARG;
    return bidir_impl(x, conv_w, conv_b, delta, z, B, C, bc_dir_stride, A, D, delta_bias, y, batch, L,
                      d_inner, d_state, dt, 0u, workspace, workspace_bytes, stream, events);
}

vim_status vim_scan_bidir_conv(const void *x, const float *conv_w, const float *conv_b,
                               const void *delta, const void *z, const void *B, const void *C,
                               int64_t bc_dir_stride, const float *A, const float *D,
                               const float *delta_bias, void *y, int batch, int L, int d_inner,
                               int d_state, vim_dtype dt, void *workspace, size_t workspace_bytes,
                               cudaStream_t stream) {
    return vim_scan_bidir_conv_events(x, conv_w, conv_b, delta, z, B, C, bc_dir_stride, A, D, delta_bias,
                                      y, batch, L, d_inner, d_state, dt, workspace, workspace_bytes,
                                      stream, nullptr);
}

vim_status vim_scan_bidir(const void *u, const void *delta, const void *z, const void *B,
                          const void *C, int64_t bc_dir_stride, const float *A, const float *D,
                          const float *delta_bias, void *y, int batch, int L, int d_inner,
                          int d_state, vim_dtype dt, void *workspace, size_t workspace_bytes,
                          cudaStream_t stream) {
    return vim_scan_bidir_events(u, delta, z, B, C, bc_dir_stride, A, D, delta_bias, y, batch, L,
                                 d_inner, d_state, dt, workspace, workspace_bytes, stream, nullptr);
}

vim_status vmamba_cross_scan4_ex(const void *u, const void *delta, const void *z, const void *B,
                                 const void *C, const float *A, const float *D, const float *delta_bias,
                                 void *y, int batch, int H, int W, int channels, int d_state, vim_dtype dt,
                                 unsigned flags, void *workspace, size_t workspace_bytes,
                                 cudaStream_t stream, cudaEvent_t *events) {
    if (H < 0 || W < 0 || (flags & ~kKnownFlags)) return VIM_ERR_INVALID_ARG;
    if ((int64_t)H * W > INT32_MAX) return VIM_ERR_UNSUPPORTED;
    const int L = H * W;
    vim_status st = check_common(batch, L, channels, d_state, dt);
    if (st != VIM_OK) return st;
    if (batch == 0 || L == 0 || channels == 0) return VIM_OK;
    if (!u || !delta || !B || !C || !A || !D || !delta_bias || !y) return VIM_ERR_INVALID_ARG;
    if (!aligned16(u) || !aligned16(delta) || !aligned16(y) || (z && !aligned16(z)))
        return VIM_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(B) | reinterpret_cast<uintptr_t>(C)) % elem_size(dt))
        return VIM_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(D) |
         reinterpret_cast<uintptr_t>(delta_bias)) % 4)
        return VIM_ERR_INVALID_ARG;
    const size_t sum_b = summary_bytes(batch, L, channels, d_state);
    const size_t need = sum_b + round_up((size_t)batch * L * channels * sizeof(float));
    if (!workspace || workspace_bytes < need) return VIM_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return VIM_ERR_WORKSPACE;

    const Plan pl = plan_for(batch, L, channels);
    float *partial = reinterpret_cast<float *>(static_cast<char *>(workspace) + sum_b);
    const size_t el = elem_size(dt);
    const size_t bc_dir = (size_t)batch * L * d_state * el;   // bytes between directions
    if (mark(events, 0, stream) != VIM_OK) return VIM_ERR_CUDA;
    vim_status rc = VIM_OK;
    for (int pair = 0; pair < 2 && rc == VIM_OK; ++pair) {
        PairArgs a;
        std::memset(&a, 0, sizeof(a));
        a.u = u; a.delta = delta; a.z = z;
        for (int k = 0; k < 2; ++k) {
            a.B[k] = static_cast<const char *>(B) + (2 * pair + k) * bc_dir;
            a.C[k] = static_cast<const char *>(C) + (2 * pair + k) * bc_dir;
        }
        a.A = A + (size_t)2 * pair * channels * d_state;
        a.D = D + (size_t)2 * pair * channels;
        a.bias = delta_bias + (size_t)2 * pair * channels;
        a.batch = batch; a.L = L; a.Di = channels; a.H = H; a.W = W;
        a.order = pair;               // pair 0: scans 1/2 (rows), pair 1: scans 3/4 (columns)
        a.chunk = pl.chunk; a.G = pl.G;
        a.zoh = (flags & VIM_FLAG_ZOH_EXACT) ? 1 : 0;
        if (pl.G > 1) {
            const size_t units = (size_t)batch * pl.G * 2 * channels;
            a.hloc = static_cast<float *>(workspace);
            a.ssum = reinterpret_cast<float *>(static_cast<char *>(workspace) +
                                               round_up(units * d_state * 4));
        }
        if (pair == 0) {
            a.partial_out = partial;
        } else {
            a.partial_in = partial;
            a.y = y;
        }
        rc = launch_pair(a, d_state, dt, stream, events ? events + 1 + 3 * pair : nullptr);
    }
    return rc;
}

vim_status vmamba_cross_scan4_events(const void *u, const void *delta, const void *z,
                                     const void *B, const void *C, const float *A, const float *D,
                                     const float *delta_bias, void *y, int batch, int H, int W,
                                     int channels, int d_state, vim_dtype dt, void *workspace,
                                     size_t workspace_bytes, cudaStream_t stream,
                                     cudaEvent_t *events) {
    return vmamba_cross_scan4_ex(u, delta, z, B, C, A, D, delta_bias, y, batch, H, W, channels, d_state,
                                 dt, 0u, workspace, workspace_bytes, stream, events);
}

vim_status vmamba_cross_scan4(const void *u, const void *delta, const void *z, const void *B,
                              const void *C, const float *A, const float *D,
                              const float *delta_bias, void *y, int batch, int H, int W,
                              int channels, int d_state, vim_dtype dt, void *workspace,
                              size_t workspace_bytes, cudaStream_t stream) {
    return vmamba_cross_scan4_ex(u, delta, z, B, C, A, D, delta_bias, y, batch, H, W, channels, d_state,
                                 dt, 0u, workspace, workspace_bytes, stream, nullptr);
}

vim_status cross_merge4(const void *ys, const void *z, void *y, int batch, int H, int W, int channels,
                        vim_dtype dt, cudaStream_t stream) {
    if (batch < 0 || H < 0 || W < 0 || channels < 0) return VIM_ERR_INVALID_ARG;
    if (dt != VIM_F32 && dt != VIM_BF16) return VIM_ERR_INVALID_ARG;
    if (channels % (dt == VIM_F32 ? 4 : 8) != 0) return VIM_ERR_UNSUPPORTED;
    if ((int64_t)H * W > INT32_MAX || (int64_t)batch * H * W * channels * 4 > INT32_MAX * (int64_t)4)
        return VIM_ERR_UNSUPPORTED;
    if (batch == 0 || H == 0 || W == 0 || channels == 0) return VIM_OK;
    if (!ys || !y) return VIM_ERR_INVALID_ARG;
    if (!aligned16(ys) || !aligned16(y) || (z && !aligned16(z))) return VIM_ERR_INVALID_ARG;
    MergeArgs a{ys, z, y, batch, H, W, channels};
    const int64_t items = (int64_t)batch * H * W * (channels / (dt == VIM_F32 ? 4 : 8));
    int blocks = (int)((items + 255) / 256);
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (dt == VIM_F32)
        merge4<float><<<blocks, 256, 0, stream>>>(a);
    else
        merge4<__nv_bfloat16><<<blocks, 256, 0, stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? VIM_OK : VIM_ERR_CUDA;
}

// ----------------------------------------------------------------------------
// the no-allocation variant of vim_scan_bidir (declared in vimscan.h)
// ----------------------------------------------------------------------------
// The built-in scratch buffer.  In host code its name only stands in for the symbol:
// the device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char vim_noalloc_scratch[VIM_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void *g_noalloc_addr[kMaxDevices] = {};

// device address of the scratch buffer on the current device (looked up on first use)
vim_status noalloc_scratch(void **addr) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return VIM_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, vim_noalloc_scratch) != cudaSuccess || !p) return VIM_ERR_CUDA;
        g_noalloc_addr[dev] = p;
    }
    *addr = g_noalloc_addr[dev];
    return VIM_OK;
}
}  // namespace

vim_status vim_scan_bidir_noalloc(const void *u, const void *delta, const void *z, const void *B,
                                  const void *C, int64_t bc_dir_stride, const float *A,
                                  const float *D, const float *delta_bias, void *y, int batch,
                                  int L, int d_inner, int d_state, vim_dtype dt,
                                  cudaStream_t stream) {
    vim_status st = check_common(batch, L, d_inner, d_state, dt);
    if (st != VIM_OK) return st;
    if (summary_bytes(batch, L, d_inner, d_state) > VIM_NOALLOC_SCRATCH_BYTES) return VIM_ERR_WORKSPACE;
    void *scratch = nullptr;
    if (batch > 0 && L > 0 && d_inner > 0) {
        st = noalloc_scratch(&scratch);
        if (st != VIM_OK) return st;
    }
    return vim_scan_bidir(u, delta, z, B, C, bc_dir_stride, A, D, delta_bias, y, batch, L, d_inner,
                          d_state, dt, scratch, VIM_NOALLOC_SCRATCH_BYTES, stream);
}

}  // extern "C"
