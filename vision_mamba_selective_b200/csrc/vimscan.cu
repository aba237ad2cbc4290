// vimscan.cu -- host side of libvimscan.so: argument checks, planning, launches.
//
// Entry points are declared (with their contracts) in include/vimscan.h.  Every
// check runs on the host before the first launch; nothing here allocates memory or
// synchronises the stream.
#include "vimscan.h"

#include <algorithm>
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

// vim_scan_bidir with an optional convolution front (conv_w/conv_b non-null: u holds x), and
// optionally the states entering every checkpoint segment (ckpt)
vim_status bidir_impl(const void *u, const float *conv_w, const float *conv_b, const void *delta,
                      const void *z, const void *B, const void *C, int64_t bc_dir_stride, const float *A,
                      const float *D, const float *delta_bias, void *y, int batch, int L, int d_inner,
                      int d_state, vim_dtype dt, unsigned flags, void *workspace, size_t workspace_bytes,
                      cudaStream_t stream, cudaEvent_t *events, float *ckpt = nullptr) {
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
    if (ckpt && reinterpret_cast<uintptr_t>(ckpt) % 8) return VIM_ERR_INVALID_ARG;
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
    a.hck = ckpt;
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

size_t vim_scan_ckpt_bytes(int batch, int L, int d_inner, int d_state) {
    if (batch <= 0 || L <= 0 || d_inner <= 0 || !supported_state(d_state)) return 0;
    return (size_t)batch * ((L + kCkTokens - 1) / kCkTokens) * 2 * d_inner * d_state * sizeof(float);
}

vim_status vim_scan_bidir_ckpt(const void *u, const void *delta, const void *z, const void *B, const void *C,
                               int64_t bc_dir_stride, const float *A, const float *D, const float *delta_bias,
                               void *y, float *ckpt, int batch, int L, int d_inner, int d_state, vim_dtype dt,
                               unsigned flags, void *workspace, size_t workspace_bytes, cudaStream_t stream,
                               cudaEvent_t *events) {
    if (batch > 0 && L > 0 && d_inner > 0 && !ckpt) return VIM_ERR_INVALID_ARG;
    return bidir_impl(u, nullptr, nullptr, delta, z, B, C, bc_dir_stride, A, D, delta_bias, y, batch, L, d_inner,
                      d_state, dt, flags, workspace, workspace_bytes, stream, events, ckpt);
}

vim_status vim_scan_bidir_conv_ckpt(const void *x, const float *conv_w, const float *conv_b, const void *delta,
                                    const void *z, const void *B, const void *C, int64_t bc_dir_stride,
                                    const float *A, const float *D, const float *delta_bias, void *y, float *ckpt,
                                    int batch, int L, int d_inner, int d_state, vim_dtype dt, unsigned flags,
                                    void *workspace, size_t workspace_bytes, cudaStream_t stream,
                                    cudaEvent_t *events) {
    if (batch > 0 && L > 0 && d_inner > 0 && (!ckpt || !conv_w || !conv_b)) return VIM_ERR_INVALID_ARG;
    return bidir_impl(x, conv_w, conv_b, delta, z, B, C, bc_dir_stride, A, D, delta_bias, y, batch, L, d_inner,
                      d_state, dt, flags, workspace, workspace_bytes, stream, events, ckpt);
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

}  // extern "C"

namespace {

// vmamba_cross_scan4, and optionally each pair's states entering every checkpoint segment
// (ckpt: [2 pairs][batch][ceil(L/32)][2][N][C], over the pair's steps)
vim_status cross_impl(const void *u, const void *delta, const void *z, const void *B, const void *C, const float *A,
                      const float *D, const float *delta_bias, void *y, int batch, int H, int W, int channels,
                      int d_state, vim_dtype dt, unsigned flags, void *workspace, size_t workspace_bytes,
                      cudaStream_t stream, cudaEvent_t *events, float *ckpt) {
    if (H < 0 || W < 0 || (flags & ~kKnownFlags)) return VIM_ERR_INVALID_ARG;
    if (ckpt && reinterpret_cast<uintptr_t>(ckpt) % 8) return VIM_ERR_INVALID_ARG;
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
        a.hdiv = div_inv((unsigned)H);
        if (ckpt)
            a.hck = ckpt + (size_t)pair * batch * ((L + kCkTokens - 1) / kCkTokens) * 2 * d_state * channels;
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
}  // namespace

extern "C" {

vim_status vmamba_cross_scan4_ex(const void *u, const void *delta, const void *z, const void *B,
                                 const void *C, const float *A, const float *D, const float *delta_bias,
                                 void *y, int batch, int H, int W, int channels, int d_state, vim_dtype dt,
                                 unsigned flags, void *workspace, size_t workspace_bytes,
                                 cudaStream_t stream, cudaEvent_t *events) {
    return cross_impl(u, delta, z, B, C, A, D, delta_bias, y, batch, H, W, channels, d_state, dt, flags, workspace,
                      workspace_bytes, stream, events, nullptr);
}

vim_status vmamba_cross_scan4_ckpt(const void *u, const void *delta, const void *z, const void *B, const void *C,
                                   const float *A, const float *D, const float *delta_bias, void *y, float *ckpt,
                                   int batch, int H, int W, int channels, int d_state, vim_dtype dt, unsigned flags,
                                   void *workspace, size_t workspace_bytes, cudaStream_t stream,
                                   cudaEvent_t *events) {
    if (batch > 0 && H > 0 && W > 0 && channels > 0 && !ckpt) return VIM_ERR_INVALID_ARG;
    return cross_impl(u, delta, z, B, C, A, D, delta_bias, y, batch, H, W, channels, d_state, dt, flags, workspace,
                      workspace_bytes, stream, events, ckpt);
}

size_t vmamba_cross_ckpt_bytes(int batch, int H, int W, int channels, int d_state) {
    if (batch <= 0 || H <= 0 || W <= 0 || channels <= 0 || !supported_state(d_state)) return 0;
    if ((int64_t)H * W > INT32_MAX) return 0;
    return 2 * vim_scan_ckpt_bytes(batch, H * W, channels, d_state);
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

// ----------------------------------------------------------------------------
// vim_scan_bidir over host activations (declared in vimscan.h)
// ----------------------------------------------------------------------------
namespace {

// the batch cut into `slices` pieces of sb items (the last one may be shorter), and the
// workspace: two staging sets (u, delta, z, y, B, C of one slice each) and the scan's
// own summaries for the largest slice
struct HostPlan {
    int slices, sb;
    size_t act, bc;        // elements of one slice's u (and delta, z, y) and of one B (or C) copy
    size_t o_u, o_d, o_z, o_y, o_B, o_C, set_bytes, o_scan, scan_bytes, total;
};

HostPlan host_plan(int batch, int L, int Di, int N, vim_dtype dt, int slices, bool two_bc) {
    HostPlan h;
    std::memset(&h, 0, sizeof(h));
    h.slices = std::max(1, std::min(slices, batch));
    h.sb = (batch + h.slices - 1) / h.slices;
    h.slices = (batch + h.sb - 1) / h.sb;
    const size_t e = elem_size(dt);
    h.act = (size_t)h.sb * L * Di;
    h.bc = (size_t)h.sb * L * N;
    size_t o = 0;
    auto take = [&](size_t bytes) { const size_t at = o; o += round_up(bytes); return at; };
    h.o_u = take(h.act * e);
    h.o_d = take(h.act * e);
    h.o_z = take(h.act * e);
    h.o_y = take(h.act * e);
    h.o_B = take(h.bc * e * (two_bc ? 2 : 1));
    h.o_C = take(h.bc * e * (two_bc ? 2 : 1));
    h.set_bytes = o;
    h.o_scan = 2 * h.set_bytes;
    const int last = batch - (h.slices - 1) * h.sb;
    h.scan_bytes = std::max(summary_bytes(h.sb, L, Di, N), summary_bytes(last, L, Di, N));
    h.total = h.o_scan + round_up(h.scan_bytes);
    return h;
}

struct Events {
    cudaEvent_t e[7] = {};   // entry, uploaded[2], scanned[2], downloaded[2]
    bool ok = true;
    Events() {
        for (auto &x : e)
            if (cudaEventCreateWithFlags(&x, cudaEventDisableTiming) != cudaSuccess) { x = nullptr; ok = false; }
    }
    ~Events() {   // pending records complete on their own; destroying them here is allowed
        for (auto &x : e)
            if (x) cudaEventDestroy(x);
    }
};

}  // namespace

extern "C" {

size_t vim_scan_host_workspace_bytes(int batch, int L, int d_inner, int d_state, vim_dtype dt, int slices,
                                     int two_bc) {
    if (check_common(batch, L, d_inner, d_state, dt) != VIM_OK || slices < 1) return 0;
    if (batch == 0 || L == 0 || d_inner == 0) return 0;
    return host_plan(batch, L, d_inner, d_state, dt, slices, two_bc != 0).total;
}

vim_status vim_scan_bidir_host(const void *u, const void *delta, const void *z, const void *B,
                               const void *C, int64_t bc_dir_stride, const float *A, const float *D,
                               const float *delta_bias, void *y, int batch, int L, int d_inner,
                               int d_state, vim_dtype dt, unsigned flags, int slices, void *workspace,
                               size_t workspace_bytes, cudaStream_t stream, cudaStream_t upload,
                               cudaStream_t download) {
    vim_status st = check_common(batch, L, d_inner, d_state, dt);
    if (st != VIM_OK) return st;
    if (bc_dir_stride < 0 || slices < 1 || (flags & ~kKnownFlags)) return VIM_ERR_INVALID_ARG;
    if (batch == 0 || L == 0 || d_inner == 0) return VIM_OK;
    if (!u || !delta || !B || !C || !A || !D || !delta_bias || !y) return VIM_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(D) |
         reinterpret_cast<uintptr_t>(delta_bias)) % 4)
        return VIM_ERR_INVALID_ARG;
    const bool two = bc_dir_stride > 0;
    const HostPlan hp = host_plan(batch, L, d_inner, d_state, dt, slices, two);
    if (!workspace || workspace_bytes < hp.total) return VIM_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return VIM_ERR_WORKSPACE;
    if (!upload) upload = stream;
    if (!download) download = stream;

    Events ev;
    if (!ev.ok) return VIM_ERR_CUDA;
    cudaEvent_t entry = ev.e[0], *up = ev.e + 1, *sc = ev.e + 3, *dn = ev.e + 5;
    const size_t e = elem_size(dt);
    char *ws = static_cast<char *>(workspace);
    const char *hu = static_cast<const char *>(u), *hd = static_cast<const char *>(delta),
               *hz = static_cast<const char *>(z), *hB = static_cast<const char *>(B),
               *hC = static_cast<const char *>(C);
    char *hy = static_cast<char *>(y);
    auto ok = [](cudaError_t r) { return r == cudaSuccess; };
    // the copy streams start after everything queued on `stream` before this call
    if (!ok(cudaEventRecord(entry, stream)) || !ok(cudaStreamWaitEvent(upload, entry, 0)) ||
        !ok(cudaStreamWaitEvent(download, entry, 0)))
        return VIM_ERR_CUDA;
    for (int k = 0; k < hp.slices; ++k) {
        const int set = k & 1, b0 = k * hp.sb, nb = std::min(hp.sb, batch - b0);
        char *base = ws + set * hp.set_bytes;
        const size_t act = (size_t)nb * L * d_inner * e, bc = (size_t)nb * L * d_state * e;
        const size_t a0 = (size_t)b0 * L * d_inner * e, c0 = (size_t)b0 * L * d_state * e;
        // slice k reuses the set of slice k - 2 once that slice's y has left the device
        if (k >= 2 && !ok(cudaStreamWaitEvent(upload, dn[set], 0))) return VIM_ERR_CUDA;
        bool good = ok(cudaMemcpyAsync(base + hp.o_u, hu + a0, act, cudaMemcpyHostToDevice, upload)) &&
                    ok(cudaMemcpyAsync(base + hp.o_d, hd + a0, act, cudaMemcpyHostToDevice, upload)) &&
                    (!z || ok(cudaMemcpyAsync(base + hp.o_z, hz + a0, act, cudaMemcpyHostToDevice, upload))) &&
                    ok(cudaMemcpyAsync(base + hp.o_B, hB + c0, bc, cudaMemcpyHostToDevice, upload)) &&
                    ok(cudaMemcpyAsync(base + hp.o_C, hC + c0, bc, cudaMemcpyHostToDevice, upload));
        if (good && two) {
            const size_t s0 = (size_t)bc_dir_stride * e;
            good = ok(cudaMemcpyAsync(base + hp.o_B + bc, hB + s0 + c0, bc, cudaMemcpyHostToDevice, upload)) &&
                   ok(cudaMemcpyAsync(base + hp.o_C + bc, hC + s0 + c0, bc, cudaMemcpyHostToDevice, upload));
        }
        if (!good || !ok(cudaEventRecord(up[set], upload)) || !ok(cudaStreamWaitEvent(stream, up[set], 0)))
            return VIM_ERR_CUDA;
        st = bidir_impl(base + hp.o_u, nullptr, nullptr, base + hp.o_d, z ? base + hp.o_z : nullptr,
                        base + hp.o_B, base + hp.o_C, two ? (int64_t)nb * L * d_state : 0, A, D, delta_bias,
                        base + hp.o_y, nb, L, d_inner, d_state, dt, flags, ws + hp.o_scan, hp.scan_bytes, stream,
                        nullptr);
        if (st != VIM_OK) return st;
        if (!ok(cudaEventRecord(sc[set], stream)) || !ok(cudaStreamWaitEvent(download, sc[set], 0)) ||
            !ok(cudaMemcpyAsync(hy + a0, base + hp.o_y, act, cudaMemcpyDeviceToHost, download)) ||
            !ok(cudaEventRecord(dn[set], download)))
            return VIM_ERR_CUDA;
    }
    // `stream` reaches the end of this call once the last slice's y is on the host
    const int last = (hp.slices - 1) & 1;
    if (!ok(cudaStreamWaitEvent(stream, dn[last], 0))) return VIM_ERR_CUDA;
    return VIM_OK;
}

}  // extern "C"
