// vimscan.cu -- host side of libvimscan.so: argument checks, planning, launches.
//
// Entry points are declared (with their contracts) in include/vimscan.h.  Every
// check runs on the host before the first launch; nothing here allocates memory or
// synchronises the stream.
#include "vimscan.h"

#include <cstdint>
#include <cstring>
#include <mutex>

#include "scan_kernels.cuh"

namespace vimscan {
namespace {

#ifndef VIMSCAN_SINGLE_CHUNK_MAX
#define VIMSCAN_SINGLE_CHUNK_MAX 256
#endif
#ifndef VIMSCAN_LONG_CHUNK
#define VIMSCAN_LONG_CHUNK 96
#endif
// sequences up to kSingleChunkMax tokens run as one chunk; longer ones in chunks of
// kLongChunk tokens (a multiple of kTile), sized so that four CTAs of the main kernel
// fit in one SM's shared memory
constexpr int kSingleChunkMax = VIMSCAN_SINGLE_CHUNK_MAX;
constexpr int kLongChunk = VIMSCAN_LONG_CHUNK;
static_assert(kLongChunk % kTile == 0, "chunks are whole tiles");
constexpr size_t kAlign = 256;

struct Plan {
    int chunk;  // tokens per chunk (multiple of kTile)
    int G;      // chunks
};

Plan plan_for(int L) {
    Plan pl;
    if (L <= kSingleChunkMax) {
        pl.chunk = ((L + kTile - 1) / kTile) * kTile;
        if (pl.chunk == 0) pl.chunk = kTile;
        pl.G = 1;
    } else {
        pl.chunk = kLongChunk;
        pl.G = (L + kLongChunk - 1) / kLongChunk;
    }
    return pl;
}

size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// summaries for one pair: hloc [batch][G][2][Di][N] + ssum [batch][G][2][Di]
size_t summary_bytes(int batch, int L, int Di, int N) {
    const Plan pl = plan_for(L);
    if (pl.G <= 1) return 0;
    const size_t units = (size_t)batch * pl.G * 2 * Di;
    return round_up(units * N * sizeof(float)) + round_up(units * sizeof(float));
}

bool supported_state(int N) { return N == 2 || N == 4 || N == 8 || N == 16; }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t elem_size(vim_dtype dt) { return dt == VIM_F32 ? 4 : 2; }

vim_status check_common(int batch, int L, int Di, int N, vim_dtype dt) {
    if (batch < 0 || L < 0 || Di < 0 || N < 0) return VIM_ERR_INVALID_ARG;
    if (dt != VIM_F32 && dt != VIM_BF16) return VIM_ERR_INVALID_ARG;
    if (!supported_state(N)) return VIM_ERR_UNSUPPORTED;
    if (Di % (dt == VIM_F32 ? 4 : 8) != 0) return VIM_ERR_UNSUPPORTED;
    if ((int64_t)batch * L * Di > INT32_MAX || (int64_t)batch * L * N > INT32_MAX)
        return VIM_ERR_UNSUPPORTED;
    return VIM_OK;
}

template <typename T, int N, bool CONV>
size_t main_smem(int chunk) {
    return 2 * (size_t)Stage<T, N, CONV>::kSlotBytes + (size_t)chunk * kDC * 4 + (size_t)kTile * kDC * 4;
}
template <typename T, int N, bool CONV>
size_t carry_smem() {
    return 2 * (size_t)Stage<T, N, CONV>::kSlotBytes;
}

// Launch of a kernel that may start while the previous kernel on the stream drains
// (programmatic dependent launch); the kernel itself waits, with
// cudaGridDependencySynchronize, before it reads anything that kernel writes.
#ifndef VIMSCAN_PDL
#define VIMSCAN_PDL 1
#endif
template <typename... Args>
cudaError_t launch_dependent(void (*kernel)(Args...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t stream, Args... args) {
    if (!VIMSCAN_PDL) {
        kernel<<<grid, block, smem, stream>>>(args...);
        return cudaGetLastError();
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// events: null, or 3 events recorded after the carry, combine and main kernels
inline vim_status mark(cudaEvent_t *events, int i, cudaStream_t stream) {
    if (!events) return VIM_OK;
    return cudaEventRecord(events[i], stream) == cudaSuccess ? VIM_OK : VIM_ERR_CUDA;
}

template <typename T, int N, bool VEC_BC, bool PIN, bool CONV>
vim_status launch_pair_v(const PairArgs &a, cudaStream_t stream, cudaEvent_t *ev) {
    const dim3 grid((a.Di + kDC - 1) / kDC, a.G, a.batch);
    if (a.G > 1) {
        const size_t sc = carry_smem<T, N, CONV>();
        if (cudaFuncSetAttribute(pair_carry<T, N, VEC_BC, CONV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)sc) != cudaSuccess)
            return VIM_ERR_CUDA;
        pair_carry<T, N, VEC_BC, CONV><<<grid, kThreads, sc, stream>>>(a);
        if (cudaGetLastError() != cudaSuccess) return VIM_ERR_CUDA;
        if (mark(ev, 0, stream) != VIM_OK) return VIM_ERR_CUDA;
        const int64_t units = (int64_t)a.batch * 2 * a.Di * N;
        if (launch_dependent(pair_combine<N>, dim3((unsigned)((units + 255) / 256)), dim3(256), 0, stream,
                             a) != cudaSuccess)
            return VIM_ERR_CUDA;
        if (mark(ev, 1, stream) != VIM_OK) return VIM_ERR_CUDA;
    } else if (ev) {
        if (mark(ev, 0, stream) != VIM_OK || mark(ev, 1, stream) != VIM_OK) return VIM_ERR_CUDA;
    }
    const size_t sm = main_smem<T, N, CONV>(a.chunk);
    auto kernel = pair_main<T, N, VEC_BC, PIN, CONV>;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) != cudaSuccess)
        return VIM_ERR_CUDA;
    if (a.G > 1) {
        if (launch_dependent(kernel, grid, dim3(kThreads), sm, stream, a) != cudaSuccess) return VIM_ERR_CUDA;
    } else {
        kernel<<<grid, kThreads, sm, stream>>>(a);
    }
    if (cudaGetLastError() != cudaSuccess) return VIM_ERR_CUDA;
    return mark(ev, 2, stream);
}

// the kernel variants a pair needs: fp32 partial_in (second pair of the cross-scan)
// and the convolution front (Vim with x as input) are never combined
template <typename T, int N, bool VEC_BC>
vim_status launch_pair_v(const PairArgs &a, cudaStream_t stream, cudaEvent_t *ev) {
    if (a.conv_w) return launch_pair_v<T, N, VEC_BC, false, true>(a, stream, ev);
    if (a.partial_in) return launch_pair_v<T, N, VEC_BC, true, false>(a, stream, ev);
    return launch_pair_v<T, N, VEC_BC, false, false>(a, stream, ev);
}

// B/C move as 16-byte vectors when their rows allow it and every base is aligned
template <typename T, int N>
vim_status launch_pair_t(const PairArgs &a, cudaStream_t stream, cudaEvent_t *ev) {
    if constexpr (bc_vectorizable<T, N>()) {
        const bool aligned = aligned16(a.B[0]) && aligned16(a.B[1]) && aligned16(a.C[0]) &&
                             aligned16(a.C[1]);
        if (aligned) return launch_pair_v<T, N, true>(a, stream, ev);
    }
    return launch_pair_v<T, N, false>(a, stream, ev);
}

template <typename T>
vim_status launch_pair_n(const PairArgs &a, int N, cudaStream_t stream, cudaEvent_t *ev) {
    switch (N) {
        case 2: return launch_pair_t<T, 2>(a, stream, ev);
        case 4: return launch_pair_t<T, 4>(a, stream, ev);
        case 8: return launch_pair_t<T, 8>(a, stream, ev);
        case 16: return launch_pair_t<T, 16>(a, stream, ev);
        default: return VIM_ERR_UNSUPPORTED;
    }
}

vim_status launch_pair(const PairArgs &a, int N, vim_dtype dt, cudaStream_t stream, cudaEvent_t *ev) {
    return dt == VIM_F32 ? launch_pair_n<float>(a, N, stream, ev)
                         : launch_pair_n<__nv_bfloat16>(a, N, stream, ev);
}

}  // namespace
}  // namespace vimscan

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
// vim_scan_bidir with an optional convolution front (conv_w/conv_b non-null: u holds x)
vim_status bidir_impl(const void *u, const float *conv_w, const float *conv_b, const void *delta,
                      const void *z, const void *B, const void *C, int64_t bc_dir_stride, const float *A,
                      const float *D, const float *delta_bias, void *y, int batch, int L, int d_inner,
                      int d_state, vim_dtype dt, void *workspace, size_t workspace_bytes,
                      cudaStream_t stream, cudaEvent_t *events) {
    vim_status st = check_common(batch, L, d_inner, d_state, dt);
    if (st != VIM_OK) return st;
    if (bc_dir_stride < 0) return VIM_ERR_INVALID_ARG;
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
    const Plan pl = plan_for(L);
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
                      d_inner, d_state, dt, workspace, workspace_bytes, stream, events);
}

vim_status vim_scan_bidir_conv_events(const void *x, const float *conv_w, const float *conv_b,
                                      const void *delta, const void *z, const void *B, const void *C,
                                      int64_t bc_dir_stride, const float *A, const float *D,
                                      const float *delta_bias, void *y, int batch, int L, int d_inner,
                                      int d_state, vim_dtype dt, void *workspace, size_t workspace_bytes,
                                      cudaStream_t stream, cudaEvent_t *events) {
    if (batch > 0 && L > 0 && d_inner > 0) {
        if (!conv_w || !conv_b) return VIM_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(conv_w) | reinterpret_cast<uintptr_t>(conv_b)) % 4)
            return VIM_ERR_INVALID_ARG;
    }
    return bidir_impl(x, conv_w, conv_b, delta, z, B, C, bc_dir_stride, A, D, delta_bias, y, batch, L,
                      d_inner, d_state, dt, workspace, workspace_bytes, stream, events);
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

vim_status vmamba_cross_scan4_events(const void *u, const void *delta, const void *z,
                                     const void *B, const void *C, const float *A, const float *D,
                                     const float *delta_bias, void *y, int batch, int H, int W,
                                     int channels, int d_state, vim_dtype dt, void *workspace,
                                     size_t workspace_bytes, cudaStream_t stream,
                                     cudaEvent_t *events) {
    if (H < 0 || W < 0) return VIM_ERR_INVALID_ARG;
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

    const Plan pl = plan_for(L);
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

vim_status vmamba_cross_scan4(const void *u, const void *delta, const void *z, const void *B,
                              const void *C, const float *A, const float *D,
                              const float *delta_bias, void *y, int batch, int H, int W,
                              int channels, int d_state, vim_dtype dt, void *workspace,
                              size_t workspace_bytes, cudaStream_t stream) {
    return vmamba_cross_scan4_events(u, delta, z, B, C, A, D, delta_bias, y, batch, H, W, channels,
                                     d_state, dt, workspace, workspace_bytes, stream, nullptr);
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
