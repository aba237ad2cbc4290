// launch.cuh -- planning and kernel launches of one pair of directions (host side).
//
// Shared by the translation units of libvimscan.so: vimscan.cu (entry points) uses the
// plan and the dispatch at the bottom; each pairs_*.cu instantiates the kernel
// variants of one element type and one discretisation through launch_pair_n.
#pragma once

#include "vimscan.h"

#include <cstdint>

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

// Chunking of a sequence.  Short sequences with few CTAs (fewer than a B200 has SMs)
// are cut into kShortChunk-token chunks anyway, so that their walks run side by side
// instead of one long walk per CTA (the latency-bound sizes).
constexpr int kShortChunk = 32;
constexpr int64_t kFewCtas = 148;

Plan plan_for(int batch, int L, int Di) {
    Plan pl;
    const int64_t ctas = (int64_t)batch * ((Di + kDC - 1) / kDC);
    if (L <= kSingleChunkMax && !(ctas < kFewCtas && L > 2 * kShortChunk)) {
        pl.chunk = ((L + kTile - 1) / kTile) * kTile;
        if (pl.chunk == 0) pl.chunk = kTile;
        pl.G = 1;
    } else {
        pl.chunk = L <= kSingleChunkMax ? kShortChunk : kLongChunk;
        pl.G = (L + pl.chunk - 1) / pl.chunk;
    }
    return pl;
}

size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// summaries for one pair: hloc [batch][G][2][Di][N] + ssum [batch][G][2][Di]
size_t summary_bytes(int batch, int L, int Di, int N) {
    const Plan pl = plan_for(batch, L, Di);
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

template <typename T, int N, bool VEC_BC, bool PIN, bool CONV, bool ZOH, bool DT>
vim_status launch_pair_v(const PairArgs &a, cudaStream_t stream, cudaEvent_t *ev) {
    const dim3 grid((a.Di + kDC - 1) / kDC, a.G, a.batch);
    if (a.G > 1) {
        const size_t sc = carry_smem<T, N, CONV>();
        if (cudaFuncSetAttribute(pair_carry<T, N, VEC_BC, CONV, ZOH, DT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)sc) != cudaSuccess)
            return VIM_ERR_CUDA;
        pair_carry<T, N, VEC_BC, CONV, ZOH, DT><<<grid, kThreads, sc, stream>>>(a);
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
    auto kernel = pair_main<T, N, VEC_BC, PIN, CONV, ZOH, DT>;
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
// and the convolution front (Vim with x as input) are never combined; the step-input
// mode (delta from the x_proj column, bf16 I/O, first-order Bbar) comes with or
// without the convolution front
template <typename T, int N, bool VEC_BC, bool ZOH>
vim_status launch_pair_v(const PairArgs &a, cudaStream_t stream, cudaEvent_t *ev) {
    if (a.dt_in) {
        if constexpr (sizeof(T) == 2 && !ZOH) {
            if (a.conv_w) return launch_pair_v<T, N, VEC_BC, false, true, false, true>(a, stream, ev);
            return launch_pair_v<T, N, VEC_BC, false, false, false, true>(a, stream, ev);
        } else {
            return VIM_ERR_UNSUPPORTED;
        }
    }
    if (a.conv_w) return launch_pair_v<T, N, VEC_BC, false, true, ZOH, false>(a, stream, ev);
    if (a.partial_in) return launch_pair_v<T, N, VEC_BC, true, false, ZOH, false>(a, stream, ev);
    return launch_pair_v<T, N, VEC_BC, false, false, ZOH, false>(a, stream, ev);
}

// B/C move as 16-byte vectors when their rows allow it and every base is aligned
template <typename T, int N, bool ZOH>
vim_status launch_pair_t(const PairArgs &a, cudaStream_t stream, cudaEvent_t *ev) {
    if constexpr (bc_vectorizable<T, N>()) {
        const bool aligned = aligned16(a.B[0]) && aligned16(a.B[1]) && aligned16(a.C[0]) &&
                             aligned16(a.C[1]);
        if (aligned) return launch_pair_v<T, N, true, ZOH>(a, stream, ev);
    }
    return launch_pair_v<T, N, false, ZOH>(a, stream, ev);
}

template <typename T, bool ZOH>
vim_status launch_pair_n(const PairArgs &a, int N, cudaStream_t stream, cudaEvent_t *ev) {
    switch (N) {
        case 2: return launch_pair_t<T, 2, ZOH>(a, stream, ev);
        case 4: return launch_pair_t<T, 4, ZOH>(a, stream, ev);
        case 8: return launch_pair_t<T, 8, ZOH>(a, stream, ev);
        case 16: return launch_pair_t<T, 16, ZOH>(a, stream, ev);
        default: return VIM_ERR_UNSUPPORTED;
    }
}

}  // namespace

// One translation unit per element type and discretisation (pairs_*.cu) instantiates
// the kernels and defines one of these.
vim_status launch_pair_f32(const PairArgs &a, int N, cudaStream_t stream, cudaEvent_t *ev);
vim_status launch_pair_bf16(const PairArgs &a, int N, cudaStream_t stream, cudaEvent_t *ev);
vim_status launch_pair_f32_zoh(const PairArgs &a, int N, cudaStream_t stream, cudaEvent_t *ev);
vim_status launch_pair_bf16_zoh(const PairArgs &a, int N, cudaStream_t stream, cudaEvent_t *ev);

inline vim_status launch_pair(const PairArgs &a, int N, vim_dtype dt, cudaStream_t stream, cudaEvent_t *ev) {
    if (a.zoh)
        return dt == VIM_F32 ? launch_pair_f32_zoh(a, N, stream, ev) : launch_pair_bf16_zoh(a, N, stream, ev);
    return dt == VIM_F32 ? launch_pair_f32(a, N, stream, ev) : launch_pair_bf16(a, N, stream, ev);
}

}  // namespace vimscan
