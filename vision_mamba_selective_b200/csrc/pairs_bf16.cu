// pairs_bf16.cu -- the pair kernels for bf16 I/O with the first-order Bbar = Delta B.
#include "launch.cuh"

namespace vimscan {

vim_status launch_pair_bf16(const PairArgs &a, int N, cudaStream_t stream, cudaEvent_t *ev) {
    return launch_pair_n<__nv_bfloat16, false>(a, N, stream, ev);
}

}  // namespace vimscan
