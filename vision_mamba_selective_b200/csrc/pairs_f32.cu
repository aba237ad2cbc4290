// pairs_f32.cu -- the pair kernels for fp32 I/O with the first-order Bbar = Delta B.
#include "launch.cuh"

namespace vimscan {

vim_status launch_pair_f32(const PairArgs &a, int N, cudaStream_t stream, cudaEvent_t *ev) {
    return launch_pair_n<float, false>(a, N, stream, ev);
}

}  // namespace vimscan
