// pairs_f32_zoh.cu -- the pair kernels for fp32 I/O with the exact zero-order-hold Bbar.
#include "launch.cuh"

namespace vimscan {

vim_status launch_pair_f32_zoh(const PairArgs &a, int N, cudaStream_t stream, cudaEvent_t *ev) {
    return launch_pair_n<float, true>(a, N, stream, ev);
}

}  // namespace vimscan
