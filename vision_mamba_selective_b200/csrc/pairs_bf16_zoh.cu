// pairs_bf16_zoh.cu -- the pair kernels for bf16 I/O with the exact zero-order-hold Bbar.
#include "launch.cuh"

namespace vimscan {

vim_status launch_pair_bf16_zoh(const PairArgs &a, int N, cudaStream_t stream, cudaEvent_t *ev) {
    return launch_pair_n<__nv_bfloat16, true>(a, N, stream, ev);
}

}  // namespace vimscan
