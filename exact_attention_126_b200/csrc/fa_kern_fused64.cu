// fa_kern_fused64.cu - the fused backward pass (dK, dV and dQ in one pass over key tiles) for
// head_dim 64, in every feature combination of ALiBi, key padding and dropout.
#include "launch_impl.cuh"

namespace fa_host {

FA_INSTANTIATE_FUSED(0) FA_INSTANTIATE_FUSED(1) FA_INSTANTIATE_FUSED(2) FA_INSTANTIATE_FUSED(3)
FA_INSTANTIATE_FUSED(8) FA_INSTANTIATE_FUSED(9) FA_INSTANTIATE_FUSED(10) FA_INSTANTIATE_FUSED(11)

int take_status_fused64() { return take_unit_status(); }

}  // namespace fa_host
