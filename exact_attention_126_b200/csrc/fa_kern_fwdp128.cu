// fa_kern_fwdp128.cu - the forward kernel for head_dim 128 on packed batches (kFeatPacked) in
// every combination of the other bf16 features.
#include "launch_impl.cuh"

namespace fa_host {

// kFeatPacked with the 16 combinations of kFeatAlibi, kFeatKpad, kFeatResidual, kFeatDropout
FA_INSTANTIATE_FWD(128, 32) FA_INSTANTIATE_FWD(128, 33) FA_INSTANTIATE_FWD(128, 34)
FA_INSTANTIATE_FWD(128, 35) FA_INSTANTIATE_FWD(128, 36) FA_INSTANTIATE_FWD(128, 37)
FA_INSTANTIATE_FWD(128, 38) FA_INSTANTIATE_FWD(128, 39) FA_INSTANTIATE_FWD(128, 40)
FA_INSTANTIATE_FWD(128, 41) FA_INSTANTIATE_FWD(128, 42) FA_INSTANTIATE_FWD(128, 43)
FA_INSTANTIATE_FWD(128, 44) FA_INSTANTIATE_FWD(128, 45) FA_INSTANTIATE_FWD(128, 46)
FA_INSTANTIATE_FWD(128, 47)

int take_status_fwdp128() { return take_unit_status(); }

}  // namespace fa_host
