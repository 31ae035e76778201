// fa_kern_fwdp64.cu - the forward kernel for head_dim 64 on packed batches (kFeatPacked) in
// every combination of the other features.
#include "launch_impl.cuh"

namespace fa_host {

// kFeatPacked with the 16 combinations of kFeatAlibi, kFeatKpad, kFeatResidual, kFeatDropout
FA_INSTANTIATE_FWD(64, 32) FA_INSTANTIATE_FWD(64, 33) FA_INSTANTIATE_FWD(64, 34)
FA_INSTANTIATE_FWD(64, 35) FA_INSTANTIATE_FWD(64, 36) FA_INSTANTIATE_FWD(64, 37)
FA_INSTANTIATE_FWD(64, 38) FA_INSTANTIATE_FWD(64, 39) FA_INSTANTIATE_FWD(64, 40)
FA_INSTANTIATE_FWD(64, 41) FA_INSTANTIATE_FWD(64, 42) FA_INSTANTIATE_FWD(64, 43)
FA_INSTANTIATE_FWD(64, 44) FA_INSTANTIATE_FWD(64, 45) FA_INSTANTIATE_FWD(64, 46)
FA_INSTANTIATE_FWD(64, 47)

int take_status_fwdp64() { return take_unit_status(); }

}  // namespace fa_host
