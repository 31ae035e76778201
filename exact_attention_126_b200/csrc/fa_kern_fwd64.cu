// fa_kern_fwd64.cu - the forward kernel for head_dim 64 in every feature combination.
#include "launch_impl.cuh"

namespace fa_host {

// the 16 combinations of kFeatAlibi, kFeatKpad, kFeatResidual, kFeatDropout
FA_INSTANTIATE_FWD(64, 0)  FA_INSTANTIATE_FWD(64, 1)  FA_INSTANTIATE_FWD(64, 2)
FA_INSTANTIATE_FWD(64, 3)  FA_INSTANTIATE_FWD(64, 4)  FA_INSTANTIATE_FWD(64, 5)
FA_INSTANTIATE_FWD(64, 6)  FA_INSTANTIATE_FWD(64, 7)  FA_INSTANTIATE_FWD(64, 8)
FA_INSTANTIATE_FWD(64, 9)  FA_INSTANTIATE_FWD(64, 10) FA_INSTANTIATE_FWD(64, 11)
FA_INSTANTIATE_FWD(64, 12) FA_INSTANTIATE_FWD(64, 13) FA_INSTANTIATE_FWD(64, 14)
FA_INSTANTIATE_FWD(64, 15)

int take_status_fwd64() { return take_unit_status(); }

}  // namespace fa_host
