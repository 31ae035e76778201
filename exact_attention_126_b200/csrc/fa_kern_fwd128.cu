// fa_kern_fwd128.cu - the forward kernel for head_dim 128 in every feature combination.
#include "launch_impl.cuh"

namespace fa_host {

// the 16 combinations of kFeatAlibi, kFeatKpad, kFeatResidual, kFeatDropout
FA_INSTANTIATE_FWD(128, 0)  FA_INSTANTIATE_FWD(128, 1)  FA_INSTANTIATE_FWD(128, 2)
FA_INSTANTIATE_FWD(128, 3)  FA_INSTANTIATE_FWD(128, 4)  FA_INSTANTIATE_FWD(128, 5)
FA_INSTANTIATE_FWD(128, 6)  FA_INSTANTIATE_FWD(128, 7)  FA_INSTANTIATE_FWD(128, 8)
FA_INSTANTIATE_FWD(128, 9)  FA_INSTANTIATE_FWD(128, 10) FA_INSTANTIATE_FWD(128, 11)
FA_INSTANTIATE_FWD(128, 12) FA_INSTANTIATE_FWD(128, 13) FA_INSTANTIATE_FWD(128, 14)
FA_INSTANTIATE_FWD(128, 15)
// the e4m3 forward (no other option)
FA_INSTANTIATE_FWD(128, 16)

int take_status_fwd128() { return take_unit_status(); }

}  // namespace fa_host
