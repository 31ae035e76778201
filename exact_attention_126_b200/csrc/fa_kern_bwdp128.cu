// fa_kern_bwdp128.cu - the dK/dV and dQ passes for head_dim 128 on packed batches
// (kFeatPacked) in every combination of the other features.
#include "launch_impl.cuh"

namespace fa_host {

// kFeatPacked with the 8 combinations of kFeatAlibi, kFeatKpad, kFeatDropout
FA_INSTANTIATE_BWD(128, 32) FA_INSTANTIATE_BWD(128, 33) FA_INSTANTIATE_BWD(128, 34)
FA_INSTANTIATE_BWD(128, 35) FA_INSTANTIATE_BWD(128, 40) FA_INSTANTIATE_BWD(128, 41)
FA_INSTANTIATE_BWD(128, 42) FA_INSTANTIATE_BWD(128, 43)

int take_status_bwdp128() { return take_unit_status(); }

}  // namespace fa_host
