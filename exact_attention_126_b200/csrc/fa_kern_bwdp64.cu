// fa_kern_bwdp64.cu - the dK/dV and dQ passes for head_dim 64 on packed batches
// (kFeatPacked) in every combination of the other features.
#include "launch_impl.cuh"

namespace fa_host {

// kFeatPacked with the 8 combinations of kFeatAlibi, kFeatKpad, kFeatDropout
FA_INSTANTIATE_BWD(64, 32) FA_INSTANTIATE_BWD(64, 33) FA_INSTANTIATE_BWD(64, 34)
FA_INSTANTIATE_BWD(64, 35) FA_INSTANTIATE_BWD(64, 40) FA_INSTANTIATE_BWD(64, 41)
FA_INSTANTIATE_BWD(64, 42) FA_INSTANTIATE_BWD(64, 43)

int take_status_bwdp64() { return take_unit_status(); }

}  // namespace fa_host
