// fa_kern_bwd128.cu - the backward kernels for head_dim 128 (delta preprocess, dK/dV pass,
// dQ pass) in every feature combination.
#include "launch_impl.cuh"

namespace fa_host {

// the 8 combinations of kFeatAlibi, kFeatKpad, kFeatDropout (bit kFeatResidual unset)
FA_INSTANTIATE_BWD(128, 0) FA_INSTANTIATE_BWD(128, 1) FA_INSTANTIATE_BWD(128, 2)
FA_INSTANTIATE_BWD(128, 3) FA_INSTANTIATE_BWD(128, 8) FA_INSTANTIATE_BWD(128, 9)
FA_INSTANTIATE_BWD(128, 10) FA_INSTANTIATE_BWD(128, 11)
template fa_status_t launch_preprocess<128>(const void*, const void*, const void*, const float*,
                                           float*, float*, const fa::SchedBuild&, const int*, int,
                                           int, int, int,
                                           cudaStream_t);
template fa_status_t launch_dq_convert<128>(const float*, void*, int, int, float, cudaStream_t);
template fa_status_t launch_fill_past_length<128>(void*, void*, void*, float*, const int*, int,
                                                 int, int, cudaStream_t);

int take_status_bwd128() { return take_unit_status(); }

}  // namespace fa_host
