// launch.h - what the host side of the C ABI (fa_api.cu) needs from the kernel units.
//
// The kernels are compiled in several translation units (fa_kern_*.cu) so that their
// many variants build in parallel; each unit defines the launchers of its kernels for
// every feature combination (explicit instantiations) and an accessor of its own copy of
// the device status word that bounded waits write.
#pragma once

#include <cuda_runtime.h>

#include "fa.h"
#include "rng.cuh"
#include "tiles.cuh"

namespace fa_host {

// Optional inputs and outputs of one call (fa_options_t, checked and resolved).
struct Extras {
  const float* alibi = nullptr;    // H slopes: the kFeatAlibi kernels
  const uint8_t* kpad = nullptr;   // (B, N) key-padding flags: the kFeatKpad kernels
  void* o_low = nullptr;           // bf16 residual of O: written by the forward, read by delta
  bool dropout = false;            // the kFeatDropout kernels, with `drop`
  bool fused = false;              // backward: the fused pass (head_dim 64) instead of the
                                   // dK/dV and dQ passes
  const int* seq_len = nullptr;    // variable-length batch: B real lengths
  const int* sched = nullptr;      // ... and the backward's schedule tables in its workspace
  const int* cu = nullptr;         // packed batch: B + 1 cumulative lengths, and ...
  int total = 0;                   // ... the tokens of its (total, H, d) tensors
  bool fp8 = false;                // forward on e4m3 Q, K, V (the kFeatFp8 kernel)
  float o_scale = 1.f;             // with fp8: the V descale, applied to O
  fa::DropoutArgs drop = {0, 0, 0, 0, 1.f};

  // A batch of sequences of their own lengths (padded or packed).
  bool varlen() const { return seq_len != nullptr || cu != nullptr; }

  // The kernel variant these options select (the backward passes ignore kFeatResidual).
  int features() const {
    return (alibi ? fa::kFeatAlibi : 0) | (kpad ? fa::kFeatKpad : 0) |
           (o_low ? fa::kFeatResidual : 0) | (dropout ? fa::kFeatDropout : 0) |
           (fp8 ? fa::kFeatFp8 : 0) | (cu ? fa::kFeatPacked : 0);
  }
};

// The problem of one launch: BH = B*H (batch, head) pairs of N rows; `left`, `right`:
// the resolved window (-1 = unbounded, right = 0 when causal).
struct Problem {
  int BH;
  int H;
  int N;
  float scale;
  int left;
  int right;
};

template <int D, int kFeat>
fa_status_t launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                       const Problem& pb, const Extras& x, int fault, cudaStream_t st);

template <int D>
fa_status_t launch_preprocess(const void* o, const void* o_low, const void* dout,
                              const float* lse, float* stats, float* dq_acc,
                              const fa::SchedBuild& sb, const int* cu, int total, int H,
                              int BH, int N, cudaStream_t st);

// The fused backward pass (head_dim 64): dK, dV, and dQ added into `dq_acc`.
template <int kFeat>
fa_status_t launch_fused(const void* q, const void* k, const void* v, const void* dout,
                         const void* ws, float* dq_acc, void* dk, void* dv, const Problem& pb,
                         const Extras& x, cudaStream_t st);

template <int D>
fa_status_t launch_dq_convert(const float* dq_acc, void* dq, int BH, int N, float scale,
                              cudaStream_t st);

template <int D, int kFeat>
fa_status_t launch_dkdv(const void* q, const void* k, const void* v, const void* dout,
                        const void* ws, void* dk, void* dv, const Problem& pb, const Extras& x,
                        cudaStream_t st);

template <int D, int kFeat>
fa_status_t launch_dq(const void* q, const void* k, const void* v, const void* dout,
                      const void* ws, void* dq, const Problem& pb, const Extras& x,
                      cudaStream_t st);

// Variable-length batches: zero rows past each entry's real length of up to three bf16
// tensors (null = absent) and set their LSE to -inf (lse null = absent).
template <int D>
fa_status_t launch_fill_past_length(void* t0, void* t1, void* t2, float* lse,
                                    const int* seq_len, int BH, int H, int N, cudaStream_t st);

// Reads and clears the device status word of each kernel unit (0 = nothing recorded);
// returns -1 if reading it failed.
int take_status_fwd64();
int take_status_fwd128();
int take_status_fwdp64();
int take_status_fwdp128();
int take_status_bwdp64();
int take_status_bwdp128();
int take_status_bwd64();
int take_status_bwd128();
int take_status_fused64();

}  // namespace fa_host
