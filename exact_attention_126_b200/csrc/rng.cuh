// rng.cuh - the counter-based generator of attention dropout.
//
// Philox4x32-10 (J. Salmon, M. Moraes, R. Dror, D. Shaw, "Parallel random numbers: as easy
// as 1, 2, 3", SC 2011): the 4-word counter goes through ten rounds of the Philox S-box,
//   (c0, c1, c2, c3) -> (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2), hi(M0 c0) ^ c3 ^ k1, lo(M0 c0)),
// with the 2-word key advanced by the Weyl increments (W0, W1) before every round but the
// first. Any counter can be evaluated on its own, so the backward regenerates exactly the
// keep flags the forward drew, in whatever order its threads need them.
//
// Layout of the flags (the pages name only `dropout_p`, page "告别OOM和训练慢…(含A100环境
// 配置)" §4.2): the weight of query i on key j of head bh = b*H + h uses the output of
// counter (j / 16, i, bh, offset) under key (seed low, seed high 32 bits); key j takes byte
// j mod 4 of word (j mod 16) / 4, and the weight is dropped iff that byte is below
// t = floor(256 p + 1/2). Kept weights are scaled by 256 / (256 - t).
#pragma once

#include <stdint.h>

namespace fa {

struct Philox4 {
  uint32_t w[4];
};

__device__ __forceinline__ Philox4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2,
                                                 uint32_t c3, uint32_t k0, uint32_t k1) {
  constexpr uint32_t kM0 = 0xD2511F53u, kM1 = 0xCD9E8D57u;
  constexpr uint32_t kW0 = 0x9E3779B9u, kW1 = 0xBB67AE85u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += kW0;
      k1 += kW1;
    }
    const uint32_t hi0 = __umulhi(kM0, c0), lo0 = kM0 * c0;
    const uint32_t hi1 = __umulhi(kM1, c2), lo1 = kM1 * c2;
    const uint32_t n0 = hi1 ^ c1 ^ k0;
    const uint32_t n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  return Philox4{{c0, c1, c2, c3}};
}

// The dropout generator's fixed inputs for one call.
struct DropoutArgs {
  uint32_t seed_lo, seed_hi;  // Philox key
  uint32_t offset;            // fourth counter word
  uint32_t threshold;         // t: a byte below it drops the weight (1 .. 255)
  float keep_scale;           // 256 / (256 - t)
};

// Keep flags of keys 16 * blk .. 16 * blk + 15 for query `row` of head bh, as 16 bits
// (bit e for key 16 * blk + e).
__device__ __forceinline__ uint32_t keep_bits16(const DropoutArgs& dr, uint32_t blk,
                                                uint32_t row, uint32_t bh) {
  const Philox4 r = philox4x32_10(blk, row, bh, dr.offset, dr.seed_lo, dr.seed_hi);
  uint32_t bits = 0;
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const uint32_t byte = (r.w[e >> 2] >> (8 * (e & 3))) & 0xFFu;
    bits |= (byte >= dr.threshold ? 1u : 0u) << e;
  }
  return bits;
}

}  // namespace fa
