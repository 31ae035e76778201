// fa_fwd.cuh - fused attention forward for sm_100a.
//
// One CTA owns one 128-row query tile of one (batch, head) and walks the key/value
// tiles it can see (page "Flash Attention 3.7 核心原理与实战" §3.1: load a Q block, iterate
// over the K, V blocks; page "告别OOM和训练慢…(含A100环境配置)" §2.1 tiling):
//
//   warp 5       TMA producer: Q once, then K_j and V_j through a ring of shared-memory
//                stages (128-byte swizzle), each stage guarded by full/empty mbarriers.
//   warp 4       MMA issuer (one thread): S_j = Q K_j^T into one of two TMEM buffers, then,
//                once the softmax has published P_j, O += P_j V_j with P_j read from TMEM.
//   warps 0..3   softmax, one thread per query row: read S_j from TMEM, apply the mask,
//                update the running max m and sum l (page "告别OOM和训练慢…" §2.2), write
//                P_j = exp2(s*scale*log2e - m) in bf16 back to TMEM, rescale O when m grew
//                by more than 2^8 (exact: O and l carry the same stale m), and at the end
//                write O / l and LSE = ln2 * (m + log2 l).
//
// S_{j+1} is computed by the tensor core while the softmax works on S_j.
#pragma once

#include <cuda_bf16.h>

#include "sm100.cuh"
#include "tiles.cuh"

namespace fa {

struct FwdArgs {
  __nv_bfloat16* o;
  float* lse;
  int N;
  int n_qtiles;
  float scale_log2;  // scale * log2(e)
  int left;
  int right;
};

template <int D>
struct FwdCfg {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static constexpr int kTile = kBlock * D * 2;  // bytes of a 128 x D bf16 tile
  static constexpr int kRegions = D / 64;       // 128-byte-wide column regions per tile
  static constexpr int kRegionBytes = kBlock * 128;
  static constexpr int kStages = (D == 64) ? 4 : 2;
  // shared memory map (offsets from a 1024-aligned base)
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTile;
  static constexpr int kV = kK + kStages * kTile;
  static constexpr int kBar = kV + kStages * kTile;
  // barrier slots
  static constexpr int bQFull = 0;
  static constexpr int bKFull = 1;
  static constexpr int bKEmpty = bKFull + kStages;
  static constexpr int bVFull = bKEmpty + kStages;
  static constexpr int bVEmpty = bVFull + kStages;
  static constexpr int bSFull = bVEmpty + kStages;  // two: one per S buffer
  static constexpr int bPFull = bSFull + 2;
  static constexpr int bODone = bPFull + 1;
  static constexpr int bMmaFin = bODone + 1;
  static constexpr int kNumBars = bMmaFin + 1;
  static constexpr int kMisc = kBar + kNumBars * 8;  // TMEM base address, abort flag
  static constexpr int kSmemBytes = kMisc + 16 + 1024;
  // tensor memory columns (128 lanes each)
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t tS0 = 0;
  static constexpr uint32_t tS1 = 128;
  static constexpr uint32_t tO = 256;
  static constexpr uint32_t tP = 256 + D;  // 64 columns: 128 bf16 per row
  static constexpr int kThreads = 192;
};

template <int D>
__global__ void __launch_bounds__(192, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdArgs a) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int m = a.n_qtiles - 1 - (int)blockIdx.x;  // within a head, longest causal rows first
  const Mask mk{a.N, a.left, a.right};
  int j_lo, j_hi;
  kv_tiles_for_q_tile(m, mk, j_lo, j_hi);
  const int n_it = j_hi - j_lo + 1;

  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMisc + 4);
  auto bar = [&](int i) -> uint32_t { return sb + C::kBar + 8u * i; };

  if (threadIdx.x == 0) {
    mbar_init(bar(C::bQFull), 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar(C::bKFull + s), 1);
      mbar_init(bar(C::bKEmpty + s), 1);
      mbar_init(bar(C::bVFull + s), 1);
      mbar_init(bar(C::bVEmpty + s), 1);
    }
    mbar_init(bar(C::bSFull + 0), 1);
    mbar_init(bar(C::bSFull + 1), 1);
    mbar_init(bar(C::bPFull), 128);
    mbar_init(bar(C::bODone), 1);
    mbar_init(bar(C::bMmaFin), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 5) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_map(&tmQ);
      tma_prefetch_map(&tmK);
      tma_prefetch_map(&tmV);
      mbar_arrive_expect_tx(bar(C::bQFull), C::kTile);
      for (int r = 0; r < C::kRegions; ++r)
        tma_load_3d(sb + C::kQ + r * C::kRegionBytes, &tmQ, bar(C::bQFull), r * 64, m * kBlock,
                    bh);
      int nk = 0, nv = 0;  // loads issued
      for (int it = 0; it < n_it; ++it) {
        const int j = j_lo + it;
        const int s = it % C::kStages;
        const uint32_t ph = (it / C::kStages) & 1;
        if (!mbar_wait(bar(C::bKEmpty + s), ph ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(C::bKFull + s), C::kTile);
        for (int r = 0; r < C::kRegions; ++r)
          tma_load_3d(sb + C::kK + s * C::kTile + r * C::kRegionBytes, &tmK, bar(C::bKFull + s),
                      r * 64, j * kBlock, bh);
        ++nk;
        if (!mbar_wait(bar(C::bVEmpty + s), ph ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(C::bVFull + s), C::kTile);
        for (int r = 0; r < C::kRegions; ++r)
          tma_load_3d(sb + C::kV + s * C::kTile + r * C::kRegionBytes, &tmV, bar(C::bVFull + s),
                      r * 64, j * kBlock, bh);
        ++nv;
      }
      // Drain: every copy issued must have landed before the CTA may exit.
      mbar_wait(bar(C::bQFull), 0, nullptr);
      for (int s = 0; s < C::kStages; ++s) {
        if (nk > s) {
          const int last = s + C::kStages * ((nk - 1 - s) / C::kStages);
          mbar_wait(bar(C::bKFull + s), (last / C::kStages) & 1, nullptr);
        }
        if (nv > s) {
          const int last = s + C::kStages * ((nv - 1 - s) / C::kStages);
          mbar_wait(bar(C::bVFull + s), (last / C::kStages) & 1, nullptr);
        }
      }
    }
    __syncwarp();
  } else if (warp == 4) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idO = idesc_bf16_f32(128, D, false, true);
      bool ok = mbar_wait(bar(C::bQFull), 0, abort_flag);
      tc_fence_after();
      for (int it = 0; ok && it <= n_it; ++it) {
        if (it < n_it) {
          const int s = it % C::kStages;
          if (!mbar_wait(bar(C::bKFull + s), (it / C::kStages) & 1, abort_flag)) break;
          tc_fence_after();
          const uint32_t dS = tmem + ((it & 1) ? C::tS1 : C::tS0);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::kRegionBytes + (kk & 3) * 32;
            mma_ss(dS, sdesc_sw128(sb + C::kQ + off, 16, 1024),
                   sdesc_sw128(sb + C::kK + s * C::kTile + off, 16, 1024), idS, kk > 0);
          }
          tc_commit(bar(C::bKEmpty + s));
          tc_commit(bar(C::bSFull + (it & 1)));
        }
        if (it > 0) {
          const int jt = it - 1;
          const int s = jt % C::kStages;
          if (!mbar_wait(bar(C::bPFull), jt & 1, abort_flag)) break;
          if (!mbar_wait(bar(C::bVFull + s), (jt / C::kStages) & 1, abort_flag)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kBlock / 16; ++kk) {
            mma_ts(tmem + C::tO, tmem + C::tP + kk * 8,
                   sdesc_sw128(sb + C::kV + s * C::kTile + kk * 2048, C::kRegionBytes, 1024), idO,
                   (jt > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(bar(C::bVEmpty + s));
          tc_commit(bar(C::bODone));
        }
      }
      // Wait for every MMA issued so far before the CTA may release tensor memory.
      tc_commit(bar(C::bMmaFin));
      mbar_wait(bar(C::bMmaFin), 0, nullptr);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax, warps 0..3
    const int t = threadIdx.x;  // query row within the tile == TMEM lane
    const int row = m * kBlock + t;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const float sl2 = a.scale_log2;
    float m_run = -INFINITY;  // running max of scale*log2e*s (the m that P and O carry)
    float l_run = 0.f;        // running sum of P
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int j = j_lo + it;
      if (!mbar_wait_warp(bar(C::bSFull + (it & 1)), (it >> 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tS = tmem + lane_base + ((it & 1) ? C::tS1 : C::tS0);
      uint32_t u[4][32];
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_ld32(tS + 32 * q, u[q]);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 4; ++q) reg_fence(u[q]);
      float x[128];
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int c = 0; c < 32; ++c) x[32 * q + c] = __uint_as_float(u[q][c]);
      if (!tile_all_visible(m, j, mk)) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (!is_visible(row, j * kBlock + c, mk)) x[c] = -INFINITY;
      }
      // row max as 8 independent chains folded by a tree (keeps the FMNMX pipe busy)
      float mx8[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) mx8[c] = fmaxf(x[c], x[c + 8]);
#pragma unroll
      for (int c = 16; c < 128; c += 8)
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = fmaxf(mx8[e], x[c + e]);
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      const float m_new = fmaxf(m_run, mx * sl2);
      const bool grow = m_new > m_run + 8.0f;
      float alpha = 1.f;
      if (grow) {
        alpha = ex2(m_run - m_new);
        m_run = m_new;
        l_run *= alpha;
      }
      const float mb = (m_run == -INFINITY) ? 0.f : m_run;
      uint32_t pk[64];
      float ls8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float p0 = ex2(fmaf(x[2 * c], sl2, -mb));
        const float p1 = ex2(fmaf(x[2 * c + 1], sl2, -mb));
        ls8[c & 7] += p0 + p1;
        pk[c] = pack_bf16x2(p0, p1);
      }
      l_run += ((ls8[0] + ls8[1]) + (ls8[2] + ls8[3])) + ((ls8[4] + ls8[5]) + (ls8[6] + ls8[7]));
      if (it > 0) {
        // O and the P buffer are busy until P_{j-1} V_{j-1} has finished.
        if (!mbar_wait_warp(bar(C::bODone), (it - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
          for (int q = 0; q < D / 32; ++q) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_base + C::tO + 32 * q, o);
            tmem_wait_ld();
            reg_fence(o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(tmem + lane_base + C::tO + 32 * q, o);
          }
        }
      }
      tmem_st32(tmem + lane_base + C::tP, pk);
      tmem_st32(tmem + lane_base + C::tP + 32, pk + 32);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(C::bPFull));
    }
    if (ok) ok = mbar_wait_warp(bar(C::bODone), (n_it - 1) & 1, abort_flag);
    if (ok) {
      tc_fence_after();
      const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
      __nv_bfloat16* orow = a.o + ((size_t)bh * a.N + row) * D;
#pragma unroll
      for (int q = 0; q < D / 32; ++q) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + C::tO + 32 * q, o);
        tmem_wait_ld();
        reg_fence(o);
        uint32_t w[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          w[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * inv_l, __uint_as_float(o[2 * c + 1]) * inv_l);
        if (row < a.N) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            st_global_v4(orow + 32 * q + 8 * v4, w[4 * v4], w[4 * v4 + 1], w[4 * v4 + 2],
                         w[4 * v4 + 3]);
        }
      }
      if (row < a.N)
        a.lse[(size_t)bh * a.N + row] =
            (l_run > 0.f) ? (m_run + log2f(l_run)) * 0.69314718055994531f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace fa
