// fa_fwd.cuh - fused attention forward for sm_100a.
//
// Each persistent CTA takes work items of two adjacent 128-row query tiles (A and B) of
// one (batch, head) and walks the key/value tiles either of them can see (page "Flash
// Attention 3.7 核心原理与实战" §3.1: load a Q block, iterate over the K, V blocks; page
// "告别OOM和训练慢…(含A100环境配置)" §2.1 tiling). Both query tiles share every K/V tile
// that is loaded. Roles:
//
//   warp 9       TMA producer: Q_A and Q_B per item, then K_j and V_j through a ring of
//                shared-memory stages (128-byte swizzle), guarded by full/empty mbarriers.
//   warps 8, 10  MMA issuers, one thread each, one per query tile t in {A, B}:
//                S_t = Q_t K_j^T into TMEM, then O_t += P_t V_j with P_t read from TMEM.
//                Two issuers let the tensor core interleave the tiles' products without
//                either tile waiting on the other's softmax.
//   warps 0..3   softmax of tile A, warps 4..7 softmax of tile B, one thread per query
//                row: read S_t from TMEM (and release the buffer at once, so the next
//                S_t is computed while this one is exponentiated), apply the mask, update
//                the running max m and sum l (page "告别OOM和训练慢…" §2.2), write
//                P_t = exp2(s*scale*log2e - m) in bf16 to TMEM, rescale O_t when m grew by
//                more than 2^8 (exact: O and l carry the same stale m), and at the end of
//                the item write O_t / l and LSE = ln2 * (m + log2 l).
//
// For head_dim 128 the four fp32 accumulators S_A, S_B, O_A, O_B fill the 512 TMEM
// columns, so P_t is written over the first half of S_t and the next S_t waits until
// P_t V_j has finished; for head_dim 64 P_t has columns of its own.
#pragma once

#include <cuda_bf16.h>

#include "sm100.cuh"
#include "tiles.cuh"

namespace fa {

struct FwdArgs {
  __nv_bfloat16* o;
  float* lse;
  int N;
  int BH;
  int n_qtiles;
  int n_pairs;       // work items per (batch, head): ceil(n_qtiles / 2)
  int n_items;       // BH * n_pairs
  int longest_first; // order items by decreasing length (masked problems)
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
  static constexpr int kQ = 0;                        // + t * kTile
  static constexpr int kK = kQ + 2 * kTile;           // + s * kTile
  static constexpr int kV = kK + kStages * kTile;     // + s * kTile
  static constexpr int kBar = kV + kStages * kTile;
  // barrier slots
  static constexpr int bQFull = 0;
  static constexpr int bQEmpty = 1;
  static constexpr int bKFull = 2;
  static constexpr int bKEmpty = bKFull + kStages;
  static constexpr int bVFull = bKEmpty + kStages;
  static constexpr int bVEmpty = bVFull + kStages;
  static constexpr int bSFull = bVEmpty + kStages;  // + t
  static constexpr int bSFree = bSFull + 2;         // + t
  static constexpr int bPFull = bSFree + 2;         // + t
  static constexpr int bODone = bPFull + 2;         // + t
  static constexpr int bOFree = bODone + 2;         // + t
  static constexpr int bMmaFin = bOFree + 2;        // + t
  static constexpr int kNumBars = bMmaFin + 2;
  // TMEM base address (+0), abort flag (+4), one exp lock per SM sub-partition (+16..+31)
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kSmemBytes = kMisc + 32 + 1024;
  // tensor memory columns (128 lanes each)
  static constexpr uint32_t kTmemCols = 512;
  static constexpr bool kAliasP = (D == 128);
  __host__ __device__ static constexpr uint32_t tS(int t) { return 128u * t; }
  __host__ __device__ static constexpr uint32_t tO(int t) { return 256u + D * t; }
  __host__ __device__ static constexpr uint32_t tP(int t) {
    return kAliasP ? tS(t) : 256u + 2 * D + 64u * t;
  }
  // 12 warps = 3 warpgroups: two softmax warpgroups and one for the producer and the
  // two MMA issuers. The CTA is launched with kLaunchRegs registers per thread (checked
  // on the host); the softmax warpgroups then take kSoftmaxRegs and the third
  // warpgroup keeps kOtherRegs: 2*128*200 + 128*96 = 63488 <= 384*168 = 64512.
  static constexpr int kThreads = 384;
  static constexpr int kLaunchRegs = 168;
  static constexpr int kSoftmaxRegs = 200;
  static constexpr int kOtherRegs = 96;
  static_assert(2 * 128 * kSoftmaxRegs + 128 * kOtherRegs <= kThreads * kLaunchRegs,
                "register split exceeds the launch allocation");
  static constexpr int kWarpProducer = 9;
  static constexpr int kWarpMmaA = 8;
  static constexpr int kWarpMmaB = 10;
};

struct FwdItem {
  int bh;
  int m[2];    // query tile index of A and B
  int lo[2];   // key tiles each query tile sees, [lo, hi] (empty when lo > hi)
  int hi[2];
  int ulo;     // union range
  int uhi;
};

__device__ __forceinline__ FwdItem fwd_item(int k, const FwdArgs& a) {
  FwdItem it;
  int p;
  if (a.longest_first) {
    p = a.n_pairs - 1 - k / a.BH;
    it.bh = k % a.BH;
  } else {
    it.bh = k / a.n_pairs;
    p = k % a.n_pairs;
  }
  const Mask mk{a.N, a.left, a.right};
  it.ulo = 1 << 30;
  it.uhi = -1;
  for (int t = 0; t < 2; ++t) {
    it.m[t] = 2 * p + t;
    if (it.m[t] < a.n_qtiles) {
      kv_tiles_for_q_tile(it.m[t], mk, it.lo[t], it.hi[t]);
      it.ulo = min(it.ulo, it.lo[t]);
      it.uhi = max(it.uhi, it.hi[t]);
    } else {
      it.lo[t] = 1;
      it.hi[t] = 0;
    }
  }
  return it;
}

template <int D>
__global__ void __launch_bounds__(384, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdArgs a) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Mask mk{a.N, a.left, a.right};

  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMisc + 4);
  int* exp_lock = reinterpret_cast<int*>(smem + C::kMisc + 16);
  auto bar = [&](int i) -> uint32_t { return sb + C::kBar + 8u * i; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) exp_lock[i] = 0;
    mbar_init(bar(C::bQFull), 1);
    mbar_init(bar(C::bQEmpty), 2);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar(C::bKFull + s), 1);
      mbar_init(bar(C::bKEmpty + s), 2);
      mbar_init(bar(C::bVFull + s), 1);
      mbar_init(bar(C::bVEmpty + s), 2);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(C::bSFull + t), 1);
      mbar_init(bar(C::bSFree + t), 128);
      mbar_init(bar(C::bPFull + t), 128);
      mbar_init(bar(C::bODone + t), 1);
      mbar_init(bar(C::bOFree + t), 128);
      mbar_init(bar(C::bMmaFin + t), 1);
    }
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

  if (warp >= 8) {
  regs_shrink<C::kOtherRegs>();
  if (warp == C::kWarpProducer) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_map(&tmQ);
      tma_prefetch_map(&tmK);
      tma_prefetch_map(&tmV);
      int n_items_done = 0;
      int kc = 0, vc = 0;  // K and V loads issued (ring positions)
      bool ok = true;
      for (int k = blockIdx.x; ok && k < a.n_items; k += gridDim.x) {
        const FwdItem it = fwd_item(k, a);
        if (!mbar_wait(bar(C::bQEmpty), (n_items_done & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(C::bQFull), 2 * C::kTile);
        for (int t = 0; t < 2; ++t)
          for (int r = 0; r < C::kRegions; ++r)
            tma_load_3d(sb + C::kQ + t * C::kTile + r * C::kRegionBytes, &tmQ, bar(C::bQFull),
                        r * 64, it.m[t] * kBlock, it.bh);
        ++n_items_done;
        for (int j = it.ulo; j <= it.uhi; ++j) {
          const int s = kc % C::kStages;
          if (!mbar_wait(bar(C::bKEmpty + s), ((kc / C::kStages) & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(C::bKFull + s), C::kTile);
          for (int r = 0; r < C::kRegions; ++r)
            tma_load_3d(sb + C::kK + s * C::kTile + r * C::kRegionBytes, &tmK, bar(C::bKFull + s),
                        r * 64, j * kBlock, it.bh);
          ++kc;
          if (!mbar_wait(bar(C::bVEmpty + s), ((vc / C::kStages) & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(C::bVFull + s), C::kTile);
          for (int r = 0; r < C::kRegions; ++r)
            tma_load_3d(sb + C::kV + s * C::kTile + r * C::kRegionBytes, &tmV, bar(C::bVFull + s),
                        r * 64, j * kBlock, it.bh);
          ++vc;
        }
      }
      // Drain: every copy issued must have landed before the CTA may exit.
      if (n_items_done > 0) mbar_wait(bar(C::bQFull), (n_items_done - 1) & 1, nullptr);
      for (int s = 0; s < C::kStages; ++s) {
        if (kc > s) {
          const int last = s + C::kStages * ((kc - 1 - s) / C::kStages);
          mbar_wait(bar(C::bKFull + s), (last / C::kStages) & 1, nullptr);
        }
        if (vc > s) {
          const int last = s + C::kStages * ((vc - 1 - s) / C::kStages);
          mbar_wait(bar(C::bVFull + s), (last / C::kStages) & 1, nullptr);
        }
      }
    }
    __syncwarp();
  } else if (warp == C::kWarpMmaA || warp == C::kWarpMmaB) {
    // ------------------------------------------------------------------ MMA issuer of tile t
    const int t = (warp == C::kWarpMmaA) ? 0 : 1;
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idO = idesc_bf16_f32(128, D, false, true);
      const uint32_t dS = tmem + C::tS(t);
      const uint32_t dO = tmem + C::tO(t);
      const uint32_t aP = tmem + C::tP(t);
      const uint32_t sQ = sb + C::kQ + t * C::kTile;
      int n_items_done = 0;
      int kc = 0, vc = 0;     // ring positions consumed
      int ns = 0, npv = 0;    // S_t and P_t V products issued so far (all items)
      int n_epi = 0;          // items of this tile whose O went through the epilogue
      bool ok = true;

      // S_t(j) for union index j (or a pass-through arrive when tile t skips j)
      auto do_s = [&](int lo, int hi, int j) -> bool {
        const int s = kc % C::kStages;
        if (!mbar_wait(bar(C::bKFull + s), (kc / C::kStages) & 1, abort_flag)) return false;
        ++kc;
        if (j < lo || j > hi) {
          mbar_arrive(bar(C::bKEmpty + s));
          return true;
        }
        // the S_t buffer is free once the softmax has read the previous S_t (and, when
        // P_t lives in it, once the previous P_t V has finished)
        if (ns > 0 && !mbar_wait(bar(C::bSFree + t), (ns - 1) & 1, abort_flag)) return false;
        if (C::kAliasP && npv > 0 && !mbar_wait(bar(C::bODone + t), (npv - 1) & 1, abort_flag))
          return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kRegionBytes + (kk & 3) * 32;
          mma_ss(dS, sdesc_sw128(sQ + off, 16, 1024),
                 sdesc_sw128(sb + C::kK + s * C::kTile + off, 16, 1024), idS, kk > 0);
        }
        tc_commit(bar(C::bKEmpty + s));
        tc_commit(bar(C::bSFull + t));
        // after this tile's last S of the item, Q_t may be replaced by the next item's
        if (j == hi) tc_commit(bar(C::bQEmpty));
        ++ns;
        return true;
      };
      // O_t += P_t V_j for union index j (or a pass-through arrive)
      auto do_pv = [&](int lo, int hi, int j) -> bool {
        const int s = vc % C::kStages;
        if (!mbar_wait(bar(C::bVFull + s), (vc / C::kStages) & 1, abort_flag)) return false;
        ++vc;
        if (j < lo || j > hi) {
          mbar_arrive(bar(C::bVEmpty + s));
          return true;
        }
        if (!mbar_wait(bar(C::bPFull + t), npv & 1, abort_flag)) return false;
        const bool first = (j == lo);
        // the first product of an item overwrites O_t: the previous item's epilogue must
        // have read it
        if (first && n_epi > 0 && !mbar_wait(bar(C::bOFree + t), (n_epi - 1) & 1, abort_flag))
          return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBlock / 16; ++kk)
          mma_ts(dO, aP + kk * 8,
                 sdesc_sw128(sb + C::kV + s * C::kTile + kk * 2048, C::kRegionBytes, 1024), idO,
                 (!first || kk > 0) ? 1u : 0u);
        tc_commit(bar(C::bVEmpty + s));
        tc_commit(bar(C::bODone + t));
        ++npv;
        return true;
      };

      for (int k = blockIdx.x; ok && k < a.n_items; k += gridDim.x) {
        const FwdItem it = fwd_item(k, a);
        const int lo = t ? it.lo[1] : it.lo[0];
        const int hi = t ? it.hi[1] : it.hi[0];
        const bool present = lo <= hi;
        if (!mbar_wait(bar(C::bQFull), n_items_done & 1, abort_flag)) break;
        ++n_items_done;
        if (!present) mbar_arrive(bar(C::bQEmpty));  // this tile reads nothing of Q_t
        if (C::kAliasP) {
          // P_t sits in S_t: the next S_t must follow P_t V
          for (int j = it.ulo; ok && j <= it.uhi; ++j) ok = do_s(lo, hi, j) && do_pv(lo, hi, j);
        } else {
          // S_t(j+1) is issued before P_t(j) V_j, so it overlaps the softmax of S_t(j)
          ok = do_s(lo, hi, it.ulo);
          for (int j = it.ulo; ok && j <= it.uhi; ++j) {
            if (j + 1 <= it.uhi) ok = do_s(lo, hi, j + 1);
            if (ok) ok = do_pv(lo, hi, j);
          }
        }
        if (!ok) break;
        if (present) ++n_epi;
      }
      // Wait for every MMA issued so far before the CTA may release tensor memory.
      tc_commit(bar(C::bMmaFin + t));
      mbar_wait(bar(C::bMmaFin + t), 0, nullptr);
    }
    __syncwarp();
  }
  } else {
    regs_grow<C::kSoftmaxRegs>();
    // ------------------------------------------------------------------ softmax of tile t
    const int t = warp >> 2;
    const int row_in_tile = threadIdx.x & 127;  // == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + C::tS(t);
    const uint32_t tO = tmem + lane_base + C::tO(t);
    const uint32_t tP = tmem + lane_base + C::tP(t);
    const float sl2 = a.scale_log2;
    int ns = 0;  // S_t tiles consumed so far (all items) == P_t published
    bool ok = true;
    for (int k = blockIdx.x; ok && k < a.n_items; k += gridDim.x) {
      const FwdItem it = fwd_item(k, a);
      const int lo = t ? it.lo[1] : it.lo[0];
      const int hi = t ? it.hi[1] : it.hi[0];
      if (lo > hi) continue;
      const int m = t ? it.m[1] : it.m[0];
      const int row = m * kBlock + row_in_tile;
      float m_run = -INFINITY;  // running max of scale*log2e*s (the m that P and O carry)
      float l_run = 0.f;        // running sum of P
      for (int j = lo; j <= hi; ++j) {
        if (!mbar_wait_warp(bar(C::bSFull + t), ns & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t u[4][32];
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_ld32(tS + 32 * q, u[q]);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) reg_fence(u[q]);
        // S_t is in registers: the tensor core may overwrite the buffer
        tc_fence_before();
        mbar_arrive(bar(C::bSFree + t));
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
        // row max as 8 independent chains folded by a tree
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
        // The warp of the other tile on this SM sub-partition shares its exp unit. With
        // head_dim 128 (P in S, so each tile's next S waits for its P V) the two tiles
        // take turns, so that one exponentiates while the other's products run; with
        // head_dim 64 the next S is already computed during the exps and turns only add
        // waiting.
        if (C::kAliasP) {
          bool got = true;
          if (lane == 0) got = smem_lock_acquire(exp_lock + (warp & 3), abort_flag);
          if (!__shfl_sync(0xffffffffu, got ? 1 : 0, 0)) {
            ok = false;
            break;
          }
        }
        // P = exp2(s*scale*log2e - m), packed to bf16 pairs as soon as it is formed
        float ls8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        uint32_t pk[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float p0 = ex2(fmaf(x[2 * c], sl2, -mb));
          const float p1 = ex2(fmaf(x[2 * c + 1], sl2, -mb));
          ls8[c & 7] += p0 + p1;
          pk[c] = pack_bf16x2(p0, p1);
        }
        if (C::kAliasP) {
          __syncwarp();
          if (lane == 0) smem_lock_release(exp_lock + (warp & 3));
        }
        l_run += ((ls8[0] + ls8[1]) + (ls8[2] + ls8[3])) + ((ls8[4] + ls8[5]) + (ls8[6] + ls8[7]));
        if (j > lo) {
          // O_t and the P_t buffer are busy until P_t(j-1) V_{j-1} has finished
          if (!mbar_wait_warp(bar(C::bODone + t), (ns - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        tmem_st32(tP, pk);
        tmem_st32(tP + 32, pk + 32);
        // rescale O_t before P_t V_j accumulates into it (that product waits for p_full)
        if (j > lo && __any_sync(0xffffffffu, grow)) {
#pragma unroll
          for (int q = 0; q < D / 32; ++q) {
            uint32_t o[32];
            tmem_ld32(tO + 32 * q, o);
            tmem_wait_ld();
            reg_fence(o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(tO + 32 * q, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(C::bPFull + t));
        ++ns;
      }
      if (!ok) break;
      // epilogue of the item: O_t / l and LSE
      if (!mbar_wait_warp(bar(C::bODone + t), (ns - 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
      __nv_bfloat16* orow = a.o + ((size_t)it.bh * a.N + row) * D;
#pragma unroll
      for (int q = 0; q < D / 32; ++q) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * q, o);
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
      // O_t has been read: the next item's first P_t V may overwrite it
      tc_fence_before();
      mbar_arrive(bar(C::bOFree + t));
      if (row < a.N)
        a.lse[(size_t)it.bh * a.N + row] =
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
