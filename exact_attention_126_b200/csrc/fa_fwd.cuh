// fa_fwd.cuh - fused attention forward for sm_100a.
//
// Each persistent CTA takes work items of one 128-row query tile of one (batch, head) and
// walks the key/value tiles the tile can see (page "Flash Attention 3.7 核心原理与实战" §3.1:
// load a Q block, iterate over the K, V blocks; page "告别OOM和训练慢…(含A100环境配置)" §2.1
// tiling). Roles:
//
//   warp 17      TMA producer: Q per item, then K_j and V_j through a ring of shared-memory
//                stages (128-byte swizzle), guarded by full/empty mbarriers.
//   warp 16      MMA issuer (one thread): S_j = Q K_j^T into one of two TMEM buffers, so that
//                S_{j+1} is computed while the softmax works on S_j; then, once P_j is
//                published, O += P_j V_j with P_j read from TMEM.
//   warps 0..15  softmax, four warpgroups that split every score row by columns: thread
//                (h, r) owns keys 32h..32h+31 of query row r (four warps per SM
//                sub-partition hide each other's latencies). They exchange their partial
//                row maxima through shared memory, update the running max m and sum l
//                (page "告别OOM和训练慢…" §2.2), write their part of P_j =
//                exp2(s*scale*log2e - m) in bf16 to TMEM, rescale their quarter of O when m
//                grew by more than 2^8 (exact: O and l carry the same stale m), and at the
//                end of the item write their quarter of O / l (and LSE = ln2 * (m + log2 l)).
//
// TMEM: S0, S1 (128 columns each), O (head_dim columns), P (64 columns).
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
  int n_items;        // BH * n_qtiles
  int longest_first;  // masked problems: chunks of `group` heads, longest items first
  int group;
  float scale_log2;   // scale * log2(e)
  int left;
  int right;
  int fault;          // test hook: 1 = the producer never loads V (waits for it run out)
};

template <int D>
struct FwdCfg {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static constexpr int kTile = kBlock * D * 2;  // bytes of a 128 x D bf16 tile
  static constexpr int kRegions = D / 64;       // 128-byte-wide column regions per tile
  static constexpr int kRegionBytes = kBlock * 128;
  static constexpr int kStages = (D == 64) ? 4 : 2;
  // shared memory map (offsets from a 1024-aligned base)
  static constexpr int kQ = 0;                        // + (item & 1) * kTile
  static constexpr int kK = kQ + 2 * kTile;           // + s * kTile
  static constexpr int kV = kK + kStages * kTile;     // + s * kTile
  static constexpr int kGroups = 4;                   // softmax warpgroups per row
  static constexpr int kCols = kBlock / kGroups;      // score columns per thread
  static constexpr int kOCols = D / kGroups;          // output columns per thread
  static constexpr int kSoftmax = 128 * kGroups;      // softmax threads
  static constexpr int kRed = kV + kStages * kTile;   // [2 slots][kGroups][128 rows] fp32
  static constexpr int kBar = kRed + 2 * kGroups * kBlock * 4;
  // barrier slots
  static constexpr int bQFull = 0;                  // + (item & 1)
  static constexpr int bQEmpty = 2;                 // + (item & 1)
  static constexpr int bKFull = 4;
  static constexpr int bKEmpty = bKFull + kStages;
  static constexpr int bVFull = bKEmpty + kStages;
  static constexpr int bVEmpty = bVFull + kStages;
  static constexpr int bSFull = bVEmpty + kStages;  // + buffer
  static constexpr int bSFree = bSFull + 2;         // + buffer
  static constexpr int bRed = bSFree + 2;           // + slot
  static constexpr int bPFull = bRed + 2;
  static constexpr int bODone = bPFull + 1;
  static constexpr int bOFree = bODone + 1;
  static constexpr int bMmaFin = bOFree + 1;
  static constexpr int kNumBars = bMmaFin + 1;
  static constexpr int kMisc = kBar + kNumBars * 8;  // TMEM base address (+0), abort flag (+4)
  static constexpr int kSmemBytes = kMisc + 16 + 1024;
  // tensor memory columns (128 lanes each)
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t tS0 = 0;
  static constexpr uint32_t tO = 256;
  static constexpr uint32_t tP = 256 + D;
  static constexpr int kThreads = kSoftmax + 64;  // softmax warps, MMA warp, producer warp
  static constexpr int kWarpMma = 4 * kGroups;
  static constexpr int kWarpProducer = 4 * kGroups + 1;
};

struct FwdItem {
  int bh;
  int m;   // query tile
  int lo;  // key tiles [lo, hi] it sees
  int hi;
};

__device__ __forceinline__ FwdItem fwd_item(int k, const FwdArgs& a) {
  FwdItem it;
  if (a.longest_first) {
    chunked_item(k, a.BH, a.n_qtiles, a.group, false, it.bh, it.m);
  } else {
    it.bh = k / a.n_qtiles;
    it.m = k % a.n_qtiles;
  }
  const Mask mk{a.N, a.left, a.right};
  kv_tiles_for_q_tile(it.m, mk, it.lo, it.hi);
  return it;
}

template <int D>
__global__ void __launch_bounds__(FwdCfg<D>::kThreads, 1)
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
  float* red = reinterpret_cast<float*>(smem + C::kRed);
  auto bar = [&](int i) -> uint32_t { return sb + C::kBar + 8u * i; };

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(C::bQFull + b), 1);
      mbar_init(bar(C::bQEmpty + b), 1);
    }
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar(C::bKFull + s), 1);
      mbar_init(bar(C::bKEmpty + s), 1);
      mbar_init(bar(C::bVFull + s), 1);
      mbar_init(bar(C::bVEmpty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(C::bSFull + b), 1);
      mbar_init(bar(C::bSFree + b), C::kSoftmax / 32);
      mbar_init(bar(C::bRed + b), C::kSoftmax / 32);
    }
    mbar_init(bar(C::bPFull), C::kSoftmax / 32);
    mbar_init(bar(C::bODone), 1);
    mbar_init(bar(C::bOFree), C::kSoftmax / 32);
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
        // two Q buffers: the next item's Q streams in while this one is being processed
        const int qb = n_items_done & 1;
        if (!mbar_wait(bar(C::bQEmpty + qb), ((n_items_done >> 1) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(C::bQFull + qb), C::kTile);
        for (int r = 0; r < C::kRegions; ++r)
          tma_load_3d(sb + C::kQ + qb * C::kTile + r * C::kRegionBytes, &tmQ, bar(C::bQFull + qb),
                      r * 64, it.m * kBlock, it.bh);
        ++n_items_done;
        for (int j = it.lo; j <= it.hi; ++j) {
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
          if (a.fault == 1) continue;
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
      for (int n = (n_items_done > 2 ? n_items_done - 2 : 0); n < n_items_done; ++n)
        mbar_wait(bar(C::bQFull + (n & 1)), (n >> 1) & 1, nullptr);
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
  } else if (warp == C::kWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idO = idesc_bf16_f32(128, D, false, true);
      int n_items_done = 0;
      int kc = 0, vc = 0;  // ring positions consumed
      int ns = 0, npv = 0; // S and P V products issued (all items)
      bool ok = true;

      // S_j = Q K_j^T into buffer ns & 1; after the item's last S, its Q may be replaced.
      auto issue_s = [&](int j, int hi, int qb) -> bool {
        const int s = kc % C::kStages;
        const int b = ns & 1;
        if (!mbar_wait(bar(C::bKFull + s), (kc / C::kStages) & 1, abort_flag)) return false;
        ++kc;
        // buffer b is free once every softmax warpgroup has read the S it held before
        if (ns >= 2 && !mbar_wait(bar(C::bSFree + b), ((ns >> 1) - 1) & 1, abort_flag))
          return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kRegionBytes + (kk & 3) * 32;
          mma_ss(tmem + C::tS0 + 128u * b, sdesc_sw128(sb + C::kQ + qb * C::kTile + off, 16, 1024),
                 sdesc_sw128(sb + C::kK + s * C::kTile + off, 16, 1024), idS, kk > 0);
        }
        tc_commit(bar(C::bKEmpty + s));
        tc_commit(bar(C::bSFull + b));
        if (j == hi) tc_commit(bar(C::bQEmpty + qb));
        ++ns;
        return true;
      };
      // O += P_j V_j
      auto issue_pv = [&](bool first, bool wait_o_free) -> bool {
        const int s = vc % C::kStages;
        if (!mbar_wait(bar(C::bVFull + s), (vc / C::kStages) & 1, abort_flag)) return false;
        ++vc;
        if (!mbar_wait(bar(C::bPFull), npv & 1, abort_flag)) return false;
        // the first product of an item overwrites O: the previous epilogue must have read it
        if (wait_o_free && !mbar_wait(bar(C::bOFree), (n_items_done - 2) & 1, abort_flag))
          return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBlock / 16; ++kk)
          mma_ts(tmem + C::tO, tmem + C::tP + kk * 8,
                 sdesc_sw128(sb + C::kV + s * C::kTile + kk * 2048, C::kRegionBytes, 1024), idO,
                 (!first || kk > 0) ? 1u : 0u);
        tc_commit(bar(C::bVEmpty + s));
        tc_commit(bar(C::bODone));
        ++npv;
        return true;
      };

      for (int k = blockIdx.x; ok && k < a.n_items; k += gridDim.x) {
        const FwdItem it = fwd_item(k, a);
        const int qb = n_items_done & 1;
        if (!mbar_wait(bar(C::bQFull + qb), (n_items_done >> 1) & 1, abort_flag)) break;
        ++n_items_done;
        ok = issue_s(it.lo, it.hi, qb);
        for (int j = it.lo; ok && j <= it.hi; ++j) {
          if (j + 1 <= it.hi) ok = issue_s(j + 1, it.hi, qb);
          if (ok) ok = issue_pv(j == it.lo, j == it.lo && n_items_done > 1);
        }
      }
      // Wait for every MMA issued so far before the CTA may release tensor memory.
      tc_commit(bar(C::bMmaFin));
      mbar_wait(bar(C::bMmaFin), 0, nullptr);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax warps
    constexpr int G = C::kGroups, NC = C::kCols, NO = C::kOCols;
    const int h = warp >> 2;                     // column group: keys NC*h .. NC*h+NC-1
    const int r = threadIdx.x & 127;             // query row in the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tO = tmem + lane_base + C::tO + NO * h;
    const uint32_t tP = tmem + lane_base + C::tP + (NC / 2) * h;
    const float sl2 = a.scale_log2;
    int ns = 0;  // S tiles consumed (all items)
    int nx = 0;  // row-statistic exchanges between the warpgroups
    bool ok = true;

    // Shares a per-row value with the other warpgroups; `all` gets the G values of the row.
    auto exchange = [&](float v, float (&all)[G]) -> bool {
      float* slot = red + (nx & 1) * (G * 128);
      slot[h * 128 + r] = v;
      mbar_arrive_warp(bar(C::bRed + (nx & 1)));
      if (!mbar_wait_warp(bar(C::bRed + (nx & 1)), (nx >> 1) & 1, abort_flag)) return false;
#pragma unroll
      for (int g = 0; g < G; ++g) all[g] = slot[g * 128 + r];
      ++nx;
      return true;
    };
    // NO accumulator columns of O: fp32 in, scaled by `mul`, back to TMEM (rescale)
    auto scale_o = [&](float mul) {
#pragma unroll
      for (int q = 0; q < NO / 16; ++q) {
        uint32_t o[16];
        tmem_ld16(tO + 16 * q, o);
        tmem_wait_ld();
        reg_fence(o);
#pragma unroll
        for (int c = 0; c < 16; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * mul);
        tmem_st16(tO + 16 * q, o);
      }
    };

    for (int k = blockIdx.x; ok && k < a.n_items; k += gridDim.x) {
      const FwdItem it = fwd_item(k, a);
      const int row = it.m * kBlock + r;
      float m_run = -INFINITY;  // running max of scale*log2e*s (the m that P and O carry)
      float l_run = 0.f;        // this group's running sum of P
      for (int j = it.lo; j <= it.hi; ++j) {
        const int b = ns & 1;
        if (!mbar_wait_warp(bar(C::bSFull + b), (ns >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t u[32];
        tmem_ld32(tmem + lane_base + C::tS0 + 128u * b + NC * h, u);
        tmem_wait_ld();
        reg_fence(u);
        // this group's part of S_j is in registers: the tensor core may reuse the buffer
        tc_fence_before();
        mbar_arrive_warp(bar(C::bSFree + b));
        float x[NC];
#pragma unroll
        for (int c = 0; c < NC; ++c) x[c] = __uint_as_float(u[c]);
        if (!tile_all_visible(it.m, j, mk)) {
#pragma unroll
          for (int c = 0; c < NC; ++c)
            if (!is_visible(row, j * kBlock + NC * h + c, mk)) x[c] = -INFINITY;
        }
        float mx8[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) mx8[c] = fmaxf(x[c], x[c + 8]);
#pragma unroll
        for (int c = 16; c < NC; c += 8)
#pragma unroll
          for (int e = 0; e < 8; ++e) mx8[e] = fmaxf(mx8[e], x[c + e]);
        float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                         fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        float mx_all[G];
        if (!exchange(mx, mx_all)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int g = 0; g < G; ++g) mx = fmaxf(mx, mx_all[g]);
        const float m_new = fmaxf(m_run, mx * sl2);
        const bool grow = m_new > m_run + 8.0f;
        float alpha = 1.f;
        if (grow) {
          alpha = ex2(m_run - m_new);
          m_run = m_new;
          l_run *= alpha;
        }
        const float mb = (m_run == -INFINITY) ? 0.f : m_run;
        // this group's part of P = exp2(s*scale*log2e - m), packed to bf16 pairs
        float ls4[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t pk[NC / 2];
#pragma unroll
        for (int c = 0; c < NC / 2; ++c) {
          const float p0 = ex2(fmaf(x[2 * c], sl2, -mb));
          const float p1 = ex2(fmaf(x[2 * c + 1], sl2, -mb));
          ls4[c & 3] += p0 + p1;
          pk[c] = pack_bf16x2(p0, p1);
        }
        l_run += (ls4[0] + ls4[1]) + (ls4[2] + ls4[3]);
        if (j > it.lo) {
          // O and the P buffer are busy until P_{j-1} V_{j-1} has finished
          if (!mbar_wait_warp(bar(C::bODone), (ns - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        tmem_st16(tP, pk);
        // rescale this group's part of O before P_j V_j accumulates into it (that waits
        // for p_full)
        if (j > it.lo && __any_sync(0xffffffffu, grow)) scale_o(alpha);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive_warp(bar(C::bPFull));
        ++ns;
      }
      if (!ok) break;
      // epilogue of the item: l of the whole row, then this group's part of O / l, and LSE
      float l_all[G];
      if (!exchange(l_run, l_all)) {
        ok = false;
        break;
      }
      float l_row = 0.f;
#pragma unroll
      for (int g = 0; g < G; ++g) l_row += l_all[g];
      if (!mbar_wait_warp(bar(C::bODone), (ns - 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float inv_l = (l_row > 0.f) ? 1.f / l_row : 0.f;
      __nv_bfloat16* orow = a.o + ((size_t)it.bh * a.N + row) * D + NO * h;
#pragma unroll
      for (int q = 0; q < NO / 16; ++q) {
        uint32_t o[16];
        tmem_ld16(tO + 16 * q, o);
        tmem_wait_ld();
        reg_fence(o);
        uint32_t w[8];
#pragma unroll
        for (int c = 0; c < 8; ++c)
          w[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * inv_l, __uint_as_float(o[2 * c + 1]) * inv_l);
        if (row < a.N) {
          st_global_v4(orow + 16 * q, w[0], w[1], w[2], w[3]);
          st_global_v4(orow + 16 * q + 8, w[4], w[5], w[6], w[7]);
        }
      }
      // O has been read: the next item's first P V may overwrite it
      tc_fence_before();
      mbar_arrive_warp(bar(C::bOFree));
      if (h == 0 && row < a.N)
        a.lse[(size_t)it.bh * a.N + row] =
            (l_row > 0.f) ? (m_run + log2f(l_row)) * 0.69314718055994531f : -INFINITY;
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
