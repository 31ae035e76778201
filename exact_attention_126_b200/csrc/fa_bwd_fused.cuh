// fa_bwd_fused.cuh - attention backward in one pass over key tiles, head_dim 64: dK and dV
// accumulate in tensor memory as in fa_bwd_dkdv_kernel, and each (query tile, key tile)
// pair also computes its share of dQ,
//   dQ_i += scale dS_ij K_j,
// which is added into an fp32 accumulator in device memory by TMA bulk reductions (performed
// at L2, asynchronously to the kernel); fa_bwd_dq_convert_kernel then writes dQ in bf16. The order of those fp32 additions varies
// from run to run, so dQ is reproducible only to fp32 rounding; the three-kernel backward
// (separate dQ pass) stays available for callers that need bit-identical results.
//
// The pages give only the idea (recompute P from the saved normalisation factors: page
// "告别OOM和训练慢…(含A100环境配置)" §2.2; page "PyTorch-CUDA-v2.9镜像中使用FlashAttention提升
// 训练速度", "3. 重计算策略"); the outer loop over key blocks with an inner loop over query
// blocks is the loop order of the first page's §2.1 block sketch.
//
// Per key tile j (item) and visible query tile i (tile t), with thread = key row:
//   S^T = K_j Q_i^T, dP^T = V_j dO_i^T                       (score issuer, warp 16)
//   P^T, dS^T = P^T o (dP^T - delta) in bf16, written to shared memory by the softmax warps
//   dV += P^T dO_i, dK += dS^T Q_i, dQ_t = dS K_j             (gradient issuer, warp 17)
// P^T and dS^T leave tensor memory right after the softmax has loaded S^T and dP^T, so both
// score buffers turn over without waiting for the gradient products. The shared-memory copy
// of dS^T (keys x queries, queries contiguous) is the K-major A operand of dK and, read
// MN-major, the A operand dS of dQ. dQ_t goes to one of two tensor-memory buffers; in the
// middle of tile t+1 (after the exponentials of P^T, by when dQ_t is complete) the softmax
// warps copy it in fp32 into the dS^T buffer, which no product reads any more, and the
// store warp (warp 19) hands it to the TMA unit as a bulk reduce-add into the accumulator;
// the next dS^T is written once that copy has been read. The last tile of an item is
// drained at the item's end.
//
// TMEM: S^T 0..127, dP^T 128..255, dK 256..319, dV 320..383, dQ 384..447 / 448..511.
#pragma once

#include <cuda_bf16.h>

#include "fa_bwd.cuh"
#include "rng.cuh"
#include "sm100.cuh"
#include "tiles.cuh"

namespace fa {

struct FusedCfg {
  static constexpr int D = 64;
  static constexpr int kTile = kBlock * D * 2;       // 16 KB: one 128 x 64 bf16 tile
  static constexpr int kRegionBytes = kBlock * 128;  // one 64-column region of a tile
  static constexpr int kStages0 = 2;                 // Q (+ statistics) ring
  static constexpr int kStages1 = 2;                 // dO ring
  static constexpr int kX = 0;                       // K_j, V_j: + xb * 2 * kTile (2 buffers)
  static constexpr int kY0 = 4 * kTile;              // + s * kTile
  static constexpr int kY1 = kY0 + kStages0 * kTile;
  static constexpr int kP = kY1 + kStages1 * kTile;  // P^T bf16, 128 keys x 128 queries (32 KB)
  static constexpr int kDS = kP + 2 * kRegionBytes;  // dS^T bf16, same layout
  static constexpr int kLse = kDS + 2 * kRegionBytes;  // + s * 512
  static constexpr int kDelta = kLse + kStages0 * 512;
  static constexpr int kBar = kDelta + kStages0 * 512;
  // barriers
  static constexpr int bXFull = 0, bXEmpty = 2;
  static constexpr int bY0Full = 4, bY0Empty = bY0Full + kStages0;
  static constexpr int bY1Full = bY0Empty + kStages0, bY1Empty = bY1Full + kStages1;
  static constexpr int bSFull = bY1Empty + kStages1, bSFree = bSFull + 1;
  static constexpr int bDPFull = bSFree + 1, bDPFree = bDPFull + 1;
  static constexpr int bPFull = bDPFree + 1, bPFree = bPFull + 1;
  static constexpr int bDSFull = bPFree + 1;
  static constexpr int bDQFull = bDSFull + 1;   // + buffer: dQ_t (and dK_t) complete
  static constexpr int bDQFree = bDQFull + 2;   // + buffer: dQ_t loaded by the softmax
  static constexpr int bDQStaged = bDQFree + 2;  // dQ_t copied into the dS^T buffer
  static constexpr int bDQRead = bDQStaged + 1;  // its bulk reduction has read the buffer
  static constexpr int bAccReady = bDQRead + 1, bAccFree = bAccReady + 1;
  static constexpr int bStaged = bAccFree + 1, bMmaFin = bStaged + 1;  // + issuer
  static constexpr int kNumBars = bMmaFin + 2;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kSmemBytes = kMisc + 16 + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t tS = 0, tDP = 128, tDK = 256, tDV = 320, tDQ = 384;  // dQ: + 64 b
  static constexpr int kGroups = 4;               // softmax warpgroups, 32 queries each
  static constexpr int kCols = kBlock / kGroups;
  static constexpr int kSoftmax = 128 * kGroups;
  static constexpr int kThreads = kSoftmax + 128;
  static constexpr int kWarpMma = 16;             // + issuer: 0 = scores, 1 = gradients
  static constexpr int kWarpProducer = 18;
  static constexpr int kWarpStore = 19;
};

// Writes 32 bf16 values (16 packed words, columns col0 .. col0 + 31 of row `row`) into a
// 128-row bf16 matrix in shared memory laid out as two 64-column regions of 128-byte rows
// with the 128-byte swizzle (16-byte chunk c of row r at chunk c ^ (r & 7)): the layout the
// tensor core reads as a K-major operand (rows = M) or an MN-major one (rows = K).
__device__ __forceinline__ void store_row32_bf16(uint32_t base, int row, int col0,
                                                 const uint32_t (&w)[16]) {
  const uint32_t region = base + (uint32_t)(col0 >> 6) * (kBlock * 128) + (uint32_t)row * 128;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int chunk = ((col0 & 63) >> 3) + k;
    st_shared_v4(region + ((uint32_t)(chunk ^ (row & 7)) << 4), w[4 * k], w[4 * k + 1],
                 w[4 * k + 2], w[4 * k + 3]);
  }
}

// Writes 16 fp32 values (columns col0 .. col0 + 15 of row `row`, col0 a multiple of 16) of
// a 128 x 64 fp32 tile held as two 32-column boxes of 128-byte rows with the 128-byte
// swizzle: the layout a TMA transfer of a {32, 128} fp32 box with SWIZZLE_128B reads.
__device__ __forceinline__ void store_row16_f32(uint32_t base, int row, int col0,
                                                const uint32_t (&w)[16]) {
  const uint32_t box = base + (uint32_t)(col0 >> 5) * (kBlock * 128) + (uint32_t)row * 128;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int chunk = ((col0 & 31) >> 2) + k;
    st_shared_v4(box + ((uint32_t)(chunk ^ (row & 7)) << 4), w[4 * k], w[4 * k + 1], w[4 * k + 2],
                 w[4 * k + 3]);
  }
}

// kFeat: kFeatAlibi, kFeatKpad and kFeatDropout as in fa_bwd_dkdv_kernel. tmDQ: the
// (B*H, Np, 64) fp32 accumulator (zeroed by the preprocess step), boxes of 32 columns x
// 128 rows, 128-byte swizzle; it receives dQ / scale (the convert kernel scales).
template <int kFeat = 0>
__global__ void __launch_bounds__(FusedCfg::kThreads, 1)
    fa_bwd_fused_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ CUtensorMap tmdO,
                        const __grid_constant__ CUtensorMap tmdK,
                        const __grid_constant__ CUtensorMap tmdV,
                        const __grid_constant__ CUtensorMap tmDQ, const BwdArgs a) {
  using C = FusedCfg;
  constexpr int D = C::D;
  constexpr bool kAlibi = (kFeat & kFeatAlibi) != 0;
  constexpr bool kKpad = (kFeat & kFeatKpad) != 0;
  constexpr bool kDropout = (kFeat & kFeatDropout) != 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMisc + 4);
  auto bar = [&](int i) -> uint32_t { return sb + C::kBar + 8u * i; };
  constexpr uint32_t kSoftWarps = C::kSoftmax / 32;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(C::bXFull + b), 1);
      mbar_init(bar(C::bXEmpty + b), 1);
      mbar_init(bar(C::bDQFull + b), 1);
      mbar_init(bar(C::bDQFree + b), kSoftWarps);
      mbar_init(bar(C::bMmaFin + b), 1);
    }
    // Q_i (with its statistics) is read by S^T and dK, dO_i by dP^T and dV
    for (int s = 0; s < C::kStages0; ++s) {
      mbar_init(bar(C::bY0Full + s), 1);
      mbar_init(bar(C::bY0Empty + s), 2);
    }
    for (int s = 0; s < C::kStages1; ++s) {
      mbar_init(bar(C::bY1Full + s), 1);
      mbar_init(bar(C::bY1Empty + s), 2);
    }
    mbar_init(bar(C::bSFull), 1);
    mbar_init(bar(C::bSFree), kSoftWarps);
    mbar_init(bar(C::bDPFull), 1);
    mbar_init(bar(C::bDPFree), kSoftWarps);
    mbar_init(bar(C::bPFull), kSoftWarps);
    mbar_init(bar(C::bPFree), 1);
    mbar_init(bar(C::bDSFull), kSoftWarps);
    mbar_init(bar(C::bDQStaged), kSoftWarps);
    mbar_init(bar(C::bDQRead), 1);
    mbar_init(bar(C::bAccReady), 1);
    mbar_init(bar(C::bAccFree), kSoftWarps);
    mbar_init(bar(C::bStaged), kSoftWarps);
    *abort_flag = 0;
    fence_mbar_init();
  }
  const uint32_t tmem = bwd_setup<C>(smem, warp);

  if (warp == C::kWarpProducer) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_map(&tmQ);
      tma_prefetch_map(&tmK);
      tma_prefetch_map(&tmV);
      tma_prefetch_map(&tmdO);
      int items = 0, n0 = 0, n1 = 0;
      bool ok = true;
      for (int k = blockIdx.x; ok && k < a.n_items; k += gridDim.x) {
        int bh, j;
        Mask mk;
        if (!bwd_item(k, a, true, bh, j, mk)) continue;
        int i_lo, i_hi;
        q_tiles_for_kv_tile(j, mk, i_lo, i_hi);
        const int xb = items & 1, xu = items >> 1;
        if (!mbar_wait(bar(C::bXEmpty + xb), (xu & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(C::bXFull + xb), 2 * C::kTile);
        tma_load_3d(sb + C::kX + xb * 2 * C::kTile, &tmK, bar(C::bXFull + xb), 0, j * kBlock, bh);
        tma_load_3d(sb + C::kX + xb * 2 * C::kTile + C::kTile, &tmV, bar(C::bXFull + xb), 0,
                    j * kBlock, bh);
        ++items;
        for (int i = i_lo; i <= i_hi; ++i) {
          const int s0 = n0 % C::kStages0, s1 = n1 % C::kStages1;
          if (!mbar_wait(bar(C::bY0Empty + s0), ((n0 / C::kStages0) & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(C::bY0Full + s0), C::kTile + 2 * 512);
          tma_load_3d(sb + C::kY0 + s0 * C::kTile, &tmQ, bar(C::bY0Full + s0), 0, i * kBlock, bh);
          const float* st = a.stats + (size_t)bh * a.Np + (size_t)i * kBlock;
          bulk_load(sb + C::kLse + s0 * 512, st, 512, bar(C::bY0Full + s0));
          bulk_load(sb + C::kDelta + s0 * 512, st + a.stat_rows, 512, bar(C::bY0Full + s0));
          ++n0;
          if (!mbar_wait(bar(C::bY1Empty + s1), ((n1 / C::kStages1) & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(C::bY1Full + s1), C::kTile);
          tma_load_3d(sb + C::kY1 + s1 * C::kTile, &tmdO, bar(C::bY1Full + s1), 0, i * kBlock,
                      bh);
          ++n1;
        }
      }
      for (int n = (items > 2 ? items - 2 : 0); n < items; ++n)
        mbar_wait(bar(C::bXFull + (n & 1)), (n >> 1) & 1, nullptr);
      drain_ring(bar(C::bY0Full), C::kStages0, n0);
      drain_ring(bar(C::bY1Full), C::kStages1, n1);
    }
    __syncwarp();
  } else if (warp == C::kWarpMma) {
    // ------------------------------------------------------------------ score products
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);
      int items = 0, t = 0;
      bool ok = true;
      for (int k = blockIdx.x; ok && k < a.n_items; k += gridDim.x) {
        int bh, j;
        Mask mk;
        if (!bwd_item(k, a, true, bh, j, mk)) continue;
        int i_lo, i_hi;
        q_tiles_for_kv_tile(j, mk, i_lo, i_hi);
        const int xb = items & 1, xu = items >> 1;
        if (!mbar_wait(bar(C::bXFull + xb), xu & 1, abort_flag)) break;
        const uint32_t xK = sb + C::kX + xb * 2 * C::kTile, xV = xK + C::kTile;
        for (int i = i_lo; i <= i_hi; ++i, ++t) {
          const int s0 = t % C::kStages0, s1 = t % C::kStages1;
          // S^T = K_j Q_i^T, once the softmax has loaded the previous S^T
          if (!mbar_wait(bar(C::bY0Full + s0), (t / C::kStages0) & 1, abort_flag) ||
              (t >= 1 && !mbar_wait(bar(C::bSFree), (t - 1) & 1, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          {
            const uint64_t dx = sdesc_sw128(xK, 16, 1024);
            const uint64_t dy = sdesc_sw128(sb + C::kY0 + s0 * C::kTile, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              mma_ss(tmem + C::tS, sdesc_add(dx, kk * 32), sdesc_add(dy, kk * 32), idS, kk > 0);
          }
          tc_commit(bar(C::bSFull));
          tc_commit(bar(C::bY0Empty + s0));
          // dP^T = V_j dO_i^T, once the softmax has loaded the previous dP^T
          if (!mbar_wait(bar(C::bY1Full + s1), (t / C::kStages1) & 1, abort_flag) ||
              (t >= 1 && !mbar_wait(bar(C::bDPFree), (t - 1) & 1, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          {
            const uint64_t dx = sdesc_sw128(xV, 16, 1024);
            const uint64_t dy = sdesc_sw128(sb + C::kY1 + s1 * C::kTile, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              mma_ss(tmem + C::tDP, sdesc_add(dx, kk * 32), sdesc_add(dy, kk * 32), idS, kk > 0);
          }
          tc_commit(bar(C::bDPFull));
          tc_commit(bar(C::bY1Empty + s1));
        }
        ++items;
      }
      tc_commit(bar(C::bMmaFin));
      mbar_wait(bar(C::bMmaFin), 0, nullptr);
    }
    __syncwarp();
  } else if (warp == C::kWarpMma + 1) {
    // ------------------------------------------------------------------ gradient products
    if (lane == 0) {
      // dV, dK: A (P^T, dS^T) K-major from shared memory, B (dO_i, Q_i) MN-major
      constexpr uint32_t idKV = idesc_bf16_f32(128, D, false, true);
      // dQ: A = dS (the dS^T copy read MN-major), B = K_j MN-major
      constexpr uint32_t idQ = idesc_bf16_f32(128, D, true, true);
      int items = 0, t = 0;
      bool ok = true;
      for (int k = blockIdx.x; ok && k < a.n_items; k += gridDim.x) {
        int bh, j;
        Mask mk;
        if (!bwd_item(k, a, true, bh, j, mk)) continue;
        int i_lo, i_hi;
        q_tiles_for_kv_tile(j, mk, i_lo, i_hi);
        const uint32_t xK = sb + C::kX + (items & 1) * 2 * C::kTile;
        for (int i = i_lo; i <= i_hi; ++i, ++t) {
          const int s0 = t % C::kStages0, s1 = t % C::kStages1;
          const bool first = i == i_lo;
          // dV += P^T dO_i; the item's first product overwrites dV (and dK), which the
          // previous item's epilogue must have read
          if (!mbar_wait(bar(C::bY1Full + s1), (t / C::kStages1) & 1, abort_flag) ||
              !mbar_wait(bar(C::bPFull), t & 1, abort_flag) ||
              (first && items > 0 &&
               !mbar_wait(bar(C::bAccFree), (items - 1) & 1, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          {
            const uint64_t dp = sdesc_sw128(sb + C::kP, 16, 1024);
            const uint64_t dy = sdesc_sw128(sb + C::kY1 + s1 * C::kTile, C::kRegionBytes, 1024);
#pragma unroll
            for (int kk = 0; kk < kBlock / 16; ++kk)
              mma_ss(tmem + C::tDV, sdesc_add(dp, (kk >> 2) * C::kRegionBytes + (kk & 3) * 32),
                     sdesc_add(dy, kk * 2048), idKV, (!first || kk > 0) ? 1u : 0u);
          }
          tc_commit(bar(C::bPFree));
          tc_commit(bar(C::bY1Empty + s1));
          // dK += dS^T Q_i, then dQ_t = dS K_j into buffer t & 1 once tile t-2's is drained
          if (!mbar_wait(bar(C::bY0Full + s0), (t / C::kStages0) & 1, abort_flag) ||
              !mbar_wait(bar(C::bDSFull), t & 1, abort_flag) ||
              (t >= 2 && !mbar_wait(bar(C::bDQFree + (t & 1)), ((t >> 1) - 1) & 1, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          {
            const uint64_t dsk = sdesc_sw128(sb + C::kDS, 16, 1024);
            const uint64_t dy = sdesc_sw128(sb + C::kY0 + s0 * C::kTile, C::kRegionBytes, 1024);
#pragma unroll
            for (int kk = 0; kk < kBlock / 16; ++kk)
              mma_ss(tmem + C::tDK, sdesc_add(dsk, (kk >> 2) * C::kRegionBytes + (kk & 3) * 32),
                     sdesc_add(dy, kk * 2048), idKV, (!first || kk > 0) ? 1u : 0u);
            const uint64_t dsm = sdesc_sw128(sb + C::kDS, C::kRegionBytes, 1024);
            const uint64_t dk = sdesc_sw128(xK, C::kRegionBytes, 1024);
#pragma unroll
            for (int kk = 0; kk < kBlock / 16; ++kk)
              mma_ss(tmem + C::tDQ + 64u * (t & 1), sdesc_add(dsm, kk * 2048),
                     sdesc_add(dk, kk * 2048), idQ, kk > 0 ? 1u : 0u);
          }
          tc_commit(bar(C::bY0Empty + s0));
          tc_commit(bar(C::bDQFull + (t & 1)));
          if (i == i_hi) tc_commit(bar(C::bAccReady));  // dK, dV (and the last dQ) complete
        }
        ++items;
      }
      tc_commit(bar(C::bMmaFin + 1));
      mbar_wait(bar(C::bMmaFin + 1), 0, nullptr);
    }
    __syncwarp();
  } else if (warp == C::kWarpStore) {
    // ------------------------------------------------------------------ bulk transfers
    // Per tile, in the order the softmax stages them: the dQ share staged in the dS^T
    // buffer goes to the accumulator as two reduce-adds of 32-column boxes, and the buffer
    // is handed back once they have read it. Per item, after its last tile: dK, dV leave
    // from the K_j, V_j buffer the softmax staged them in, which then goes back to the
    // producer.
    if (lane == 0) {
      tma_prefetch_map(&tmDQ);
      int items = 0, t = 0;
      bool ok = true;
      for (int k = blockIdx.x; ok && k < a.n_items; k += gridDim.x) {
        int bh, j;
        Mask mk;
        if (!bwd_item(k, a, true, bh, j, mk)) continue;
        int i_lo, i_hi;
        q_tiles_for_kv_tile(j, mk, i_lo, i_hi);
        for (int i = i_lo; i <= i_hi; ++i, ++t) {
          if (!mbar_wait(bar(C::bDQStaged), t & 1, abort_flag)) {
            ok = false;
            break;
          }
          tma_reduce_add_3d(&tmDQ, sb + C::kDS, 0, i * kBlock, bh);
          tma_reduce_add_3d(&tmDQ, sb + C::kDS + C::kRegionBytes, 32, i * kBlock, bh);
          bulk_commit();
          bulk_wait_read();
          mbar_arrive(bar(C::bDQRead));
        }
        if (!ok) break;
        const int xb = items & 1;
        if (!mbar_wait(bar(C::bStaged), items & 1, abort_flag)) break;
        ++items;
        tma_store_3d(&tmdK, sb + C::kX + xb * 2 * C::kTile, 0, j * kBlock, bh);
        tma_store_3d(&tmdV, sb + C::kX + xb * 2 * C::kTile + C::kTile, 0, j * kBlock, bh);
        bulk_commit();
        bulk_wait_read();
        mbar_arrive(bar(C::bXEmpty + xb));
      }
      bulk_wait_all();
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax warps
    constexpr int NC = C::kCols;
    static_assert(NC == 32, "one lane per query of the warp's 32");
    const int h = warp >> 2;              // queries NC*h .. NC*h+NC-1 of each query tile
    const int quad = warp & 3;            // TMEM lane quadrant
    const int t_row = threadIdx.x & 127;  // key row of the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const float sl2 = a.scale_log2;
    int g = 0, items = 0;
    bool ok = true;
    // Copies tile tt's dQ share from tensor memory into the dS^T buffer (fp32, as two
    // 32-column boxes) for the store warp's bulk reduction: this warp's 32 query rows (its
    // lane quadrant), columns 16h .. 16h+15. DQFull(tt) also means that dK and dQ of tile
    // tt, the last readers of the buffer, are complete.
    auto stage_dq = [&](int tt) -> bool {
      if (!mbar_wait_warp(bar(C::bDQFull + (tt & 1)), (tt >> 1) & 1, abort_flag)) return false;
      tc_fence_after();
      uint32_t r[16];
      tmem_ld16(tmem + lane_base + C::tDQ + 64u * (tt & 1) + 16u * h, r);
      tmem_wait_ld();
      reg_fence(r);
      tc_fence_before();
      mbar_arrive_warp(bar(C::bDQFree + (tt & 1)));
      store_row16_f32(sb + C::kDS, quad * 32 + lane, 16 * h, r);
      fence_async_smem();
      mbar_arrive_warp(bar(C::bDQStaged));
      return true;
    };
    for (int k = blockIdx.x; ok && k < a.n_items; k += gridDim.x) {
      int bh, j;
      Mask mk;
      if (!bwd_item(k, a, true, bh, j, mk)) continue;
      int i_lo, i_hi;
      q_tiles_for_kv_tile(j, mk, i_lo, i_hi);
      const int n_it = i_hi - i_lo + 1;
      const int c = j * kBlock + t_row;  // this thread's key
      const float slope2 = kAlibi ? a.alibi[bh % a.H] * kLog2e : 0.f;
      const bool key_padded = kKpad && c < a.N && a.kpad[(size_t)(bh / a.H) * a.N + c] != 0;
      for (int it = 0; it < n_it; ++it) {
        const int i = i_lo + it;
        const int t = g + it;
        const int s = t % C::kStages0;
        uint32_t keep = ~0u;
        if (kDropout) {
          const uint32_t blk = (uint32_t)(8 * j + 2 * quad);
          const uint32_t qrow = (uint32_t)(i * kBlock + NC * h + lane);
          const uint32_t mine = keep_bits16(a.drop, blk, qrow, (uint32_t)bh) |
                                (keep_bits16(a.drop, blk + 1, qrow, (uint32_t)bh) << 16);
#pragma unroll
          for (int b = 0; b < 32; ++b) {
            const uint32_t col = __ballot_sync(0xffffffffu, (mine >> b) & 1u);
            keep = (lane == b) ? col : keep;
          }
        }
        if (!mbar_wait_warp(bar(C::bY0Full + s), (t / C::kStages0) & 1, abort_flag) ||
            !mbar_wait_warp(bar(C::bSFull), t & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float p[NC];
        load_cols32(tmem + lane_base + C::tS + NC * h, p);
        // S^T is in registers: the next tile's S^T may overwrite it
        tc_fence_before();
        mbar_arrive_warp(bar(C::bSFree));
        const float* lse_s = reinterpret_cast<const float*>(smem + C::kLse + s * 512) + NC * h;
        const float* del_s = reinterpret_cast<const float*>(smem + C::kDelta + s * 512) + NC * h;
#pragma unroll
        for (int r = 0; r < NC; r += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(lse_s + r);
          float b4[4] = {0.f, 0.f, 0.f, 0.f};
          if (kAlibi) {
            const float base = (float)((long long)i * kBlock + NC * h + r - c);
#pragma unroll
            for (int e = 0; e < 4; ++e) b4[e] = -slope2 * fabsf(base + (float)e);
          }
          p[r] = ex2(fmaf(p[r], sl2, kAlibi ? b4[0] - l4.x : -l4.x));
          p[r + 1] = ex2(fmaf(p[r + 1], sl2, kAlibi ? b4[1] - l4.y : -l4.y));
          p[r + 2] = ex2(fmaf(p[r + 2], sl2, kAlibi ? b4[2] - l4.z : -l4.z));
          p[r + 3] = ex2(fmaf(p[r + 3], sl2, kAlibi ? b4[3] - l4.w : -l4.w));
        }
        if (!tile_all_visible(i, j, mk)) {
          int r_lo, r_hi;
          visible_queries(c, (long long)i * kBlock + NC * h, NC, mk, r_lo, r_hi);
#pragma unroll
          for (int r = 0; r < NC; ++r) p[r] = (r >= r_lo && r <= r_hi) ? p[r] : 0.f;
        }
        if (kKpad) {
#pragma unroll
          for (int r = 0; r < NC; ++r) p[r] = key_padded ? 0.f : p[r];
        }
        {
          // P^T (with dropout: P o Z / (1 - p')) in bf16 to shared memory, once the previous
          // tile's dV has read it
          uint32_t pk[NC / 2];
          if (kDropout) {
            const float ks = a.drop.keep_scale;
#pragma unroll
            for (int r = 0; r < NC / 2; ++r)
              pk[r] = pack_bf16x2(((keep >> (2 * r)) & 1u) ? p[2 * r] * ks : 0.f,
                                  ((keep >> (2 * r + 1)) & 1u) ? p[2 * r + 1] * ks : 0.f);
          } else {
#pragma unroll
            for (int r = 0; r < NC / 2; ++r) pk[r] = pack_bf16x2(p[2 * r], p[2 * r + 1]);
          }
          // the previous tile's dQ share is complete by now (its product followed the
          // previous dS): stage it for the bulk reduction
          if (it > 0 && !stage_dq(t - 1)) {
            ok = false;
            break;
          }
          if (t >= 1 && !mbar_wait_warp(bar(C::bPFree), (t - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          store_row32_bf16(sb + C::kP, t_row, NC * h, pk);
          fence_async_smem();
          mbar_arrive_warp(bar(C::bPFull));
        }
        if (!mbar_wait_warp(bar(C::bDPFull), t & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float dp[NC];
        load_cols32(tmem + lane_base + C::tDP + NC * h, dp);
        tc_fence_before();
        mbar_arrive_warp(bar(C::bDPFree));
        if (kDropout) {
          const float ks = a.drop.keep_scale;
#pragma unroll
          for (int r = 0; r < NC; ++r) dp[r] = ((keep >> r) & 1u) ? dp[r] * ks : 0.f;
        }
        {
          uint32_t w[NC / 2];
#pragma unroll
          for (int e = 0; e < NC / 2; e += 2) {
            const int r0 = 2 * e;
            const float4 d4 = *reinterpret_cast<const float4*>(del_s + r0);
            w[e] = pack_bf16x2(p[r0] * (dp[r0] - d4.x), p[r0 + 1] * (dp[r0 + 1] - d4.y));
            w[e + 1] = pack_bf16x2(p[r0 + 2] * (dp[r0 + 2] - d4.z), p[r0 + 3] * (dp[r0 + 3] - d4.w));
          }
          // dS^T to shared memory, once the previous tile's dQ share staged there has been
          // read by its bulk reduction (which also means its dK and dQ are complete)
          if (t >= 1 && !mbar_wait_warp(bar(C::bDQRead), (t - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          store_row32_bf16(sb + C::kDS, t_row, NC * h, w);
          fence_async_smem();
          mbar_arrive_warp(bar(C::bDSFull));
        }
      }
      if (!ok) break;
      g += n_it;
      // the item's last dQ share
      if (!stage_dq(g - 1)) {
        ok = false;
        break;
      }
      // once per item, after its last dK (which follows its last dV)
      if (!mbar_wait_warp(bar(C::bAccReady), items & 1, abort_flag)) {
        ok = false;
        break;
      }
      // dK, dV go out through the item's K_j, V_j buffer, which no product reads any more
      // (its last reader, the last dQ, is complete: AccReady follows it)
      const int xb = items & 1;
      const uint32_t tK = sb + C::kX + xb * 2 * C::kTile, tV = tK + C::kTile;
      ++items;
      tc_fence_after();
      constexpr int NO = D / C::kGroups;
      stage_acc_cols<NO>(tmem + lane_base + C::tDV + NO * h, 1.f, tV, t_row, NO * h);
      stage_acc_cols<NO>(tmem + lane_base + C::tDK + NO * h, a.scale, tK, t_row, NO * h);
      fence_async_smem();
      tc_fence_before();
      mbar_arrive_warp(bar(C::bAccFree));
      mbar_arrive_warp(bar(C::bStaged));
    }
  }
  bwd_teardown<C>(tmem, warp);
}

// ------------------------------------------------------------------------------------
// dQ = scale * accumulator in bf16, for the rows r < N of every (batch, head); 8 values per
// thread (two 16-byte loads, one 16-byte store).
// ------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256)
    fa_bwd_dq_convert_kernel(const float* __restrict__ dq_acc, __nv_bfloat16* __restrict__ dq,
                             long long rows, int N, int Np, float scale) {
  constexpr int kPerRow = D / 8;  // threads per row
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long row = idx / kPerRow;  // over B*H*N output rows
  if (row >= rows) return;
  const int part = (int)(idx - row * kPerRow);
  const long long bh = row / N;
  const long long r = row - bh * N;
  const float4* src =
      reinterpret_cast<const float4*>(dq_acc + ((size_t)bh * Np + (size_t)r) * D + part * 8);
  const float4 x = src[0], y = src[1];
  st_global_v4(dq + (size_t)row * D + part * 8, pack_bf16x2(x.x * scale, x.y * scale),
               pack_bf16x2(x.z * scale, x.w * scale), pack_bf16x2(y.x * scale, y.y * scale),
               pack_bf16x2(y.z * scale, y.w * scale));
}

}  // namespace fa
