// fa_fwd.cuh - fused attention forward for sm_100a.
//
// Each persistent CTA takes work items of two consecutive 128-row query tiles (A and B)
// of one (batch, head) and walks the key/value tiles they can see (page "Flash Attention
// 3.7 核心原理与实战" §3.1: load a Q block, iterate over the K, V blocks; page
// "告别OOM和训练慢…(含A100环境配置)" §2.1 tiling). The two query tiles are independent
// streams that share every K/V tile: while the softmax of one works on its scores, the
// tensor core computes the other's products, so neither the special-function unit nor
// the tensor core waits for the other. Roles:
//
//   warp 10      TMA producer: Q_A, Q_B per item, then K_j and V_j through a ring of
//                shared-memory stages (128-byte swizzle), guarded by full/empty mbarriers.
//   warps 8, 9   MMA issuers (one thread each), for stream A and B: per key tile j,
//                S_s = Q_s K_j^T, and O_s += P_s V_j once P_s is published. At head_dim 64
//                P_s has its own columns and the next S_s is issued one key tile ahead, as
//                soon as the softmax has loaded S_s. At head_dim 128 P_s must lie over
//                S_s, so each key tile is processed as two 64-key halves: S of half h of
//                the next tile waits only for the P V product of half h, which runs while
//                the softmax works on the other half.
//   warps 0..3   softmax of stream A, warps 4..7 of stream B: thread r owns query row r
//                of its tile (TMEM lane r) and the scores of it. Per key tile (head_dim
//                64) or half tile (head_dim 128) it updates the running max m and sum l
//                (page "告别OOM和训练慢…" §2.2), rescales its row of O when m grew by more
//                than 2^8 (exact: O and l carry the same stale m), and writes
//                P = exp2(s*scale*log2e - m) in bf16 to TMEM, where the P V product reads
//                it (with ALiBi, the linear bias -m_h |i - j| joins every scaled score
//                first). At the end of an item it writes O / l and LSE = ln2 * (m + log2 l).
//
// TMEM: S_A (128 columns), S_B (128), O_A (head_dim), O_B (head_dim), and for head_dim 64
// P_A, P_B (64 each); for head_dim 128 P of half h goes over the first 32 (e4m3: 16)
// columns of half h of S_s.
#pragma once

#include <cuda_bf16.h>

#include "rng.cuh"
#include "sm100.cuh"
#include "tiles.cuh"

namespace fa {

struct FwdArgs {
  __nv_bfloat16* o;
  float* lse;
  int N;
  int BH;
  int n_qtiles;
  int n_pairs;        // items per (batch, head): query tiles taken per_item at a time
  int per_item;       // query tiles per item: 2 (streams A and B), or 1 when pairs would
                      // leave SMs idle (stream B then has no tile)
  int n_items;        // BH * n_pairs
  int longest_first;  // masked problems: chunks of `group` heads, longest items first
  int group;
  int paired;         // causal problems: complementary items paired per CTA (paired_item)
  int n_double;       // ... over n_double pairs; n_items then counts the schedule's slots
  float scale_log2;   // scale * log2(e)
  int left;
  int right;
  int fault;          // test hook: 1 = the producer never loads V (waits for it run out)
  const float* alibi; // ALiBi kernels: one slope per head (heads = H)
  int H;              // heads per batch entry (batch entry of bh = bh / H)
  const uint8_t* kpad;       // (B, N) key-padding flags (nonzero = padded key), or null
  __nv_bfloat16* o_low;      // (B, H, N, d) bf16 residual O - bf16(O), or null
  DropoutArgs drop;          // kFeatDropout kernels
  const int* seq_len;        // variable-length batch: B real lengths, or null
  const int* cu;             // packed batch: B + 1 cumulative lengths (tensors (total, H, D),
  int total;                 // LSE (H, total)), or null
  int sorted;                // variable-length batch: the schedule of varlen_item, whose
                             // tables each CTA builds in shared memory after kMisc
  float o_scale;             // kFeatFp8: the V descale, applied to O in the epilogue
};

// kFp8: 8-bit (e4m3) Q, K, V tiles (head_dim 128 only: one 128-byte row per token).
template <int D, bool kFp8 = false>
struct FwdCfg {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(!kFp8 || D == 128, "the e4m3 forward is for head_dim 128");
  static constexpr int kElemBytes = kFp8 ? 1 : 2;
  static constexpr int kTile = kBlock * D * kElemBytes;  // bytes of a 128 x D tile
  static constexpr int kRegions = D * kElemBytes / 128;  // 128-byte-wide column regions per tile
  static constexpr int kRegionBytes = kBlock * 128;
  // K_j and V_j share a ring stage, released by one commit per stream after its P V_j
  static constexpr int kStagesK = (D == 64) ? 4 : 2;
  static constexpr int kStagesV = kStagesK;
  // shared memory map (offsets from a 1024-aligned base)
  // Q buffers per stream: with head_dim 64 two, so that the next item's Q_s loads while
  // the current one is in use
  static constexpr int kQBufs = (D == 64) ? 2 : 1;
  static constexpr int kQ = 0;                        // + (stream * kQBufs + buffer) * kTile
  static constexpr int kK = kQ + 2 * kQBufs * kTile;  // + stage * kTile
  static constexpr int kV = kK + kStagesK * kTile;    // + stage * kTile
  static constexpr int kBar = kV + kStagesV * kTile;
  // barrier slots
  static constexpr int bQFull = 0;                  // + stream * 2 + buffer
  static constexpr int bQEmpty = 4;                 // + stream * 2 + buffer
  static constexpr int bKFull = 8;                  // + stage
  static constexpr int bKEmpty = bKFull + kStagesK;
  static constexpr int bVFull = bKEmpty + kStagesK;
  static constexpr int bVEmpty = bVFull + kStagesV;
  static constexpr int bSFull = bVEmpty + kStagesV;  // + stream: S_s computed
  static constexpr int bPFull = bSFull + 2;          // + stream: P_s published (4 warps)
  static constexpr int bODone = bPFull + 2;          // + stream: a P_s V product completed
  static constexpr int bOFree = bODone + 2;          // + stream: O_s read by the epilogue
  static constexpr int bSFree = bOFree + 2;          // + stream: S_s loaded (separate P)
  // head_dim 128 works in 64-key halves of each key tile: the barriers above serve half 0,
  // these half 1
  static constexpr int bSFull2 = bSFree + 2;         // + stream
  static constexpr int bPFull2 = bSFull2 + 2;        // + stream
  static constexpr int bODone2 = bPFull2 + 2;        // + stream
  static constexpr int bMmaFin = bODone2 + 2;        // + stream
  static constexpr int kNumBars = bMmaFin + 2;
  static constexpr int kMisc = kBar + kNumBars * 8;  // TMEM base address (+0), abort flag (+4)
  static constexpr int kSmemBytes = kMisc + 16 + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
  // tensor memory columns (128 lanes each)
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t tS = 0;    // + 128 * stream
  static constexpr uint32_t tO = 256;  // + D * stream
  // With head_dim 64 there is room for P in its own columns: S_s of the next key tile may
  // then be computed as soon as the softmax has loaded S_s, instead of waiting for the
  // P V product that reads P from the columns of S_s.
  static constexpr bool kSepP = (D == 64);
  // Without room for P (head_dim 128), each key tile is processed as two 64-key halves:
  // P of half h goes over the first columns of half h of S_s, so S of half h of the next
  // key tile waits only for the P V product of half h, which runs while the softmax works
  // on the other half.
  static constexpr bool kHalves = !kSepP;
  static constexpr uint32_t tP = 256 + 2 * D;  // + 64 * stream, when kSepP
  static constexpr int kThreads = 352;  // 8 softmax warps, 2 MMA warps, producer warp
  static constexpr int kWarpMma = 8;     // + stream
  static constexpr int kWarpProducer = 10;
};

// One work item: query tiles m[0] = 2p and m[1] = 2p + 1 (absent past the last tile) of
// one (batch, head), and the key tiles [lo[s], hi[s]] each of them sees. The producer
// walks [first, last], the union (the ranges of consecutive query tiles overlap or touch).
struct FwdItem {
  int bh;
  int n;        // the sequence's real length (N unless the batch is variable-length)
  int m[2];
  bool has_a;   // query tile A lies within the real length (else the item has no work)
  bool has_b;
  int lo[2];
  int hi[2];
  int first;
  int last;
};

__device__ __forceinline__ FwdItem no_fwd_item() {
  FwdItem it;
  it.bh = 0;
  it.n = 0;
  it.m[0] = it.m[1] = 0;
  it.has_a = it.has_b = false;
  it.lo[0] = it.lo[1] = 1;
  it.hi[0] = it.hi[1] = 0;
  it.first = 1;
  it.last = 0;
  return it;
}

// `sched`: the varlen_item tables (shared memory) when a.sorted; kPacked: a packed batch
// (a.cu), else a.cu is not looked at.
template <bool kPacked>
__device__ __forceinline__ FwdItem fwd_item(int k, const FwdArgs& a, const int* sched) {
  const int* const cu = kPacked ? a.cu : nullptr;
  FwdItem it;
  int pair;
  if (a.paired) {
    // a slot past the last pair: no work
    if (!paired_item(k, (int)gridDim.x, a.n_double, a.n_pairs, false, it.bh, pair))
      return no_fwd_item();
  } else if (a.sorted) {
    if (!varlen_item(k, (int)gridDim.x, sched, a.n_pairs, a.H, it.bh, pair)) return no_fwd_item();
  } else if (a.longest_first) {
    chunked_item(k, a.BH, a.n_pairs, a.group, false, it.bh, pair);
  } else {
    it.bh = k / a.n_pairs;
    pair = k % a.n_pairs;
  }
  it.n = real_length(a.seq_len, cu, it.bh, a.H, a.N);
  const Mask mk{it.n, a.left, a.right};
  const int n_qtiles = num_tiles(it.n);
  it.m[0] = a.per_item * pair;
  it.m[1] = it.m[0] + 1;
  it.has_a = it.m[0] < n_qtiles;
  it.has_b = a.per_item == 2 && it.m[1] < n_qtiles;
  kv_tiles_for_q_tile(it.m[0], mk, it.lo[0], it.hi[0]);
  if (it.has_b) {
    kv_tiles_for_q_tile(it.m[1], mk, it.lo[1], it.hi[1]);
  } else {
    it.lo[1] = 1;
    it.hi[1] = 0;
  }
  it.first = it.lo[0];
  it.last = it.hi[0];
  if (it.has_b) {
    if (it.lo[1] < it.first) it.first = it.lo[1];
    if (it.hi[1] > it.last) it.last = it.hi[1];
  }
  return it;
}

// Stream s's query tile and key range of item `it`, as scalars (s need not be a constant).
struct FwdRange {
  bool has;  // stream s has a query tile in this item
  int m;
  int lo;
  int hi;
};

__device__ __forceinline__ FwdRange fwd_range(const FwdItem& it, int s) {
  FwdRange r;
  r.has = s == 0 ? it.has_a : it.has_b;
  r.m = s ? it.m[1] : it.m[0];
  r.lo = s ? it.lo[1] : it.lo[0];
  r.hi = s ? it.hi[1] : it.hi[0];
  return r;
}

// kFeat: kFeatAlibi adds the linear bias -m_h |i - j| (m_h = alibi[bh % H]) to every
// scaled score; kFeatKpad masks the keys a.kpad flags; kFeatResidual also writes
// O - bf16(O) to a.o_low; kFeatDropout zeroes the weights whose Philox keep flag is
// clear before the P V product (the row sum l keeps them: dropout follows the softmax)
// and scales O by 1 / (1 - p'); kFeatFp8 takes e4m3 Q, K, V (S = Q K^T and P V as
// kind::f8f6f4 products, P rounded to e4m3, four per tensor-memory column; the Q and K
// descales are folded into scale_log2, the V descale into O).
// 352 threads (11 warps, three of them on one SM sub-partition with its 16K registers): at
// most 168 registers per thread.
template <int D, int kFeat = 0>
__global__ void __launch_bounds__(FwdCfg<D, (kFeat & kFeatFp8) != 0>::kThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdArgs a) {
  constexpr bool kFp8 = (kFeat & kFeatFp8) != 0;
  using C = FwdCfg<D, kFp8>;
  constexpr bool kAlibi = (kFeat & kFeatAlibi) != 0;
  constexpr bool kKpad = (kFeat & kFeatKpad) != 0;
  constexpr bool kResidual = (kFeat & kFeatResidual) != 0;
  constexpr bool kDropout = (kFeat & kFeatDropout) != 0;
  constexpr bool kPacked = (kFeat & kFeatPacked) != 0;
  const int* const cu = kPacked ? a.cu : nullptr;  // a packed batch's cumulative lengths
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMisc + 4);
  auto bar = [&](int i) -> uint32_t { return sb + C::kBar + 8u * i; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(C::bQFull + 2 * s), 1);
      mbar_init(bar(C::bQEmpty + 2 * s), 1);
      mbar_init(bar(C::bQFull + 2 * s + 1), 1);
      mbar_init(bar(C::bQEmpty + 2 * s + 1), 1);
      mbar_init(bar(C::bSFull + s), 1);
      mbar_init(bar(C::bPFull + s), 4);
      mbar_init(bar(C::bODone + s), 1);
      mbar_init(bar(C::bOFree + s), 4);
      mbar_init(bar(C::bSFree + s), 4);
      mbar_init(bar(C::bSFull2 + s), 1);
      mbar_init(bar(C::bPFull2 + s), 4);
      mbar_init(bar(C::bODone2 + s), 1);
    }
    // a K/V stage is released by one commit per stream after its P V product of the
    // stage's key tile (which the stream's S product of that tile precedes); each commit
    // holds its issuing thread for a few hundred clocks, so K and V are not released
    // separately
    for (int s = 0; s < C::kStagesK; ++s) {
      mbar_init(bar(C::bKFull + s), 1);
      mbar_init(bar(C::bVFull + s), 1);
      mbar_init(bar(C::bKEmpty + s), 2);
    }
    mbar_init(bar(C::bMmaFin), 1);
    mbar_init(bar(C::bMmaFin + 1), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  int* sched = reinterpret_cast<int*>(smem + C::kMisc + 16);
  if (a.sorted && warp == 1)
    build_varlen_sched(a.seq_len, cu, a.BH / a.H, a.H, a.N, a.per_item, a.n_pairs, sched);
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
      int nq[2] = {0, 0};  // Q loads per stream
      int kc = 0, vc = 0;  // K and V loads issued (ring positions)
      bool ok = true;
      for (int k = blockIdx.x; ok && k < a.n_items; k += gridDim.x) {
        const FwdItem it = fwd_item<kPacked>(k, a, sched);
        if (!it.has_a) continue;  // past the real length: nothing to load
        const int base = seq_base(cu, it.bh, a.H);
        for (int s = 0; s < 2; ++s) {
          if (s == 1 && !it.has_b) break;
          // Q_s of this item replaces the previous item's once its last S_s has been read
          const int qb = 2 * s + nq[s] % C::kQBufs, qu = nq[s] / C::kQBufs;
          if (!mbar_wait(bar(C::bQEmpty + qb), (qu & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(C::bQFull + qb), C::kTile);
          const int qslot = s * C::kQBufs + nq[s] % C::kQBufs;
          for (int r = 0; r < C::kRegions; ++r)
            tma_load_3d(sb + C::kQ + qslot * C::kTile + r * C::kRegionBytes, &tmQ, bar(C::bQFull + qb),
                        r * 64, tma_y(cu, it.bh, a.H, it.m[s] * kBlock),
                        tma_z(cu, it.bh, base, it.m[s] * kBlock));
          ++nq[s];
        }
        for (int j = it.first; ok && j <= it.last; ++j) {
          const int sk = kc % C::kStagesK;
          if (!mbar_wait(bar(C::bKEmpty + sk), ((kc / C::kStagesK) & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(C::bKFull + sk), C::kTile);
          for (int r = 0; r < C::kRegions; ++r)
            tma_load_3d(sb + C::kK + sk * C::kTile + r * C::kRegionBytes, &tmK,
                        bar(C::bKFull + sk), r * 64, tma_y(cu, it.bh, a.H, j * kBlock),
                        tma_z(cu, it.bh, base, j * kBlock));
          ++kc;
          if (a.fault == 1) continue;
          mbar_arrive_expect_tx(bar(C::bVFull + sk), C::kTile);
          for (int r = 0; r < C::kRegions; ++r)
            tma_load_3d(sb + C::kV + sk * C::kTile + r * C::kRegionBytes, &tmV,
                        bar(C::bVFull + sk), r * 64, tma_y(cu, it.bh, a.H, j * kBlock),
                        tma_z(cu, it.bh, base, j * kBlock));
          ++vc;
        }
      }
      // Drain: every copy issued must have landed before the CTA may exit.
      for (int s = 0; s < 2; ++s)
        for (int n = (nq[s] > C::kQBufs ? nq[s] - C::kQBufs : 0); n < nq[s]; ++n)
          mbar_wait(bar(C::bQFull + 2 * s + n % C::kQBufs), (n / C::kQBufs) & 1, nullptr);
      for (int s = 0; s < C::kStagesK; ++s) {
        if (kc > s) {
          const int last = s + C::kStagesK * ((kc - 1 - s) / C::kStagesK);
          mbar_wait(bar(C::bKFull + s), (last / C::kStagesK) & 1, nullptr);
        }
      }
      for (int s = 0; s < C::kStagesV; ++s) {
        if (vc > s) {
          const int last = s + C::kStagesV * ((vc - 1 - s) / C::kStagesV);
          mbar_wait(bar(C::bVFull + s), (last / C::kStagesV) & 1, nullptr);
        }
      }
    }
    __syncwarp();
  } else if (warp == C::kWarpMma || warp == C::kWarpMma + 1) {
    // ------------------------------------------------------------------ MMA issuers
    // One issuing thread per stream, so that a stream whose softmax is late never holds
    // up the other's products (issuing a product group occupies its thread for about as
    // long as the tensor core takes to run it). Each steps through every K/V ring position
    // of every item in order, issuing S or P V where its query tile sees the key tile and
    // only passing where it does not; a ring slot is released by one arrival per stream.
    if (lane == 0) {
      const int s = warp - C::kWarpMma;
      constexpr uint32_t idS = kFp8 ? idesc_e4m3_f32(128, 128, false, false)
                                    : idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idO = kFp8 ? idesc_e4m3_f32(128, D, false, true)
                                    : idesc_bf16_f32(128, D, false, true);
      int nq = 0;     // Q tiles consumed
      int nsi = 0;    // S products issued (all items)
      int npv = 0;    // P V products issued (all items)
      int nitem = 0;  // items whose last P V has been issued
      int pos = 0;    // K/V ring position
      int pend = -1;  // K/V stage whose release waits for the next S product, or -1
      bool ok = true;
      // Commits the pending release of a K/V stage. Without separate P the next S product
      // waits for the P V product to complete, so the release is committed after that S
      // product, off the path from P V to S.
      auto release = [&]() {
        if (pend >= 0) tc_commit(bar(C::bKEmpty + pend));
        pend = -1;
      };
      // K step of key tile j (ring position p): S_s = Q_s K_j^T if the stream sees j
      auto k_step = [&](const FwdItem& it, const FwdRange& rg, int j, int p) -> bool {
        const bool sees = rg.has && rg.lo <= j && j <= rg.hi;
        const bool first = j == rg.lo;
        const int sk = p % C::kStagesK;
        if (!mbar_wait(bar(C::bKFull + sk), (p / C::kStagesK) & 1, abort_flag)) return false;
        if (sees) {
          // S_s overwrites the stream's previous scores, which the softmax must have
          // loaded, and (without separate P) P_s, whose P V must be complete
          const bool free_s =
              C::kSepP ? (nsi == 0 || mbar_wait(bar(C::bSFree + s), (nsi - 1) & 1, abort_flag))
                       : (npv == 0 || mbar_wait(bar(C::bODone + s), (npv - 1) & 1, abort_flag));
          const int qb = 2 * s + nq % C::kQBufs;
          if ((first && !mbar_wait(bar(C::bQFull + qb), (nq / C::kQBufs) & 1, abort_flag)) ||
              !free_s)
            return false;
          tc_fence_after();
          const uint32_t qbase = sb + C::kQ + (s * C::kQBufs + nq % C::kQBufs) * C::kTile;
          const uint64_t dq = sdesc_sw128(qbase, 16, 1024);
          const uint64_t dk = sdesc_sw128(sb + C::kK + sk * C::kTile, 16, 1024);
          if constexpr (kFp8) {
            // K-steps of 32 e4m3 values: 32 bytes of the 128-byte rows
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk)
              mma_ss_f8(tmem + C::tS + 128u * s, sdesc_add(dq, kk * 32), sdesc_add(dk, kk * 32),
                        idS, kk > 0);
          } else {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * C::kRegionBytes + (kk & 3) * 32;
              mma_ss(tmem + C::tS + 128u * s, sdesc_add(dq, off), sdesc_add(dk, off), idS,
                     kk > 0);
            }
          }
          tc_commit(bar(C::bSFull + s));
          ++nsi;
          release();
          if (j == rg.hi) {
            tc_commit(bar(C::bQEmpty + qb));  // last read of this Q_s buffer
            ++nq;
          }
        }
        return true;
      };
      // V step of key tile j (ring position p): O_s += P_s V_j if the stream sees j
      auto v_step = [&](const FwdItem& it, const FwdRange& rg, int j, int p) -> bool {
        const bool sees = rg.has && rg.lo <= j && j <= rg.hi;
        const bool first = j == rg.lo;
        const int sv = p % C::kStagesV;
        if (!mbar_wait(bar(C::bVFull + sv), (p / C::kStagesV) & 1, abort_flag)) return false;
        if (sees) {
          // the first product of an item overwrites O_s: the previous epilogue must have
          // read it
          if (!mbar_wait(bar(C::bPFull + s), npv & 1, abort_flag) ||
              (first && nitem > 0 && !mbar_wait(bar(C::bOFree + s), (nitem - 1) & 1, abort_flag)))
            return false;
          tc_fence_after();
          const uint32_t pcol = tmem + (C::kSepP ? C::tP + 64u * s : C::tS + 128u * s);
          const uint64_t dv = sdesc_sw128(sb + C::kV + sv * C::kTile, C::kRegionBytes, 1024);
          if constexpr (kFp8) {
            // K-steps of 32 keys: 8 columns of P (four e4m3 per column), 32 rows of V
#pragma unroll
            for (int kk = 0; kk < kBlock / 32; ++kk)
              mma_ts_f8(tmem + C::tO + D * s, pcol + kk * 8, sdesc_add(dv, kk * 4096), idO,
                        (!first || kk > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int kk = 0; kk < kBlock / 16; ++kk)
              mma_ts(tmem + C::tO + D * s, pcol + kk * 8, sdesc_add(dv, kk * 2048), idO,
                     (!first || kk > 0) ? 1u : 0u);
          }
          tc_commit(bar(C::bODone + s));
          ++npv;
          if (j == rg.hi) ++nitem;
        }
        release();  // a stage whose release is still pending goes now
        pend = sv;
        if (C::kSepP) release();
        return true;
      };

      // head_dim 128, in 64-key halves: products issued per half, S_h overwrites P_h
      int nsh[2] = {0, 0};  // S products issued per half
      int nph[2] = {0, 0};  // P V products issued per half
      constexpr uint32_t idS64 = kFp8 ? idesc_e4m3_f32(128, 64, false, false)
                                      : idesc_bf16_f32(128, 64, false, false);
      // S_h = Q_s K_j[64h .. 64h+63]^T of key tile j (ring position p), if the stream sees j
      auto s_half = [&](const FwdRange& rg, int j, int p, int h) -> bool {
        const int sk = p % C::kStagesK;
        if (h == 0 && !mbar_wait(bar(C::bKFull + sk), (p / C::kStagesK) & 1, abort_flag))
          return false;
        if (!(rg.has && rg.lo <= j && j <= rg.hi)) return true;
        const bool first = j == rg.lo;
        const int qb = 2 * s + nq % C::kQBufs;
        // S_h overwrites P_h of the previous key tile, whose P V must have completed
        if ((nsh[h] > 0 &&
             !mbar_wait(bar((h ? C::bODone2 : C::bODone) + s), (nph[h] - 1) & 1, abort_flag)) ||
            (first && h == 0 && !mbar_wait(bar(C::bQFull + qb), (nq / C::kQBufs) & 1, abort_flag)))
          return false;
        tc_fence_after();
        const uint32_t qbase = sb + C::kQ + (s * C::kQBufs + nq % C::kQBufs) * C::kTile;
        const uint64_t dq = sdesc_sw128(qbase, 16, 1024);
        // rows 64h .. of K_j: 64 rows of 128 bytes into each 128-byte-wide region
        const uint64_t dk = sdesc_sw128(sb + C::kK + sk * C::kTile + 64 * 128 * h, 16, 1024);
        const uint32_t td = tmem + C::tS + 128u * s + 64u * h;
        if constexpr (kFp8) {
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)
            mma_ss_f8(td, sdesc_add(dq, kk * 32), sdesc_add(dk, kk * 32), idS64, kk > 0);
        } else {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::kRegionBytes + (kk & 3) * 32;
            mma_ss(td, sdesc_add(dq, off), sdesc_add(dk, off), idS64, kk > 0);
          }
        }
        tc_commit(bar((h ? C::bSFull2 : C::bSFull) + s));
        ++nsh[h];
        if (h == 1 && j == rg.hi) {
          tc_commit(bar(C::bQEmpty + qb));  // last read of this Q_s buffer
          ++nq;
        }
        return true;
      };
      // O_s += P_h V_j[64h .. 64h+63] of key tile j, if the stream sees j; after half 1 the
      // stream's share of the K/V stage is released
      auto v_half = [&](const FwdRange& rg, int j, int p, int h) -> bool {
        const int sv = p % C::kStagesV;
        if (h == 0 && !mbar_wait(bar(C::bVFull + sv), (p / C::kStagesV) & 1, abort_flag))
          return false;
        if (rg.has && rg.lo <= j && j <= rg.hi) {
          const bool first = j == rg.lo;
          // the item's first product overwrites O_s: the previous epilogue must have read it
          if (!mbar_wait(bar((h ? C::bPFull2 : C::bPFull) + s), nph[h] & 1, abort_flag) ||
              (first && h == 0 && nitem > 0 &&
               !mbar_wait(bar(C::bOFree + s), (nitem - 1) & 1, abort_flag)))
            return false;
          tc_fence_after();
          const uint32_t pcol = tmem + C::tS + 128u * s + 64u * h;
          const uint64_t dv = sdesc_sw128(sb + C::kV + sv * C::kTile, C::kRegionBytes, 1024);
          if constexpr (kFp8) {
            // K-steps of 32 keys: 8 columns of P (four e4m3 per column), 32 rows of V
#pragma unroll
            for (int kk = 0; kk < 2; ++kk)
              mma_ts_f8(tmem + C::tO + D * s, pcol + kk * 8, sdesc_add(dv, (2 * h + kk) * 4096),
                        idO, (!first || h > 0 || kk > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ts(tmem + C::tO + D * s, pcol + kk * 8, sdesc_add(dv, (4 * h + kk) * 2048),
                     idO, (!first || h > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(bar((h ? C::bODone2 : C::bODone) + s));
          ++nph[h];
          if (h == 1 && j == rg.hi) ++nitem;
        }
        if (h == 1) tc_commit(bar(C::bKEmpty + sv));
        return true;
      };

      for (int k = blockIdx.x; ok && k < a.n_items; k += gridDim.x) {
        const FwdItem it = fwd_item<kPacked>(k, a, sched);
        if (!it.has_a) continue;  // past the real length: no products
        const FwdRange rg = fwd_range(it, s);
        const int n = it.last - it.first + 1;
        if (C::kSepP) {
          // S one key tile ahead of P V: S_s(j+1) is computed while the softmax works on j
          ok = k_step(it, rg, it.first, pos);
          for (int t = 0; ok && t < n; ++t) {
            if (t + 1 < n) ok = k_step(it, rg, it.first + t + 1, pos + t + 1);
            if (ok) ok = v_step(it, rg, it.first + t, pos + t);
          }
        } else {
          // halves: S_0, S_1 of the first key tile, then P V of half h of tile t followed
          // by S of half h of tile t + 1
          ok = s_half(rg, it.first, pos, 0) && s_half(rg, it.first, pos, 1);
          for (int t = 0; ok && t < n; ++t) {
            ok = v_half(rg, it.first + t, pos + t, 0);
            if (ok && t + 1 < n) ok = s_half(rg, it.first + t + 1, pos + t + 1, 0);
            if (ok) ok = v_half(rg, it.first + t, pos + t, 1);
            if (ok && t + 1 < n) ok = s_half(rg, it.first + t + 1, pos + t + 1, 1);
          }
        }
        pos += n;
      }
      release();
      // Wait for every MMA this thread issued before the CTA may release tensor memory.
      tc_commit(bar(C::bMmaFin + s));
      mbar_wait(bar(C::bMmaFin + s), 0, nullptr);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax warps
    const int s = warp >> 2;                     // stream: query tile A or B of the item
    const int r = threadIdx.x & 127;             // query row in the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + C::tS + 128u * s;
    const uint32_t tP = C::kSepP ? tmem + lane_base + C::tP + 64u * s : tS;
    const uint32_t tO = tmem + lane_base + C::tO + D * s;
    const float sl2 = a.scale_log2;
    int ns = 0;  // S tiles of this stream consumed (all items)
    int nsh[2] = {0, 0};   // kHalves: S halves consumed, per half
    int npub[2] = {0, 0};  // kHalves: P halves published, per half
    bool ok = true;


    for (int k = blockIdx.x; ok && k < a.n_items; k += gridDim.x) {
      const FwdItem it = fwd_item<kPacked>(k, a, sched);
      const FwdRange rg = fwd_range(it, s);
      if (!rg.has) continue;
      const Mask mk{it.n, a.left, a.right};
      const int row = rg.m * kBlock + r;
      // with ALiBi the scores are scaled and biased as they are loaded (in log2 units), so
      // the later steps take them as they are
      const float slope2 = kAlibi ? a.alibi[it.bh % a.H] * kLog2e : 0.f;
      const float xs = kAlibi ? 1.f : sl2;
      float m_run = -INFINITY;  // running max of scale*log2e*s (the m that P and O carry)
      float l_run = 0.f;        // running sum of P
      for (int j = rg.lo; j <= rg.hi; ++j) {
        if constexpr (C::kHalves) {
          // the key tile as two 64-key halves, each its own step of the online softmax
          for (int h = 0; h < 2; ++h) {
            // keep flags of this row's 64 weights: bit c of keep[g] for key 64h + 32g + c
            uint32_t keep[2] = {~0u, ~0u};
            if (kDropout) {
#pragma unroll
              for (int g = 0; g < 2; ++g) {
                const uint32_t blk = (uint32_t)(8 * j + 4 * h + 2 * g);
                keep[g] = keep_bits16(a.drop, blk, (uint32_t)row, (uint32_t)it.bh) |
                          (keep_bits16(a.drop, blk + 1, (uint32_t)row, (uint32_t)it.bh) << 16);
              }
            }
            if (!mbar_wait_warp(bar((h ? C::bSFull2 : C::bSFull) + s), nsh[h] & 1, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t tSh = tS + 64u * h;
            float x[64];
            {
              uint32_t u[64];
              tmem_ld32(tSh, *reinterpret_cast<uint32_t(*)[32]>(u));
              tmem_ld32(tSh + 32, *reinterpret_cast<uint32_t(*)[32]>(u + 32));
              tmem_wait_ld();
              reg_fence(u);
#pragma unroll
              for (int c = 0; c < 64; ++c) x[c] = __uint_as_float(u[c]);
            }
            if (kAlibi) {
              // key minus query index at column 0 of the half
              const long long kq = (long long)j * kBlock + 64 * h - row;
              const float base = (float)kq;
              const bool below = __all_sync(0xffffffffu, kq + 63 <= 0);
              const bool above = __all_sync(0xffffffffu, kq >= 0);
              if (below || above) {
                const float s2 = below ? slope2 : -slope2;
                const float c0 = s2 * base;
#pragma unroll
                for (int c = 0; c < 64; ++c) x[c] = fmaf(x[c], sl2, fmaf(s2, (float)c, c0));
              } else {
#pragma unroll
                for (int c = 0; c < 64; ++c)
                  x[c] = fmaf(x[c], sl2, -slope2 * fabsf(base + (float)c));
              }
            }
            if (!tile_all_visible(rg.m, j, mk)) {
              int c_lo, c_hi;
              visible_keys(row, (long long)j * kBlock + 64 * h, 64, mk, c_lo, c_hi);
#pragma unroll
              for (int c = 0; c < 64; ++c) x[c] = (c >= c_lo && c <= c_hi) ? x[c] : -INFINITY;
            }
            if (kKpad) {
              uint32_t pm[2];
              const uint8_t* fl = a.kpad + (size_t)(it.bh / a.H) * a.N;
#pragma unroll
              for (int g = 0; g < 2; ++g) {
                const int col = j * kBlock + 64 * h + 32 * g + lane;
                pm[g] = __ballot_sync(0xffffffffu, col < a.N && fl[col] != 0);
              }
              if ((pm[0] | pm[1]) != 0u) {
#pragma unroll
                for (int c = 0; c < 64; ++c)
                  x[c] = ((pm[c >> 5] >> (c & 31)) & 1u) ? -INFINITY : x[c];
              }
            }
            float mx;
            {
              float t[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) t[e] = fmax3(x[e], x[e + 16], x[e + 32]);
#pragma unroll
              for (int e = 0; e < 16; ++e) t[e] = fmaxf(t[e], x[48 + e]);
#pragma unroll
              for (int e = 0; e < 4; ++e) t[e] = fmax3(t[e], t[e + 4], t[e + 8]);
              mx = fmax3(fmax3(t[0], t[1], t[2]), fmax3(t[3], t[12], t[13]),
                         fmaxf(t[14], t[15]));
            }
            const float m_new = fmaxf(m_run, mx * xs);
            const bool grow = m_new > m_run + 8.0f;
            float alpha = 1.f;
            if (grow) {
              alpha = ex2(m_run - m_new);
              m_run = m_new;
              l_run *= alpha;
            }
            const float mb = (m_run == -INFINITY) ? 0.f : m_run;
            // P over the first columns of this half of S_s, 32 keys at a time
            float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              if constexpr (kFp8) {
                uint32_t pk[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                  float p4[4];
#pragma unroll
                  for (int e = 0; e < 4; ++e) p4[e] = ex2(fmaf(x[32 * hh + 4 * c + e], xs, -mb));
                  ls[c & 3] += (p4[0] + p4[1]) + (p4[2] + p4[3]);
                  pk[c] = pack_e4m3x4(p4[0], p4[1], p4[2], p4[3]);
                }
                tmem_st8(tSh + 8 * hh, pk);
              } else {
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                  float p0 = ex2(fmaf(x[32 * hh + 2 * c], xs, -mb));
                  float p1 = ex2(fmaf(x[32 * hh + 2 * c + 1], xs, -mb));
                  ls[c & 3] += p0 + p1;
                  if (kDropout) {
                    p0 = ((keep[hh] >> (2 * c)) & 1u) ? p0 : 0.f;
                    p1 = ((keep[hh] >> (2 * c + 1)) & 1u) ? p1 : 0.f;
                  }
                  pk[c] = pack_bf16x2(p0, p1);
                }
                tmem_st16(tSh + 16 * hh, pk);
              }
            }
            l_run += (ls[0] + ls[1]) + (ls[2] + ls[3]);
            // rescale this row of O before P_h V accumulates into it, once the previous
            // half's P V (the last product into O) has completed
            if (!(j == rg.lo && h == 0) && __any_sync(0xffffffffu, grow)) {
              const int hp = h ^ 1;
              if (!mbar_wait_warp(bar((hp ? C::bODone2 : C::bODone) + s), (npub[hp] - 1) & 1,
                                  abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
#pragma unroll
              for (int q = 0; q < D / 32; ++q) {
                uint32_t o[32];
                tmem_ld32(tO + 32 * q, o);
                tmem_wait_ld();
                reg_fence(o);
#pragma unroll
                for (int c = 0; c < 32; ++c)
                  o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                tmem_st32(tO + 32 * q, o);
              }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive_warp(bar((h ? C::bPFull2 : C::bPFull) + s));
            ++nsh[h];
            ++npub[h];
          }
          if (!ok) break;
          continue;
        }
        // keep flags of this row's 128 weights (they depend on no score, so they are drawn
        // before S is ready): bit c of keep[g] for key 32g + c of the tile
        uint32_t keep[4] = {~0u, ~0u, ~0u, ~0u};
        if (kDropout) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const uint32_t blk = (uint32_t)(8 * j + 2 * g);
            keep[g] = keep_bits16(a.drop, blk, (uint32_t)row, (uint32_t)it.bh) |
                      (keep_bits16(a.drop, blk + 1, (uint32_t)row, (uint32_t)it.bh) << 16);
          }
        }
        if (!mbar_wait_warp(bar(C::bSFull + s), ns & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float x[kBlock];
        {
          // all four loads in flight before one wait
          uint32_t u[kBlock];
#pragma unroll
          for (int q = 0; q < 4; ++q)
            tmem_ld32(tS + 32 * q, *reinterpret_cast<uint32_t(*)[32]>(u + 32 * q));
          tmem_wait_ld();
          reg_fence(u);
#pragma unroll
          for (int c = 0; c < kBlock; ++c) x[c] = __uint_as_float(u[c]);
        }
        if (C::kSepP) {
          // S_s is in registers: the next key tile's S_s may overwrite it
          tc_fence_before();
          mbar_arrive_warp(bar(C::bSFree + s));
        }
        if (kAlibi) {
          // key minus query index at column 0 of the tile
          const long long kq = (long long)j * kBlock - row;
          const float base = (float)kq;
          // off the diagonal the distance is linear in the column: -m|k - q| is
          // s2 * (base + c) with s2 = +m below it (keys before the query) and -m above
          const bool below = __all_sync(0xffffffffu, kq + kBlock - 1 <= 0);
          const bool above = __all_sync(0xffffffffu, kq >= 0);
          if (below || above) {
            const float s2 = below ? slope2 : -slope2;
            const float c0 = s2 * base;
#pragma unroll
            for (int c = 0; c < kBlock; ++c) x[c] = fmaf(x[c], sl2, fmaf(s2, (float)c, c0));
          } else {
#pragma unroll
            for (int c = 0; c < kBlock; ++c)
              x[c] = fmaf(x[c], sl2, -slope2 * fabsf(base + (float)c));
          }
        }
        if (!tile_all_visible(rg.m, j, mk)) {
          int c_lo, c_hi;
          visible_keys(row, (long long)j * kBlock, kBlock, mk, c_lo, c_hi);
#pragma unroll
          for (int c = 0; c < kBlock; ++c) x[c] = (c >= c_lo && c <= c_hi) ? x[c] : -INFINITY;
        }
        if (kKpad) {
          // padded keys of this tile: lane l reads the flag of key 32g + l, one ballot per
          // 32 keys; the same 128 bits for every row
          uint32_t pm[4];
          const uint8_t* fl = a.kpad + (size_t)(it.bh / a.H) * a.N;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int col = j * kBlock + 32 * g + lane;
            pm[g] = __ballot_sync(0xffffffffu, col < a.N && fl[col] != 0);
          }
          if ((pm[0] | pm[1] | pm[2] | pm[3]) != 0u) {
#pragma unroll
            for (int c = 0; c < kBlock; ++c)
              x[c] = ((pm[c >> 5] >> (c & 31)) & 1u) ? -INFINITY : x[c];
          }
        }
        float mx;
        {
          // 16 partial maxima: x[0..47], then two columns at a time up to x[111], then x[112..127]
          float t[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) t[e] = fmax3(x[e], x[e + 16], x[e + 32]);
#pragma unroll
          for (int c = 48; c + 32 <= kBlock; c += 32)
#pragma unroll
            for (int e = 0; e < 16; ++e) t[e] = fmax3(t[e], x[c + e], x[c + 16 + e]);
          static_assert(kBlock == 128, "the tail below covers columns 112..127");
#pragma unroll
          for (int e = 0; e < 16; ++e) t[e] = fmaxf(t[e], x[112 + e]);
#pragma unroll
          for (int e = 0; e < 4; ++e) t[e] = fmax3(t[e], t[e + 4], t[e + 8]);
          // t[0..3] and t[12..15] remain
          mx = fmax3(fmax3(t[0], t[1], t[2]), fmax3(t[3], t[12], t[13]), fmaxf(t[14], t[15]));
        }
        // O_s is stable once the stream's previous P V product has completed: implied by
        // S_full when P shares the columns of S_s, waited for below otherwise.
        const float m_new = fmaxf(m_run, mx * xs);
        const bool grow = m_new > m_run + 8.0f;
        float alpha = 1.f;
        if (grow) {
          alpha = ex2(m_run - m_new);
          m_run = m_new;
          l_run *= alpha;
        }
        const float mb = (m_run == -INFINITY) ? 0.f : m_run;
        // with separate P, P_s and O_s are free once the previous P V has completed
        if (C::kSepP && ns > 0) {
          if (!mbar_wait_warp(bar(C::bODone + s), (ns - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        // P = exp2(s*scale*log2e - m) in bf16 pairs (over columns 0..63 of S_s without
        // separate P)
        float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          if constexpr (kFp8) {
            // e4m3 P, four per column: keys 32h .. 32h+31 in columns 8h .. 8h+7
            uint32_t pk[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              float p4[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) p4[e] = ex2(fmaf(x[32 * h + 4 * c + e], xs, -mb));
              ls[c & 3] += (p4[0] + p4[1]) + (p4[2] + p4[3]);
              pk[c] = pack_e4m3x4(p4[0], p4[1], p4[2], p4[3]);
            }
            tmem_st8(tP + 8 * h, pk);
          } else {
            uint32_t pk[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              float p0 = ex2(fmaf(x[32 * h + 2 * c], xs, -mb));
              float p1 = ex2(fmaf(x[32 * h + 2 * c + 1], xs, -mb));
              ls[c & 3] += p0 + p1;
              if (kDropout) {
                p0 = ((keep[h] >> (2 * c)) & 1u) ? p0 : 0.f;
                p1 = ((keep[h] >> (2 * c + 1)) & 1u) ? p1 : 0.f;
              }
              pk[c] = pack_bf16x2(p0, p1);
            }
            tmem_st16(tP + 16 * h, pk);
          }
        }
        l_run += (ls[0] + ls[1]) + (ls[2] + ls[3]);
        // rescale this row of O before P_s V_j accumulates into it (that waits for p_full)
        if (j > rg.lo && __any_sync(0xffffffffu, grow)) {
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
        mbar_arrive_warp(bar(C::bPFull + s));
        ++ns;
      }
      if (!ok) break;
      // epilogue of the item: O / l and LSE, once the last P V product has completed
      if (!(C::kHalves ? mbar_wait_warp(bar(C::bODone2 + s), (npub[1] - 1) & 1, abort_flag)
                       : mbar_wait_warp(bar(C::bODone + s), (ns - 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
      if (kDropout) inv_l *= a.drop.keep_scale;
      if (kFp8) inv_l *= a.o_scale;
      // (the (B*H, N, d) layout forms its row pointer directly: through the packed helpers
      // the same expression compiled to a measurably slower d = 64 kernel)
      const int base = kPacked ? seq_base(cu, it.bh, a.H) : 0;
      const bool written = kPacked ? row_written(cu, a.total, a.N, it.n, base, row) : row < a.N;
      __nv_bfloat16* orow =
          kPacked ? a.o + row_at(cu, it.bh, a.H, a.N, base, written ? row : 0, D)
                  : a.o + ((size_t)it.bh * a.N + (row < a.N ? row : 0)) * D;
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
        if (written) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            st_global_v4(orow + 32 * q + 8 * v4, w[4 * v4], w[4 * v4 + 1], w[4 * v4 + 2],
                         w[4 * v4 + 3]);
        }
        if (kResidual) {
          // what rounding to bf16 left out: O - bf16(O), itself rounded to bf16, so that
          // the backward can form rowsum(dO o O) from O to about 16 significant bits
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float r0 = __uint_as_float(o[2 * c]) * inv_l - __uint_as_float(w[c] << 16);
            const float r1 =
                __uint_as_float(o[2 * c + 1]) * inv_l - __uint_as_float(w[c] & 0xFFFF0000u);
            w[c] = pack_bf16x2(r0, r1);
          }
          if (written) {
            __nv_bfloat16* lrow = a.o_low + row_at(cu, it.bh, a.H, a.N, base, row, D);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              st_global_v4(lrow + 32 * q + 8 * v4, w[4 * v4], w[4 * v4 + 1], w[4 * v4 + 2],
                           w[4 * v4 + 3]);
          }
        }
      }
      // O_s has been read: the next item's first P V may overwrite it
      tc_fence_before();
      mbar_arrive_warp(bar(C::bOFree + s));
      if (written)
        a.lse[lse_at(cu, a.total, it.bh, a.H, a.N, base, row)] =
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
