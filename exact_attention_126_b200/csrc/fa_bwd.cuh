// fa_bwd.cuh - attention backward for sm_100a: recompute P from the saved LSE.
//
// The pages give only the idea: keep the per-row normalisation factors and recompute
// the attention matrix in the backward (page "告别OOM和训练慢…(含A100环境配置)" §2.2; page
// "PyTorch-CUDA-v2.9镜像中使用FlashAttention提升训练速度", "3. 重计算策略"). The steps are the
// chain rule of softmax attention for the loss L = <O, dO>:
//
//   delta_i = sum_c dO_ic O_ic                     fa_bwd_preprocess_kernel (with LSE*log2e,
//                                                  both padded to whole 128-row tiles)
//   P_ij    = exp(scale q_i.k_j - LSE_i)           (recomputed, masked entries 0)
//   dP_ij   = dO_i . v_j
//   dS_ij   = P_ij (dP_ij - delta_i)
//   dV_j    = sum_i P_ij dO_i ;  dK_j = scale sum_i dS_ij q_i      fa_bwd_dkdv_kernel
//   dQ_i    = scale sum_j dS_ij k_j                                  fa_bwd_dq_kernel
//
// dK/dV are accumulated in TMEM by one CTA per 128-row key tile that walks the query
// tiles it is visible from; it computes the transposed products S^T = K Q^T and
// dP^T = V dO^T, so that each thread owns one key row and P^T, dS^T can go straight
// back into TMEM as the A operand of dV += P^T dO and dK += dS^T Q. dQ is accumulated
// the same way by one CTA per query tile walking its key tiles (S, dP, then
// dQ += dS K). Nothing is reduced across CTAs, so the results are deterministic.
//
// In both kernels four warpgroups share every row: warpgroup h takes the 32 columns
// 32h..32h+31 of it (query columns for dK/dV, key columns for dQ), so that four warps
// per SM sub-partition hide each other's latencies. P needs no row maximum here (the
// LSE is known), so the groups never wait for each other. Two MMA issuers (warps 16 and
// 17) work side by side: one computes the score products S and dP tile after tile, the
// other the gradient products as soon as the softmax publishes P and dS. Issuing a
// product group occupies its thread for about as long as the tensor core takes to run
// it, so one issuer for both would serialise them. Warp 18 issues the TMA loads and
// warp 19 the bulk stores of staged outputs.
#pragma once

#include <cuda_bf16.h>

#include "rng.cuh"
#include "sm100.cuh"
#include "tiles.cuh"

namespace fa {


// ------------------------------------------------------------------------------------
// Row statistics of the backward, over B*H rows of Np (N rounded up to 128) entries:
//   stats[bh*Np + r]             = LSE_r * log2(e)        (+inf for r >= N)
//   stats[BH*Np + bh*Np + r]     = rowsum(dO_r * O_r)     (0 for r >= N), summed in fp32
// With o_low (the residual O - bf16(O) the forward can write), O_r is taken as
// o_r + o_low_r, which carries about 16 significant bits instead of 8: for rows whose
// softmax is nearly one-hot, dS = P (dP - delta) cancels almost completely and the
// rounding of a bf16 O would dominate dQ and dK.
// With dq_acc (the fused backward's fp32 dQ accumulator, (B*H, Np, D)), each block also
// zeroes the accumulator rows it covers.
// Block b covers rows 64x .. 64x+63 of head bh, with (bh, x) = divmod(b, Np/64), 8 rows
// per warp; G = D/8 lanes share a row, 16 bytes of O and dO per lane, and a warp's loads
// for its 8 rows are all issued before any is used. In a packed batch (cu: B + 1 cumulative
// lengths; O, dO (total, H, D), LSE (H, total)) the rows are those of the sequence, and
// rows at or past its real length count as padding (+inf and 0).
// ------------------------------------------------------------------------------------
template <int D, bool kPacked>
__global__ void __launch_bounds__(256)
    fa_bwd_preprocess_kernel(const __nv_bfloat16* __restrict__ o,
                             const __nv_bfloat16* __restrict__ o_low,
                             const __nv_bfloat16* __restrict__ dout, const float* __restrict__ lse,
                             float* __restrict__ stats, float* __restrict__ dq_acc, SchedBuild sb,
                             const int* __restrict__ cu_in, int total, int H, int BH, int N,
                             int Np) {
  const int* const cu = kPacked ? cu_in : nullptr;
  constexpr int G = D / 8;                      // lanes per row
  constexpr int kRowsPerPass = 32 / G;          // rows a warp covers per load
  constexpr int kPasses = 8 / kRowsPerPass;     // 8 rows per warp
  const int blocks_per_head = Np / 64;
  if ((int)blockIdx.x >= BH * blocks_per_head) {
    if (threadIdx.x < 32)
      build_varlen_sched(sb.seq_len, sb.cu, sb.B, sb.H, sb.N, 1, sb.U, sb.tables);
    return;
  }
  const int bh = blockIdx.x / blocks_per_head;
  const int xb = blockIdx.x - bh * blocks_per_head;
  const int lane = threadIdx.x & 31;
  const int sub = lane / G;                     // row within the pass
  const int part = lane % G;                    // 16-byte slice of the row
  const int row0 = xb * 64 + (threadIdx.x >> 5) * 8;
  if (dq_acc != nullptr) {
    // the fused backward's dQ accumulator: this block's 64 rows (D fp32 each) start at zero
    float4* z = reinterpret_cast<float4*>(dq_acc + ((size_t)bh * Np + (size_t)xb * 64) * D);
    constexpr int kVec = 64 * D / 4;
#pragma unroll
    for (int e = threadIdx.x; e < kVec; e += 256) z[e] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // rows this head holds: N, or in a packed batch its real length (and no row past the
  // tensor's end)
  const int base = seq_base(cu, bh, H);
  int n_rows = N;
  if (cu != nullptr) {
    n_rows = real_length(nullptr, cu, bh, H, N);
    if (base < 0) n_rows = 0;  // offsets outside [0, total] read nothing
    if (total - base < n_rows) n_rows = total - base < 0 ? 0 : total - base;
  }
  uint4 a[kPasses], b[kPasses], c[kPasses];
#pragma unroll
  for (int p = 0; p < kPasses; ++p) {
    const int r = row0 + p * kRowsPerPass + sub;
    a[p] = make_uint4(0, 0, 0, 0);
    b[p] = make_uint4(0, 0, 0, 0);
    c[p] = make_uint4(0, 0, 0, 0);
    if (r < n_rows) {
      const size_t src = row_at(cu, bh, H, N, base, r, D) + part * 8;
      a[p] = *reinterpret_cast<const uint4*>(o + src);
      b[p] = *reinterpret_cast<const uint4*>(dout + src);
      if (o_low != nullptr) c[p] = *reinterpret_cast<const uint4*>(o_low + src);
    }
  }
  const size_t rows = (size_t)BH * Np;
#pragma unroll
  for (int p = 0; p < kPasses; ++p) {
    const uint32_t aw[4] = {a[p].x, a[p].y, a[p].z, a[p].w};
    const uint32_t bw[4] = {b[p].x, b[p].y, b[p].z, b[p].w};
    const uint32_t cw[4] = {c[p].x, c[p].y, c[p].z, c[p].w};
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float d0 = __uint_as_float(bw[w] << 16), d1 = __uint_as_float(bw[w] & 0xFFFF0000u);
      acc = fmaf(__uint_as_float(aw[w] << 16), d0, acc);
      acc = fmaf(__uint_as_float(aw[w] & 0xFFFF0000u), d1, acc);
      // the residual is zero without o_low
      acc = fmaf(__uint_as_float(cw[w] << 16), d0, acc);
      acc = fmaf(__uint_as_float(cw[w] & 0xFFFF0000u), d1, acc);
    }
#pragma unroll
    for (int off = G / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    const int r = row0 + p * kRowsPerPass + sub;
    if (part == 0 && r < Np) {
      const size_t rp = (size_t)bh * Np + r;
      stats[rp] = r < n_rows ? lse[lse_at(cu, total, bh, H, N, base, r)] * kLog2e : INFINITY;
      stats[rows + rp] = acc;
    }
  }
}

// ------------------------------------------------------------------------------------
// Variable-length batches: rows r >= L_b (the real length of the row's batch entry) of up to
// three bf16 (B*H, N, D) tensors become zero and, with `lse`, their LSE becomes -inf. The
// attention kernels skip every tile that lies wholly past the real length; this fills what
// they leave. Block b covers rows 128x .. 128x+127 of head bh, (bh, x) = divmod(b, tiles):
// a block whose rows are all below L_b returns at once, the others write 16 bytes per
// thread and step, the 256 threads of a step covering 256 / (D / 8) consecutive rows.
// ------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256)
    fa_fill_past_length_kernel(__nv_bfloat16* __restrict__ t0, __nv_bfloat16* __restrict__ t1,
                               __nv_bfloat16* __restrict__ t2, float* __restrict__ lse,
                               const int* __restrict__ seq_len, int N, int H) {
  constexpr int kPerRow = D / 8;
  const int tiles = num_tiles(N);
  const int bh = blockIdx.x / tiles;
  const int r0 = (blockIdx.x - bh * tiles) * kBlock;
  const int L = real_length(seq_len, nullptr, bh, H, N);
  const int r_end = r0 + kBlock < N ? r0 + kBlock : N;
  const int r_begin = r0 > L ? r0 : L;
  if (r_begin >= r_end) return;
  const size_t base = (size_t)bh * N;
  for (int e = r_begin * kPerRow - r0 * kPerRow + threadIdx.x;
       e < (r_end - r0) * kPerRow; e += blockDim.x) {
    const int r = r0 + e / kPerRow;
    const int part = e % kPerRow;
    const size_t off = (base + r) * D + part * 8;
    if (t0 != nullptr) st_global_v4(t0 + off, 0u, 0u, 0u, 0u);
    if (t1 != nullptr) st_global_v4(t1 + off, 0u, 0u, 0u, 0u);
    if (t2 != nullptr) st_global_v4(t2 + off, 0u, 0u, 0u, 0u);
    if (lse != nullptr && part == 0) lse[base + r] = -INFINITY;
  }
}

// Whether the output tile of rows r0 .. r0+127 of a sequence of real length L (first token
// `base`) leaves through a bulk store of the whole tile: always, except in a packed batch
// (cu) the last, partial tile of a sequence, whose rows past L are the next sequence's, and
// a tile not wholly inside the tensor's `total` tokens; those are written row by row
// (row_written).
__device__ __forceinline__ bool whole_tile_store(const int* cu, int total, int L, int base,
                                                 int r0) {
  return cu == nullptr || (r0 + kBlock <= L && base >= 0 && base + r0 + kBlock <= total);
}

struct BwdArgs {
  const float* stats;   // row statistics written by fa_bwd_preprocess_kernel
  __nv_bfloat16* out0;  // dkdv: dK ; dq: dQ (written directly when outputs are not staged)
  __nv_bfloat16* out1;  // dkdv: dV
  long long stat_rows;  // B*H*Np: offset of delta after LSE*log2e
  int N;
  int Np;               // N rounded up to a multiple of 128
  int BH;
  int n_tiles;
  int n_items;          // BH * n_tiles: one item per (batch*head, stationary tile)
  int longest_first;    // masked problems: chunks of `group` heads, longest items first
  int group;
  int paired;           // causal problems: complementary items paired per CTA (paired_item)
  int n_double;         // ... over n_double pairs; n_items then counts the schedule's slots
  float scale;
  float scale_log2;
  int left;
  int right;
  const float* alibi;   // ALiBi kernels: one slope per head (heads = H)
  int H;                // heads per batch entry (batch entry of bh = bh / H)
  const uint8_t* kpad;  // (B, N) key-padding flags (nonzero = padded key), or null
  DropoutArgs drop;     // kFeatDropout kernels
  const int* seq_len;   // variable-length batch: B real lengths, or null
  const int* cu;        // packed batch: B + 1 cumulative lengths (tensors (total, H, D),
  int total;            // LSE (H, total)), or null
  int sorted;           // variable-length batch: the schedule of varlen_item, with ...
  const int* sched;     // ... its tables, written by fa_bwd_preprocess_kernel
};

// Shared layout of both backward kernels: the stationary tiles X0, X1 of an item (in XB
// buffers, so that the next item's can load while this one runs) and two rings of
// streamed tiles, Y0 (with per-stage row statistics when kStats) and Y1, each with its own
// full/empty barriers so a tile is released right after its last product.
// dK/dV: X = K, V; Y0 = Q (+ LSE, delta), Y1 = dO. dQ: X = Q, dO; Y0 = K, Y1 = V.
template <int D, int XB, int S0, int S1, bool kStats>
struct BwdCfgT {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static constexpr int kTile = kBlock * D * 2;
  static constexpr int kRegions = D / 64;
  static constexpr int kRegionBytes = kBlock * 128;
  static constexpr int kXBufs = XB;
  static constexpr int kStages0 = S0;
  static constexpr int kStages1 = S1;
  static constexpr int kX0 = 0;                              // + xb * 2 * kTile
  static constexpr int kX1 = kTile;                          // + xb * 2 * kTile
  static constexpr int kY0 = XB * 2 * kTile;                 // + s * kTile
  static constexpr int kY1 = kY0 + S0 * kTile;               // + s * kTile
  static constexpr int kLse = kY1 + S1 * kTile;              // + s * 512 (128 fp32), ring 0
  static constexpr int kDelta = kLse + (kStats ? S0 * 512 : 0);
  static constexpr int kBar = kDelta + (kStats ? S0 * 512 : 0);
  static constexpr int bXFull = 0;                           // + xb
  static constexpr int bXEmpty = 2;                          // + xb
  static constexpr int bY0Full = 4;
  static constexpr int bY0Empty = bY0Full + S0;
  static constexpr int bY1Full = bY0Empty + S0;
  static constexpr int bY1Empty = bY1Full + S1;
  static constexpr int bA = bY1Empty + S1;  // 16 kernel-specific barriers
  static constexpr int bMmaFin = bA + 16;   // + issuer
  static constexpr int kNumBars = bMmaFin + 2;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kSmemBytes = kMisc + 16 + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
  static constexpr uint32_t kTmemCols = 512;
  static constexpr int kGroups = 4;               // softmax warpgroups per row
  static constexpr int kCols = kBlock / kGroups;  // columns of a row per thread
  static constexpr int kSoftmax = 128 * kGroups;  // softmax threads
  static constexpr int kThreads = kSoftmax + 128;  // softmax, 2 MMA, producer, store warps
  static constexpr int kWarpMma = 4 * kGroups;     // + issuer: 0 = score products, 1 = gradients
  static constexpr int kWarpProducer = 4 * kGroups + 2;
  static constexpr int kWarpStore = 4 * kGroups + 3;  // bulk stores of the staged outputs
  // Outputs are staged in the finished item's stationary buffer and leave by bulk stores
  // when there are two such buffers; with one, waiting for the stores would hold up the
  // next item's loads, so the softmax warps write their rows directly instead.
  static constexpr bool kStageOut = XB >= 2;
};

template <int D>
using DkdvCfg = BwdCfgT<D, (D == 64) ? 2 : 1, (D == 64) ? 4 : 2, (D == 64) ? 4 : 2, true>;
template <int D>
using DqCfg = BwdCfgT<D, (D == 64) ? 2 : 1, (D == 64) ? 5 : 3, (D == 64) ? 5 : 2, false>;

// Waits until every copy a ring's producer issued (n uses of stages 0..S-1) has landed.
__device__ __forceinline__ void drain_ring(uint32_t full_bar0, int S, int n) {
  for (int s = 0; s < S; ++s) {
    if (n > s) {
      const int last = s + S * ((n - 1 - s) / S);
      mbar_wait(full_bar0 + 8u * s, (last / S) & 1, nullptr);
    }
  }
}

// Writes this thread's NC fp32 accumulator columns (columns col0 .. col0+NC-1 of row `row`
// of a 128-row output tile), times `mul`, in bf16 to the shared-memory tile at `tile`, in
// the layout a TMA load of the tile's 64-column boxes leaves (128-byte rows; 16-byte chunks
// swizzled by the row's low three bits), ready for tma_store_3d. Writing the tile through
// one bulk store keeps each warp's stores from touching 32 separate rows of global memory.
template <int NC>
__device__ __forceinline__ void stage_acc_cols(uint32_t taddr, float mul, uint32_t tile, int row,
                                               int col0) {
  static_assert(NC % 16 == 0, "whole 16-column steps");
#pragma unroll
  for (int q = 0; q < NC / 16; ++q) {
    uint32_t o[16];
    tmem_ld16(taddr + 16 * q, o);
    tmem_wait_ld();
    reg_fence(o);
    uint32_t w[8];
#pragma unroll
    for (int c = 0; c < 8; ++c)
      w[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * mul, __uint_as_float(o[2 * c + 1]) * mul);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int col = col0 + 16 * q + 8 * k;
      const uint32_t addr = tile + (uint32_t)(col >> 6) * (kBlock * 128) + (uint32_t)row * 128 +
                            ((uint32_t)(((col & 63) >> 3) ^ (row & 7)) << 4);
      st_shared_v4(addr, w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
    }
  }
}

// Writes this thread's NC fp32 accumulator columns starting at `taddr`, times `mul`, as
// bf16 straight to global memory at `dst` (16 columns, 32 bytes, per step); used where no
// shared-memory buffer is free to stage the tile in.
template <int NC>
__device__ __forceinline__ void store_acc_cols(uint32_t taddr, float mul, __nv_bfloat16* dst,
                                               bool valid) {
  static_assert(NC % 16 == 0, "whole 16-column steps");
#pragma unroll
  for (int q = 0; q < NC / 16; ++q) {
    uint32_t o[16];
    tmem_ld16(taddr + 16 * q, o);
    tmem_wait_ld();
    reg_fence(o);
    uint32_t w[8];
#pragma unroll
    for (int c = 0; c < 8; ++c)
      w[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * mul, __uint_as_float(o[2 * c + 1]) * mul);
    if (valid) {
      st_global_v4(dst + 16 * q, w[0], w[1], w[2], w[3]);
      st_global_v4(dst + 16 * q + 8, w[4], w[5], w[6], w[7]);
    }
  }
}

// Loads 32 consecutive fp32 TMEM columns of this thread's lane.
__device__ __forceinline__ void load_cols32(uint32_t taddr, float (&x)[32]) {
  uint32_t u[32];
  tmem_ld32(taddr, u);
  tmem_wait_ld();
  reg_fence(u);
#pragma unroll
  for (int c = 0; c < 32; ++c) x[c] = __uint_as_float(u[c]);
}

// TMEM column (from the buffer base) of K-step kk of a bf16 A operand that the softmax
// warpgroups packed: group h holds its 32 bf16 entries (16 columns) over the first half
// of its own 32 fp32 columns, so K-steps 2h and 2h+1 sit at columns 32h and 32h+8.
__device__ __forceinline__ constexpr uint32_t packed_col(int kk) {
  return 8u * kk + 16u * (kk >> 1);
}

// Item k of the persistent schedule: the (batch*head, stationary tile). Masked problems
// use chunks of heads with the longest items first (see chunked_item): key tiles in
// increasing order for dK/dV, query tiles in decreasing order for dQ.
// Returns false when the stationary tile lies past the sequence's real length (a
// variable-length batch): such an item has no work, and every role skips it without
// advancing its counters. `mk` is the item's mask, over the real length.
template <bool kPacked = false>
__device__ __forceinline__ bool bwd_item(int k, const BwdArgs& a, bool rising, int& bh,
                                         int& tile, Mask& mk) {
  const int* const cu = kPacked ? a.cu : nullptr;
  if (a.paired) {
    if (!paired_item(k, (int)gridDim.x, a.n_double, a.n_tiles, rising, bh, tile)) return false;
  } else if (a.sorted) {
    int u;
    if (!varlen_item(k, (int)gridDim.x, a.sched, a.n_tiles, a.H, bh, u)) return false;
    const int n = real_length(a.seq_len, cu, bh, a.H, a.N);
    mk = Mask{n, a.left, a.right};
    // key tiles count from the end of the sequence, query tiles from its start
    tile = rising ? num_tiles(n) - 1 - u : u;
    return true;
  } else if (a.longest_first) {
    chunked_item(k, a.BH, a.n_tiles, a.group, rising, bh, tile);
  } else {
    bh = k / a.n_tiles;
    tile = k % a.n_tiles;
  }
  const int n = real_length(a.seq_len, cu, bh, a.H, a.N);
  mk = Mask{n, a.left, a.right};
  return tile < num_tiles(n);
}

template <typename C>
__device__ __forceinline__ uint32_t bwd_setup(uint8_t* smem, int warp) {
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMisc);
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  return *tmem_slot;
}

template <typename C>
__device__ __forceinline__ void bwd_teardown(uint32_t tmem, int warp) {
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------------------------------------------------
// dK, dV: persistent CTAs over items (batch*head, key tile j). X0 = K_j, X1 = V_j; per
// stage Y0 = Q_i with the LSE (log2 units) and delta of its 128 rows, Y1 = dO_i.
// TMEM: S^T in kSBufs buffers (two for head_dim 64, so that S^T of the next query tile
// is computed while the softmax works on this one), dP^T, dK, dV. Warpgroup h writes its
// bf16 part of P^T over the first 16 of its own 32 fp32 columns of S^T, so the A operand
// of dV takes K-step kk from column packed_col(kk). With two S^T buffers, dS^T goes over
// the other 16 of those columns (packed_col(kk) + 16), whose scores are in registers by
// then: dP^T is free as soon as the softmax has loaded it, and dP^T of the next query
// tile is computed while dS^T and dK of this one are. With one buffer, dS^T goes over
// the first half of the group's dP^T columns and dP^T waits for dK.
// Two MMA issuers: one computes S^T and dP^T of each query tile in order, the other
// dV += P^T dO and dK += dS^T Q as soon as the softmax publishes P^T and dS^T. Tile
// counters (for barrier parities) run over all items of the CTA.
// ------------------------------------------------------------------------------------
// kFeat: kFeatAlibi, the scores carry the linear bias -m_h |i - j| (m_h = alibi[bh % H]);
// kFeatKpad, keys flagged in a.kpad get no attention; kFeatDropout, the forward's keep
// flags Z are regenerated: dV += (P o Z / (1-p'))^T dO and dS = P o (dP o Z / (1-p') - delta).
// A warp owns 32 keys and 32 queries of each tile; lane l draws the flags of query l for
// all 32 keys (two Philox calls), and 32 ballots hand each lane the flags of its own key.
template <int D, int kFeat = 0>
__global__ void __launch_bounds__(DkdvCfg<D>::kThreads, 1)
    fa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmdO,
                       const __grid_constant__ CUtensorMap tmdK,
                       const __grid_constant__ CUtensorMap tmdV, const BwdArgs a) {
  using C = DkdvCfg<D>;
  static_assert(C::kStages0 == C::kStages1, "one ring of (Q, dO) stages");
  constexpr bool kAlibi = (kFeat & kFeatAlibi) != 0;
  constexpr bool kKpad = (kFeat & kFeatKpad) != 0;
  constexpr bool kDropout = (kFeat & kFeatDropout) != 0;
  constexpr bool kPacked = (kFeat & kFeatPacked) != 0;
  const int* const cu = kPacked ? a.cu : nullptr;  // a packed batch's cumulative lengths
  constexpr int kSBufs = (D == 64) ? 2 : 1;
  constexpr bool kDsInS = kSBufs == 2;               // dS^T over the second half of S^T
  // With one S^T buffer (head_dim 128) the products go in two 64-query halves: S^T, dP^T,
  // dV and dK of half h have barriers of their own, so S^T of half h of the next tile waits
  // only for dV of half h (and dP^T for dK of half h), while the other half's products
  // run. Softmax warpgroups 0, 1 own half 0 of the query columns, 2, 3 half 1.
  constexpr bool kHalves = !kDsInS;
  constexpr uint32_t tS = 0;                         // + 128 * buffer
  constexpr uint32_t tDP = 128 * kSBufs, tDK = tDP + 128, tDV = tDK + D;
  static_assert(tDV + D <= C::kTmemCols, "tensor memory columns");
  // per S^T buffer: S^T full, P^T full, buffer free (the last product that reads it, dV
  // or with kDsInS dK, has completed); dP^T full, dS^T full, dP^T free (loaded by the
  // softmax with kDsInS, else read by dK), dK/dV read by the epilogue, dK/dV of the item
  // complete. Every barrier that one side may complete twice before the other has waited
  // once is kept per buffer, so that no parity wait can mistake a later phase for the one
  // it wants.
  // With kDsInS, dS^T full is kept per buffer (a second tile's dS^T may be published before
  // dK has waited for the first), in the slots of S^T free, which kDsInS does not use (the
  // ring stage of tile t - 2 frees its S^T buffer).
  constexpr int bSFull = C::bA + 0, bPFull = C::bA + 2, bSFree = C::bA + 4,
                bDPFull = C::bA + 6, bDSFull = kDsInS ? C::bA + 4 : C::bA + 7,
                bDPFree = C::bA + 8, bAccFree = C::bA + 9, bAccReady = C::bA + 10,
                bStaged = C::bA + 11;
  // kHalves: dP^T full, dS^T full and dP^T free of half 1 (those above serve half 0; S^T
  // full, P^T full and S^T free are kept per half in their two slots)
  constexpr int bDPFull1 = C::bA + 12, bDSFull1 = C::bA + 13, bDPFree1 = C::bA + 14;
  auto half_bar = [](int b0, int b1, int h) { return h ? b1 : b0; };
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMisc + 4);
  auto bar = [&](int i) -> uint32_t { return sb + C::kBar + 8u * i; };

  if (threadIdx.x == 0) {
    for (int b = 0; b < C::kXBufs; ++b) {
      mbar_init(bar(C::bXFull + b), 1);
      mbar_init(bar(C::bXEmpty + b), 1);
    }
    // One stage of the ring holds Q_i (with its statistics) and dO_i; it is released by
    // one commit after dK(i), the last product of the query tile: by then S^T, dP^T and dV
    // of the tile have completed too (the softmax consumed S^T and dP^T before it
    // published dS^T, and dV was issued before dK by the same thread). Each commit holds
    // its issuing thread for a few hundred clocks, so releases are not made separately.
    for (int s = 0; s < C::kStages0; ++s) {
      mbar_init(bar(C::bY0Full + s), 1);
      mbar_init(bar(C::bY1Full + s), 1);
      mbar_init(bar(C::bY0Empty + s), 1);
    }
    // softmax warps that publish a P^T or dS^T: all of them, or with kHalves those of a half
    constexpr int kPub = kHalves ? C::kSoftmax / 64 : C::kSoftmax / 32;
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(bSFull + b), 1);
      mbar_init(bar(bPFull + b), kPub);
      mbar_init(bar(bSFree + b), kDsInS ? C::kSoftmax / 32 : 1);  // dS^T full with kDsInS
      mbar_init(bar(C::bMmaFin + b), 1);
    }
    mbar_init(bar(bDPFull), 1);
    if (!kDsInS) mbar_init(bar(bDSFull), kPub);
    mbar_init(bar(bDPFree), kDsInS ? C::kSoftmax / 32 : 1);
    if (kHalves) {
      mbar_init(bar(bDPFull1), 1);
      mbar_init(bar(bDSFull1), kPub);
      mbar_init(bar(bDPFree1), 1);
    }
    mbar_init(bar(bAccFree), C::kSoftmax / 32);
    mbar_init(bar(bAccReady), 1);
    mbar_init(bar(bStaged), C::kSoftmax / 32);
    *abort_flag = 0;
    fence_mbar_init();
  }
  const uint32_t tmem = bwd_setup<C>(smem, warp);

  if (warp == C::kWarpProducer) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_map(&tmQ);
      tma_prefetch_map(&tmK);
      tma_prefetch_map(&tmV);
      tma_prefetch_map(&tmdO);
      int items = 0, n = 0;  // items started; query tiles loaded into the ring
      bool ok = true;
      for (int k = blockIdx.x; ok && k < a.n_items; k += gridDim.x) {
        int bh, j;
        Mask mk;
        if (!bwd_item<kPacked>(k, a, true, bh, j, mk)) continue;
        int i_lo, i_hi;
        q_tiles_for_kv_tile(j, mk, i_lo, i_hi);
        const int xb = items % C::kXBufs, xu = items / C::kXBufs;
        const int base = seq_base(cu, bh, a.H), ty = tma_y(cu, bh, a.H, j * kBlock);
        if (!mbar_wait(bar(C::bXEmpty + xb), (xu & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(C::bXFull + xb), 2 * C::kTile);
        for (int r = 0; r < C::kRegions; ++r) {
          tma_load_3d(sb + C::kX0 + xb * 2 * C::kTile + r * C::kRegionBytes, &tmK,
                      bar(C::bXFull + xb), r * 64, ty, tma_z(cu, bh, base, j * kBlock));
          tma_load_3d(sb + C::kX1 + xb * 2 * C::kTile + r * C::kRegionBytes, &tmV,
                      bar(C::bXFull + xb), r * 64, ty, tma_z(cu, bh, base, j * kBlock));
        }
        ++items;
        for (int i = i_lo; i <= i_hi; ++i, ++n) {
          const int s = n % C::kStages0;
          if (!mbar_wait(bar(C::bY0Empty + s), ((n / C::kStages0) & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(C::bY0Full + s), C::kTile + 2 * 512);
          const int yi = tma_y(cu, bh, a.H, i * kBlock), zi = tma_z(cu, bh, base, i * kBlock);
          for (int r = 0; r < C::kRegions; ++r)
            tma_load_3d(sb + C::kY0 + s * C::kTile + r * C::kRegionBytes, &tmQ,
                        bar(C::bY0Full + s), r * 64, yi, zi);
          // LSE*log2e and delta of the 128 rows of query tile i (512 bytes each)
          const float* st = a.stats + (size_t)bh * a.Np + (size_t)i * kBlock;
          bulk_load(sb + C::kLse + s * 512, st, 512, bar(C::bY0Full + s));
          bulk_load(sb + C::kDelta + s * 512, st + a.stat_rows, 512, bar(C::bY0Full + s));
          mbar_arrive_expect_tx(bar(C::bY1Full + s), C::kTile);
          for (int r = 0; r < C::kRegions; ++r)
            tma_load_3d(sb + C::kY1 + s * C::kTile + r * C::kRegionBytes, &tmdO,
                        bar(C::bY1Full + s), r * 64, yi, zi);
        }
      }
      // Drain: every copy issued must have landed before the CTA may exit.
      for (int x = (items > C::kXBufs ? items - C::kXBufs : 0); x < items; ++x)
        mbar_wait(bar(C::bXFull + x % C::kXBufs), (x / C::kXBufs) & 1, nullptr);
      drain_ring(bar(C::bY0Full), C::kStages0, n);
      drain_ring(bar(C::bY1Full), C::kStages0, n);
    }
    __syncwarp();
  } else if (warp == C::kWarpMma) {
    // ------------------------------------------------------------------ score products
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);
      int items = 0, t = 0;  // items and query tiles started (all items)
      bool ok = true;
      for (int k = blockIdx.x; ok && k < a.n_items; k += gridDim.x) {
        int bh, j;
        Mask mk;
        if (!bwd_item<kPacked>(k, a, true, bh, j, mk)) continue;
        int i_lo, i_hi;
        q_tiles_for_kv_tile(j, mk, i_lo, i_hi);
        const int xb = items % C::kXBufs, xu = items / C::kXBufs;
        if (!mbar_wait(bar(C::bXFull + xb), xu & 1, abort_flag)) break;
        for (int i = i_lo; i <= i_hi; ++i, ++t) {
          const int b = t % kSBufs, s0 = t % C::kStages0, s1 = s0;
          if constexpr (kHalves) {
            // S^T_h = K_j Q_i[64h ..]^T, then dP^T_h = V_j dO_i[64h ..]^T, each once the
            // previous tile's product that read its columns (dV_h, dK_h) has completed
            constexpr uint32_t idS64 = idesc_bf16_f32(128, 64, false, false);
            if (!mbar_wait(bar(C::bY0Full + s0), (t / C::kStages0) & 1, abort_flag)) {
              ok = false;
              break;
            }
            for (int h = 0; h < 2 && ok; ++h) {
              if (t >= 1 && !mbar_wait(bar(bSFree + h), (t - 1) & 1, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint64_t dx = sdesc_sw128(sb + C::kX0 + xb * 2 * C::kTile, 16, 1024);
              const uint64_t dy = sdesc_sw128(sb + C::kY0 + s0 * C::kTile + 64 * 128 * h, 16, 1024);
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = (kk >> 2) * C::kRegionBytes + (kk & 3) * 32;
                mma_ss(tmem + tS + 64u * h, sdesc_add(dx, off), sdesc_add(dy, off), idS64,
                       kk > 0);
              }
              tc_commit(bar(bSFull + h));
            }
            if (!ok) break;
            if (!mbar_wait(bar(C::bY1Full + s1), (t / C::kStages1) & 1, abort_flag)) {
              ok = false;
              break;
            }
            for (int h = 0; h < 2 && ok; ++h) {
              if (t >= 1 &&
                  !mbar_wait(bar(half_bar(bDPFree, bDPFree1, h)), (t - 1) & 1, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint64_t dx = sdesc_sw128(sb + C::kX1 + xb * 2 * C::kTile, 16, 1024);
              const uint64_t dy = sdesc_sw128(sb + C::kY1 + s1 * C::kTile + 64 * 128 * h, 16, 1024);
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = (kk >> 2) * C::kRegionBytes + (kk & 3) * 32;
                mma_ss(tmem + tDP + 64u * h, sdesc_add(dx, off), sdesc_add(dy, off), idS64,
                       kk > 0);
              }
              tc_commit(bar(half_bar(bDPFull, bDPFull1, h)));
            }
            if (!ok) break;
            if (!C::kStageOut && i == i_hi) tc_commit(bar(C::bXEmpty + xb));
            continue;
          }
          // S^T = K_j Q_i^T, once the products that read its buffer's P^T (and dS^T) have
          // completed: dV of the previous tile, or with kDsInS dK of tile t - 2, whose
          // completion releases that tile's ring stage
          const int tp = t - kSBufs;
          if (!mbar_wait(bar(C::bY0Full + s0), (t / C::kStages0) & 1, abort_flag) ||
              (tp >= 0 && !(kDsInS ? mbar_wait(bar(C::bY0Empty + tp % C::kStages0),
                                               (tp / C::kStages0) & 1, abort_flag)
                                   : mbar_wait(bar(bSFree + b), ((t / kSBufs) - 1) & 1,
                                               abort_flag)))) {
            ok = false;
            break;
          }
          tc_fence_after();
          {
            const uint64_t dx = sdesc_sw128(sb + C::kX0 + xb * 2 * C::kTile, 16, 1024);
            const uint64_t dy = sdesc_sw128(sb + C::kY0 + s0 * C::kTile, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * C::kRegionBytes + (kk & 3) * 32;
              mma_ss(tmem + tS + 128u * b, sdesc_add(dx, off), sdesc_add(dy, off), idS, kk > 0);
            }
          }
          tc_commit(bar(bSFull + b));
          // dP^T = V_j dO_i^T, once the previous tile's dP^T is free
          if (!mbar_wait(bar(C::bY1Full + s1), (t / C::kStages1) & 1, abort_flag) ||
              (t >= 1 && !mbar_wait(bar(bDPFree), (t - 1) & 1, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          {
            const uint64_t dx = sdesc_sw128(sb + C::kX1 + xb * 2 * C::kTile, 16, 1024);
            const uint64_t dy = sdesc_sw128(sb + C::kY1 + s1 * C::kTile, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * C::kRegionBytes + (kk & 3) * 32;
              mma_ss(tmem + tDP, sdesc_add(dx, off), sdesc_add(dy, off), idS, kk > 0);
            }
          }
          tc_commit(bar(bDPFull));
          // without staged outputs, K_j and V_j are free after their last product
          if (!C::kStageOut && i == i_hi) tc_commit(bar(C::bXEmpty + xb));
        }
        ++items;
      }
      tc_commit(bar(C::bMmaFin));
      mbar_wait(bar(C::bMmaFin), 0, nullptr);
    }
    __syncwarp();
  } else if (warp == C::kWarpMma + 1) {
    // ------------------------------------------------------------------ dV, dK products
    if (lane == 0) {
      constexpr uint32_t idA = idesc_bf16_f32(128, D, false, true);
      int items = 0, t = 0;
      bool ok = true;
      for (int k = blockIdx.x; ok && k < a.n_items; k += gridDim.x) {
        int bh, j;
        Mask mk;
        if (!bwd_item<kPacked>(k, a, true, bh, j, mk)) continue;
        int i_lo, i_hi;
        q_tiles_for_kv_tile(j, mk, i_lo, i_hi);
        for (int i = i_lo; i <= i_hi; ++i, ++t) {
          const int b = t % kSBufs, s0 = t % C::kStages0, s1 = s0;
          const bool first = i == i_lo;
          if constexpr (kHalves) {
            // dV += P^T_h dO_i[64h ..] (K-steps 4h .. 4h+3) as each half of P^T is
            // published, then dK += dS^T_h Q_i[64h ..] likewise; the item's first product
            // overwrites dV (dK), which the previous item's epilogue must have read
            if (!mbar_wait(bar(C::bY1Full + s1), (t / C::kStages1) & 1, abort_flag) ||
                (first && items > 0 && !mbar_wait(bar(bAccFree), (items - 1) & 1, abort_flag))) {
              ok = false;
              break;
            }
            const uint64_t dyo = sdesc_sw128(sb + C::kY1 + s1 * C::kTile, C::kRegionBytes, 1024);
            for (int h = 0; h < 2 && ok; ++h) {
              if (!mbar_wait(bar(bPFull + h), t & 1, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
#pragma unroll
              for (int kq = 0; kq < 4; ++kq) {
                const int kk = 4 * h + kq;
                mma_ts(tmem + tDV, tmem + tS + packed_col(kk), sdesc_add(dyo, kk * 2048), idA,
                       (!first || kk > 0) ? 1u : 0u);
              }
              tc_commit(bar(bSFree + h));
            }
            if (!ok) break;
            if (!mbar_wait(bar(C::bY0Full + s0), (t / C::kStages0) & 1, abort_flag)) {
              ok = false;
              break;
            }
            const uint64_t dyq = sdesc_sw128(sb + C::kY0 + s0 * C::kTile, C::kRegionBytes, 1024);
            for (int h = 0; h < 2 && ok; ++h) {
              if (!mbar_wait(bar(half_bar(bDSFull, bDSFull1, h)), t & 1, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
#pragma unroll
              for (int kq = 0; kq < 4; ++kq) {
                const int kk = 4 * h + kq;
                mma_ts(tmem + tDK, tmem + tDP + packed_col(kk), sdesc_add(dyq, kk * 2048), idA,
                       (!first || kk > 0) ? 1u : 0u);
              }
              tc_commit(bar(half_bar(bDPFree, bDPFree1, h)));
            }
            if (!ok) break;
            // the tile's ring stage is free
            tc_commit(bar(C::bY0Empty + s0));
            if (i == i_hi) tc_commit(bar(bAccReady));  // dK, dV of the item are complete
            continue;
          }
          // dV += P^T dO_i; the item's first product overwrites dV, which the previous
          // item's epilogue must have read
          if (!mbar_wait(bar(C::bY1Full + s1), (t / C::kStages1) & 1, abort_flag) ||
              !mbar_wait(bar(bPFull + b), (t / kSBufs) & 1, abort_flag) ||
              (first && items > 0 && !mbar_wait(bar(bAccFree), (items - 1) & 1, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          {
            const uint64_t dy = sdesc_sw128(sb + C::kY1 + s1 * C::kTile, C::kRegionBytes, 1024);
#pragma unroll
            for (int kk = 0; kk < kBlock / 16; ++kk)
              mma_ts(tmem + tDV, tmem + tS + 128u * b + packed_col(kk), sdesc_add(dy, kk * 2048),
                     idA, (!first || kk > 0) ? 1u : 0u);
          }
          if (!kDsInS) tc_commit(bar(bSFree + b));
          // dK += dS^T Q_i
          if (!mbar_wait(bar(C::bY0Full + s0), (t / C::kStages0) & 1, abort_flag) ||
              !mbar_wait(bar(bDSFull + (kDsInS ? b : 0)), (kDsInS ? t / 2 : t) & 1,
                         abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          {
            const uint64_t dy = sdesc_sw128(sb + C::kY0 + s0 * C::kTile, C::kRegionBytes, 1024);
            const uint32_t ta = tmem + (kDsInS ? tS + 128u * b + 16u : tDP);
#pragma unroll
            for (int kk = 0; kk < kBlock / 16; ++kk)
              mma_ts(tmem + tDK, ta + packed_col(kk), sdesc_add(dy, kk * 2048), idA,
                     (!first || kk > 0) ? 1u : 0u);
          }
          // the tile's ring stage (and with kDsInS its S^T buffer) is free
          tc_commit(bar(C::bY0Empty + s0));
          if (!kDsInS) tc_commit(bar(bDPFree));
          if (i == i_hi) tc_commit(bar(bAccReady));  // dK, dV of the item are complete
        }
        ++items;
      }
      tc_commit(bar(C::bMmaFin + 1));
      mbar_wait(bar(C::bMmaFin + 1), 0, nullptr);
    }
    __syncwarp();
  } else if (warp == C::kWarpStore) {
    // ------------------------------------------------------------------ output stores
    // dK, dV of each item leave through two bulk stores from the buffer the softmax warps
    // staged them in; the buffer goes back to the producer once the stores have read it.
    if (lane == 0 && C::kStageOut) {
      int items = 0;
      for (int k = blockIdx.x; k < a.n_items; k += gridDim.x) {
        int bh, j;
        Mask mk;
        if (!bwd_item<kPacked>(k, a, true, bh, j, mk)) continue;
        const int xb = items % C::kXBufs;
        if (!mbar_wait(bar(bStaged), items & 1, abort_flag)) break;
        ++items;
        // (a partial tile of a packed batch was written row by row)
        if (whole_tile_store(cu, a.total, mk.N, seq_base(cu, bh, a.H), j * kBlock)) {
          const int base = seq_base(cu, bh, a.H);
          const int ty = tma_y(cu, bh, a.H, j * kBlock), tz = tma_z(cu, bh, base, j * kBlock);
          for (int r = 0; r < C::kRegions; ++r) {
            tma_store_3d(&tmdK, sb + C::kX0 + xb * 2 * C::kTile + r * C::kRegionBytes, r * 64,
                         ty, tz);
            tma_store_3d(&tmdV, sb + C::kX1 + xb * 2 * C::kTile + r * C::kRegionBytes, r * 64,
                         ty, tz);
          }
        }
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
    const int h = warp >> 2;              // query columns NC*h .. NC*h+NC-1 of each tile
    const int t_row = threadIdx.x & 127;  // key row in the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const float sl2 = a.scale_log2;
    int g = 0, items = 0;
    bool ok = true;
    for (int k = blockIdx.x; ok && k < a.n_items; k += gridDim.x) {
      int bh, j;
      Mask mk;
      if (!bwd_item<kPacked>(k, a, true, bh, j, mk)) continue;
      int i_lo, i_hi;
      q_tiles_for_kv_tile(j, mk, i_lo, i_hi);
      const int n_it = i_hi - i_lo + 1;
      const int c = j * kBlock + t_row;  // this thread's key
      const float slope2 = kAlibi ? a.alibi[bh % a.H] * kLog2e : 0.f;
      // a padded key gets no attention from any query: its rows of P^T and dS^T are zero
      const bool key_padded = kKpad && c < a.N && a.kpad[(size_t)(bh / a.H) * a.N + c] != 0;
      for (int it = 0; it < n_it; ++it) {
        const int i = i_lo + it;
        const int t = g + it;
        const int s = t % C::kStages0;
        // keep flags of this thread's key for the queries NC*h + r of tile i (bit r)
        uint32_t keep = ~0u;
        if (kDropout) {
          const uint32_t blk = (uint32_t)(8 * j + 2 * (warp & 3));
          const uint32_t qrow = (uint32_t)(i * kBlock + NC * h + lane);
          const uint32_t mine = keep_bits16(a.drop, blk, qrow, (uint32_t)bh) |
                                (keep_bits16(a.drop, blk + 1, qrow, (uint32_t)bh) << 16);
          static_assert(NC == 32, "one lane per query of the warp's 32");
#pragma unroll
          for (int b = 0; b < 32; ++b) {
            const uint32_t col = __ballot_sync(0xffffffffu, (mine >> b) & 1u);
            keep = (lane == b) ? col : keep;
          }
        }
        if (!mbar_wait_warp(bar(C::bY0Full + s), (t / C::kStages0) & 1, abort_flag) ||
            !mbar_wait_warp(bar(bSFull + (kHalves ? (h >> 1) : t % kSBufs)), (t / kSBufs) & 1,
                            abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float* lse_s = reinterpret_cast<const float*>(smem + C::kLse + s * 512) + NC * h;
        const float* del_s = reinterpret_cast<const float*>(smem + C::kDelta + s * 512) + NC * h;
        float p[NC];
        const uint32_t tSb = tmem + lane_base + tS + 128u * (t % kSBufs) + NC * h;
        load_cols32(tSb, p);
#pragma unroll
        for (int r = 0; r < NC; r += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(lse_s + r);
          float b4[4] = {0.f, 0.f, 0.f, 0.f};
          if (kAlibi) {
            // -m |query - key| in log2 units for the queries of these four columns
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
          uint32_t pk[NC / 2];
          if (kDropout) {
            // the weights that multiplied V: P o Z / (1 - p')
            const float ks = a.drop.keep_scale;
#pragma unroll
            for (int r = 0; r < NC / 2; ++r)
              pk[r] = pack_bf16x2(((keep >> (2 * r)) & 1u) ? p[2 * r] * ks : 0.f,
                                  ((keep >> (2 * r + 1)) & 1u) ? p[2 * r + 1] * ks : 0.f);
          } else {
#pragma unroll
            for (int r = 0; r < NC / 2; ++r) pk[r] = pack_bf16x2(p[2 * r], p[2 * r + 1]);
          }
          tmem_st16(tSb, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive_warp(bar(bPFull + (kHalves ? (h >> 1) : t % kSBufs)));
        if (!mbar_wait_warp(bar(kHalves ? half_bar(bDPFull, bDPFull1, h >> 1) : bDPFull), t & 1,
                            abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float dp[NC];
        load_cols32(tmem + lane_base + tDP + NC * h, dp);
        if (kDsInS) {
          // dP^T is in registers: the next query tile's dP^T may overwrite it
          tc_fence_before();
          mbar_arrive_warp(bar(bDPFree));
        }
        if (kDropout) {
          // dP o Z / (1 - p'): the gradient reaching the weights before dropout
          const float ks = a.drop.keep_scale;
#pragma unroll
          for (int r = 0; r < NC; ++r) dp[r] = ((keep >> r) & 1u) ? dp[r] * ks : 0.f;
        }
        uint32_t w[NC / 2];
#pragma unroll
        for (int e = 0; e < NC / 2; e += 2) {
          const int r0 = 2 * e;
          const float4 d4 = *reinterpret_cast<const float4*>(del_s + r0);
          // two columns per instruction (packed fp32 add and multiply of sm_100): the same
          // roundings as the scalar form, half the issue slots
          const float2 v0 = __fmul2_rn(make_float2(p[r0], p[r0 + 1]),
                                       __fadd2_rn(make_float2(dp[r0], dp[r0 + 1]),
                                                  make_float2(-d4.x, -d4.y)));
          const float2 v1 = __fmul2_rn(make_float2(p[r0 + 2], p[r0 + 3]),
                                       __fadd2_rn(make_float2(dp[r0 + 2], dp[r0 + 3]),
                                                  make_float2(-d4.z, -d4.w)));
          w[e] = pack_bf16x2(v0.x, v0.y);
          w[e + 1] = pack_bf16x2(v1.x, v1.y);
        }
        // bf16 dS^T goes over the second half of this warpgroup's own fp32 S^T columns
        // (kDsInS) or the first half of its dP^T columns
        tmem_st16(kDsInS ? tSb + 16 : tmem + lane_base + tDP + NC * h, w);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive_warp(bar(kHalves ? half_bar(bDSFull, bDSFull1, h >> 1)
                                     : bDSFull + (kDsInS ? t % kSBufs : 0)));
      }
      if (!ok) break;
      g += n_it;
      // once per item, after its last dK (which follows its last dV)
      if (!mbar_wait_warp(bar(bAccReady), items & 1, abort_flag)) {
        ok = false;
        break;
      }
      // With staged outputs, dK and dV go through the item's K_j, V_j buffer, which no
      // product reads any more; the store warp writes them out and hands the buffer back to
      // the producer. Otherwise each thread writes its part of its row directly.
      const int xb = items % C::kXBufs;
      const uint32_t tK = sb + C::kX0 + xb * 2 * C::kTile, tV = sb + C::kX1 + xb * 2 * C::kTile;
      ++items;
      tc_fence_after();
      constexpr int NO = D / C::kGroups;
      if (C::kStageOut && whole_tile_store(cu, a.total, mk.N, seq_base(cu, bh, a.H), j * kBlock)) {
        stage_acc_cols<NO>(tmem + lane_base + tDV + NO * h, 1.f, tV, t_row, NO * h);
        stage_acc_cols<NO>(tmem + lane_base + tDK + NO * h, a.scale, tK, t_row, NO * h);
        fence_async_smem();
      } else {
        const int base = seq_base(cu, bh, a.H);
        const bool valid = row_written(cu, a.total, a.N, mk.N, base, c);
        const size_t off = row_at(cu, bh, a.H, a.N, base, valid ? c : 0, D) + NO * h;
        store_acc_cols<NO>(tmem + lane_base + tDV + NO * h, 1.f, a.out1 + off, valid);
        store_acc_cols<NO>(tmem + lane_base + tDK + NO * h, a.scale, a.out0 + off, valid);
      }
      // dK, dV have been read: the next item's first products may overwrite them
      tc_fence_before();
      mbar_arrive_warp(bar(bAccFree));
      if (C::kStageOut) mbar_arrive_warp(bar(bStaged));
    }
  }
  bwd_teardown<C>(tmem, warp);
}

// ------------------------------------------------------------------------------------
// dQ: persistent CTAs over items (batch*head, query tile i). X0 = Q_i, X1 = dO_i; per
// stage Y0 = K_j, Y1 = V_j. TMEM: S in two buffers at 0 and 128 (bf16 dS goes over S,
// each warpgroup over the first half of its own 32 columns), dP at 256, dQ at 384. Two
// MMA issuers: one computes S and dP of each key tile in order, the other dQ += dS K_j
// as soon as the softmax publishes dS. Tile counters run over all items.
// ------------------------------------------------------------------------------------
// kFeat: kFeatAlibi, the scores carry the linear bias -m_h |i - j| (m_h = alibi[bh % H]);
// kFeatKpad, keys flagged in a.kpad get no attention; kFeatDropout, the forward's keep
// flags Z are regenerated and dS = P o (dP o Z / (1-p') - delta).
template <int D, int kFeat = 0>
__global__ void __launch_bounds__(DqCfg<D>::kThreads, 1)
    fa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmdO,
                     const __grid_constant__ CUtensorMap tmdQ, const BwdArgs a) {
  using C = DqCfg<D>;
  // With equal rings, one stage holds K_j and V_j and is released by one commit after
  // dQ(j), the last product of the key tile (S and dP of the tile have completed by then:
  // the softmax consumed both before it published dS); the S buffer of tile t - 2 is free
  // with that tile's stage. Otherwise K_j is released by S and dQ, V_j by dP, and the S
  // buffer by its own barrier.
  constexpr bool kOneRelease = C::kStages0 == C::kStages1;
  constexpr bool kAlibi = (kFeat & kFeatAlibi) != 0;
  constexpr bool kKpad = (kFeat & kFeatKpad) != 0;
  constexpr bool kDropout = (kFeat & kFeatDropout) != 0;
  constexpr bool kPacked = (kFeat & kFeatPacked) != 0;
  const int* const cu = kPacked ? a.cu : nullptr;  // a packed batch's cumulative lengths
  constexpr uint32_t tS0 = 0, tDP = 256, tDQ = 384;
  // per S buffer: S full, dS full, dQ done (dQ read that buffer's dS); dP full, dP free;
  // dQ read by the epilogue, dQ of the item complete
  constexpr int bSFull = C::bA + 0, bDSFull = C::bA + 2, bDQDone = C::bA + 4,
                bDPFull = C::bA + 6, bDPFree = C::bA + 7, bAccFree = C::bA + 8,
                bAccReady = C::bA + 9, bStaged = C::bA + 10;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMisc + 4);
  auto bar = [&](int k) -> uint32_t { return sb + C::kBar + 8u * k; };

  if (threadIdx.x == 0) {
    for (int b = 0; b < C::kXBufs; ++b) {
      mbar_init(bar(C::bXFull + b), 1);
      mbar_init(bar(C::bXEmpty + b), 1);
    }
    for (int s = 0; s < C::kStages0; ++s) {
      mbar_init(bar(C::bY0Full + s), 1);
      mbar_init(bar(C::bY0Empty + s), kOneRelease ? 1 : 2);
    }
    for (int s = 0; s < C::kStages1; ++s) {
      mbar_init(bar(C::bY1Full + s), 1);
      mbar_init(bar(C::bY1Empty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(bSFull + b), 1);
      mbar_init(bar(bDSFull + b), C::kSoftmax / 32);
      mbar_init(bar(bDQDone + b), 1);
      mbar_init(bar(C::bMmaFin + b), 1);
    }
    mbar_init(bar(bDPFull), 1);
    mbar_init(bar(bDPFree), C::kSoftmax / 32);
    mbar_init(bar(bAccFree), C::kSoftmax / 32);
    mbar_init(bar(bAccReady), 1);
    mbar_init(bar(bStaged), C::kSoftmax / 32);
    *abort_flag = 0;
    fence_mbar_init();
  }
  const uint32_t tmem = bwd_setup<C>(smem, warp);

  if (warp == C::kWarpProducer) {
    if (lane == 0) {
      tma_prefetch_map(&tmQ);
      tma_prefetch_map(&tmK);
      tma_prefetch_map(&tmV);
      tma_prefetch_map(&tmdO);
      int items = 0, n0 = 0, n1 = 0;
      bool ok = true;
      for (int k = blockIdx.x; ok && k < a.n_items; k += gridDim.x) {
        int bh, i;
        Mask mk;
        if (!bwd_item<kPacked>(k, a, false, bh, i, mk)) continue;
        int j_lo, j_hi;
        kv_tiles_for_q_tile(i, mk, j_lo, j_hi);
        const int xb = items % C::kXBufs, xu = items / C::kXBufs;
        const int base = seq_base(cu, bh, a.H);
        if (!mbar_wait(bar(C::bXEmpty + xb), (xu & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(C::bXFull + xb), 2 * C::kTile);
        const int yi = tma_y(cu, bh, a.H, i * kBlock), zi = tma_z(cu, bh, base, i * kBlock);
        for (int r = 0; r < C::kRegions; ++r) {
          tma_load_3d(sb + C::kX0 + xb * 2 * C::kTile + r * C::kRegionBytes, &tmQ,
                      bar(C::bXFull + xb), r * 64, yi, zi);
          tma_load_3d(sb + C::kX1 + xb * 2 * C::kTile + r * C::kRegionBytes, &tmdO,
                      bar(C::bXFull + xb), r * 64, yi, zi);
        }
        ++items;
        for (int jj = j_lo; jj <= j_hi; ++jj) {
          const int s0 = n0 % C::kStages0, s1 = n1 % C::kStages1;
          if (!mbar_wait(bar(C::bY0Empty + s0), ((n0 / C::kStages0) & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(C::bY0Full + s0), C::kTile);
          for (int r = 0; r < C::kRegions; ++r)
            tma_load_3d(sb + C::kY0 + s0 * C::kTile + r * C::kRegionBytes, &tmK,
                        bar(C::bY0Full + s0), r * 64, tma_y(cu, bh, a.H, jj * kBlock),
                        tma_z(cu, bh, base, jj * kBlock));
          ++n0;
          if (!kOneRelease &&
              !mbar_wait(bar(C::bY1Empty + s1), ((n1 / C::kStages1) & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(C::bY1Full + s1), C::kTile);
          for (int r = 0; r < C::kRegions; ++r)
            tma_load_3d(sb + C::kY1 + s1 * C::kTile + r * C::kRegionBytes, &tmV,
                        bar(C::bY1Full + s1), r * 64, tma_y(cu, bh, a.H, jj * kBlock),
                        tma_z(cu, bh, base, jj * kBlock));
          ++n1;
        }
      }
      for (int n = (items > C::kXBufs ? items - C::kXBufs : 0); n < items; ++n)
        mbar_wait(bar(C::bXFull + n % C::kXBufs), (n / C::kXBufs) & 1, nullptr);
      drain_ring(bar(C::bY0Full), C::kStages0, n0);
      drain_ring(bar(C::bY1Full), C::kStages1, n1);
    }
    __syncwarp();
  } else if (warp == C::kWarpMma) {
    // ------------------------------------------------------------------ S, dP products
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);
      int items = 0, t = 0;
      bool ok = true;
      for (int k = blockIdx.x; ok && k < a.n_items; k += gridDim.x) {
        int bh, i;
        Mask mk;
        if (!bwd_item<kPacked>(k, a, false, bh, i, mk)) continue;
        int j_lo, j_hi;
        kv_tiles_for_q_tile(i, mk, j_lo, j_hi);
        const int xb = items % C::kXBufs, xu = items / C::kXBufs;
        if (!mbar_wait(bar(C::bXFull + xb), xu & 1, abort_flag)) break;
        for (int jj = j_lo; jj <= j_hi; ++jj, ++t) {
          const int s0 = t % C::kStages0, s1 = t % C::kStages1;
          // S(t) = Q_i K_j^T into buffer t & 1, which held dS(t-2): dQ(t-2) must have read it
          const int tp = t - 2;
          if (!mbar_wait(bar(C::bY0Full + s0), (t / C::kStages0) & 1, abort_flag) ||
              (tp >= 0 && !(kOneRelease ? mbar_wait(bar(C::bY0Empty + tp % C::kStages0),
                                                    (tp / C::kStages0) & 1, abort_flag)
                                        : mbar_wait(bar(bDQDone + (t & 1)), ((t >> 1) - 1) & 1,
                                                    abort_flag)))) {
            ok = false;
            break;
          }
          tc_fence_after();
          {
            const uint64_t dx = sdesc_sw128(sb + C::kX0 + xb * 2 * C::kTile, 16, 1024);
            const uint64_t dy = sdesc_sw128(sb + C::kY0 + s0 * C::kTile, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * C::kRegionBytes + (kk & 3) * 32;
              mma_ss(tmem + tS0 + 128u * (t & 1), sdesc_add(dx, off), sdesc_add(dy, off), idS,
                     kk > 0);
            }
          }
          tc_commit(bar(bSFull + (t & 1)));
          if (!kOneRelease) tc_commit(bar(C::bY0Empty + s0));
          // dP(t) = dO_i V_j^T, once the softmax has loaded dP(t-1); V_j is then free
          if (!mbar_wait(bar(C::bY1Full + s1), (t / C::kStages1) & 1, abort_flag) ||
              (t >= 1 && !mbar_wait(bar(bDPFree), (t - 1) & 1, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          {
            const uint64_t dx = sdesc_sw128(sb + C::kX1 + xb * 2 * C::kTile, 16, 1024);
            const uint64_t dy = sdesc_sw128(sb + C::kY1 + s1 * C::kTile, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * C::kRegionBytes + (kk & 3) * 32;
              mma_ss(tmem + tDP, sdesc_add(dx, off), sdesc_add(dy, off), idS, kk > 0);
            }
          }
          tc_commit(bar(bDPFull));
          if (!kOneRelease) tc_commit(bar(C::bY1Empty + s1));
          // without a staged output, Q_i and dO_i are free after their last product
          if (!C::kStageOut && jj == j_hi) tc_commit(bar(C::bXEmpty + xb));
        }
        ++items;
      }
      tc_commit(bar(C::bMmaFin));
      mbar_wait(bar(C::bMmaFin), 0, nullptr);
    }
    __syncwarp();
  } else if (warp == C::kWarpMma + 1) {
    // ------------------------------------------------------------------ dQ products
    if (lane == 0) {
      constexpr uint32_t idA = idesc_bf16_f32(128, D, false, true);
      int items = 0, t = 0;
      bool ok = true;
      for (int k = blockIdx.x; ok && k < a.n_items; k += gridDim.x) {
        int bh, i;
        Mask mk;
        if (!bwd_item<kPacked>(k, a, false, bh, i, mk)) continue;
        int j_lo, j_hi;
        kv_tiles_for_q_tile(i, mk, j_lo, j_hi);
        for (int jj = j_lo; jj <= j_hi; ++jj, ++t) {
          const int s0 = t % C::kStages0;
          const bool first = jj == j_lo;
          // dQ += dS K_j; the item's first product overwrites dQ, which the previous
          // item's epilogue must have read
          if (!mbar_wait(bar(C::bY0Full + s0), (t / C::kStages0) & 1, abort_flag) ||
              !mbar_wait(bar(bDSFull + (t & 1)), (t >> 1) & 1, abort_flag) ||
              (first && items > 0 && !mbar_wait(bar(bAccFree), (items - 1) & 1, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          {
            const uint64_t dy = sdesc_sw128(sb + C::kY0 + s0 * C::kTile, C::kRegionBytes, 1024);
            const uint32_t ta = tmem + tS0 + 128u * (t & 1);
#pragma unroll
            for (int kk = 0; kk < kBlock / 16; ++kk)
              mma_ts(tmem + tDQ, ta + packed_col(kk), sdesc_add(dy, kk * 2048), idA,
                     (!first || kk > 0) ? 1u : 0u);
          }
          tc_commit(bar(C::bY0Empty + s0));
          if (!kOneRelease) tc_commit(bar(bDQDone + (t & 1)));
          if (jj == j_hi) tc_commit(bar(bAccReady));  // dQ of the item is complete
        }
        ++items;
      }
      tc_commit(bar(C::bMmaFin + 1));
      mbar_wait(bar(C::bMmaFin + 1), 0, nullptr);
    }
    __syncwarp();
  } else if (warp == C::kWarpStore) {
    // ------------------------------------------------------------------ output stores
    if (lane == 0 && C::kStageOut) {
      int items = 0;
      for (int k = blockIdx.x; k < a.n_items; k += gridDim.x) {
        int bh, i;
        Mask mk;
        if (!bwd_item<kPacked>(k, a, false, bh, i, mk)) continue;
        const int xb = items % C::kXBufs;
        if (!mbar_wait(bar(bStaged), items & 1, abort_flag)) break;
        ++items;
        // (a partial tile of a packed batch was written row by row)
        if (whole_tile_store(cu, a.total, mk.N, seq_base(cu, bh, a.H), i * kBlock)) {
          const int base = seq_base(cu, bh, a.H);
          for (int rg = 0; rg < C::kRegions; ++rg)
            tma_store_3d(&tmdQ, sb + C::kX0 + xb * 2 * C::kTile + rg * C::kRegionBytes,
                         rg * 64, tma_y(cu, bh, a.H, i * kBlock),
                         tma_z(cu, bh, base, i * kBlock));
        }
        bulk_commit();
        bulk_wait_read();
        mbar_arrive(bar(C::bXEmpty + xb));
      }
      bulk_wait_all();
    }
    __syncwarp();
  } else {
    constexpr int NC = C::kCols;
    const int h = warp >> 2;          // key columns NC*h .. NC*h+NC-1 of each key tile
    const int t_row = threadIdx.x & 127;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const float sl2 = a.scale_log2;
    int g = 0, items = 0;
    bool ok = true;
    for (int k = blockIdx.x; ok && k < a.n_items; k += gridDim.x) {
      int bh, i;
      Mask mk;
      if (!bwd_item<kPacked>(k, a, false, bh, i, mk)) continue;
      int j_lo, j_hi;
      kv_tiles_for_q_tile(i, mk, j_lo, j_hi);
      const int n_it = j_hi - j_lo + 1;
      const int r = i * kBlock + t_row;  // this thread's query row
      // rows past N carry +inf and 0 in the padded statistics, which zero their P and dS
      const float lse2 = a.stats[(size_t)bh * a.Np + r];
      const float dl = a.stats[a.stat_rows + (size_t)bh * a.Np + r];
      const float slope2 = kAlibi ? a.alibi[bh % a.H] * kLog2e : 0.f;
      for (int it = 0; it < n_it; ++it) {
        const int jj = j_lo + it;
        const int t = g + it;
        const int b = t & 1;
        // keep flags of this row for keys NC*h + c of tile jj (bit c)
        uint32_t keep = ~0u;
        if (kDropout) {
          const uint32_t blk = (uint32_t)(8 * jj + 2 * h);
          keep = keep_bits16(a.drop, blk, (uint32_t)r, (uint32_t)bh) |
                 (keep_bits16(a.drop, blk + 1, (uint32_t)r, (uint32_t)bh) << 16);
        }
        if (!mbar_wait_warp(bar(bSFull + b), (t >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float p[NC];
        load_cols32(tmem + lane_base + tS0 + 128u * b + NC * h, p);
        {
          // with ALiBi, -m |key - query| in log2 units joins the exponent
          const float base = (float)((long long)jj * kBlock + NC * h - r);
          if constexpr (kAlibi) {
#pragma unroll
            for (int c = 0; c < NC; ++c) {
              const float arg = -slope2 * fabsf(base + (float)c) - lse2;
              p[c] = ex2(fmaf(p[c], sl2, arg));
            }
          } else {
            // exponent arguments two at a time (packed fp32 FMA), rounded as fmaf rounds
            const float2 s2 = make_float2(sl2, sl2), a2 = make_float2(-lse2, -lse2);
#pragma unroll
            for (int c = 0; c < NC; c += 2) {
              const float2 x = __ffma2_rn(make_float2(p[c], p[c + 1]), s2, a2);
              p[c] = ex2(x.x);
              p[c + 1] = ex2(x.y);
            }
          }
        }
        if (!tile_all_visible(i, jj, mk)) {
          int c_lo, c_hi;
          visible_keys(r, (long long)jj * kBlock + NC * h, NC, mk, c_lo, c_hi);
#pragma unroll
          for (int c = 0; c < NC; ++c) p[c] = (c >= c_lo && c <= c_hi) ? p[c] : 0.f;
        }
        if (kKpad) {
          // lane l reads the flag of key NC*h + l of the tile; the ballot gives all 32
          static_assert(NC == 32, "one ballot covers a warpgroup's columns");
          const int col = jj * kBlock + NC * h + lane;
          const uint32_t pm = __ballot_sync(
              0xffffffffu, col < a.N && a.kpad[(size_t)(bh / a.H) * a.N + col] != 0);
          if (pm != 0u) {
#pragma unroll
            for (int c = 0; c < NC; ++c) p[c] = ((pm >> c) & 1u) ? 0.f : p[c];
          }
        }
        if (!mbar_wait_warp(bar(bDPFull), t & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float dp[NC];
        load_cols32(tmem + lane_base + tDP + NC * h, dp);
        tc_fence_before();
        mbar_arrive_warp(bar(bDPFree));
        if (kDropout) {
          const float ks = a.drop.keep_scale;
#pragma unroll
          for (int c = 0; c < NC; ++c) dp[c] = ((keep >> c) & 1u) ? dp[c] * ks : 0.f;
        }
        uint32_t w[NC / 2];
        {
          const float2 ndl = make_float2(-dl, -dl);
#pragma unroll
          for (int e = 0; e < NC / 2; ++e) {
            const float2 v = __fmul2_rn(make_float2(p[2 * e], p[2 * e + 1]),
                                        __fadd2_rn(make_float2(dp[2 * e], dp[2 * e + 1]), ndl));
            w[e] = pack_bf16x2(v.x, v.y);
          }
        }
        // bf16 dS goes over the first half of this warpgroup's own fp32 S columns
        tmem_st16(tmem + lane_base + tS0 + 128u * b + NC * h, w);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive_warp(bar(bDSFull + b));
      }
      if (!ok) break;
      g += n_it;
      // once per item, after its last dQ product
      if (!mbar_wait_warp(bar(bAccReady), items & 1, abort_flag)) {
        ok = false;
        break;
      }
      // With a staged output, dQ goes through the item's Q_i buffer, which no product reads
      // any more; the store warp writes it out and hands the buffer back to the producer.
      // Otherwise each thread writes its part of its row directly.
      const int xb = items % C::kXBufs;
      const uint32_t tQ = sb + C::kX0 + xb * 2 * C::kTile;
      ++items;
      tc_fence_after();
      constexpr int NO = D / C::kGroups;
      if (C::kStageOut && whole_tile_store(cu, a.total, mk.N, seq_base(cu, bh, a.H), i * kBlock)) {
        stage_acc_cols<NO>(tmem + lane_base + tDQ + NO * h, a.scale, tQ, t_row, NO * h);
        fence_async_smem();
      } else {
        const int base = seq_base(cu, bh, a.H);
        const bool valid = row_written(cu, a.total, a.N, mk.N, base, r);
        const size_t off = row_at(cu, bh, a.H, a.N, base, valid ? r : 0, D) + NO * h;
        store_acc_cols<NO>(tmem + lane_base + tDQ + NO * h, a.scale, a.out0 + off, valid);
      }
      // dQ has been read: the next item's first product may overwrite it
      tc_fence_before();
      mbar_arrive_warp(bar(bAccFree));
      if (C::kStageOut) mbar_arrive_warp(bar(bStaged));
    }
  }
  bwd_teardown<C>(tmem, warp);
}

}  // namespace fa
