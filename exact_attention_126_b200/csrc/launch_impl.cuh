// launch_impl.cuh - the launchers of the kernels (included by the kernel units only).
//
// Each launcher encodes one TMA tensor map per tensor ((B*H, N, d) viewed as a 3-D tensor,
// so that rows past N of a (batch, head) read as zeros instead of the next head's rows),
// fills the kernel's argument block and launches persistent CTAs on the caller's stream.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "fa_bwd.cuh"
#include "fa_bwd_fused.cuh"
#include "fa_fwd.cuh"
#include "launch.h"

namespace fa_host {

using fa::kBlock;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's cuTensorMapEncodeTiled, looked up once (thread-safe static initialisation).
inline EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(p);
    return nullptr;
  }();
  return fn;
}

// The fused backward's dQ accumulator: (B*H, Np, 64) fp32, boxes of 32 columns (128 bytes)
// x 128 rows, 128-byte swizzle.
inline bool make_acc_map(CUtensorMap* map, float* base, int BH, int Np) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {64, (cuuint64_t)Np, (cuuint64_t)BH};
  const cuuint64_t strides[2] = {64 * 4, (cuuint64_t)Np * 64 * 4};
  const cuuint32_t box[3] = {32, (cuuint32_t)kBlock, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// (B*H, N, d) e4m3 tensor (one byte per value), box of 128 rows x 128 columns (128 bytes),
// 128-byte swizzle.
inline bool make_map_u8(CUtensorMap* map, const void* base, int BH, int N, int d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  const cuuint64_t strides[2] = {(cuuint64_t)d, (cuuint64_t)N * d};
  const cuuint32_t box[3] = {128, (cuuint32_t)kBlock, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// (B*H, N, d) bf16 tensor, box of 128 rows x 64 columns (128 bytes), 128-byte swizzle.
inline bool make_map(CUtensorMap* map, const void* base, int BH, int N, int d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)N * d * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)kBlock, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A packed (total, H, d) bf16 tensor viewed as (d, H, total): a box of 1 head x 128 tokens x
// 64 columns lands in shared memory as the (B*H, N, d) view's 128 x 64 box does.
inline bool make_map_packed(CUtensorMap* map, const void* base, int total, int H, int d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)total};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2};
  const cuuint32_t box[3] = {64, 1, (cuuint32_t)kBlock};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The map of a bf16 attention tensor of the problem: (B*H, N, d), or packed (total, H, d)
// when the options carry cumulative lengths.
inline bool map_rows(CUtensorMap* map, const void* base, const Problem& pb, const Extras& x,
                     int d) {
  return x.cu != nullptr ? make_map_packed(map, base, x.total, pb.H, d)
                         : make_map(map, base, pb.BH, pb.N, d);
}

constexpr int kMaxSmemPerBlock = 232448;  // the opt-in limit of sm_100

template <typename Kernel>
fa_status_t set_smem(Kernel k, int bytes) {
  // Per device and kernel; cheap enough to repeat, but only needed once per device.
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess
             ? FA_OK
             : FA_ERR_CUDA;
}

inline int sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
  int n = 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 148;
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

// Heads per chunk of the masked schedules: enough for about one item per SM.
inline int head_group(int BH, int tiles) {
  int g = (sm_count() + tiles - 1) / tiles;
  if (g < 1) g = 1;
  if (g > BH) g = BH;
  return g;
}

// The causal schedule of paired_item: for a causal mask (no window), an even number T of
// tiles per head and one length for every batch entry, items go in complementary pairs
// (with real lengths the pairs would not weigh the same). Sets paired, n_double and n_items
// (the slots of whole round pairs over the grid that persistent_grid() returns).
template <typename Args>
inline void pair_schedule(Args& a, int BH, int T, int left, int right, bool varlen) {
  a.paired = (left < 0 && right == 0 && T % 2 == 0 && !varlen) ? 1 : 0;
  a.n_double = 0;
  if (a.paired) {
    a.n_double = BH * (T / 2);
    const int P = a.n_double < sm_count() ? a.n_double : sm_count();
    a.n_items = 2 * ((a.n_double + P - 1) / P) * P;
  }
}

// The schedule of a variable-length batch (varlen_item) over U units per head: the slots of
// whole rounds of the persistent grid, so that both directions of the last round are
// visited. Sets sorted and n_items.
template <typename Args>
inline void varlen_schedule(Args& a, int BH, int U) {
  a.sorted = 1;
  const int P = BH * U < sm_count() ? BH * U : sm_count();
  a.n_items = (BH * U + P - 1) / P * P;
}

// Persistent CTAs: one per SM, or one per item (one per pair of items with the causal
// schedule) when there are fewer.
template <typename Args>
inline int persistent_grid(const Args& a) {
  const int units = a.paired ? a.n_double : a.n_items;
  return units < sm_count() ? units : sm_count();
}

inline fa_status_t launched() {
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}


template <int D, int kFeat>
fa_status_t launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                       const Problem& pb, const Extras& x, int fault, cudaStream_t st) {
  const int BH = pb.BH, H = pb.H, N = pb.N, left = pb.left, right = pb.right;
  const float scale = pb.scale;
  constexpr bool kFp8 = (kFeat & fa::kFeatFp8) != 0;
  CUtensorMap mq, mkk, mv;
  if (kFp8) {
    if (!make_map_u8(&mq, q, BH, N, D) || !make_map_u8(&mkk, k, BH, N, D) ||
        !make_map_u8(&mv, v, BH, N, D))
      return FA_ERR_CUDA;
  } else if (!map_rows(&mq, q, pb, x, D) || !map_rows(&mkk, k, pb, x, D) ||
             !map_rows(&mv, v, pb, x, D)) {
    return FA_ERR_CUDA;
  }
  using C = fa::FwdCfg<D, kFp8>;
  fa::FwdArgs a;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.N = N;
  a.BH = BH;
  a.n_qtiles = fa::num_tiles(N);
  // two query tiles per item, unless that leaves SMs without an item
  a.per_item = (BH * ((a.n_qtiles + 1) / 2) < sm_count() && a.n_qtiles > 1) ? 1 : 2;
  a.n_pairs = (a.n_qtiles + a.per_item - 1) / a.per_item;
  a.n_items = BH * a.n_pairs;
  a.longest_first = (left >= 0 || right >= 0) ? 1 : 0;
  a.group = head_group(BH, a.n_pairs);
  pair_schedule(a, BH, a.n_pairs, left, right, x.varlen());
  // a variable-length batch: the varlen_item schedule, its tables in shared memory
  a.sorted = 0;
  int smem = C::kSmemBytes;
  const int sched_bytes = 4 * fa::varlen_sched_ints(BH / H, a.n_pairs);
  if (x.varlen() && BH / H <= fa::kVarlenSchedMaxB &&
      C::kSmemBytes + sched_bytes <= kMaxSmemPerBlock) {
    varlen_schedule(a, BH, a.n_pairs);
    smem += sched_bytes;
  }
  if (set_smem(fa::fa_fwd_kernel<D, kFeat>, smem) != FA_OK) return FA_ERR_CUDA;
  a.scale_log2 = scale * fa::kLog2e;
  a.left = left;
  a.right = right;
  a.fault = fault;
  a.alibi = x.alibi;
  a.H = H;
  a.kpad = x.kpad;
  a.o_low = static_cast<__nv_bfloat16*>(x.o_low);
  a.drop = x.drop;
  a.seq_len = x.seq_len;
  a.cu = x.cu;
  a.total = x.total;
  a.o_scale = x.o_scale;
  const int grid = persistent_grid(a);
  fa::fa_fwd_kernel<D, kFeat><<<grid, C::kThreads, smem, st>>>(mq, mkk, mv, a);
  return launched();
}

inline int padded_rows(int N) { return fa::num_tiles(N) * kBlock; }

template <int D>
fa_status_t launch_preprocess(const void* o, const void* o_low, const void* dout,
                              const float* lse, float* stats, float* dq_acc,
                              const fa::SchedBuild& sb, const int* cu, int total, int H,
                              int BH, int N, cudaStream_t st) {
  const int Np = padded_rows(N);
  // 64 rows per block, blocks of one head consecutive; BH * Np / 64 < 2^31 because every
  // tensor has fewer than 2^31 elements (d >= 64); one more block builds the tables of sb
  const long long blocks = (long long)BH * (Np / 64) + (sb.tables != nullptr ? 1 : 0);
  auto kernel = cu != nullptr ? fa::fa_bwd_preprocess_kernel<D, true>
                              : fa::fa_bwd_preprocess_kernel<D, false>;
  kernel<<<(unsigned)blocks, 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(o_low),
      static_cast<const __nv_bfloat16*>(dout), lse, stats, dq_acc, sb, cu, total, H, BH, N, Np);
  return launched();
}

// Arguments both backward passes share.
inline fa::BwdArgs bwd_args(const void* ws, const Problem& pb, const Extras& x) {
  const int BH = pb.BH, H = pb.H, N = pb.N, left = pb.left, right = pb.right;
  const float scale = pb.scale;
  fa::BwdArgs a;
  a.stats = static_cast<const float*>(ws);
  a.out0 = nullptr;
  a.out1 = nullptr;
  a.stat_rows = (long long)BH * padded_rows(N);
  a.Np = padded_rows(N);
  a.N = N;
  a.n_tiles = fa::num_tiles(N);
  a.scale = scale;
  a.scale_log2 = scale * fa::kLog2e;
  a.left = left;
  a.right = right;
  a.BH = BH;
  a.n_items = BH * a.n_tiles;
  a.longest_first = (left >= 0 || right >= 0) ? 1 : 0;
  a.group = head_group(BH, a.n_tiles);
  pair_schedule(a, BH, a.n_tiles, left, right, x.varlen());
  a.sorted = 0;
  a.sched = x.sched;
  if (x.sched != nullptr) varlen_schedule(a, BH, a.n_tiles);
  a.alibi = x.alibi;
  a.H = H;
  a.kpad = x.kpad;
  a.drop = x.drop;
  a.seq_len = x.seq_len;
  a.cu = x.cu;
  a.total = x.total;
  return a;
}

template <int D, int kFeat>
fa_status_t launch_dkdv(const void* q, const void* k, const void* v, const void* dout,
                        const void* ws, void* dk, void* dv, const Problem& pb, const Extras& x,
                        cudaStream_t st) {
  CUtensorMap mq, mkk, mv, mdo, mdk, mdv;
  if (!map_rows(&mq, q, pb, x, D) || !map_rows(&mkk, k, pb, x, D) ||
      !map_rows(&mv, v, pb, x, D) || !map_rows(&mdo, dout, pb, x, D) ||
      !map_rows(&mdk, dk, pb, x, D) || !map_rows(&mdv, dv, pb, x, D))
    return FA_ERR_CUDA;
  using C = fa::DkdvCfg<D>;
  if (set_smem(fa::fa_bwd_dkdv_kernel<D, kFeat>, C::kSmemBytes) != FA_OK) return FA_ERR_CUDA;
  fa::BwdArgs a = bwd_args(ws, pb, x);
  a.out0 = static_cast<__nv_bfloat16*>(dk);
  a.out1 = static_cast<__nv_bfloat16*>(dv);
  const int grid = persistent_grid(a);
  fa::fa_bwd_dkdv_kernel<D, kFeat><<<grid, C::kThreads, C::kSmemBytes, st>>>(mq, mkk, mv, mdo,
                                                                               mdk, mdv, a);
  return launched();
}

template <int D, int kFeat>
fa_status_t launch_dq(const void* q, const void* k, const void* v, const void* dout,
                      const void* ws, void* dq, const Problem& pb, const Extras& x,
                      cudaStream_t st) {
  CUtensorMap mq, mkk, mv, mdo, mdq;
  if (!map_rows(&mq, q, pb, x, D) || !map_rows(&mkk, k, pb, x, D) ||
      !map_rows(&mv, v, pb, x, D) || !map_rows(&mdo, dout, pb, x, D) ||
      !map_rows(&mdq, dq, pb, x, D))
    return FA_ERR_CUDA;
  using C = fa::DqCfg<D>;
  if (set_smem(fa::fa_bwd_dq_kernel<D, kFeat>, C::kSmemBytes) != FA_OK) return FA_ERR_CUDA;
  fa::BwdArgs a = bwd_args(ws, pb, x);
  a.out0 = static_cast<__nv_bfloat16*>(dq);
  const int grid = persistent_grid(a);
  fa::fa_bwd_dq_kernel<D, kFeat><<<grid, C::kThreads, C::kSmemBytes, st>>>(mq, mkk, mv, mdo, mdq,
                                                                             a);
  return launched();
}

template <int kFeat>
fa_status_t launch_fused(const void* q, const void* k, const void* v, const void* dout,
                         const void* ws, float* dq_acc, void* dk, void* dv, const Problem& pb,
                         const Extras& x, cudaStream_t st) {
  constexpr int D = 64;
  const int BH = pb.BH, N = pb.N;
  CUtensorMap mq, mkk, mv, mdo, mdk, mdv, macc;
  if (!make_map(&mq, q, BH, N, D) || !make_map(&mkk, k, BH, N, D) ||
      !make_map(&mv, v, BH, N, D) || !make_map(&mdo, dout, BH, N, D) ||
      !make_map(&mdk, dk, BH, N, D) || !make_map(&mdv, dv, BH, N, D) ||
      !make_acc_map(&macc, dq_acc, BH, padded_rows(N)))
    return FA_ERR_CUDA;
  using C = fa::FusedCfg;
  if (set_smem(fa::fa_bwd_fused_kernel<kFeat>, C::kSmemBytes) != FA_OK) return FA_ERR_CUDA;
  fa::BwdArgs a = bwd_args(ws, pb, x);
  a.out0 = static_cast<__nv_bfloat16*>(dk);
  a.out1 = static_cast<__nv_bfloat16*>(dv);
  const int grid = persistent_grid(a);
  fa::fa_bwd_fused_kernel<kFeat><<<grid, C::kThreads, C::kSmemBytes, st>>>(mq, mkk, mv, mdo, mdk,
                                                                           mdv, macc, a);
  return launched();
}

template <int D>
fa_status_t launch_dq_convert(const float* dq_acc, void* dq, int BH, int N, float scale,
                              cudaStream_t st) {
  const long long rows = (long long)BH * N;
  const long long threads = rows * (D / 8);
  const long long blocks = (threads + 255) / 256;
  fa::fa_bwd_dq_convert_kernel<D><<<(unsigned)blocks, 256, 0, st>>>(
      dq_acc, static_cast<__nv_bfloat16*>(dq), rows, N, padded_rows(N), scale);
  return launched();
}

template <int D>
fa_status_t launch_fill_past_length(void* t0, void* t1, void* t2, float* lse,
                                    const int* seq_len, int BH, int H, int N, cudaStream_t st) {
  // one block per 128-row tile: BH * tiles < 2^31 (every tensor has < 2^31 elements)
  const long long blocks = (long long)BH * fa::num_tiles(N);
  fa::fa_fill_past_length_kernel<D><<<(unsigned)blocks, 256, 0, st>>>(
      static_cast<__nv_bfloat16*>(t0), static_cast<__nv_bfloat16*>(t1),
      static_cast<__nv_bfloat16*>(t2), lse, seq_len, N, H);
  return launched();
}

// Reads and clears this unit's copy of the device status word.
inline int take_unit_status() {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, fa::g_fa_status, sizeof(int)) != cudaSuccess) return -1;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(fa::g_fa_status, &zero, sizeof(int)) != cudaSuccess) return -1;
  }
  return v;
}

// Explicit instantiation definitions of the launchers (one line per feature set).
#define FA_INSTANTIATE_FWD(D, F)                                                            \
  template fa_status_t launch_fwd<D, F>(const void*, const void*, const void*, void*, float*, \
                                        const Problem&, const Extras&, int, cudaStream_t);
#define FA_INSTANTIATE_BWD(D, F)                                                             \
  template fa_status_t launch_dkdv<D, F>(const void*, const void*, const void*, const void*,   \
                                         const void*, void*, void*, const Problem&,            \
                                         const Extras&, cudaStream_t);                         \
  template fa_status_t launch_dq<D, F>(const void*, const void*, const void*, const void*,     \
                                       const void*, void*, const Problem&, const Extras&,      \
                                       cudaStream_t);
#define FA_INSTANTIATE_FUSED(F)                                                               \
  template fa_status_t launch_fused<F>(const void*, const void*, const void*, const void*,    \
                                       const void*, float*, void*, void*, const Problem&,      \
                                       const Extras&, cudaStream_t);

}  // namespace fa_host
