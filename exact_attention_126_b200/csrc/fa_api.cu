// fa_api.cu - host side of the C ABI declared in include/fa.h.
//
// Validates every argument before touching the GPU, encodes one TMA tensor map per input
// tensor ((B*H, N, d) viewed as a 3-D tensor so that the rows past N of a (batch, head)
// read as zeros instead of the next head's rows), and launches the kernels of
// fa_fwd.cuh / fa_bwd.cuh on the caller's stream.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "fa.h"
#include "fa_bwd.cuh"
#include "fa_fwd.cuh"

namespace {

using fa::kBlock;

// Test hook set by fa_debug_set_fault(); 0 in normal operation.
std::atomic<int> g_fault{0};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// (B*H, N, d) bf16 tensor, box of 128 rows x 64 columns (128 bytes), 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, int BH, int N, int d) {
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

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shared validation. Returns FA_OK and sets *empty when there is nothing to do.
fa_status_t check_problem(int B, int H, int N, int d, bool* empty) {
  *empty = false;
  if (B < 0 || H < 0 || N < 0) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || N == 0) {
    *empty = true;
    return FA_OK;
  }
  const long long elems = (long long)B * H * N * d;
  if (elems >= (1ll << 31)) return FA_ERR_UNSUPPORTED;
  if ((long long)B * H > 65535) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

fa_status_t check_mask(float scale, fa_window_t w) {
  if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (w.left < -1 || w.right < -1) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

fa_status_t check_ptrs(std::initializer_list<const void*> ptrs) {
  for (const void* p : ptrs)
    if (p == nullptr) return FA_ERR_INVALID_ARG;
  for (const void* p : ptrs)
    if (!aligned16(p)) return FA_ERR_MISALIGNED;
  return FA_OK;
}

template <typename Kernel>
fa_status_t set_smem(Kernel k, int bytes) {
  // Per device and kernel; cheap enough to repeat, but only needed once per device.
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess
             ? FA_OK
             : FA_ERR_CUDA;
}

template <typename Kernel>
int launch_regs(Kernel k) {
  cudaFuncAttributes attr;
  if (cudaFuncGetAttributes(&attr, k) != cudaSuccess) return -1;
  return attr.numRegs;
}

int sm_count() {
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
int head_group(int BH, int tiles) {
  int g = (sm_count() + tiles - 1) / tiles;
  if (g < 1) g = 1;
  if (g > BH) g = BH;
  return g;
}

fa_status_t launched() {
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}


// alibi: H slopes for the ALiBi kernels (kAlibi), unused otherwise.
template <int D, bool kAlibi>
fa_status_t launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int BH,
                       int H, int N, float scale, int left, int right, const float* alibi,
                       cudaStream_t st) {
  CUtensorMap mq, mkk, mv;
  if (!make_map(&mq, q, BH, N, D) || !make_map(&mkk, k, BH, N, D) || !make_map(&mv, v, BH, N, D))
    return FA_ERR_CUDA;
  using C = fa::FwdCfg<D>;
  if (set_smem(fa::fa_fwd_kernel<D, kAlibi>, C::kSmemBytes) != FA_OK) return FA_ERR_CUDA;
  fa::FwdArgs a;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.N = N;
  a.BH = BH;
  a.n_qtiles = fa::num_tiles(N);
  a.n_pairs = (a.n_qtiles + 1) / 2;
  a.n_items = BH * a.n_pairs;
  a.longest_first = (left >= 0 || right >= 0) ? 1 : 0;
  a.group = head_group(BH, a.n_pairs);
  a.scale_log2 = scale * fa::kLog2e;
  a.left = left;
  a.right = right;
  a.fault = g_fault.load(std::memory_order_relaxed);
  a.alibi = alibi;
  a.H = H;
  const int grid = a.n_items < sm_count() ? a.n_items : sm_count();
  fa::fa_fwd_kernel<D, kAlibi><<<grid, C::kThreads, C::kSmemBytes, st>>>(mq, mkk, mv, a);
  return launched();
}

int padded_rows(int N) { return fa::num_tiles(N) * kBlock; }

template <int D>
fa_status_t launch_preprocess(const void* o, const void* dout, const float* lse, float* stats,
                              int BH, int N, cudaStream_t st) {
  const int Np = padded_rows(N);
  const dim3 grid(Np / 64, BH);  // 64 rows per block; Np is a multiple of 128, BH <= 65535
  fa::fa_bwd_preprocess_kernel<D><<<grid, 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse, stats,
      BH, N, Np);
  return launched();
}

template <int D, bool kAlibi>
fa_status_t launch_dkdv(const void* q, const void* k, const void* v, const void* dout,
                        const void* ws, void* dk, void* dv, int BH, int H, int N,
                        float scale, int left, int right, const float* alibi, cudaStream_t st) {
  CUtensorMap mq, mkk, mv, mdo, mdk, mdv;
  if (!make_map(&mq, q, BH, N, D) || !make_map(&mkk, k, BH, N, D) ||
      !make_map(&mv, v, BH, N, D) || !make_map(&mdo, dout, BH, N, D) ||
      !make_map(&mdk, dk, BH, N, D) || !make_map(&mdv, dv, BH, N, D))
    return FA_ERR_CUDA;
  using C = fa::DkdvCfg<D>;
  if (set_smem(fa::fa_bwd_dkdv_kernel<D, kAlibi>, C::kSmemBytes) != FA_OK) return FA_ERR_CUDA;
  fa::BwdArgs a;
  a.stats = static_cast<const float*>(ws);
  a.out0 = static_cast<__nv_bfloat16*>(dk);
  a.out1 = static_cast<__nv_bfloat16*>(dv);
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
  const int grid = a.n_items < sm_count() ? a.n_items : sm_count();
  a.alibi = alibi;
  a.H = H;
  fa::fa_bwd_dkdv_kernel<D, kAlibi><<<grid, C::kThreads, C::kSmemBytes, st>>>(mq, mkk, mv, mdo,
                                                                               mdk, mdv, a);
  return launched();
}

template <int D, bool kAlibi>
fa_status_t launch_dq(const void* q, const void* k, const void* v, const void* dout,
                      const void* ws, void* dq, int BH, int H, int N, float scale,
                      int left, int right, const float* alibi, cudaStream_t st) {
  CUtensorMap mq, mkk, mv, mdo, mdq;
  if (!make_map(&mq, q, BH, N, D) || !make_map(&mkk, k, BH, N, D) ||
      !make_map(&mv, v, BH, N, D) || !make_map(&mdo, dout, BH, N, D) ||
      !make_map(&mdq, dq, BH, N, D))
    return FA_ERR_CUDA;
  using C = fa::DqCfg<D>;
  if (set_smem(fa::fa_bwd_dq_kernel<D, kAlibi>, C::kSmemBytes) != FA_OK) return FA_ERR_CUDA;
  fa::BwdArgs a;
  a.stats = static_cast<const float*>(ws);
  a.out0 = static_cast<__nv_bfloat16*>(dq);
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
  const int grid = a.n_items < sm_count() ? a.n_items : sm_count();
  a.alibi = alibi;
  a.H = H;
  fa::fa_bwd_dq_kernel<D, kAlibi><<<grid, C::kThreads, C::kSmemBytes, st>>>(mq, mkk, mv, mdo, mdq,
                                                                             a);
  return launched();
}

size_t workspace_bytes(int B, int H, int N) {
  const size_t raw = 2 * (size_t)B * H * padded_rows(N) * sizeof(float);
  return (raw + 255) & ~size_t(255);
}

// ------------------------------------------------------------------------------------
// Backward without caller workspace (fa_bwd_noalloc): a fixed array in device memory
// holds the row statistics instead. Every GPU that loads the library keeps this array
// until the process exits.
// ------------------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {nullptr};

// Device address of g_noalloc_scratch on the current device. The symbol names a
// host-side stand-in, not device memory, so the address is looked up once per device
// (with that device current) and cached.
fa_status_t noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return FA_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return FA_OK;
}

}  // namespace

fa_status_t check_slopes(const float* alibi) {
  if (alibi == nullptr) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(alibi) & 3u) != 0) return FA_ERR_MISALIGNED;
  return FA_OK;
}

// fa_fwd and fa_fwd_alibi (alibi != nullptr)
fa_status_t forward(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                    int N, int d, float scale, int causal, fa_window_t window, const float* alibi,
                    void* stream) {
  bool empty;
  fa_status_t s = check_problem(B, H, N, d, &empty);
  if (s != FA_OK || empty) return s;
  if ((s = check_mask(scale, window)) != FA_OK) return s;
  if ((s = check_ptrs({q, k, v, o, lse})) != FA_OK) return s;
  const int right = fa::resolve_right(causal, window.right);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int l = window.left, BH = B * H;
  if (alibi != nullptr)
    return d == 64 ? launch_fwd<64, true>(q, k, v, o, lse, BH, H, N, scale, l, right, alibi, st)
                   : launch_fwd<128, true>(q, k, v, o, lse, BH, H, N, scale, l, right, alibi, st);
  return d == 64 ? launch_fwd<64, false>(q, k, v, o, lse, BH, H, N, scale, l, right, nullptr, st)
                 : launch_fwd<128, false>(q, k, v, o, lse, BH, H, N, scale, l, right, nullptr, st);
}

// The two passes of the backward after the preprocess step, with or without ALiBi.
fa_status_t backward_passes(const void* q, const void* k, const void* v, const void* dout,
                            const void* ws, void* dq, void* dk, void* dv, int B, int H, int N,
                            int d, float scale, int causal, fa_window_t window,
                            const float* alibi, void* stream) {
  const int right = fa::resolve_right(causal, window.right);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int l = window.left, BH = B * H;
  fa_status_t s;
  if (alibi != nullptr) {
    s = d == 64 ? launch_dkdv<64, true>(q, k, v, dout, ws, dk, dv, BH, H, N, scale, l, right,
                                        alibi, st)
                : launch_dkdv<128, true>(q, k, v, dout, ws, dk, dv, BH, H, N, scale, l, right,
                                         alibi, st);
    if (s != FA_OK) return s;
    return d == 64 ? launch_dq<64, true>(q, k, v, dout, ws, dq, BH, H, N, scale, l, right,
                                         alibi, st)
                   : launch_dq<128, true>(q, k, v, dout, ws, dq, BH, H, N, scale, l, right,
                                          alibi, st);
  }
  s = d == 64 ? launch_dkdv<64, false>(q, k, v, dout, ws, dk, dv, BH, H, N, scale, l, right,
                                       nullptr, st)
              : launch_dkdv<128, false>(q, k, v, dout, ws, dk, dv, BH, H, N, scale, l, right,
                                        nullptr, st);
  if (s != FA_OK) return s;
  return d == 64 ? launch_dq<64, false>(q, k, v, dout, ws, dq, BH, H, N, scale, l, right,
                                        nullptr, st)
                 : launch_dq<128, false>(q, k, v, dout, ws, dq, BH, H, N, scale, l, right,
                                         nullptr, st);
}

extern "C" {

fa_status_t fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                   int N, int d, float scale, int causal, fa_window_t window, void* stream) {
  return forward(q, k, v, o, lse, B, H, N, d, scale, causal, window, nullptr, stream);
}

fa_status_t fa_fwd_alibi(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int H, int N, int d, float scale, int causal, fa_window_t window,
                         const float* alibi_slopes, void* stream) {
  bool empty;
  fa_status_t s = check_problem(B, H, N, d, &empty);
  if (s != FA_OK || empty) return s;
  if ((s = check_slopes(alibi_slopes)) != FA_OK) return s;
  return forward(q, k, v, o, lse, B, H, N, d, scale, causal, window, alibi_slopes, stream);
}

size_t fa_bwd_workspace_bytes(int B, int H, int N, int d) {
  bool empty;
  if (check_problem(B, H, N, d, &empty) != FA_OK || empty) return 0;
  return workspace_bytes(B, H, N);
}

fa_status_t fa_bwd_preprocess(const void* o, const void* dout, const float* lse,
                              void* workspace, int B, int H, int N, int d, void* stream) {
  bool empty;
  fa_status_t s = check_problem(B, H, N, d, &empty);
  if (s != FA_OK || empty) return s;
  if ((s = check_ptrs({o, dout, lse, workspace})) != FA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* stats = static_cast<float*>(workspace);
  return d == 64 ? launch_preprocess<64>(o, dout, lse, stats, B * H, N, st)
                 : launch_preprocess<128>(o, dout, lse, stats, B * H, N, st);
}

fa_status_t fa_bwd_dkdv(const void* q, const void* k, const void* v, const void* dout,
                        const void* workspace, void* dk, void* dv, int B, int H, int N, int d,
                        float scale, int causal, fa_window_t window, void* stream) {
  bool empty;
  fa_status_t s = check_problem(B, H, N, d, &empty);
  if (s != FA_OK || empty) return s;
  if ((s = check_mask(scale, window)) != FA_OK) return s;
  if ((s = check_ptrs({q, k, v, dout, workspace, dk, dv})) != FA_OK) return s;
  const int right = fa::resolve_right(causal, window.right);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return d == 64 ? launch_dkdv<64, false>(q, k, v, dout, workspace, dk, dv, B * H, H, N, scale,
                                          window.left, right, nullptr, st)
                 : launch_dkdv<128, false>(q, k, v, dout, workspace, dk, dv, B * H, H, N, scale,
                                           window.left, right, nullptr, st);
}

fa_status_t fa_bwd_dq(const void* q, const void* k, const void* v, const void* dout,
                      const void* workspace, void* dq, int B, int H, int N, int d, float scale,
                      int causal, fa_window_t window, void* stream) {
  bool empty;
  fa_status_t s = check_problem(B, H, N, d, &empty);
  if (s != FA_OK || empty) return s;
  if ((s = check_mask(scale, window)) != FA_OK) return s;
  if ((s = check_ptrs({q, k, v, dout, workspace, dq})) != FA_OK) return s;
  const int right = fa::resolve_right(causal, window.right);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return d == 64 ? launch_dq<64, false>(q, k, v, dout, workspace, dq, B * H, H, N, scale,
                                        window.left, right, nullptr, st)
                 : launch_dq<128, false>(q, k, v, dout, workspace, dq, B * H, H, N, scale,
                                         window.left, right, nullptr, st);
}

fa_status_t fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                   const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                   float scale, int causal, fa_window_t window, void* workspace,
                   size_t workspace_bytes_given, void* stream) {
  bool empty;
  fa_status_t s = check_problem(B, H, N, d, &empty);
  if (s != FA_OK || empty) return s;
  if ((s = check_mask(scale, window)) != FA_OK) return s;
  if ((s = check_ptrs({q, k, v, o, dout, lse, dq, dk, dv, workspace})) != FA_OK) return s;
  if (workspace_bytes_given < workspace_bytes(B, H, N)) return FA_ERR_WORKSPACE;
  if ((s = fa_bwd_preprocess(o, dout, lse, workspace, B, H, N, d, stream)) != FA_OK) return s;
  if ((s = fa_bwd_dkdv(q, k, v, dout, workspace, dk, dv, B, H, N, d, scale, causal, window,
                       stream)) != FA_OK)
    return s;
  return fa_bwd_dq(q, k, v, dout, workspace, dq, B, H, N, d, scale, causal, window, stream);
}

fa_status_t fa_bwd_alibi(const void* q, const void* k, const void* v, const void* o,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                         int H, int N, int d, float scale, int causal, fa_window_t window,
                         const float* alibi_slopes, void* workspace,
                         size_t workspace_bytes_given, void* stream) {
  bool empty;
  fa_status_t s = check_problem(B, H, N, d, &empty);
  if (s != FA_OK || empty) return s;
  if ((s = check_mask(scale, window)) != FA_OK) return s;
  if ((s = check_slopes(alibi_slopes)) != FA_OK) return s;
  if ((s = check_ptrs({q, k, v, o, dout, lse, dq, dk, dv, workspace})) != FA_OK) return s;
  if (workspace_bytes_given < workspace_bytes(B, H, N)) return FA_ERR_WORKSPACE;
  if ((s = fa_bwd_preprocess(o, dout, lse, workspace, B, H, N, d, stream)) != FA_OK) return s;
  return backward_passes(q, k, v, dout, workspace, dq, dk, dv, B, H, N, d, scale, causal, window,
                         alibi_slopes, stream);
}

fa_status_t fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                           const void* dout, const float* lse, void* dq, void* dk, void* dv,
                           int B, int H, int N, int d, float scale, int causal,
                           fa_window_t window, void* stream) {
  bool empty;
  fa_status_t s = check_problem(B, H, N, d, &empty);
  if (s != FA_OK || empty) return s;
  if ((s = check_mask(scale, window)) != FA_OK) return s;
  if ((s = check_ptrs({q, k, v, o, dout, lse, dq, dk, dv})) != FA_OK) return s;
  if (workspace_bytes(B, H, N) > kNoAllocScratchBytes) return FA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if ((s = noalloc_scratch(&scratch)) != FA_OK) return s;
  // The statistics are rewritten in full by the preprocess step, so nothing needs clearing.
  if ((s = fa_bwd_preprocess(o, dout, lse, scratch, B, H, N, d, stream)) != FA_OK) return s;
  if ((s = fa_bwd_dkdv(q, k, v, dout, scratch, dk, dv, B, H, N, d, scale, causal, window,
                       stream)) != FA_OK)
    return s;
  return fa_bwd_dq(q, k, v, dout, scratch, dq, B, H, N, d, scale, causal, window, stream);
}

const char* fa_status_string(fa_status_t status) {
  switch (status) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG: null pointer, negative size, bad scale or window";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: head_dim must be 64 or 128 and tensors < 2^31 elements";
    case FA_ERR_MISALIGNED: return "FA_ERR_MISALIGNED: pointers must be 16-byte aligned";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE: workspace smaller than fa_bwd_workspace_bytes()";
    case FA_ERR_CUDA: return "FA_ERR_CUDA: a CUDA call failed";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT: a kernel abandoned a bounded wait";
  }
  return "FA_ERR_UNKNOWN";
}

fa_status_t fa_debug_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, fa::g_fa_status, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(fa::g_fa_status, &zero, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
    return FA_ERR_TIMEOUT;
  }
  return FA_OK;
}

fa_status_t fa_debug_set_fault(int fault) {
  if (fault < 0 || fault > 1) return FA_ERR_INVALID_ARG;
  g_fault.store(fault, std::memory_order_relaxed);
  return FA_OK;
}

int fa_version(void) { return 100; }

}  // extern "C"
