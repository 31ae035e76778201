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


// Optional inputs and outputs of one call (fa_options_t, checked and resolved).
struct Extras {
  const float* alibi = nullptr;    // H slopes: the kAlibi kernels
  const uint8_t* kpad = nullptr;   // (B, N) key-padding flags
  void* o_low = nullptr;           // bf16 residual of O: written by the forward, read by delta
};

template <int D, bool kAlibi>
fa_status_t launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int BH,
                       int H, int N, float scale, int left, int right, const Extras& x,
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
  a.alibi = x.alibi;
  a.H = H;
  a.kpad = x.kpad;
  a.o_low = static_cast<__nv_bfloat16*>(x.o_low);
  const int grid = a.n_items < sm_count() ? a.n_items : sm_count();
  fa::fa_fwd_kernel<D, kAlibi><<<grid, C::kThreads, C::kSmemBytes, st>>>(mq, mkk, mv, a);
  return launched();
}

int padded_rows(int N) { return fa::num_tiles(N) * kBlock; }

template <int D>
fa_status_t launch_preprocess(const void* o, const void* o_low, const void* dout,
                              const float* lse, float* stats, int BH, int N, cudaStream_t st) {
  const int Np = padded_rows(N);
  // 64 rows per block, blocks of one head consecutive; BH * Np / 64 < 2^31 because every
  // tensor has fewer than 2^31 elements (d >= 64)
  const long long blocks = (long long)BH * (Np / 64);
  fa::fa_bwd_preprocess_kernel<D><<<(unsigned)blocks, 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(o_low),
      static_cast<const __nv_bfloat16*>(dout), lse, stats, BH, N, Np);
  return launched();
}

// Arguments both backward passes share.
fa::BwdArgs bwd_args(const void* ws, int BH, int H, int N, float scale, int left, int right,
                     const Extras& x) {
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
  a.alibi = x.alibi;
  a.H = H;
  a.kpad = x.kpad;
  return a;
}

template <int D, bool kAlibi>
fa_status_t launch_dkdv(const void* q, const void* k, const void* v, const void* dout,
                        const void* ws, void* dk, void* dv, int BH, int H, int N, float scale,
                        int left, int right, const Extras& x, cudaStream_t st) {
  CUtensorMap mq, mkk, mv, mdo, mdk, mdv;
  if (!make_map(&mq, q, BH, N, D) || !make_map(&mkk, k, BH, N, D) ||
      !make_map(&mv, v, BH, N, D) || !make_map(&mdo, dout, BH, N, D) ||
      !make_map(&mdk, dk, BH, N, D) || !make_map(&mdv, dv, BH, N, D))
    return FA_ERR_CUDA;
  using C = fa::DkdvCfg<D>;
  if (set_smem(fa::fa_bwd_dkdv_kernel<D, kAlibi>, C::kSmemBytes) != FA_OK) return FA_ERR_CUDA;
  fa::BwdArgs a = bwd_args(ws, BH, H, N, scale, left, right, x);
  a.out0 = static_cast<__nv_bfloat16*>(dk);
  a.out1 = static_cast<__nv_bfloat16*>(dv);
  const int grid = a.n_items < sm_count() ? a.n_items : sm_count();
  fa::fa_bwd_dkdv_kernel<D, kAlibi><<<grid, C::kThreads, C::kSmemBytes, st>>>(mq, mkk, mv, mdo,
                                                                               mdk, mdv, a);
  return launched();
}

template <int D, bool kAlibi>
fa_status_t launch_dq(const void* q, const void* k, const void* v, const void* dout,
                      const void* ws, void* dq, int BH, int H, int N, float scale, int left,
                      int right, const Extras& x, cudaStream_t st) {
  CUtensorMap mq, mkk, mv, mdo, mdq;
  if (!make_map(&mq, q, BH, N, D) || !make_map(&mkk, k, BH, N, D) ||
      !make_map(&mv, v, BH, N, D) || !make_map(&mdo, dout, BH, N, D) ||
      !make_map(&mdq, dq, BH, N, D))
    return FA_ERR_CUDA;
  using C = fa::DqCfg<D>;
  if (set_smem(fa::fa_bwd_dq_kernel<D, kAlibi>, C::kSmemBytes) != FA_OK) return FA_ERR_CUDA;
  fa::BwdArgs a = bwd_args(ws, BH, H, N, scale, left, right, x);
  a.out0 = static_cast<__nv_bfloat16*>(dq);
  const int grid = a.n_items < sm_count() ? a.n_items : sm_count();
  fa::fa_bwd_dq_kernel<D, kAlibi><<<grid, C::kThreads, C::kSmemBytes, st>>>(mq, mkk, mv, mdo, mdq,
                                                                             a);
  return launched();
}

size_t workspace_bytes(int B, int H, int N) {
  const size_t raw = 2 * (size_t)B * H * padded_rows(N) * sizeof(float);
  return (raw + 255) & ~size_t(255);
}

// Checks the optional arguments of an _ex call and resolves them; a null `opt` means none.
fa_status_t resolve_options(const fa_options_t* opt, Extras* x) {
  *x = Extras();
  if (opt == nullptr) return FA_OK;
  if (opt->alibi_slopes != nullptr && (reinterpret_cast<uintptr_t>(opt->alibi_slopes) & 3u) != 0)
    return FA_ERR_MISALIGNED;
  if (opt->o_low != nullptr && !aligned16(opt->o_low)) return FA_ERR_MISALIGNED;
  if (!(opt->dropout_p == 0.f)) return FA_ERR_UNSUPPORTED;
  x->alibi = opt->alibi_slopes;
  x->kpad = opt->key_padding;
  x->o_low = opt->o_low;
  return FA_OK;
}

fa_status_t check_slopes(const float* alibi) {
  if (alibi == nullptr) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(alibi) & 3u) != 0) return FA_ERR_MISALIGNED;
  return FA_OK;
}

// The forward for every entry point: checks, then the kernel for (d, ALiBi or not).
fa_status_t forward(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                    int N, int d, float scale, int causal, fa_window_t window, const Extras& x,
                    void* stream) {
  bool empty;
  fa_status_t s = check_problem(B, H, N, d, &empty);
  if (s != FA_OK || empty) return s;
  if ((s = check_mask(scale, window)) != FA_OK) return s;
  if ((s = check_ptrs({q, k, v, o, lse})) != FA_OK) return s;
  const int right = fa::resolve_right(causal, window.right);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int l = window.left, BH = B * H;
  if (x.alibi != nullptr)
    return d == 64 ? launch_fwd<64, true>(q, k, v, o, lse, BH, H, N, scale, l, right, x, st)
                   : launch_fwd<128, true>(q, k, v, o, lse, BH, H, N, scale, l, right, x, st);
  return d == 64 ? launch_fwd<64, false>(q, k, v, o, lse, BH, H, N, scale, l, right, x, st)
                 : launch_fwd<128, false>(q, k, v, o, lse, BH, H, N, scale, l, right, x, st);
}

// Step 1 of the backward: the row statistics in `workspace`.
fa_status_t preprocess(const void* o, const void* dout, const float* lse, void* workspace, int B,
                       int H, int N, int d, const Extras& x, void* stream) {
  bool empty;
  fa_status_t s = check_problem(B, H, N, d, &empty);
  if (s != FA_OK || empty) return s;
  if ((s = check_ptrs({o, dout, lse, workspace})) != FA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* stats = static_cast<float*>(workspace);
  return d == 64 ? launch_preprocess<64>(o, x.o_low, dout, lse, stats, B * H, N, st)
                 : launch_preprocess<128>(o, x.o_low, dout, lse, stats, B * H, N, st);
}

// Step 2: dK, dV.
fa_status_t dkdv_pass(const void* q, const void* k, const void* v, const void* dout,
                      const void* workspace, void* dk, void* dv, int B, int H, int N, int d,
                      float scale, int causal, fa_window_t window, const Extras& x,
                      void* stream) {
  bool empty;
  fa_status_t s = check_problem(B, H, N, d, &empty);
  if (s != FA_OK || empty) return s;
  if ((s = check_mask(scale, window)) != FA_OK) return s;
  if ((s = check_ptrs({q, k, v, dout, workspace, dk, dv})) != FA_OK) return s;
  const int right = fa::resolve_right(causal, window.right);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int l = window.left, BH = B * H;
  if (x.alibi != nullptr)
    return d == 64 ? launch_dkdv<64, true>(q, k, v, dout, workspace, dk, dv, BH, H, N, scale, l,
                                           right, x, st)
                   : launch_dkdv<128, true>(q, k, v, dout, workspace, dk, dv, BH, H, N, scale, l,
                                            right, x, st);
  return d == 64 ? launch_dkdv<64, false>(q, k, v, dout, workspace, dk, dv, BH, H, N, scale, l,
                                          right, x, st)
                 : launch_dkdv<128, false>(q, k, v, dout, workspace, dk, dv, BH, H, N, scale, l,
                                           right, x, st);
}

// Step 3: dQ.
fa_status_t dq_pass(const void* q, const void* k, const void* v, const void* dout,
                    const void* workspace, void* dq, int B, int H, int N, int d, float scale,
                    int causal, fa_window_t window, const Extras& x, void* stream) {
  bool empty;
  fa_status_t s = check_problem(B, H, N, d, &empty);
  if (s != FA_OK || empty) return s;
  if ((s = check_mask(scale, window)) != FA_OK) return s;
  if ((s = check_ptrs({q, k, v, dout, workspace, dq})) != FA_OK) return s;
  const int right = fa::resolve_right(causal, window.right);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int l = window.left, BH = B * H;
  if (x.alibi != nullptr)
    return d == 64 ? launch_dq<64, true>(q, k, v, dout, workspace, dq, BH, H, N, scale, l, right,
                                         x, st)
                   : launch_dq<128, true>(q, k, v, dout, workspace, dq, BH, H, N, scale, l,
                                          right, x, st);
  return d == 64 ? launch_dq<64, false>(q, k, v, dout, workspace, dq, BH, H, N, scale, l, right,
                                        x, st)
                 : launch_dq<128, false>(q, k, v, dout, workspace, dq, BH, H, N, scale, l, right,
                                         x, st);
}

// The three steps of the backward, with the statistics in `stats` (caller workspace or the
// fixed array of fa_bwd_noalloc).
fa_status_t backward(const void* q, const void* k, const void* v, const void* o, const void* dout,
                     const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                     float scale, int causal, fa_window_t window, const Extras& x, void* stats,
                     void* stream) {
  fa_status_t s;
  if ((s = preprocess(o, dout, lse, stats, B, H, N, d, x, stream)) != FA_OK) return s;
  if ((s = dkdv_pass(q, k, v, dout, stats, dk, dv, B, H, N, d, scale, causal, window, x,
                     stream)) != FA_OK)
    return s;
  return dq_pass(q, k, v, dout, stats, dq, B, H, N, d, scale, causal, window, x, stream);
}

// Checks shared by every full backward before anything is launched.
fa_status_t check_backward(const void* q, const void* k, const void* v, const void* o,
                           const void* dout, const float* lse, void* dq, void* dk, void* dv,
                           int B, int H, int N, int d, float scale, fa_window_t window,
                           bool* empty) {
  fa_status_t s = check_problem(B, H, N, d, empty);
  if (s != FA_OK || *empty) return s;
  if ((s = check_mask(scale, window)) != FA_OK) return s;
  return check_ptrs({q, k, v, o, dout, lse, dq, dk, dv});
}

// ------------------------------------------------------------------------------------
// Backward without caller workspace (fa_bwd_noalloc): a fixed array in device memory
// holds the row statistics instead. Every GPU that loads the library keeps this array
// until the process exits.
// ------------------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// The driver's identifier of the calling thread's current context: unique for the life of
// the process, so that a context created after a cudaDeviceReset never matches an earlier
// one. Returns false if the driver cannot tell.
bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (get_current == nullptr || get_id == nullptr) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

constexpr int kMaxContexts = 64;
std::mutex g_noalloc_mu;
unsigned long long g_noalloc_ctx[kMaxContexts] = {0};
void* g_noalloc_ptr[kMaxContexts] = {nullptr};
int g_noalloc_used = 0;

// Device address of g_noalloc_scratch in the calling thread's current context. In host
// code the symbol names a host-side stand-in, not device memory, so the address is looked
// up with cudaGetSymbolAddress, once per context (a module is loaded per context, so the
// address belongs to the context: a cache by device number alone would go stale after a
// cudaDeviceReset or in a second context on the same device), and cached by context id.
// If no context is current yet (the runtime creates it lazily), the lookup below creates
// it and the address is cached from the next call on.
fa_status_t noalloc_scratch(void** out) {
  unsigned long long id = 0;
  const bool have_id = current_context_id(&id);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (have_id) {
    for (int i = 0; i < g_noalloc_used; ++i) {
      if (g_noalloc_ctx[i] == id) {
        *out = g_noalloc_ptr[i];
        return FA_OK;
      }
    }
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
    return FA_ERR_CUDA;
  if (have_id && g_noalloc_used < kMaxContexts) {
    g_noalloc_ctx[g_noalloc_used] = id;
    g_noalloc_ptr[g_noalloc_used] = p;
    ++g_noalloc_used;
  }
  *out = p;
  return FA_OK;
}

}  // namespace

extern "C" {

fa_status_t fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                   int N, int d, float scale, int causal, fa_window_t window, void* stream) {
  return forward(q, k, v, o, lse, B, H, N, d, scale, causal, window, Extras(), stream);
}

fa_status_t fa_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                      int H, int N, int d, float scale, int causal, fa_window_t window,
                      const fa_options_t* options, void* stream) {
  bool empty;
  fa_status_t s = check_problem(B, H, N, d, &empty);
  if (s != FA_OK || empty) return s;
  Extras x;
  if ((s = resolve_options(options, &x)) != FA_OK) return s;
  return forward(q, k, v, o, lse, B, H, N, d, scale, causal, window, x, stream);
}

fa_status_t fa_fwd_alibi(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int H, int N, int d, float scale, int causal, fa_window_t window,
                         const float* alibi_slopes, void* stream) {
  bool empty;
  fa_status_t s = check_problem(B, H, N, d, &empty);
  if (s != FA_OK || empty) return s;
  if ((s = check_slopes(alibi_slopes)) != FA_OK) return s;
  Extras x;
  x.alibi = alibi_slopes;
  return forward(q, k, v, o, lse, B, H, N, d, scale, causal, window, x, stream);
}

size_t fa_bwd_workspace_bytes(int B, int H, int N, int d) {
  bool empty;
  if (check_problem(B, H, N, d, &empty) != FA_OK || empty) return 0;
  return workspace_bytes(B, H, N);
}

fa_status_t fa_bwd_preprocess(const void* o, const void* dout, const float* lse,
                              void* workspace, int B, int H, int N, int d,
                              const fa_options_t* options, void* stream) {
  Extras x;
  fa_status_t s = resolve_options(options, &x);
  if (s != FA_OK) return s;
  return preprocess(o, dout, lse, workspace, B, H, N, d, x, stream);
}

fa_status_t fa_bwd_dkdv(const void* q, const void* k, const void* v, const void* dout,
                        const void* workspace, void* dk, void* dv, int B, int H, int N, int d,
                        float scale, int causal, fa_window_t window,
                        const fa_options_t* options, void* stream) {
  Extras x;
  fa_status_t s = resolve_options(options, &x);
  if (s != FA_OK) return s;
  return dkdv_pass(q, k, v, dout, workspace, dk, dv, B, H, N, d, scale, causal, window, x,
                   stream);
}

fa_status_t fa_bwd_dq(const void* q, const void* k, const void* v, const void* dout,
                      const void* workspace, void* dq, int B, int H, int N, int d, float scale,
                      int causal, fa_window_t window, const fa_options_t* options,
                      void* stream) {
  Extras x;
  fa_status_t s = resolve_options(options, &x);
  if (s != FA_OK) return s;
  return dq_pass(q, k, v, dout, workspace, dq, B, H, N, d, scale, causal, window, x, stream);
}

fa_status_t fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                   const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                   float scale, int causal, fa_window_t window, void* workspace,
                   size_t workspace_bytes_given, void* stream) {
  return fa_bwd_ex(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale, causal, window, nullptr,
                   workspace, workspace_bytes_given, stream);
}

fa_status_t fa_bwd_ex(const void* q, const void* k, const void* v, const void* o,
                      const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                      int H, int N, int d, float scale, int causal, fa_window_t window,
                      const fa_options_t* options, void* workspace,
                      size_t workspace_bytes_given, void* stream) {
  bool empty;
  fa_status_t s =
      check_backward(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale, window, &empty);
  if (s != FA_OK || empty) return s;
  Extras x;
  if ((s = resolve_options(options, &x)) != FA_OK) return s;
  if ((s = check_ptrs({workspace})) != FA_OK) return s;
  if (workspace_bytes_given < workspace_bytes(B, H, N)) return FA_ERR_WORKSPACE;
  return backward(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale, causal, window, x,
                  workspace, stream);
}

fa_status_t fa_bwd_alibi(const void* q, const void* k, const void* v, const void* o,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                         int H, int N, int d, float scale, int causal, fa_window_t window,
                         const float* alibi_slopes, void* workspace,
                         size_t workspace_bytes_given, void* stream) {
  bool empty;
  fa_status_t s =
      check_backward(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale, window, &empty);
  if (s != FA_OK || empty) return s;
  if ((s = check_slopes(alibi_slopes)) != FA_OK) return s;
  if ((s = check_ptrs({workspace})) != FA_OK) return s;
  if (workspace_bytes_given < workspace_bytes(B, H, N)) return FA_ERR_WORKSPACE;
  Extras x;
  x.alibi = alibi_slopes;
  return backward(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale, causal, window, x,
                  workspace, stream);
}

fa_status_t fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                           const void* dout, const float* lse, void* dq, void* dk, void* dv,
                           int B, int H, int N, int d, float scale, int causal,
                           fa_window_t window, void* stream) {
  bool empty;
  fa_status_t s =
      check_backward(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale, window, &empty);
  if (s != FA_OK || empty) return s;
  if (workspace_bytes(B, H, N) > kNoAllocScratchBytes) return FA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if ((s = noalloc_scratch(&scratch)) != FA_OK) return s;
  // The statistics are rewritten in full by the preprocess step, so nothing needs clearing.
  return backward(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale, causal, window, Extras(),
                  scratch, stream);
}

const char* fa_status_string(fa_status_t status) {
  switch (status) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG: null pointer, negative size, bad scale or window";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: head_dim must be 64 or 128, tensors < 2^31 elements, options as documented";
    case FA_ERR_MISALIGNED: return "FA_ERR_MISALIGNED: tensor pointers must be 16-byte aligned, slopes 4-byte aligned";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE: the workspace (or fa_bwd_noalloc's fixed 8 MiB array) is too small for this problem";
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

int fa_version(void) { return 200; }

}  // extern "C"
