// fa_api.cu - host side of the C ABI declared in include/fa.h.
//
// Validates every argument before touching the GPU, resolves the options into a kernel
// variant and calls the launchers of the kernel units (fa_kern_*.cu) on the caller's
// stream. Holds the fixed device array of fa_bwd_noalloc.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>
#include <utility>

#include <cuda.h>
#include <cuda_runtime.h>

#include "fa.h"
#include "launch.h"

namespace {

using fa_host::Extras;
using fa_host::Problem;

// Test hook set by fa_debug_set_fault(); 0 in normal operation.
std::atomic<int> g_fault{0};

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

// check_problem, and for a packed batch (cumulative lengths) its token count: a (total, H, d)
// tensor must also have fewer than 2^31 elements; no tokens is an empty problem.
fa_status_t check_problem_x(int B, int H, int N, int d, const Extras& x, bool* empty) {
  const fa_status_t s = check_problem(B, H, N, d, empty);
  if (s != FA_OK || *empty || x.cu == nullptr) return s;
  if ((long long)x.total * H * d >= (1ll << 31)) return FA_ERR_UNSUPPORTED;
  if (x.total == 0) *empty = true;
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

// Calls L::template run<F>(args...) for the compile-time F in Fs... equal to `feat`; the
// lists below are the feature sets each kernel family is instantiated for.
template <typename L, int... Fs, typename... Args>
fa_status_t dispatch_features(std::integer_sequence<int, Fs...>, int feat, Args&&... args) {
  fa_status_t s = FA_ERR_UNSUPPORTED;
  const bool found = ((feat == Fs ? (s = L::template run<Fs>(std::forward<Args>(args)...), true)
                                  : false) || ...);
  return found ? s : FA_ERR_UNSUPPORTED;
}

// forward: every combination of ALiBi, key padding, residual and dropout, in the (B, H, N, d)
// layout and packed (kFeatPacked = 32); at head_dim 128 also the e4m3 forward
using FwdFeatures64 = std::integer_sequence<int, 0, 1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 12, 13, 14,
                                            15, 32, 33, 34, 35, 36, 37, 38, 39, 40, 41, 42, 43,
                                            44, 45, 46, 47>;
using FwdFeatures128 = std::integer_sequence<int, 0, 1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 12, 13,
                                             14, 15, 16, 32, 33, 34, 35, 36, 37, 38, 39, 40, 41,
                                             42, 43, 44, 45, 46, 47>;
// backward passes: ALiBi, key padding and dropout (the residual only changes delta), in both
// layouts; the fused pass only in the (B, H, N, d) layout
using BwdFeatures = std::integer_sequence<int, 0, 1, 2, 3, 8, 9, 10, 11, 32, 33, 34, 35, 40, 41,
                                          42, 43>;
using FusedFeatures = std::integer_sequence<int, 0, 1, 2, 3, 8, 9, 10, 11>;

// The launchers as class templates over the feature flags, for dispatch_features.
template <int D>
struct FwdLaunch {
  template <int F, typename... Args>
  static fa_status_t run(Args&&... args) {
    return fa_host::launch_fwd<D, F>(std::forward<Args>(args)...);
  }
};
template <int D>
struct DkdvLaunch {
  template <int F, typename... Args>
  static fa_status_t run(Args&&... args) {
    return fa_host::launch_dkdv<D, F>(std::forward<Args>(args)...);
  }
};
template <int D>
struct DqLaunch {
  template <int F, typename... Args>
  static fa_status_t run(Args&&... args) {
    return fa_host::launch_dq<D, F>(std::forward<Args>(args)...);
  }
};

struct FusedLaunch {
  template <int F, typename... Args>
  static fa_status_t run(Args&&... args) {
    return fa_host::launch_fused<F>(std::forward<Args>(args)...);
  }
};

int padded_rows(int N) { return fa::num_tiles(N) * fa::kBlock; }

// Workspace of the backward: the row statistics (two fp32 arrays of B*H*Np), then, for the
// fused pass (head_dim 64), the fp32 dQ accumulator (B*H*Np rows of 64), each part rounded
// up to 256 bytes.
size_t stats_bytes(int B, int H, int N) {
  const size_t raw = 2 * (size_t)B * H * padded_rows(N) * sizeof(float);
  return (raw + 255) & ~size_t(255);
}

bool uses_fused(int d, const Extras& x) { return d == 64 && x.fused; }

size_t dq_acc_bytes(int B, int H, int N, int d) {
  return (size_t)B * H * padded_rows(N) * (size_t)d * sizeof(float);
}

// A variable-length batch (up to kVarlenSchedMaxB entries) adds, last, the tables of its
// schedule (varlen_item), which the preprocess step writes.
size_t sched_bytes(int B, int N, const Extras& x) {
  if (!x.varlen() || B > fa::kVarlenSchedMaxB) return 0;
  const size_t raw = 4 * (size_t)fa::varlen_sched_ints(B, fa::num_tiles(N));
  return (raw + 255) & ~size_t(255);
}

size_t workspace_bytes(int B, int H, int N, int d, const Extras& x) {
  return stats_bytes(B, H, N) + (uses_fused(d, x) ? dq_acc_bytes(B, H, N, d) : 0) +
         sched_bytes(B, N, x);
}

float* dq_acc_of(void* workspace, int B, int H, int N) {
  return reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + stats_bytes(B, H, N));
}

// The schedule tables in `workspace`, or null without them.
int* sched_of(const void* workspace, int B, int H, int N, int d, const Extras& x) {
  if (sched_bytes(B, N, x) == 0) return nullptr;
  const size_t off = stats_bytes(B, H, N) + (uses_fused(d, x) ? dq_acc_bytes(B, H, N, d) : 0);
  return reinterpret_cast<int*>(static_cast<uint8_t*>(const_cast<void*>(workspace)) + off);
}

// x with the schedule tables of `workspace` (a variable-length batch).
Extras with_sched(const Extras& x, const void* workspace, int B, int H, int N, int d) {
  Extras xs = x;
  xs.sched = sched_of(workspace, B, H, N, d, x);
  return xs;
}

// Checks the optional arguments of an _ex call and resolves them; a null `opt` means none.
fa_status_t resolve_options(const fa_options_t* opt, Extras* x) {
  *x = Extras();
  if (opt == nullptr) return FA_OK;
  if (opt->alibi_slopes != nullptr && (reinterpret_cast<uintptr_t>(opt->alibi_slopes) & 3u) != 0)
    return FA_ERR_MISALIGNED;
  if (opt->o_low != nullptr && !aligned16(opt->o_low)) return FA_ERR_MISALIGNED;
  // dropout: t = floor(256 p + 1/2) must leave some weights (t <= 255); the offset is the
  // fourth 32-bit counter word
  const float p = opt->dropout_p;
  if (!(p >= 0.f && p < 1.f) || opt->dropout_offset > 0xFFFFFFFFull) return FA_ERR_INVALID_ARG;
  const int t = (int)std::floor(256.0 * (double)p + 0.5);
  if (t > 255) return FA_ERR_INVALID_ARG;
  if ((opt->flags & ~(unsigned)FA_BWD_FUSED) != 0) return FA_ERR_INVALID_ARG;
  x->alibi = opt->alibi_slopes;
  x->kpad = opt->key_padding;
  x->o_low = opt->o_low;
  x->fused = (opt->flags & FA_BWD_FUSED) != 0;
  if (opt->seq_lengths != nullptr && (reinterpret_cast<uintptr_t>(opt->seq_lengths) & 3u) != 0)
    return FA_ERR_MISALIGNED;
  x->seq_len = opt->seq_lengths;
  // a packed batch: exclusive with seq_lengths, a token count >= 0, not the fused backward
  // (its dQ conversion takes no options)
  if (opt->cu_seqlens != nullptr) {
    if ((reinterpret_cast<uintptr_t>(opt->cu_seqlens) & 3u) != 0) return FA_ERR_MISALIGNED;
    if (opt->seq_lengths != nullptr || opt->total_tokens < 0) return FA_ERR_INVALID_ARG;
    if (x->fused) return FA_ERR_UNSUPPORTED;
    x->cu = opt->cu_seqlens;
    x->total = opt->total_tokens;
  }
  if (t > 0) {
    x->dropout = true;
    x->drop.seed_lo = (uint32_t)(opt->dropout_seed & 0xFFFFFFFFull);
    x->drop.seed_hi = (uint32_t)(opt->dropout_seed >> 32);
    x->drop.offset = (uint32_t)opt->dropout_offset;
    x->drop.threshold = (uint32_t)t;
    x->drop.keep_scale = (float)(256.0 / (256.0 - t));
  }
  return FA_OK;
}

fa_status_t check_slopes(const float* alibi) {
  if (alibi == nullptr) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(alibi) & 3u) != 0) return FA_ERR_MISALIGNED;
  return FA_OK;
}

// Variable-length batches: what the kernels leave past each entry's real length.
fa_status_t fill(void* t0, void* t1, void* t2, float* lse, int d, int BH, int H, int N,
                 const Extras& x, cudaStream_t st) {
  return d == 64 ? fa_host::launch_fill_past_length<64>(t0, t1, t2, lse, x.seq_len, BH, H, N, st)
                 : fa_host::launch_fill_past_length<128>(t0, t1, t2, lse, x.seq_len, BH, H, N, st);
}

// The forward for every entry point: checks, then the kernel for (d, ALiBi or not).
fa_status_t forward(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                    int N, int d, float scale, int causal, fa_window_t window, const Extras& x,
                    void* stream) {
  bool empty;
  fa_status_t s = check_problem_x(B, H, N, d, x, &empty);
  if (s != FA_OK || empty) return s;
  if ((s = check_mask(scale, window)) != FA_OK) return s;
  if ((s = check_ptrs({q, k, v, o, lse})) != FA_OK) return s;
  const int right = fa::resolve_right(causal, window.right);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int l = window.left, BH = B * H;
  const Problem pb{BH, H, N, scale, l, right};
  const int fault = g_fault.load(std::memory_order_relaxed);
  s = d == 64 ? dispatch_features<FwdLaunch<64>>(FwdFeatures64(), x.features(), q, k, v, o, lse,
                                                 pb, x, fault, st)
              : dispatch_features<FwdLaunch<128>>(FwdFeatures128(), x.features(), q, k, v, o,
                                                  lse, pb, x, fault, st);
  if (s != FA_OK || x.seq_len == nullptr) return s;
  return fill(o, x.o_low, nullptr, lse, d, BH, H, N, x, st);
}

// Step 1 of the backward: the row statistics in `workspace`.
fa_status_t preprocess(const void* o, const void* dout, const float* lse, void* workspace, int B,
                       int H, int N, int d, const Extras& x, void* stream) {
  bool empty;
  fa_status_t s = check_problem_x(B, H, N, d, x, &empty);
  if (s != FA_OK || empty) return s;
  if ((s = check_ptrs({o, dout, lse, workspace})) != FA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* stats = static_cast<float*>(workspace);
  // the fused pass accumulates dQ: its accumulator starts at zero
  float* acc = uses_fused(d, x) ? dq_acc_of(workspace, B, H, N) : nullptr;
  // and with real lengths, the tables of the passes' schedule
  const fa::SchedBuild sb{x.seq_len, x.cu, sched_of(workspace, B, H, N, d, x), B, H, N,
                          fa::num_tiles(N)};
  return d == 64
             ? fa_host::launch_preprocess<64>(o, x.o_low, dout, lse, stats, acc, sb, x.cu,
                                              x.total, H, B * H, N, st)
             : fa_host::launch_preprocess<128>(o, x.o_low, dout, lse, stats, acc, sb, x.cu,
                                               x.total, H, B * H, N, st);
}

// The fused pass (head_dim 64): dK, dV, and dQ added into the workspace's accumulator.
fa_status_t fused_pass(const void* q, const void* k, const void* v, const void* dout,
                       void* workspace, void* dk, void* dv, int B, int H, int N, int d,
                       float scale, int causal, fa_window_t window, const Extras& x,
                       void* stream) {
  bool empty;
  fa_status_t s = check_problem_x(B, H, N, d, x, &empty);
  if (s != FA_OK || empty) return s;
  if (d != 64) return FA_ERR_UNSUPPORTED;
  if ((s = check_mask(scale, window)) != FA_OK) return s;
  if ((s = check_ptrs({q, k, v, dout, workspace, dk, dv})) != FA_OK) return s;
  const int right = fa::resolve_right(causal, window.right);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Problem pb{B * H, H, N, scale, window.left, right};
  const int feat = x.features() & ~fa::kFeatResidual;
  const Extras xs = with_sched(x, workspace, B, H, N, d);
  s = dispatch_features<FusedLaunch>(FusedFeatures(), feat, q, k, v, dout, workspace,
                                     dq_acc_of(workspace, B, H, N), dk, dv, pb, xs, st);
  // rows of dQ past the real length stay zero in the accumulator
  if (s != FA_OK || x.seq_len == nullptr) return s;
  return fill(dk, dv, nullptr, nullptr, d, B * H, H, N, x, st);
}

// dQ from the fused pass's accumulator.
fa_status_t dq_convert(void* workspace, void* dq, int B, int H, int N, int d, float scale,
                       void* stream) {
  bool empty;
  fa_status_t s = check_problem(B, H, N, d, &empty);
  if (s != FA_OK || empty) return s;
  if (d != 64) return FA_ERR_UNSUPPORTED;
  if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
  if ((s = check_ptrs({workspace, dq})) != FA_OK) return s;
  return fa_host::launch_dq_convert<64>(dq_acc_of(workspace, B, H, N), dq, B * H, N, scale,
                                        static_cast<cudaStream_t>(stream));
}

// Step 2: dK, dV.
fa_status_t dkdv_pass(const void* q, const void* k, const void* v, const void* dout,
                      const void* workspace, void* dk, void* dv, int B, int H, int N, int d,
                      float scale, int causal, fa_window_t window, const Extras& x,
                      void* stream) {
  bool empty;
  fa_status_t s = check_problem_x(B, H, N, d, x, &empty);
  if (s != FA_OK || empty) return s;
  if ((s = check_mask(scale, window)) != FA_OK) return s;
  if ((s = check_ptrs({q, k, v, dout, workspace, dk, dv})) != FA_OK) return s;
  const int right = fa::resolve_right(causal, window.right);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int l = window.left, BH = B * H;
  const int feat = x.features() & ~fa::kFeatResidual;
  const Problem pb{BH, H, N, scale, l, right};
  const Extras xs = with_sched(x, workspace, B, H, N, d);
  s = d == 64 ? dispatch_features<DkdvLaunch<64>>(BwdFeatures(), feat, q, k, v, dout, workspace,
                                                  dk, dv, pb, xs, st)
              : dispatch_features<DkdvLaunch<128>>(BwdFeatures(), feat, q, k, v, dout, workspace,
                                                   dk, dv, pb, xs, st);
  if (s != FA_OK || x.seq_len == nullptr) return s;
  return fill(dk, dv, nullptr, nullptr, d, BH, H, N, x, st);
}

// Step 3: dQ.
fa_status_t dq_pass(const void* q, const void* k, const void* v, const void* dout,
                    const void* workspace, void* dq, int B, int H, int N, int d, float scale,
                    int causal, fa_window_t window, const Extras& x, void* stream) {
  bool empty;
  fa_status_t s = check_problem_x(B, H, N, d, x, &empty);
  if (s != FA_OK || empty) return s;
  if ((s = check_mask(scale, window)) != FA_OK) return s;
  if ((s = check_ptrs({q, k, v, dout, workspace, dq})) != FA_OK) return s;
  const int right = fa::resolve_right(causal, window.right);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int l = window.left, BH = B * H;
  const int feat = x.features() & ~fa::kFeatResidual;
  const Problem pb{BH, H, N, scale, l, right};
  const Extras xs = with_sched(x, workspace, B, H, N, d);
  s = d == 64 ? dispatch_features<DqLaunch<64>>(BwdFeatures(), feat, q, k, v, dout, workspace,
                                                dq, pb, xs, st)
              : dispatch_features<DqLaunch<128>>(BwdFeatures(), feat, q, k, v, dout, workspace,
                                                 dq, pb, xs, st);
  if (s != FA_OK || x.seq_len == nullptr) return s;
  return fill(dq, nullptr, nullptr, nullptr, d, BH, H, N, x, st);
}

// The three steps of the backward, with the statistics in `stats` (caller workspace or the
// fixed array of fa_bwd_noalloc).
fa_status_t backward(const void* q, const void* k, const void* v, const void* o, const void* dout,
                     const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                     float scale, int causal, fa_window_t window, const Extras& x, void* stats,
                     void* stream) {
  fa_status_t s;
  if ((s = preprocess(o, dout, lse, stats, B, H, N, d, x, stream)) != FA_OK) return s;
  if (uses_fused(d, x)) {
    if ((s = fused_pass(q, k, v, dout, stats, dk, dv, B, H, N, d, scale, causal, window, x,
                        stream)) != FA_OK)
      return s;
    return dq_convert(stats, dq, B, H, N, d, scale, stream);
  }
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

// The library is compiled with hidden visibility: only the entry points of include/fa.h
// are exported.
#pragma GCC visibility push(default)
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

fa_status_t fa_fwd_fp8(const void* q, const void* k, const void* v, float q_scale, float k_scale,
                       float v_scale, void* o, float* lse, int B, int H, int N, int d,
                       float scale, int causal, fa_window_t window, void* stream) {
  bool empty;
  fa_status_t s = check_problem(B, H, N, d, &empty);
  if (s != FA_OK || empty) return s;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  for (float f : {q_scale, k_scale, v_scale})
    if (!std::isfinite(f) || !(f > 0.f)) return FA_ERR_INVALID_ARG;
  if ((s = check_mask(scale, window)) != FA_OK) return s;
  const float s_all = scale * q_scale * k_scale;  // the descales of Q and K join the scale
  if (!std::isfinite(s_all) || !(s_all > 0.f)) return FA_ERR_INVALID_ARG;
  Extras x;
  x.fp8 = true;
  x.o_scale = v_scale;
  return forward(q, k, v, o, lse, B, H, N, d, s_all, causal, window, x, stream);
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
  return workspace_bytes(B, H, N, d, Extras());
}

size_t fa_bwd_workspace_bytes_ex(int B, int H, int N, int d, const fa_options_t* options) {
  bool empty;
  if (check_problem(B, H, N, d, &empty) != FA_OK || empty) return 0;
  Extras x;
  if (resolve_options(options, &x) != FA_OK) return 0;
  return workspace_bytes(B, H, N, d, x);
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

fa_status_t fa_bwd_fused(const void* q, const void* k, const void* v, const void* dout,
                         void* workspace, void* dk, void* dv, int B, int H, int N, int d,
                         float scale, int causal, fa_window_t window, const fa_options_t* options,
                         void* stream) {
  Extras x;
  fa_status_t s = resolve_options(options, &x);
  if (s != FA_OK) return s;
  return fused_pass(q, k, v, dout, workspace, dk, dv, B, H, N, d, scale, causal, window, x,
                    stream);
}

fa_status_t fa_bwd_dq_convert(void* workspace, void* dq, int B, int H, int N, int d, float scale,
                              void* stream) {
  return dq_convert(workspace, dq, B, H, N, d, scale, stream);
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
  if (workspace_bytes_given < workspace_bytes(B, H, N, d, x)) return FA_ERR_WORKSPACE;
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
  Extras x;
  x.alibi = alibi_slopes;
  if (workspace_bytes_given < workspace_bytes(B, H, N, d, x)) return FA_ERR_WORKSPACE;
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
  // the three-kernel backward, whose only scratch is the row statistics
  Extras x;
  if (workspace_bytes(B, H, N, d, x) > kNoAllocScratchBytes) return FA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if ((s = noalloc_scratch(&scratch)) != FA_OK) return s;
  // The statistics are rewritten in full by the preprocess step, so nothing needs clearing.
  return backward(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale, causal, window, x,
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
  // every kernel unit has its own copy of the status word: read and clear them all
  const int words[9] = {fa_host::take_status_fwd64(),  fa_host::take_status_fwd128(),
                        fa_host::take_status_bwd64(),  fa_host::take_status_bwd128(),
                        fa_host::take_status_fused64(), fa_host::take_status_fwdp64(),
                        fa_host::take_status_fwdp128(), fa_host::take_status_bwdp64(),
                        fa_host::take_status_bwdp128()};
  bool timeout = false;
  for (int w : words) {
    if (w < 0) return FA_ERR_CUDA;
    if (w != 0) timeout = true;
  }
  return timeout ? FA_ERR_TIMEOUT : FA_OK;
}

fa_status_t fa_debug_set_fault(int fault) {
  if (fault < 0 || fault > 1) return FA_ERR_INVALID_ARG;
  g_fault.store(fault, std::memory_order_relaxed);
  return FA_OK;
}

int fa_version(void) { return 200; }

}  // extern "C"
#pragma GCC visibility pop
