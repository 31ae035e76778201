// tiles.cuh - which (query tile, key tile) pairs carry work, and which scores are masked.
//
// A tile is 128 consecutive rows of one (batch, head). Key j is visible from query i iff
// i - left <= j <= i + right (-1 = unbounded), both < N; causal masking forces right = 0
// (page "告别OOM和训练慢…(含A100环境配置)" §4.2, `causal`, `window_size=(-1,-1)`; page
// "Flash Attention 3.7 核心原理与实战" §3.2, "mask future positions"). Tiles whose every
// score is masked are never visited; tiles whose every score is visible skip the
// element-wise test.
#pragma once

namespace fa {

constexpr int kBlock = 128;  // rows of a tile; the M (and N) extent of every MMA

// Optional parts of the computation, compiled in as template flags so that a kernel
// without them carries no trace of them (one bit each, combined into `kFeat`).
constexpr int kFeatAlibi = 1;     // linear bias -m_h |i - j| on the scaled scores
constexpr int kFeatKpad = 2;      // (B, N) key-padding flags
constexpr int kFeatResidual = 4;  // forward also writes O - bf16(O)
constexpr int kFeatDropout = 8;   // attention weights dropped with Philox keep flags
constexpr int kFeatFp8 = 16;      // forward on e4m3 Q, K, V (P in e4m3 for the P V product)
constexpr int kFeatPacked = 32;   // a packed batch: (total, H, D) tensors, cumulative lengths
constexpr float kLog2e = 1.4426950408889634f;

struct Mask {
  int N;      // sequence length
  int left;   // -1 = unbounded
  int right;  // -1 = unbounded, 0 when causal
};

__host__ __device__ inline int resolve_right(int causal, int right) {
  return causal ? 0 : right;
}

__host__ __device__ inline int num_tiles(int N) { return (N + kBlock - 1) / kBlock; }

#ifdef __CUDACC__
// The real length of (batch, head) bh's sequence in a variable-length batch: seq_len[bh / H],
// or in a packed batch (cumulative lengths cu) cu[b + 1] - cu[b], clamped to [0, N]; N when
// the batch is not variable-length (both null).
__device__ __forceinline__ int real_length(const int* seq_len, const int* cu, int bh, int H,
                                           int N) {
  int L;
  if (cu != nullptr) {
    const int b = bh / H;
    L = __ldg(cu + b + 1) - __ldg(cu + b);
  } else if (seq_len != nullptr) {
    L = __ldg(seq_len + bh / H);
  } else {
    return N;
  }
  return L < 0 ? 0 : (L > N ? N : L);
}

// Where the rows of (batch, head) bh lie. Without cumulative lengths the tensors are
// (B*H, N, D) and the LSE (B*H, N). A packed batch (cu = B + 1 cumulative lengths, `total`
// tokens) stores the tensors as (total, H, D) and the LSE as (H, total): row r of sequence
// b is token cu[b] + r. `base` is seq_base() of the head.
__device__ __forceinline__ int seq_base(const int* cu, int bh, int H) {
  return cu != nullptr ? __ldg(cu + bh / H) : 0;
}
// element offset of row r in a D-wide tensor
__device__ __forceinline__ size_t row_at(const int* cu, int bh, int H, int N, int base, int r,
                                         int D) {
  return cu != nullptr ? ((size_t)(base + r) * H + (size_t)(bh % H)) * D
                       : ((size_t)bh * N + r) * D;
}
// index of row r in the LSE
__device__ __forceinline__ size_t lse_at(const int* cu, int total, int bh, int H, int N,
                                         int base, int r) {
  return cu != nullptr ? (size_t)(bh % H) * total + base + r : (size_t)bh * N + r;
}
// whether the kernels write row r: below N, or in a packed batch below the real length L
// and inside the tensor (a row past L is the next sequence's; offsets outside [0, total]
// write nothing)
__device__ __forceinline__ bool row_written(const int* cu, int total, int N, int L, int base,
                                            int r) {
  return cu != nullptr ? (r < L && base + r >= 0 && base + r < total) : r < N;
}
// the (y, z) coordinates of row r for a TMA copy: (r, bh) in the (D, N, B*H) view of a
// (B*H, N, D) tensor, (h, cu[b] + r) in the (D, H, total) view of a packed one
__device__ __forceinline__ int tma_y(const int* cu, int bh, int H, int r) {
  return cu != nullptr ? bh % H : r;
}
__device__ __forceinline__ int tma_z(const int* cu, int bh, int base, int r) {
  return cu != nullptr ? base + r : bh;
}
#endif

// Key tiles [lo, hi] holding at least one key visible from some valid row of query tile m.
__host__ __device__ inline void kv_tiles_for_q_tile(int m, const Mask& k, int& lo, int& hi) {
  const long long r0 = (long long)m * kBlock;
  const long long r1 = (r0 + kBlock < k.N ? r0 + kBlock : k.N) - 1;
  long long c0 = 0, c1 = k.N - 1;
  if (k.left >= 0 && r0 - k.left > c0) c0 = r0 - k.left;
  if (k.right >= 0 && r1 + k.right < c1) c1 = r1 + k.right;
  lo = (int)(c0 / kBlock);
  hi = (int)(c1 / kBlock);
}

// Query tiles [lo, hi] holding at least one valid row that sees some key of key tile j.
__host__ __device__ inline void q_tiles_for_kv_tile(int j, const Mask& k, int& lo, int& hi) {
  const long long c0 = (long long)j * kBlock;
  const long long c1 = (c0 + kBlock < k.N ? c0 + kBlock : k.N) - 1;
  long long r0 = 0, r1 = k.N - 1;
  if (k.right >= 0 && c0 - k.right > r0) r0 = c0 - k.right;
  if (k.left >= 0 && c1 + k.left < r1) r1 = c1 + k.left;
  lo = (int)(r0 / kBlock);
  hi = (int)(r1 / kBlock);
}

// True when every (row, key) of the pair (query tile qt, key tile kt) is visible and valid.
__host__ __device__ inline bool tile_all_visible(int qt, int kt, const Mask& k) {
  const long long r0 = (long long)qt * kBlock, r1 = r0 + kBlock - 1;
  const long long c0 = (long long)kt * kBlock, c1 = c0 + kBlock - 1;
  if (r1 >= k.N || c1 >= k.N) return false;
  if (k.right >= 0 && c1 - r0 > k.right) return false;
  if (k.left >= 0 && r1 - c0 > k.left) return false;
  return true;
}

__host__ __device__ inline bool is_visible(int r, int c, const Mask& k) {
  return r < k.N && c < k.N && (k.left < 0 || r - c <= k.left) &&
         (k.right < 0 || c - r <= k.right);
}

// Keys col_base + [c_lo, c_hi] of the `width` keys from col_base that query `row` sees
// (c_lo > c_hi when none): the per-row form of is_visible, for masking a row of scores
// with two compares per element.
__host__ __device__ inline void visible_keys(int row, long long col_base, int width,
                                             const Mask& k, int& c_lo, int& c_hi) {
  long long lo = 0, hi = width - 1;
  if (k.left >= 0 && row - k.left - col_base > lo) lo = row - k.left - col_base;
  if (k.right >= 0 && row + (long long)k.right - col_base < hi) hi = row + (long long)k.right - col_base;
  if (k.N - 1 - col_base < hi) hi = k.N - 1 - col_base;
  if (row >= k.N) hi = -1;
  c_lo = (int)(lo > width ? width : lo);
  c_hi = (int)(hi < -1 ? -1 : hi);
}

// Queries row_base + [r_lo, r_hi] of the `width` queries from row_base that see key `col`
// (r_lo > r_hi when none): the per-key form of is_visible.
__host__ __device__ inline void visible_queries(int col, long long row_base, int width,
                                                const Mask& k, int& r_lo, int& r_hi) {
  long long lo = 0, hi = width - 1;
  if (k.right >= 0 && col - k.right - row_base > lo) lo = col - k.right - row_base;
  if (k.left >= 0 && col + (long long)k.left - row_base < hi) hi = col + (long long)k.left - row_base;
  if (k.N - 1 - row_base < hi) hi = k.N - 1 - row_base;
  if (col >= k.N) hi = -1;
  r_lo = (int)(lo > width ? width : lo);
  r_hi = (int)(hi < -1 ? -1 : hi);
}

// Work item k of a persistent schedule over BH heads of T tiles each, for masked problems
// (tiles of different lengths). Heads go in chunks of `group` (chosen so that a chunk has
// about one item per SM): every CTA works on a few heads at a time, whose K/V (or Q/dO)
// tiles then stay in L2 while all of them are read. Inside a chunk, items go longest
// first: tile index increasing when `rising` (dK/dV: key tile 0 is seen by the most query
// tiles), decreasing otherwise (forward, dQ: the last query tile sees the most keys).
__host__ __device__ inline void chunked_item(int k, int BH, int T, int group, bool rising,
                                             int& bh, int& tile) {
  const int per_chunk = group * T;
  const int chunk = k / per_chunk;
  const int r = k - chunk * per_chunk;
  const int heads = (BH - chunk * group) < group ? (BH - chunk * group) : group;
  const int step = r / heads;
  bh = chunk * group + (r - step * heads);
  tile = rising ? step : T - 1 - step;
}

// Work item of slot k of a persistent schedule for causal problems, where tile t of a head
// has work growing linearly with t (or with T - 1 - t): the items go in pairs of a tile and
// its complement T - 1 - t of the same head, whose work adds up to the same for every pair.
// CTA c (of P) takes pair q = (r / 2) P + c of its rounds r = 2m, 2m + 1: the longer item in
// round 2m, the shorter in 2m + 1. Every CTA then gets nearly the same work, and the two
// items of a pair read the same head's tiles one after the other (from L2 the second time).
// Returns false for the slots past the last pair (n_double = BH T / 2 pairs, T even).
// `rising`: tile 0 is the longest (dK/dV), else tile T - 1 (forward, dQ).
__host__ __device__ inline bool paired_item(int k, int P, int n_double, int T, bool rising,
                                            int& bh, int& tile) {
  const int r = k / P;
  const int c = k - r * P;
  const int q = (r >> 1) * P + c;
  if (q >= n_double) return false;
  const int half = T / 2;
  bh = q / half;
  const int p = q - bh * half;
  const int longer = rising ? p : T - 1 - p;
  tile = (r & 1) ? T - 1 - longer : longer;
  return true;
}

// ---- The schedule of a variable-length batch ----
// With real lengths L_b the work of an item is set by the distance u of its tile from the
// start of the sequence (query tiles: a causal query tile i sees i + 1 key tiles) or from
// its end (key tiles: causal key tile j is seen by T_b - j query tiles, T_b the tiles of
// L_b); u counts units, a unit being a tile or, in the forward, the per_item query tiles
// of an item. Items go in order of u, largest first. Bucket u holds the H heads of every
// batch entry with more than u units, and those entries are the first M_u of the batch
// entries ordered by units, most first (ties by index), so that an item's position is
// resolved by one search over the buckets. Slot k of a grid of P persistent CTAs takes
// position p of that order, the rounds of P positions alternating in direction (CTA c
// takes positions c, 2P - 1 - c, 2P + c, ...), which evens out what the CTAs add up along
// a decreasing sequence. Entries past a sequence's last unit are never scheduled.
//
// Tables, in ints: start[0 .. U] (start[q] = position of the first item of bucket
// u = U - 1 - q; start[U] = the number of items), sigma[0 .. B) (the ordered batch
// entries), then U + 1 ints of scratch for building them.
__host__ __device__ inline int varlen_sched_ints(int B, int U) { return 2 * (U + 1) + B; }

// What the backward's preprocess kernel needs to build the tables of the schedule above
// (one unit per tile) in one block past its row blocks; `tables` null = none.
struct SchedBuild {
  const int* seq_len;
  const int* cu;  // or cumulative lengths (a packed batch)
  int* tables;
  int B;
  int H;
  int N;
  int U;  // tiles per head
};

// Largest batch for which the schedule above is built (the build is one warp's pass over
// the batch); larger batches keep the chunked schedule.
constexpr int kVarlenSchedMaxB = 8192;

#ifdef __CUDACC__
__device__ __forceinline__ int varlen_units(const int* seq_len, const int* cu, int b, int N,
                                            int per_item) {
  int L = cu != nullptr ? cu[b + 1] - cu[b] : seq_len[b];
  L = L < 0 ? 0 : (L > N ? N : L);
  return (num_tiles(L) + per_item - 1) / per_item;
}

// Builds the tables of the schedule above from the lengths seq_len (or the cumulative
// lengths cu); called by all 32 lanes of one warp.
__device__ __forceinline__ void build_varlen_sched(const int* seq_len, const int* cu, int B,
                                                   int H, int N, int per_item, int U,
                                                   int* tables) {
  int* start = tables;
  int* sigma = tables + U + 1;
  int* cnt = sigma + B;  // cnt[v], v in [0, U]: entries with v units, then a running count
  const int lane = threadIdx.x & 31;
  for (int v = lane; v <= U; v += 32) cnt[v] = 0;
  __syncwarp();
  // counted without atomics (the tables may be in global memory): the lowest lane of each
  // group of lanes with equal units adds the group's size
  for (int b0 = 0; b0 < B; b0 += 32) {
    const int b = b0 + lane;
    const int u = b < B ? varlen_units(seq_len, cu, b, N, per_item) : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, u);
    if (b < B && (peers & ((1u << lane) - 1u)) == 0) cnt[u] += __popc(peers);
    __syncwarp();
  }
  // M(q) = entries with more than u = U - 1 - q units = sum of cnt[v] over v >= U - q;
  // bucket q has H M(q) items: start is the exclusive prefix sum of H M
  int carry_m = 0, carry_s = 0;
  if (lane == 0) start[0] = 0;
  for (int q0 = 0; q0 < U; q0 += 32) {
    const int q = q0 + lane;
    int m = q < U ? cnt[U - q] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, m, off);
      if (lane >= off) m += t;
    }
    m += carry_m;
    int s = q < U ? H * m : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, s, off);
      if (lane >= off) s += t;
    }
    s += carry_s;
    if (q < U) start[q + 1] = s;
    carry_m = __shfl_sync(0xffffffffu, m, 31);
    carry_s = __shfl_sync(0xffffffffu, s, 31);
  }
  __syncwarp();
  for (int v = lane; v <= U; v += 32) cnt[v] = 0;
  __syncwarp();
  // rank of entry b = (entries with more units) + (earlier entries with as many units)
  for (int b0 = 0; b0 < B; b0 += 32) {
    const int b = b0 + lane;
    const int u = b < B ? varlen_units(seq_len, cu, b, N, per_item) : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, u);
    const int before = __popc(peers & ((1u << lane) - 1u));
    const int seen = b < B ? cnt[u] : 0;
    __syncwarp();
    if (b < B) {
      const int more = u >= U ? 0 : (start[U - u] - start[U - 1 - u]) / H;
      sigma[more + seen + before] = b;
      if (before == 0) cnt[u] = seen + __popc(peers);
    }
    __syncwarp();
  }
}

#endif

// Slot k of the schedule above over a grid of P CTAs: the item's (batch*head) and its unit
// distance u, or false past the last item.
__host__ __device__ inline bool varlen_item(int k, int P, const int* tables, int U, int H,
                                            int& bh, int& u) {
  const int* start = tables;
  const int* sigma = tables + U + 1;
  const int r = k / P;
  const int c = k - r * P;
  const int p = r * P + ((r & 1) ? P - 1 - c : c);
  if (p >= start[U]) return false;
  int lo = 0, hi = U - 1;  // the last bucket q with start[q] <= p (it is not empty)
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (start[mid] <= p) {
      lo = mid;
    } else {
      hi = mid - 1;
    }
  }
  const int idx = p - start[lo];
  const int e = idx / H;
  u = U - 1 - lo;
  bh = sigma[e] * H + (idx - e * H);
  return true;
}

}  // namespace fa
