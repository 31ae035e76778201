// Host-side check of the tile and mask logic the kernels share (tiles.cuh), against
// brute force over every (query, key) pair: the key-tile ranges of a query tile and the
// query-tile ranges of a key tile hold exactly the tiles with a visible pair, the
// per-row and per-key column ranges equal the element-wise visibility test, and the
// chunked schedule visits every (head, tile) item exactly once. Prints "OK" or the first
// mismatch and exits non-zero.
#define __host__
#define __device__
#include <algorithm>
#include <cstdio>
#include <vector>
#include "tiles.cuh"

using namespace fa;

static int fail(const char* what, int a, int b, int c, int d) {
  std::printf("FAIL %s (%d %d %d %d)\n", what, a, b, c, d);
  return 1;
}

static int check_mask(const Mask& mk) {
  const int N = mk.N, T = num_tiles(N);
  for (int m = 0; m < T; ++m) {
    int lo, hi;
    kv_tiles_for_q_tile(m, mk, lo, hi);
    for (int j = 0; j < T; ++j) {
      bool any = false, all = true;
      for (int r = m * kBlock; r < m * kBlock + kBlock; ++r)
        for (int c = j * kBlock; c < j * kBlock + kBlock; ++c) {
          const bool v = is_visible(r, c, mk);
          any = any || v;
          all = all && v;
        }
      if (any != (lo <= j && j <= hi)) return fail("kv_tiles_for_q_tile", N, mk.left, m, j);
      if (all != tile_all_visible(m, j, mk)) return fail("tile_all_visible", N, mk.left, m, j);
    }
  }
  for (int j = 0; j < T; ++j) {
    int lo, hi;
    q_tiles_for_kv_tile(j, mk, lo, hi);
    for (int m = 0; m < T; ++m) {
      bool any = false;
      for (int r = m * kBlock; r < m * kBlock + kBlock && !any; ++r)
        for (int c = j * kBlock; c < j * kBlock + kBlock && !any; ++c) any = is_visible(r, c, mk);
      if (any != (lo <= m && m <= hi)) return fail("q_tiles_for_kv_tile", N, mk.left, j, m);
    }
  }
  const int widths[3] = {32, 64, 128};
  for (int w : widths)
    for (int base = 0; base < T * kBlock; base += w)
      for (int x = 0; x < T * kBlock; ++x) {
        int lo, hi;
        visible_keys(x, base, w, mk, lo, hi);
        for (int c = 0; c < w; ++c)
          if ((lo <= c && c <= hi) != is_visible(x, base + c, mk))
            return fail("visible_keys", N, x, base, c);
        visible_queries(x, base, w, mk, lo, hi);
        for (int r = 0; r < w; ++r)
          if ((lo <= r && r <= hi) != is_visible(base + r, x, mk))
            return fail("visible_queries", N, x, base, r);
      }
  return 0;
}

int main() {
  const int Ns[5] = {1, 127, 128, 300, 640};
  const int windows[7][2] = {{-1, -1}, {-1, 0}, {0, 0}, {100, 0}, {0, 37}, {200, 129}, {5, -1}};
  for (int N : Ns)
    for (auto& w : windows) {
      const Mask mk{N, w[0], w[1]};
      if (check_mask(mk)) return 1;
    }
  for (int BH = 1; BH <= 7; ++BH)
    for (int T = 1; T <= 9; ++T)
      for (int group = 1; group <= BH; ++group)
        for (int rising = 0; rising < 2; ++rising) {
          std::vector<int> seen(BH * T, 0);
          for (int k = 0; k < BH * T; ++k) {
            int bh, tile;
            chunked_item(k, BH, T, group, rising != 0, bh, tile);
            if (bh < 0 || bh >= BH || tile < 0 || tile >= T) return fail("chunked_item range", BH, T, group, k);
            ++seen[bh * T + tile];
          }
          for (int v : seen)
            if (v != 1) return fail("chunked_item cover", BH, T, group, rising);
        }
  // paired_item: over the whole round pairs of P CTAs every (head, tile) appears exactly
  // once, each CTA's two items of a round pair are a tile and its complement of one head
  // (longer first), and with work t + 1 (or T - t) per tile every pair weighs T + 1.
  for (int BH = 1; BH <= 9; ++BH)
    for (int T = 2; T <= 12; T += 2)
      for (int P = 1; P <= 13; ++P)
        for (int rising = 0; rising < 2; ++rising) {
          const int n_double = BH * (T / 2);
          const int Pg = n_double < P ? n_double : P;
          const int slots = 2 * ((n_double + Pg - 1) / Pg) * Pg;
          std::vector<int> seen(BH * T, 0);
          for (int k = 0; k < slots; ++k) {
            int bh, tile;
            if (!paired_item(k, Pg, n_double, T, rising != 0, bh, tile)) continue;
            if (bh < 0 || bh >= BH || tile < 0 || tile >= T) return fail("paired_item range", BH, T, Pg, k);
            ++seen[bh * T + tile];
            const int r = k / Pg;
            if (r % 2 == 1) {
              int bh0, tile0;
              if (!paired_item(k - Pg, Pg, n_double, T, rising != 0, bh0, tile0))
                return fail("paired_item partner", BH, T, Pg, k);
              const int w0 = rising ? T - tile0 : tile0 + 1, w1 = rising ? T - tile : tile + 1;
              if (bh0 != bh || tile0 + tile != T - 1 || w0 < w1 || w0 + w1 != T + 1)
                return fail("paired_item pair", BH, T, Pg, k);
            }
          }
          for (int v : seen)
            if (v != 1) return fail("paired_item cover", BH, T, Pg, rising);
        }
  // varlen_item: with the tables built here by a plain sort (the kernels build them with a
  // warp; the GPU parity tests cover that), the slots of whole rounds of P CTAs visit every
  // (head, unit) of every sequence exactly once, units in decreasing order of position.
  const int lens_sets[4][6] = {{0, 1, 128, 129, 640, 300},
                               {640, 640, 640, 640, 640, 640},
                               {5, 0, 0, 700, 256, 1},
                               {0, 0, 0, 0, 0, 0}};
  for (auto& lens : lens_sets)
    for (int B = 1; B <= 6; ++B)
      for (int H = 1; H <= 3; ++H)
        for (int per_item = 1; per_item <= 2; ++per_item)
          for (int P = 1; P <= 11; ++P) {
            const int N = 700, U = (num_tiles(N) + per_item - 1) / per_item;
            std::vector<int> units(B), sigma(B), start(U + 1, 0);
            for (int b = 0; b < B; ++b)
              units[b] = (num_tiles(lens[b] < N ? lens[b] : N) + per_item - 1) / per_item;
            for (int b = 0; b < B; ++b) sigma[b] = b;
            std::stable_sort(sigma.begin(), sigma.end(),
                             [&](int x, int y) { return units[x] > units[y]; });
            for (int q = 0; q < U; ++q) {
              int m = 0;
              for (int b = 0; b < B; ++b) m += units[b] > U - 1 - q;
              start[q + 1] = start[q] + H * m;
            }
            std::vector<int> tables(start);
            tables.insert(tables.end(), sigma.begin(), sigma.end());
            const int slots = (B * H * U + P - 1) / P * P;
            std::vector<int> seen(B * H * U, 0), by_pos(slots, -1);
            for (int k = 0; k < slots; ++k) {
              int bh, u;
              if (!varlen_item(k, P, tables.data(), U, H, bh, u)) continue;
              if (bh < 0 || bh >= B * H || u < 0 || u >= units[bh / H])
                return fail("varlen_item range", B, H, P, k);
              ++seen[bh * U + u];
              const int r = k / P, c = k % P;
              by_pos[r * P + ((r & 1) ? P - 1 - c : c)] = u;
            }
            for (int bh = 0; bh < B * H; ++bh)
              for (int u = 0; u < U; ++u)
                if (seen[bh * U + u] != (u < units[bh / H] ? 1 : 0))
                  return fail("varlen_item cover", B, H, P, bh * U + u);
            for (int p = 1; p < slots; ++p)
              if (by_pos[p] > by_pos[p - 1]) return fail("varlen_item order", B, H, P, p);
          }
  std::printf("OK\n");
  return 0;
}
