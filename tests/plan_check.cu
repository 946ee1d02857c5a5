// Host check of the split-KV planner's arithmetic (worker_of_tile,
// worker_begin, for_each_piece from the library's own header), run on the
// CPU: no kernel is launched.  The prefix sums plan_kernel computes on the
// device are restated here as plain loops.  For random batches it checks
// that the workers' pieces cover every tile once, that partial slots are
// distinct and fill [0, seg_start[B]), and that the rule the few-head
// attention kernel uses to load the next piece's Q ahead (a next piece
// exists iff sequence b + 1 starts before the worker's last tile) matches
// the pieces for_each_piece yields.  Prints "ok" and exits 0, or prints the
// first failure and exits 1.
#include <cstdio>
#include <cstdlib>
#include <random>
#include <vector>

#include "simt.cuh"

using mla::Piece;

static int fail(const char* what, int B, int W, int w) {
  std::printf("FAIL %s (B=%d W=%d worker %d)\n", what, B, W, w);
  return 1;
}

static int check(const std::vector<int>& L, int W, int tile_tokens) {
  const int B = static_cast<int>(L.size());
  std::vector<int> tile_start(B + 1, 0), seg_start(B + 1, 0);
  for (int b = 0; b < B; ++b) tile_start[b + 1] = tile_start[b] + (L[b] + 1 + tile_tokens - 1) / tile_tokens;
  const long long T = tile_start[B];
  const int We = static_cast<int>(T < W ? T : W);
  for (int b = 0; b < B; ++b) {
    const int pieces = mla::worker_of_tile(tile_start[b + 1] - 1, T, We) - mla::worker_of_tile(tile_start[b], T, We) + 1;
    seg_start[b + 1] = seg_start[b] + pieces;
  }
  std::vector<int> tile_seen(T, 0), slot_seen(seg_start[B], 0);
  for (int w = 0; w < W; ++w) {
    std::vector<Piece> ps;
    mla::for_each_piece(w, W, B, tile_start.data(), seg_start.data(), [&](const Piece& p) { ps.push_back(p); });
    if (w >= We) {
      if (!ps.empty()) return fail("a worker past min(W, T) got work", B, W, w);
      continue;
    }
    if (ps.empty()) return fail("a worker below min(W, T) got no tile", B, W, w);
    const long long r1 = mla::worker_begin(w + 1, T, We);
    for (size_t i = 0; i < ps.size(); ++i) {
      const Piece& p = ps[i];
      if (p.t1 <= p.t0) return fail("empty piece", B, W, w);
      if (i > 0 && p.b != ps[i - 1].b + 1) return fail("pieces of a worker are not consecutive sequences", B, W, w);
      for (int t = p.t0; t < p.t1; ++t) {
        const long long g = tile_start[p.b] + t;
        if (g < 0 || g >= T || tile_seen[g]++) return fail("a tile covered twice or out of range", B, W, w);
      }
      if (p.slot < seg_start[p.b] || p.slot >= seg_start[p.b + 1]) return fail("slot outside its sequence", B, W, w);
      if (slot_seen[p.slot]++) return fail("slot used twice", B, W, w);
      const bool next_rule = p.b + 1 < B && tile_start[p.b + 1] < r1;
      if (next_rule != (i + 1 < ps.size())) return fail("next-piece rule disagrees with the pieces", B, W, w);
    }
  }
  for (long long g = 0; g < T; ++g)
    if (tile_seen[g] != 1) return fail("a tile not covered", B, W, -1);
  for (int s = 0; s < seg_start[B]; ++s)
    if (slot_seen[s] != 1) return fail("a slot not written", B, W, -1);
  return 0;
}

int main() {
  std::mt19937_64 rng(7);
  const int Ws[] = {1, 3, 74, 148, 296};
  const int Bs[] = {1, 2, 5, 16, 64, 128, 700};
  int cases = 0;
  for (int rep = 0; rep < 6; ++rep)
    for (int W : Ws)
      for (int B : Bs) {
        std::vector<int> L(B);
        for (int b = 0; b < B; ++b) {
          switch ((rep + b) % 4) {
            case 0: L[b] = 0; break;                                        // empty cache: one tile (the new token)
            case 1: L[b] = static_cast<int>(rng() % 200); break;            // short
            case 2: L[b] = 64 * static_cast<int>(1 + rng() % 40) - 1; break;  // tile-aligned totals
            default: L[b] = static_cast<int>(rng() % 131072); break;        // long
          }
        }
        if (check(L, W, 64)) return 1;
        ++cases;
      }
  std::printf("ok %d cases\n", cases);
  return 0;
}
