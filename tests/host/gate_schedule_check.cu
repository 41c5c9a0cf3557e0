// Host-side check of the streaming gate's tile schedule (gate_stream_schedule): the per-CTA ranges
// that the host cuts, walked the way the kernel's producer warp walks them (heads and 128-row
// pieces of a block, then the next block, kv head, non-empty sequence; rows whose selection is
// fixed are published as one run per block and head), must cover every (query head, 128-row
// piece) of every block exactly once, and each range must start at the right first block of its
// sequence. Built and run by tests/test_gate_schedule.py; no GPU is used.
#include <algorithm>
#include <cstdio>
#include <map>
#include <tuple>
#include <vector>

#include "../../block_sparse_long_moba_b200/csrc/launch.h"

using moba::GateSched;

static int check(const std::vector<int>& cu, int H, int G, int d, int B, int topk, int ctas) {
  const int nseq = static_cast<int>(cu.size()) - 1;
  const int r = H / G, ksel = topk - 1;
  static GateSched S;
  const int grid = moba::gate_stream_schedule(cu.data(), nseq, H, G, d, B, topk, ctas, &S);
  std::map<std::tuple<int, int>, int> want, got;  // (head, first token of the piece) -> count
  for (int s = 0; s < nseq; ++s) {
    const int L = cu[s + 1] - cu[s];
    for (int i = 0; i * B < L; ++i)
      for (int h = 0; h < H; ++h)
        for (int t = 0; t < std::min(B, L - i * B); t += 128) want[{h, cu[s] + i * B + t}] = 1;
  }
  if (grid < 1 || grid > ctas || grid != S.n_cta) return 1;
  for (int c = 0; c < grid; ++c) {
    int seg = S.seg[c], i = S.blk[c], p = S.pos[c], base = S.base[c], left = S.count[c];
    int s = seg / G, g = seg % G;
    int seq0 = cu[s], L = cu[s + 1] - seq0, nb = (L + B - 1) / B;
    while (left > 0) {
      int expect_base = 0;
      for (int x = 0; x < s; ++x) expect_base += (cu[x + 1] - cu[x] + B - 1) / B;
      if (i >= nb || base != expect_base) return 2;
      const int blen = std::min(B, L - i * B), ntt = (blen + 127) / 128;
      const int hh = p / ntt, tt = p % ntt;
      const bool scored = ksel > 0 && i > ksel;
      const int run = scored ? 1 : std::min(left, ntt - tt);
      for (int q = 0; q < run; ++q) got[{g * r + hh, seq0 + i * B + (tt + q) * 128}] += 1;
      left -= run;
      p += run;
      if (p == r * ntt) {
        p = 0;
        if (++i == nb) {
          i = 0;
          if (++g == G) {
            g = 0;
            base += nb;
            do {
              ++s;
              if (s >= nseq) break;
              seq0 = cu[s];
              L = cu[s + 1] - seq0;
              nb = (L + B - 1) / B;
            } while (nb == 0);
          }
        }
      }
    }
  }
  if (got != want) return 3;
  return 0;
}

int main() {
  struct Case { std::vector<int> cu; int H, G, d, B, topk, ctas; };
  std::vector<int> many{0};
  for (int x = 0; x < 300; ++x) many.push_back(many.back() + (x * 37) % 900);
  const std::vector<Case> cases = {
      {{0, 131072}, 32, 8, 128, 4096, 12, 148},     // Llama-3.1-8B at 128K
      {{0, 1048576}, 32, 8, 128, 4096, 12, 148},    // and at 1M
      {{0, 1024}, 1, 1, 64, 128, 3, 148},           // fewer tiles than CTAs
      {{0, 700, 700, 1600}, 4, 2, 128, 128, 4, 148},
      {{0, 300, 300, 1000, 1100}, 4, 2, 64, 64, 5, 148},
      {{0, 0, 0, 5000, 5000, 9000, 9000}, 8, 2, 128, 192, 6, 7},  // empty sequences, 192-key blocks
      {{0, 1}, 2, 2, 64, 64, 2, 148},
      {{0, 2048}, 2, 1, 128, 128, 1, 148},          // topk = 1: every row fixed
      {{0, 65536}, 16, 16, 64, 4096, 16, 148},
      {{0, 20000, 20000, 40000}, 2, 1, 128, 256, 33, 148},
      {many, 4, 4, 64, 128, 8, 148},
  };
  int bad = 0;
  for (size_t n = 0; n < cases.size(); ++n) {
    const Case& c = cases[n];
    const int rc = check(c.cu, c.H, c.G, c.d, c.B, c.topk, c.ctas);
    std::printf("case %zu: %s (%d)\n", n, rc == 0 ? "ok" : "FAIL", rc);
    bad |= rc;
  }
  return bad ? 1 : 0;
}
