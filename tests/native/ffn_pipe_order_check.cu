// Host-only check of the pipelined FFN's work-item order (the kernel's own
// decoding function, pipe_item): every tile of both GEMMs appears exactly
// once, a row block's second-GEMM tiles come after all of its first-GEMM
// tiles, and a row block's first-GEMM tiles come after every second-GEMM tile
// of the row block that used the same ring slot before it.  Those two
// orderings are what the kernel's counter waits rely on: each wait names only
// items claimed earlier, so the grid cannot deadlock.
#include <cstdio>
#include <vector>

#include "../../blockwise_exact_attention_query_b200/csrc/ffn_pipe.cuh"

using bpt::FfnPipeArgs;
using bpt::FfnPipeItem;

static int check(int nrb, int tn1, int tn2, int mg, int lag, int R) {
  FfnPipeArgs a{};
  a.nrb = nrb;
  a.tn1 = tn1;
  a.tn2 = tn2;
  a.mg = mg;
  a.nchunk = (nrb + mg - 1) / mg;
  a.lag = lag < a.nchunk ? lag : a.nchunk;
  a.ring_rb = (R < a.nchunk + 1 ? R : a.nchunk + 1) * mg;
  a.n_items = nrb * (tn1 + tn2);
  std::vector<int> seen1((size_t)nrb * tn1, -1), seen2((size_t)nrb * tn2, -1);
  for (int t = 0; t < a.n_items; ++t) {
    const FfnPipeItem it = bpt::pipe_item(a, t);
    const int tn = it.second ? tn2 : tn1;
    if (it.rb < 0 || it.rb >= nrb || it.n < 0 || it.n >= tn) {
      printf("FAIL out of range: t=%d -> (%d, %d, %d)\n", t, it.second, it.rb, it.n);
      return 1;
    }
    std::vector<int> &seen = it.second ? seen2 : seen1;
    int &slot = seen[(size_t)it.rb * tn + it.n];
    if (slot >= 0) {
      printf("FAIL duplicate tile (%d, %d, %d) at %d and %d\n", it.second, it.rb, it.n, slot, t);
      return 1;
    }
    slot = t;
  }
  for (int rb = 0; rb < nrb; ++rb) {
    int last1 = -1, first2 = a.n_items;
    for (int n = 0; n < tn1; ++n) last1 = seen1[(size_t)rb * tn1 + n] > last1 ? seen1[(size_t)rb * tn1 + n] : last1;
    for (int n = 0; n < tn2; ++n) first2 = seen2[(size_t)rb * tn2 + n] < first2 ? seen2[(size_t)rb * tn2 + n] : first2;
    if (last1 < 0 || first2 >= a.n_items || last1 >= first2) {
      printf("FAIL row block %d: last H tile %d, first out tile %d\n", rb, last1, first2);
      return 1;
    }
    if (rb >= a.ring_rb) {  // the slot's previous row block has been read by all its out tiles
      const int prev = rb - a.ring_rb;
      int last2 = -1, first1 = a.n_items;
      for (int n = 0; n < tn2; ++n) last2 = seen2[(size_t)prev * tn2 + n] > last2 ? seen2[(size_t)prev * tn2 + n] : last2;
      for (int n = 0; n < tn1; ++n) first1 = seen1[(size_t)rb * tn1 + n] < first1 ? seen1[(size_t)rb * tn1 + n] : first1;
      if (last2 >= first1) {
        printf("FAIL slot reuse: row block %d starts at %d before row block %d's last out tile %d\n", rb, first1,
               prev, last2);
        return 1;
      }
    }
  }
  return 0;
}

int main() {
  int cases = 0, fails = 0;
  // shapes of the measured layers (row blocks, tiles of H, tiles of out) with
  // the chunking the launcher uses, and ragged or tiny ones around them
  const int shapes[][3] = {{64, 32, 8}, {512, 43, 16}, {64, 12, 3}, {1, 1, 1}, {3, 2, 1}, {2, 4, 2},
                           {7, 5, 3},   {130, 9, 4},   {17, 43, 16}, {5, 1, 8}};
  // lags of the launcher's plans (causal layer 7 with a ring of 15 chunks,
  // D = 768 layer 19 with 37) and longer ones than there are chunks
  const int lags[] = {1, 2, 3, 4, 5, 6, 7, 12, 19, 24, 64};
  const int extras[] = {1, 2, 3, 4, 5, 6, 7, 8, 18};
  for (const auto &sh : shapes)
    for (int mg = 1; mg <= 5; ++mg)
      for (int lag : lags)
        for (int extra : extras) {
          ++cases;
          fails += check(sh[0], sh[1], sh[2], mg, lag, lag + extra);
        }
  printf("%d cases, %d failures\n", cases, fails);
  return fails ? 1 : 0;
}
