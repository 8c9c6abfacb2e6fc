// Host check of the visible-range helpers the kernels mask with (fa_internal.h): for every
// query row i, [key_lo(i), key_hi(i)] must be exactly the keys j < N with
//   (!causal || j <= i) && (left < 0 || j >= i - left) && (right < 0 || j <= i + right),
// and for every key j, [query_lo(j), query_hi(j)] clipped to [0, N) must be exactly the rows
// that see j -- the forward / dQ kernels use the first form, the dK/dV kernel the second.
// Prints the number of ranges checked, or the first mismatch, and exits non-zero on one.
#include <cstdio>

#include "fa_internal.h"

static bool visible(int i, int j, int causal, int left, int right) {
  return (!causal || j <= i) && (left < 0 || j >= i - left) && (right < 0 || j <= i + right);
}

int main() {
  const int Ns[] = {1, 2, 3, 7, 64, 127, 128, 129, 255, 300};
  const int ws[] = {-1, 0, 1, 2, 5, 63, 64, 127, 128, 300};
  long long checked = 0;
  for (int N : Ns)
    for (int causal = 0; causal < 2; ++causal)
      for (int left : ws)
        for (int right : ws) {
          for (int i = 0; i < N; ++i) {  // keys seen by row i
            const int lo = fa::key_lo(i, N, left), hi = fa::key_hi(i, N, causal, right);
            for (int j = 0; j < N; ++j) {
              const bool in = j >= lo && j <= hi;
              if (in != visible(i, j, causal, left, right)) {
                std::printf("key range mismatch N=%d causal=%d left=%d right=%d row=%d key=%d\n", N, causal, left,
                            right, i, j);
                return 1;
              }
            }
            if (!(lo <= i && i <= hi)) {
              std::printf("row %d does not see itself (N=%d)\n", i, N);
              return 1;
            }
            ++checked;
          }
          for (int j = 0; j < N; ++j) {  // rows that see key j
            const int lo = fa::query_lo(j, causal, right), hi = fa::query_hi(j, N, left);
            for (int i = 0; i < N; ++i) {
              const bool in = i >= lo && i <= hi;
              if (in != visible(i, j, causal, left, right)) {
                std::printf("query range mismatch N=%d causal=%d left=%d right=%d key=%d row=%d\n", N, causal,
                            left, right, j, i);
                return 1;
              }
            }
            ++checked;
          }
        }
  std::printf("ok %lld\n", checked);
  return 0;
}
