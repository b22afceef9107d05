// Host check of the sequence-parallel row map used by the GEMM producers: SeqCursor::row must
// equal seq_row for every token of every sweep, and seq_row must be a bijection from token
// order onto the shard-major layout [p][b][s/p]. Exit status 0 on success.
#include <cstdio>
#include <vector>

#include "../../tensor_transformer_layer_megatron_b200/csrc/mgt_internal.h"

int main() {
  const int cases[][3] = {{1024, 2, 2}, {256, 2, 2}, {512, 3, 4}, {2048, 1, 8},
                          {128, 5, 1}, {4096, 2, 4}, {384, 3, 3}};
  int bad = 0;
  for (const auto& c : cases) {
    mgt::GemmArgs a{};
    a.sp_seq = c[0];
    a.sp_b = c[1];
    a.sp_len = c[0] / c[2];
    const int T = c[0] * c[1];
    std::vector<int> seen(T, 0);
    for (int m = 0; m < T; ++m) {
      const int r = mgt::seq_row(a, m);
      const int bb = m / c[0], pos = m % c[0], t = pos / a.sp_len;
      const int want = (t * c[1] + bb) * a.sp_len + pos % a.sp_len;
      if (r != want || r < 0 || r >= T) ++bad;
      else ++seen[r];
    }
    for (int r = 0; r < T; ++r) bad += seen[r] != 1;
    // three sweeps with a fresh cursor per tile, as the producer runs them; every row of a
    // 64-token step must also be contiguous in the shard-major layout
    mgt::SeqCursor cur{0, 0};
    for (int sweep = 0; sweep < 3; ++sweep)
      for (int k = 0; k < T; k += 64) {
        const int r = cur.row(a, k);
        for (int j = 0; j < 64 && k + j < T; ++j) bad += (r + j) != mgt::seq_row(a, k + j);
      }
  }
  std::printf("%s (%d mismatches)\n", bad ? "FAIL" : "ok", bad);
  return bad ? 1 : 0;
}
