// Test-only host build of bwdc::slot_chunk (csrc/ckda_bwd_split.cuh), the
// map from a checkpoint slot g to (sequence n, chunk ci) that the chunked
// kernels' per-chunk grids use. Prints one line "g n ci ok" per slot
// g < floor(T_total / 16) + N; the test compares it with an enumeration of the
// chunks.
//
// usage: emu_slot_map N T cu_0 ... cu_N    (cu given: varlen offsets)
//        emu_slot_map N T                  (N sequences of T tokens)
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "ckda_bwd_split.cuh"

int main(int argc, char **argv) {
  if (argc < 3) return 1;
  const int N = std::atoi(argv[1]), T = std::atoi(argv[2]);
  const bool varlen = argc > 3;
  if (varlen && argc != 4 + N) return 1;
  std::vector<int> cu(N + 1);
  for (int i = 0; varlen && i <= N; ++i) cu[i] = std::atoi(argv[3 + i]);
  const int T_total = varlen ? cu[N] : N * T;
  const int slots = T_total / ckda::bwdc::C + N;
  for (int g = 0; g < slots; ++g) {
    int n = -1, ci = -1;
    const bool ok = ckda::bwdc::slot_chunk(varlen ? cu.data() : nullptr, N, T, g, n, ci);
    std::printf("%d %d %d %d\n", g, n, ci, ok ? 1 : 0);
  }
  return 0;
}
