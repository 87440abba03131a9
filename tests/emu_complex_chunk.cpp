// Test-only host build of the complex-phase gate's chunked forward programs
// (csrc/ckda_complex_chunk.cuh): every CTA of the prep grid and then of the
// scan grid runs in turn, each phase as a plain loop over its work items,
// the same set of calls the GPU makes between two barriers. It checks the
// programs' index arithmetic and algebra on the CPU (built with
// AddressSanitizer by the test, every workspace piece its own allocation);
// it is not a product path and no library calls it.
//
// usage: emu_complex_chunk DIR N T H d_k d_v scale varlen has_s0
// DIR holds q k v (complex64 as interleaved float32), alpha theta beta
// (float32), s0 (complex64, optional) and cu (int32, varlen) as raw .bin
// files; writes o and sf (complex64) there.
#include <cstdio>
#include <cstdlib>
#include <deque>
#include <string>
#include <utility>
#include <vector>

#include "ckda_bwd_split.cuh"
#include "ckda_complex_chunk.cuh"

namespace {

// Runs a phase's items in index order, or in reverse when `reverse` is set:
// the two orders give bit-identical results only if no item reads what
// another item of the same phase writes, which is what the GPU's concurrent
// threads need.
struct HostExec {
  bool reverse = false;
  template <int N, class F>
  void run(F f) {
    for (int i = 0; i < N; ++i) f(reverse ? N - 1 - i : i);
  }
  // Asynchronous copies as the GPU may see them: each lands only when a
  // wait_copies that covers its group runs, so a program that reads a copy's
  // destination before waiting for it reads the old contents here too.
  std::vector<std::pair<float *, const float *>> open_group;
  std::deque<std::vector<std::pair<float *, const float *>>> groups;
  void acopy4(float *dst, const float *src) { open_group.emplace_back(dst, src); }
  void commit() {
    groups.push_back(std::move(open_group));
    open_group.clear();
  }
  template <int pending>
  void wait_copies() {
    while (groups.size() > (size_t)pending) {
      for (auto &c : groups.front()) *c.first = *c.second;
      groups.pop_front();
    }
  }
};

std::vector<float> load(const std::string &path, size_t n) {
  std::vector<float> x(n);
  FILE *f = std::fopen(path.c_str(), "rb");
  if (!f || std::fread(x.data(), sizeof(float), n, f) != n) {
    std::fprintf(stderr, "cannot read %s\n", path.c_str());
    std::exit(2);
  }
  std::fclose(f);
  return x;
}

void save(const std::string &path, const std::vector<float> &x) {
  FILE *f = std::fopen(path.c_str(), "wb");
  if (!f || std::fwrite(x.data(), sizeof(float), x.size(), f) != x.size()) std::exit(3);
  std::fclose(f);
}

template <int DK, int DVT>
void run(const std::string &dir, int N, int T, int H, int DV, float scale, bool varlen,
         bool has_s0) {
  using namespace ckda;
  constexpr int C = bwdc::C;
  std::vector<int> cu(N + 1);
  int T_total = N * T;
  if (varlen) {
    FILE *f = std::fopen((dir + "/cu.bin").c_str(), "rb");
    if (!f || std::fread(cu.data(), sizeof(int), N + 1, f) != (size_t)N + 1) std::exit(2);
    std::fclose(f);
    T_total = T;
  }
  const size_t TH = (size_t)T_total * H, st = (size_t)N * H * DK * DV;
  auto q = load(dir + "/q.bin", 2 * TH * DK), k = load(dir + "/k.bin", 2 * TH * DK);
  auto v = load(dir + "/v.bin", 2 * TH * DV), al = load(dir + "/alpha.bin", TH * DK);
  auto th = load(dir + "/theta.bin", TH * DK), be = load(dir + "/beta.bin", TH);
  std::vector<float> s0;
  if (has_s0) s0 = load(dir + "/s0.bin", 2 * st);
  std::vector<float> o(2 * TH * DV), sf(2 * st);
  const size_t slots = (size_t)T_total / C + N;
  std::vector<float> wt(2 * TH * DK), kb(2 * TH * DK), qh(2 * TH * DK), ut(2 * TH * DV),
      mm(2 * slots * H * C * C), gc(2 * slots * H * DK);
  cplx::Args a{q.data(), k.data(), v.data(), al.data(), th.data(), be.data(),
               has_s0 ? s0.data() : nullptr, sf.data(), o.data(), H, DV, scale};
  cplx::Ws w{wt.data(), kb.data(), qh.data(), ut.data(), mm.data(), gc.data()};
  auto bounds = [&](int n, int &bos, int &eos) {
    bos = varlen ? cu[n] : n * T;
    eos = varlen ? cu[n + 1] : bos + T;
  };
  HostExec x;
  x.reverse = std::getenv("EMU_REVERSE_ITEMS") != nullptr;
  std::vector<float> psm(cplx::PrepLayout<DK, DVT>::FLOATS);
  std::vector<float> ssm(cplx::ScanLayout<DK, DVT>::FLOATS);
  for (int h = 0; h < H; ++h)
    for (int g = 0; g < (int)slots; ++g) {
      int n, ci, bos, eos;
      if (!bwdc::slot_chunk(varlen ? cu.data() : nullptr, N, T, g, n, ci)) continue;
      bounds(n, bos, eos);
      if (ci >= (eos - bos + C - 1) / C) continue;
      const int t0 = bos + C * ci, L = eos - t0 < C ? eos - t0 : C;
      cplx::prep_program<HostExec, DK, DVT>(x, a, w, psm.data(), h, t0, L, g);
    }
  for (int tile = 0; tile < DV / DVT; ++tile)
    for (int n = 0; n < N; ++n)
      for (int h = 0; h < H; ++h) {
        int bos, eos;
        bounds(n, bos, eos);
        cplx::scan_program<HostExec, DK, DVT>(x, a, w, ssm.data(), h, n, tile, bos, eos,
                                              bos / C + n);
      }
  save(dir + "/o.bin", o);
  save(dir + "/sf.bin", sf);
}

}  // namespace

int main(int argc, char **argv) {
  if (argc != 10) {
    std::fprintf(stderr, "usage: %s DIR N T H d_k d_v scale varlen has_s0\n", argv[0]);
    return 1;
  }
  const std::string dir = argv[1];
  const int N = std::atoi(argv[2]), T = std::atoi(argv[3]), H = std::atoi(argv[4]);
  const int dk = std::atoi(argv[5]), dv = std::atoi(argv[6]);
  const float scale = (float)std::atof(argv[7]);
  const bool varlen = std::atoi(argv[8]), s0 = std::atoi(argv[9]);
#define EMU_CASE(DK, DVT)                                   \
  if (dk == DK && (dv < 32 ? dv : 32) == DVT) {             \
    run<DK, DVT>(dir, N, T, H, dv, scale, varlen, s0);      \
    return 0;                                               \
  }
  EMU_CASE(16, 16) EMU_CASE(16, 32) EMU_CASE(32, 16) EMU_CASE(32, 32)
  EMU_CASE(64, 16) EMU_CASE(64, 32) EMU_CASE(128, 16) EMU_CASE(128, 32)
#undef EMU_CASE
  std::fprintf(stderr, "unsupported d_k=%d d_v=%d\n", dk, dv);
  return 1;
}
