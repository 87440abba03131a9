// Test-only host build of the chunkwise backward's per-CTA programs
// (csrc/ckda_bwd_split.cuh): every CTA of each of the four launch grids runs
// in turn, the launches in their stream order, each phase as a plain loop over
// its work items, which is the same set of calls the GPU makes between two
// barriers. It checks the programs' index arithmetic and algebra on the
// CPU (built with AddressSanitizer by the test, every workspace piece its own
// allocation); it is not a product path and no library calls it.
//
// usage: emu_bwd_chunk DIR N T H d_k d_v scale varlen has_s0 has_dsf
// DIR holds float32 q k v alpha beta do [s0] [dsf] and int32 cu (varlen) as
// raw .bin files; writes dq dk dv dalpha dbeta ds0 (.bin, float32) there.
#include <cstdio>
#include <cstdlib>
#include <deque>
#include <string>
#include <utility>
#include <vector>

#include "ckda_bwd_split.cuh"

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

struct HostIO {
  static float ld(const float *p) { return *p; }
  static float ldg(const float *p) { return *p; }
  static void st(float *p, float x) { *p = x; }
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
         bool has_s0, bool has_dsf) {
  using namespace ckda::bwdc;
  std::vector<int> cu(N + 1);
  int T_total = N * T;
  if (varlen) {
    FILE *f = std::fopen((dir + "/cu.bin").c_str(), "rb");
    if (!f || std::fread(cu.data(), sizeof(int), N + 1, f) != (size_t)N + 1) std::exit(2);
    std::fclose(f);
    T_total = T;
  }
  const size_t TH = (size_t)T_total * H;
  auto q = load(dir + "/q.bin", TH * DK), k = load(dir + "/k.bin", TH * DK);
  auto v = load(dir + "/v.bin", TH * DV), al = load(dir + "/alpha.bin", TH * DK);
  auto be = load(dir + "/beta.bin", TH), d_o = load(dir + "/do.bin", TH * DV);
  const size_t st = (size_t)N * H * DK * DV;
  std::vector<float> s0, dsf;
  if (has_s0) s0 = load(dir + "/s0.bin", st);
  if (has_dsf) dsf = load(dir + "/dsf.bin", st);
  const int ntile = DV / DVT;
  const size_t slots = (size_t)T_total / C + N;
  std::vector<float> dq(TH * DK), dk(TH * DK), dv(TH * DV), da(TH * DK), db(TH), ds0(st);
  Args<float> a{q.data(),  k.data(),  v.data(),  al.data(), be.data(),
                has_s0 ? s0.data() : nullptr, d_o.data(), has_dsf ? dsf.data() : nullptr,
                dq.data(), dk.data(), dv.data(), da.data(), db.data(), ds0.data(), H, DV, scale};
  HostExec x;
  x.reverse = std::getenv("EMU_REVERSE_ITEMS") != nullptr;
  auto bounds = [&](int n, int &bos, int &eos) {
    bos = varlen ? cu[n] : n * T;
    eos = varlen ? cu[n + 1] : bos + T;
  };
  {
    const size_t sl = slots * H;
    std::vector<float> cks(sl * DK * DV), ckd(sl * DK * DV), gc(sl * DK), ab(sl * C * C);
    std::vector<float> wt(TH * DK), kb(TH * DK), wb(TH * DK), qs(TH * DK), bk(TH * DK);
    std::vector<float> ut(TH * DV), xt(TH * DV), uu(TH * DV), dr(TH * DV);
    SplitWs w{cks.data(), ckd.data(), gc.data(), ab.data(), wt.data(), kb.data(), wb.data(),
              qs.data(), bk.data(), ut.data(), xt.data(), uu.data(), dr.data()};
    // the chunk of slot g, as the kernels find it
    auto slot_rows = [&](int g, int &t0, int &L) {
      int n, ci, bos, eos;
      if (!slot_chunk(varlen ? cu.data() : nullptr, N, T, g, n, ci)) return false;
      bounds(n, bos, eos);
      if (ci >= (eos - bos + C - 1) / C) return false;
      t0 = bos + C * ci;
      L = eos - t0 < C ? eos - t0 : C;
      return true;
    };
    constexpr int GT = 16;  // columns per tile of the gradient program
    std::vector<float> psm(PrepLayout<DK, DVT>::FLOATS), ssm(ScanLayout<DK, DVT>::FLOATS),
        gsm(GradLayout<DK, GT>::FLOATS);
    int t0, L;
    for (int h = 0; h < H; ++h)
      for (int g = 0; g < (int)slots; ++g)
        if (slot_rows(g, t0, L))
          prep_program<HostExec, HostIO, float, DK, DVT>(x, a, w, psm.data(), h, t0, L, g);
    for (int pass = 0; pass < 2; ++pass)
      for (int tile = 0; tile < ntile; ++tile)
        for (int n = 0; n < N; ++n)
          for (int h = 0; h < H; ++h) {
            int bos, eos;
            bounds(n, bos, eos);
            if (pass == 0)
              scan1_program<HostExec, HostIO, float, DK, DVT>(x, a, w, ssm.data(), h, n, tile,
                                                             bos, eos, bos / C + n);
            else
              scan2_program<HostExec, HostIO, float, DK, DVT>(x, a, w, ssm.data(), h, n, tile,
                                                             bos, eos, bos / C + n);
          }
    for (int h = 0; h < H; ++h)
      for (int g = 0; g < (int)slots; ++g)
        if (slot_rows(g, t0, L))
          grads_program<HostExec, HostIO, float, DK, GT>(x, a, w, gsm.data(), h, t0, L, g);
  }
  save(dir + "/dq.bin", dq);
  save(dir + "/dk.bin", dk);
  save(dir + "/dv.bin", dv);
  save(dir + "/dalpha.bin", da);
  save(dir + "/dbeta.bin", db);
  save(dir + "/ds0.bin", ds0);
}

}  // namespace

int main(int argc, char **argv) {
  if (argc != 11) {
    std::fprintf(stderr, "usage: %s DIR N T H d_k d_v scale varlen has_s0 has_dsf\n", argv[0]);
    return 1;
  }
  const std::string dir = argv[1];
  const int N = std::atoi(argv[2]), T = std::atoi(argv[3]), H = std::atoi(argv[4]);
  const int dk = std::atoi(argv[5]), dv = std::atoi(argv[6]);
  const float scale = (float)std::atof(argv[7]);
  const bool varlen = std::atoi(argv[8]), s0 = std::atoi(argv[9]), dsf = std::atoi(argv[10]);
#define EMU_CASE(DK)                                          \
  if (dk == DK) { /* 16-column scan tiles, as the kernels */  \
    run<DK, 16>(dir, N, T, H, dv, scale, varlen, s0, dsf);    \
    return 0;                                                 \
  }
  EMU_CASE(16) EMU_CASE(32) EMU_CASE(64) EMU_CASE(128)
#undef EMU_CASE
  std::fprintf(stderr, "unsupported d_k=%d d_v=%d\n", dk, dv);
  return 1;
}
