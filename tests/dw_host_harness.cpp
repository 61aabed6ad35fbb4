// Host build of the BF16 depthwise kernels' per-thread code: every thread
// index of a launch, run in order on the CPU, with the geometry the library
// plans.  Test infrastructure; the library itself never runs this.
//
//   dw_host_harness OP N C H W Kh Kw stride pad A_FILE B_FILE OUT_FILE
//
// OP 0: out = fwd(w = A, x = B); 1: out = dgrad(w = A, gy = B);
// 2: out = wgrad(gy = A, x = B).  A and B hold raw bfloat16 bit patterns in
// the library's layouts; OUT receives raw fp32.  Every buffer is allocated
// at its exact size, so a build with an address sanitizer reports any
// access outside it.
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "mqv_depthwise_core.h"

template <typename T>
static std::vector<T> read_all(const char* path) {
  std::FILE* f = std::fopen(path, "rb");
  if (!f) std::exit(3);
  std::fseek(f, 0, SEEK_END);
  const long n = std::ftell(f);
  std::fseek(f, 0, SEEK_SET);
  std::vector<T> v(static_cast<size_t>(n) / sizeof(T));
  if (std::fread(v.data(), sizeof(T), v.size(), f) != v.size()) std::exit(4);
  std::fclose(f);
  return v;
}

int main(int argc, char** argv) {
  if (argc != 13) return 2;
  int64_t d[8];
  for (int i = 0; i < 8; ++i) d[i] = std::atoll(argv[2 + i]);
  const int op = std::atoi(argv[1]);
  const mqv::DwGeom g = mqv::dw_geom(d[0], d[1], d[2], d[3], d[4], d[5], d[6], d[7]);
  const std::vector<uint16_t> a = read_all<uint16_t>(argv[10]), b = read_all<uint16_t>(argv[11]);
  std::vector<float> out;
  if (op == 0) {
    out.assign(static_cast<size_t>(g.Ho * g.Wo * g.C * g.N), 0.0f);
    for (int64_t t = 0; t < mqv::dw_fwd_threads(g); ++t) mqv::dw_fwd_thread(g, t, a.data(), b.data(), out.data());
  } else if (op == 1) {
    out.assign(static_cast<size_t>(g.H * g.W * g.C * g.N), 0.0f);
    for (int64_t t = 0; t < mqv::dw_dgrad_threads(g); ++t)
      mqv::dw_dgrad_thread(g, t, a.data(), b.data(), out.data());
  } else {
    std::vector<float> ws(static_cast<size_t>(mqv::dw_wgrad_threads(g)), 0.0f);
    out.assign(static_cast<size_t>(g.C * g.Kh * g.Kw), 0.0f);
    for (int64_t t = 0; t < mqv::dw_wgrad_threads(g); ++t)
      mqv::dw_wgrad_thread(g, t, a.data(), b.data(), ws.data());
    for (int64_t t = 0; t < g.C * g.Kh * g.Kw; ++t) mqv::dw_wgrad_reduce_thread(g, t, ws.data(), out.data());
  }
  std::FILE* f = std::fopen(argv[12], "wb");
  if (!f || std::fwrite(out.data(), sizeof(float), out.size(), f) != out.size()) return 5;
  std::fclose(f);
  return 0;
}
