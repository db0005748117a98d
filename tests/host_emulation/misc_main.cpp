// Runs the bucket search's expansion kernel (expand_kernel) and the causal
// eligible-count kernel (causal_counts_kernel) of the library's source, made
// host-compilable by cuda_shim.h and the test's preprocessing, on files of
// inputs: one OS thread per CUDA thread, one CTA at a time.  Test
// infrastructure only.
//   DIR expand T top_p P budget   picked.bin [T][top_p] i32, off.bin [P+1] i32,
//                                 mem.bin [off[P]] i32 -> cand.bin [T][budget] i32
//   DIR counts T stride n_total   pos.bin [T] i64 -> cnt.bin [T] i32
//   DIR fold n blocks             w.bin, qs.bin [n] f32 -> out.bin [n] f32 (fold_scales_kernel)
#include "misc_host.h"

#include <cstdio>
#include <cstdlib>
#include <string>
#include <thread>
#include <vector>

thread_local Dim3 threadIdx, blockIdx;
Dim3 blockDim{256, 1, 1}, gridDim{1, 1, 1};
std::barrier<>* g_block_bar;
std::barrier<>* g_warp_bar[32];
float g_xbuf[32][32];
std::mutex g_atomic_mu;
unsigned char* g_smem;
namespace lsi { int g_fault = 0; }

template <class T>
static std::vector<T> load(const char* dir, const char* name, size_t n) {
  char p[1024];
  std::snprintf(p, sizeof p, "%s/%s", dir, name);
  std::vector<T> v(n);
  FILE* f = std::fopen(p, "rb");
  if (!f || std::fread(v.data(), sizeof(T), n, f) != n) { std::fprintf(stderr, "cannot read %s\n", p); std::exit(2); }
  std::fclose(f);
  return v;
}

template <class T>
static void save(const char* dir, const char* name, const std::vector<T>& v) {
  char p[1024];
  std::snprintf(p, sizeof p, "%s/%s", dir, name);
  FILE* f = std::fopen(p, "wb");
  std::fwrite(v.data(), sizeof(T), v.size(), f);
  std::fclose(f);
}

// Launches `body` over `blocks` CTAs of 256 threads, as the launchers do.
template <class F>
static void launch(int blocks, F body) {
  const int NT = 256;
  blockDim = {static_cast<unsigned>(NT), 1, 1};
  gridDim = {static_cast<unsigned>(blocks), 1, 1};
  for (int w = 0; w < NT / 32; ++w) g_warp_bar[w] = new std::barrier<>(32);
  for (int b = 0; b < blocks; ++b) {
    std::barrier<> bar(NT);
    g_block_bar = &bar;
    std::vector<std::thread> th;
    for (int t = 0; t < NT; ++t)
      th.emplace_back([&, t, b] {
        threadIdx = {static_cast<unsigned>(t), 0, 0};
        blockIdx = {static_cast<unsigned>(b), 0, 0};
        body();
      });
    for (auto& x : th) x.join();
  }
  for (int w = 0; w < NT / 32; ++w) delete g_warp_bar[w];
}

int main(int argc, char** argv) {
  if (argc < 5) return 2;
  const char* dir = argv[1];
  const std::string mode = argv[2];
  const int T = std::atoi(argv[3]);
  if (mode == "expand" && argc == 7) {
    const int top_p = std::atoi(argv[4]), P = std::atoi(argv[5]), budget = std::atoi(argv[6]);
    auto picked = load<int32_t>(dir, "picked.bin", static_cast<size_t>(T) * top_p);
    auto off = load<int32_t>(dir, "off.bin", static_cast<size_t>(P) + 1);
    auto mem = load<int32_t>(dir, "mem.bin", static_cast<size_t>(off[P]));
    std::vector<int32_t> cand(static_cast<size_t>(T) * budget, 777);
    launch((T * 32 + 255) / 256, [&] {
      lsi::expand_kernel(picked.data(), T, top_p, off.data(), mem.data(), P, budget, cand.data());
    });
    save(dir, "cand.bin", cand);
    return 0;
  }
  if (mode == "fold" && argc == 5) {
    const int64_t n = std::atoll(argv[3]);
    const int blocks = std::atoi(argv[4]);
    auto w = load<float>(dir, "w.bin", static_cast<size_t>(n));
    auto qs = load<float>(dir, "qs.bin", static_cast<size_t>(n));
    std::vector<float> out(static_cast<size_t>(n), 777.f);
    launch(blocks, [&] { lsi::fold_scales_kernel(w.data(), qs.data(), n, out.data()); });
    save(dir, "out.bin", out);
    return 0;
  }
  if (mode == "counts" && argc == 6) {
    const int stride = std::atoi(argv[4]), n_total = std::atoi(argv[5]);
    auto pos = load<int64_t>(dir, "pos.bin", static_cast<size_t>(T));
    std::vector<int32_t> cnt(static_cast<size_t>(T), 777);
    launch((T + 255) / 256, [&] { lsi::causal_counts_kernel(pos.data(), T, stride, n_total, cnt.data()); });
    save(dir, "cnt.bin", cnt);
    return 0;
  }
  return 2;
}
