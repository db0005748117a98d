// Runs the LSA read-list kernel (lsa_expand_kernel, the library's source made
// host-compilable by cuda_shim.h and the test's preprocessing) on files of
// inputs, one OS thread per CUDA thread, one query (CTA) at a time.  Test
// infrastructure only.
//   DIR T top_p P M block_keys n_sink budget
//   inputs: picked.bin [T][top_p] i32, qpos.bin [T] i64, off.bin [P+1] i32, mem.bin [M] i32
//   outputs: keys.bin [T][n_sink + block_keys + budget] i32, n.bin [T] i32
#include "lsa_expand_host.h"

#include <cstdio>
#include <cstdlib>
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

int main(int argc, char** argv) {
  if (argc < 9) return 2;
  const char* dir = argv[1];
  const int T = std::atoi(argv[2]), top_p = std::atoi(argv[3]), P = std::atoi(argv[4]), M = std::atoi(argv[5]);
  const int block_keys = std::atoi(argv[6]), n_sink = std::atoi(argv[7]), budget = std::atoi(argv[8]);
  const int row_len = n_sink + block_keys + budget;
  auto picked = load<int32_t>(dir, "picked.bin", static_cast<size_t>(T) * top_p);
  auto qpos = load<int64_t>(dir, "qpos.bin", static_cast<size_t>(T));
  auto off = load<int32_t>(dir, "off.bin", static_cast<size_t>(P) + 1);
  auto mem = load<int32_t>(dir, "mem.bin", static_cast<size_t>(M));
  std::vector<int32_t> keys(static_cast<size_t>(T) * row_len, 777), n(T, 777);
  const int NT = lsi::kExpandThreads;
  blockDim = {static_cast<unsigned>(NT), 1, 1};
  gridDim = {static_cast<unsigned>(T), 1, 1};
  for (int w = 0; w < NT / 32; ++w) g_warp_bar[w] = new std::barrier<>(32);
  for (int b = 0; b < T; ++b) {
    std::barrier<> bar(NT);
    g_block_bar = &bar;
    std::vector<std::thread> th;
    for (int t = 0; t < NT; ++t)
      th.emplace_back([&, t, b] {
        threadIdx = {static_cast<unsigned>(t), 0, 0};
        blockIdx = {static_cast<unsigned>(b), 0, 0};
        lsi::lsa_expand_kernel(picked.data(), qpos.data(), T, top_p, off.data(), mem.data(), P, block_keys, n_sink,
                               budget, keys.data(), row_len, n.data());
      });
    for (auto& x : th) x.join();
  }
  for (int w = 0; w < NT / 32; ++w) delete g_warp_bar[w];
  save(dir, "keys.bin", keys);
  save(dir, "n.bin", n);
  return 0;
}
