// Runs the shard-merge pack kernel of the library's source (made
// host-compilable by cuda_shim.h and the test's preprocessing) on files of
// inputs.  Test infrastructure only.
//   DIR S T k_in  (vals.bin, idx.bin, offs.bin) -> pv.bin, pl.bin, nv.bin
#include "merge_host.h"

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
  if (argc < 5) return 2;
  const char* dir = argv[1];
  const int S = std::atoi(argv[2]), T = std::atoi(argv[3]), k_in = std::atoi(argv[4]);
  const size_t n = static_cast<size_t>(S) * T * k_in;
  auto vals = load<float>(dir, "vals.bin", n);
  auto idx = load<int32_t>(dir, "idx.bin", n);
  auto offs = load<int32_t>(dir, "offs.bin", S);
  std::vector<float> pv(n, 777.f);
  std::vector<int32_t> pl(n, 777), nv(T, 777);
  for (int b = 0; b < T; ++b) {
    std::barrier<> bar(256);
    g_block_bar = &bar;
    std::vector<std::thread> th;
    for (int t = 0; t < 256; ++t)
      th.emplace_back([&, t] {
        threadIdx = {static_cast<unsigned>(t), 0, 0};
        blockIdx = {static_cast<unsigned>(b), 0, 0};
        lsi::merge_pack_kernel(vals.data(), idx.data(), offs.data(), S, T, k_in, pv.data(), pl.data(), nv.data());
      });
    for (auto& x : th) x.join();
  }
  save(dir, "pv.bin", pv);
  save(dir, "pl.bin", pl);
  save(dir, "nv.bin", nv);
  return 0;
}
