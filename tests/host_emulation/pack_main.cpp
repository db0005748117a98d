// Runs the running prefill selection's segment-pack kernel of the library's
// source (made host-compilable by cuda_shim.h and the test's preprocessing)
// on files of inputs.  Test infrastructure only.
//   DIR T ld k S cap  (val.bin, lab.bin [T][ld], cnt.bin, over.bin [S][T])
//   -> val.bin, lab.bin rewritten in place, nv.bin
#include "pack_host.h"

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
  if (argc < 7) return 2;
  const char* dir = argv[1];
  const int T = std::atoi(argv[2]);
  const long long ld = std::atoll(argv[3]);
  const int k = std::atoi(argv[4]), S = std::atoi(argv[5]), cap = std::atoi(argv[6]);
  auto val = load<float>(dir, "val.bin", static_cast<size_t>(T) * ld);
  auto lab = load<int32_t>(dir, "lab.bin", static_cast<size_t>(T) * ld);
  auto cnt = load<uint32_t>(dir, "cnt.bin", static_cast<size_t>(S) * T);
  auto over = load<int32_t>(dir, "over.bin", static_cast<size_t>(S) * T);
  std::vector<int32_t> nv(T, 777);
  gridDim = {static_cast<unsigned>(T), 1, 1};
  for (int b = 0; b < T; ++b) {
    std::barrier<> bar(256);
    g_block_bar = &bar;
    std::vector<std::thread> th;
    for (int t = 0; t < 256; ++t)
      th.emplace_back([&, t] {
        threadIdx = {static_cast<unsigned>(t), 0, 0};
        blockIdx = {static_cast<unsigned>(b), 0, 0};
        lsi::pack_segments_kernel(val.data(), lab.data(), ld, T, k, S, cap, cnt.data(), over.data(), nv.data());
      });
    for (auto& x : th) x.join();
  }
  save(dir, "val.bin", val);
  save(dir, "lab.bin", lab);
  save(dir, "nv.bin", nv);
  return 0;
}
