// Runs the LSA tree search's candidate-scoring kernel (lsa_tree_candidates_kernel,
// the library's source made host-compilable by cuda_shim.h and the test's
// preprocessing) on files of inputs, one OS thread per CUDA thread, one
// query (CTA) at a time.  Test infrastructure only.
//   DIR T R beam_w fanout cap
//   inputs: q.bin [T][64] u16 (bf16), c.bin [R][64] u16, beam.bin [T][beam_w] i32,
//           vis.bin [T] i32, visn.bin [T] i32
//   outputs: cval.bin [T][cap] f32, clab.bin [T][cap] i32, nv.bin [T] i32
#include "tree_cand_host.h"

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
  const int T = std::atoi(argv[2]), R = std::atoi(argv[3]), beam_w = std::atoi(argv[4]);
  const int fanout = std::atoi(argv[5]), cap = std::atoi(argv[6]);
  auto q = load<uint16_t>(dir, "q.bin", static_cast<size_t>(T) * 64);
  auto c = load<uint16_t>(dir, "c.bin", static_cast<size_t>(R) * 64);
  auto beam = load<int32_t>(dir, "beam.bin", static_cast<size_t>(T) * beam_w);
  auto vis = load<int32_t>(dir, "vis.bin", static_cast<size_t>(T));
  auto visn = load<int32_t>(dir, "visn.bin", static_cast<size_t>(T));
  std::vector<float> cval(static_cast<size_t>(T) * cap, 777.f);
  std::vector<int32_t> clab(static_cast<size_t>(T) * cap, 777), nv(T, 777);
  const int NT = 256;
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
        lsi::lsa_tree_candidates_kernel(q.data(), c.data(), beam.data(), beam_w, vis.data(), visn.data(), fanout, cap,
                                        cval.data(), clab.data(), nv.data());
      });
    for (auto& x : th) x.join();
  }
  for (int w = 0; w < NT / 32; ++w) delete g_warp_bar[w];
  save(dir, "cval.bin", cval);
  save(dir, "clab.bin", clab);
  save(dir, "nv.bin", nv);
  return 0;
}
