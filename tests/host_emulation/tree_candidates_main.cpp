// Runs the LSA tree search's candidate-scoring kernel (lsa_tree_candidates_kernel)
// and its level-visibility kernel (lsa_tree_levels_visible_kernel), the library's
// source made host-compilable by cuda_shim.h and the test's preprocessing, on
// files of inputs, one OS thread per CUDA thread, one CTA at a time.  Test
// infrastructure only.
//   DIR T R beam_w fanout cap
//   inputs: q.bin [T][64] u16 (bf16), c.bin [R][64] u16, beam.bin [T][beam_w] i32,
//           vis.bin [T] i32, visn.bin [T] i32
//   outputs: cval.bin [T][cap] f32, clab.bin [T][cap] i32, nv.bin [T] i32
//   DIR vis T block_keys bpb node_block fanout n size_0 .. size_n
//   inputs: pos.bin [T] i64; output: lvis.bin [n + 1][T] i32
// and the one-level tree's and the flat search's visibility kernels
// (lsa_tree_visible_kernel, lsa_visible_kernel):
//   DIR vis1 T block_keys bpb P node_block fanout P1   pos.bin -> lvis.bin [2][T] i32
//   DIR visflat T block_keys bpb P stride              pos.bin -> lvis.bin [2][T] i32 (vis, samples)
#include "tree_cand_host.h"

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

static int run_visible(const char* dir, int argc, char** argv) {
  const int T = std::atoi(argv[3]), block_keys = std::atoi(argv[4]), bpb = std::atoi(argv[5]);
  const int node_block = std::atoi(argv[6]), fanout = std::atoi(argv[7]), n = std::atoi(argv[8]);
  if (n < 1 || n > lsi::kMaxTreeLevels || argc != 10 + n) return 2;
  lsi::TreeLevels lv;
  lv.n = n;
  for (int l = 0; l <= n; ++l) lv.size[l] = std::atoi(argv[9 + l]);
  auto pos = load<int64_t>(dir, "pos.bin", static_cast<size_t>(T));
  std::vector<int32_t> vis(static_cast<size_t>(n + 1) * T, 777);
  const int NT = 256, NB = (T + NT - 1) / NT;
  blockDim = {static_cast<unsigned>(NT), 1, 1};
  gridDim = {static_cast<unsigned>(NB), 1, 1};
  for (int b = 0; b < NB; ++b) {
    std::vector<std::thread> th;
    for (int t = 0; t < NT; ++t)
      th.emplace_back([&, t, b] {
        threadIdx = {static_cast<unsigned>(t), 0, 0};
        blockIdx = {static_cast<unsigned>(b), 0, 0};
        lsi::lsa_tree_levels_visible_kernel(pos.data(), T, block_keys, bpb, node_block, fanout, lv, vis.data());
      });
    for (auto& x : th) x.join();
  }
  save(dir, "lvis.bin", vis);
  return 0;
}

// One thread per query over ceil(T / 256) CTAs of 256 threads.
template <class F>
static void run_per_query(int T, F body) {
  const int NT = 256, NB = (T + NT - 1) / NT;
  blockDim = {static_cast<unsigned>(NT), 1, 1};
  gridDim = {static_cast<unsigned>(NB), 1, 1};
  for (int b = 0; b < NB; ++b) {
    std::vector<std::thread> th;
    for (int t = 0; t < NT; ++t)
      th.emplace_back([&, t, b] {
        threadIdx = {static_cast<unsigned>(t), 0, 0};
        blockIdx = {static_cast<unsigned>(b), 0, 0};
        body();
      });
    for (auto& x : th) x.join();
  }
}

int main(int argc, char** argv) {
  if (argc < 7) return 2;
  const char* dir = argv[1];
  const std::string mode = argv[2];
  if (mode == "vis") return run_visible(dir, argc, argv);
  if (mode == "vis1" || mode == "visflat") {
    const int T = std::atoi(argv[3]), block_keys = std::atoi(argv[4]), bpb = std::atoi(argv[5]), P = std::atoi(argv[6]);
    auto pos = load<int64_t>(dir, "pos.bin", static_cast<size_t>(T));
    std::vector<int32_t> out(static_cast<size_t>(2) * T, 777);
    if (mode == "vis1" && argc == 10) {
      const int node_block = std::atoi(argv[7]), fanout = std::atoi(argv[8]), P1 = std::atoi(argv[9]);
      run_per_query(T, [&] {
        lsi::lsa_tree_visible_kernel(pos.data(), T, block_keys, bpb, P, node_block, fanout, P1, out.data(),
                                     out.data() + T);
      });
    } else if (mode == "visflat" && argc == 8) {
      const int stride = std::atoi(argv[7]);
      run_per_query(T, [&] { lsi::lsa_visible_kernel(pos.data(), T, block_keys, bpb, P, stride, out.data(), out.data() + T); });
    } else {
      return 2;
    }
    save(dir, "lvis.bin", out);
    return 0;
  }
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
