// Runs the attention kernels of the library's source (made host-compilable by
// cuda_shim.h and the test's preprocessing) on files of inputs.  Test
// infrastructure only.
//   attn  DIR T H k n_rows scale has_row_off foreign   -> out.bin, lse.bin; prints the fault word
//   merge DIR S rows d_v blocks                         -> mo.bin, ml.bin
#include "kernel_host.h"

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

static int run_attn(char** a) {
  const char* dir = a[0];
  const int T = std::atoi(a[1]), H = std::atoi(a[2]), k = std::atoi(a[3]);
  const long long n_rows = std::atoll(a[4]);
  const float scale = static_cast<float>(std::atof(a[5]));
  const int has_off = std::atoi(a[6]), foreign = std::atoi(a[7]);
  auto q = load<uint16_t>(dir, "q.bin", static_cast<size_t>(T) * H * 576);
  auto lat = load<uint16_t>(dir, "lat.bin", static_cast<size_t>(n_rows) * 576);
  auto idx = load<int32_t>(dir, "idx.bin", static_cast<size_t>(T) * k);
  std::vector<int64_t> off;
  if (has_off) off = load<int64_t>(dir, "off.bin", T);
  std::vector<float> out(static_cast<size_t>(T) * H * 512, 12345.f), lse(static_cast<size_t>(T) * H, 12345.f);
  const size_t smem = lsi::attn_smem_bytes();
  std::vector<unsigned char> smem_buf(smem);
  g_smem = smem_buf.data();
  const int blocks = T * (H / 8);
  for (int b = 0; b < blocks; ++b) {
    std::barrier<> bar(256);
    std::vector<std::barrier<>*> wb;
    for (int w = 0; w < 8; ++w) {
      wb.push_back(new std::barrier<>(32));
      g_warp_bar[w] = wb.back();
    }
    g_block_bar = &bar;
    std::memset(g_smem, 0xA5, smem);   // stale contents, as on the device
    std::vector<std::thread> th;
    for (int t = 0; t < 256; ++t)
      th.emplace_back([&, t] {
        threadIdx = {static_cast<unsigned>(t), 0, 0};
        blockIdx = {static_cast<unsigned>(b), 0, 0};
        lsi::sparse_attn_kernel(q.data(), lat.data(), idx.data(), has_off ? off.data() : nullptr, H, k, n_rows, scale,
                                foreign, out.data(), lse.data());
      });
    for (auto& x : th) x.join();
    for (auto* x : wb) delete x;
  }
  save(dir, "out.bin", out);
  save(dir, "lse.bin", lse);
  std::printf("%d\n", lsi::g_fault);
  return 0;
}

static int run_merge(char** a) {
  const char* dir = a[0];
  const int S = std::atoi(a[1]);
  const long long rows = std::atoll(a[2]);
  const int d_v = std::atoi(a[3]), blocks = std::atoi(a[4]);
  auto op = load<float>(dir, "op.bin", static_cast<size_t>(S) * rows * d_v);
  auto lp = load<float>(dir, "lp.bin", static_cast<size_t>(S) * rows);
  std::vector<float> o(static_cast<size_t>(rows) * d_v, 777.f), l(rows, 777.f);
  gridDim = {static_cast<unsigned>(blocks), 1, 1};
  for (int b = 0; b < blocks; ++b)   // no barriers: the threads of a block run one after another
    for (int t = 0; t < 256; ++t) {
      threadIdx = {static_cast<unsigned>(t), 0, 0};
      blockIdx = {static_cast<unsigned>(b), 0, 0};
      lsi::attn_merge_kernel(op.data(), lp.data(), S, rows, d_v, o.data(), l.data());
    }
  save(dir, "mo.bin", o);
  save(dir, "ml.bin", l);
  return 0;
}

int main(int argc, char** argv) {
  if (argc >= 10 && std::strcmp(argv[1], "attn") == 0) return run_attn(argv + 2);
  if (argc >= 7 && std::strcmp(argv[1], "merge") == 0) return run_merge(argv + 2);
  std::fprintf(stderr, "usage: attn DIR T H k n_rows scale has_row_off foreign | merge DIR S rows d_v blocks\n");
  return 2;
}
