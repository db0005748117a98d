// Runs the LSA threshold form's compaction kernel and its missed-row list
// kernel (the library's source, made host-compilable by cuda_shim.h and the
// test's preprocessing) on files of inputs, one OS thread per CUDA thread,
// one CTA at a time.  Test infrastructure only.
//   DIR T P cap2 slack nseg grid top_p cap rows n_chunks
//   inputs:  slist.bin [T][ld] uint2 (ld = cap2 + slack * nseg), cnt.bin
//            [T][nseg][4] u32, vis.bin [T] i32
//   outputs: cval.bin, clab.bin [T][cap], nv.bin [T], over.bin [T] (+ any),
//            list.bin [T], count.bin, run.bin [n_chunks]
#include "lsa_compact_host.h"

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

template <class F>
static void run_grid(int blocks, int threads, F body) {
  blockDim = {static_cast<unsigned>(threads), 1, 1};
  gridDim = {static_cast<unsigned>(blocks), 1, 1};
  for (int w = 0; w < threads / 32; ++w) g_warp_bar[w] = new std::barrier<>(32);
  for (int b = 0; b < blocks; ++b) {
    std::barrier<> bar(threads);
    g_block_bar = &bar;
    std::vector<std::thread> th;
    for (int t = 0; t < threads; ++t)
      th.emplace_back([&, t, b] {
        threadIdx = {static_cast<unsigned>(t), 0, 0};
        blockIdx = {static_cast<unsigned>(b), 0, 0};
        body();
      });
    for (auto& x : th) x.join();
  }
  for (int w = 0; w < threads / 32; ++w) delete g_warp_bar[w];
}

int main(int argc, char** argv) {
  if (argc < 12) return 2;
  const char* dir = argv[1];
  const int T = std::atoi(argv[2]), P = std::atoi(argv[3]), cap2 = std::atoi(argv[4]), slack = std::atoi(argv[5]);
  const int nseg = std::atoi(argv[6]), grid = std::atoi(argv[7]), top_p = std::atoi(argv[8]), cap = std::atoi(argv[9]);
  const int rows = std::atoi(argv[10]), n_chunks = std::atoi(argv[11]);
  const int64_t ld = cap2 + static_cast<int64_t>(slack) * nseg;
  const int NT = (P + 127) / 128;
  const long long units = static_cast<long long>((T + 255) / 256) * NT;
  // exactly-sized heap blocks: reads past a row or an array are reported
  auto slist = load<uint2>(dir, "slist.bin", static_cast<size_t>(T) * ld);
  auto cnt = load<uint32_t>(dir, "cnt.bin", static_cast<size_t>(T) * nseg * 4);
  auto vis = load<int32_t>(dir, "vis.bin", static_cast<size_t>(T));
  std::vector<float> cval(static_cast<size_t>(T) * cap, 777.f);
  std::vector<int32_t> clab(static_cast<size_t>(T) * cap, 777), nv(T, 777), over(T, 0);
  int any = 0;
  run_grid(T, 256, [&] {
    lsi::lsa_compact_kernel(slist.data(), cnt.data(), ld, nseg, cap2, slack, grid, NT, units, vis.data(), top_p, cap,
                            cval.data(), clab.data(), nv.data(), over.data(), &any);
  });
  std::vector<int32_t> list(T, 777), count(1, 777), run(n_chunks, 777);
  run_grid(1, 1024, [&] {
    lsi::lsa_flag_list_kernel(over.data(), T, rows, n_chunks, list.data(), count.data(), run.data());
  });
  // the missed rows' queries and visible counts, gathered once for all
  // chunks; a second gather with its run flag clear must write nothing
  auto q = load<uint16_t>(dir, "q.bin", static_cast<size_t>(T) * 64);
  std::vector<uint16_t> qbuf(static_cast<size_t>(T) * 64, 0x7777), qidle(static_cast<size_t>(T) * 64, 0x7777);
  std::vector<int32_t> vbuf(T, 777), vidle(T, 777);
  const int zero = 0;
  run_grid((T * 8 + 255) / 256, 256, [&] {
    lsi::lsa_gather_rows_kernel(list.data(), count.data(), T, q.data(), vis.data(), &any, qbuf.data(), vbuf.data());
  });
  run_grid((T * 8 + 255) / 256, 256, [&] {
    lsi::lsa_gather_rows_kernel(list.data(), count.data(), T, q.data(), vis.data(), &zero, qidle.data(), vidle.data());
  });
  save(dir, "qbuf.bin", qbuf);
  save(dir, "vbuf.bin", vbuf);
  save(dir, "qidle.bin", qidle);
  save(dir, "vidle.bin", vidle);
  over.push_back(any);
  save(dir, "cval.bin", cval);
  save(dir, "clab.bin", clab);
  save(dir, "nv.bin", nv);
  save(dir, "over.bin", over);
  save(dir, "list.bin", list);
  save(dir, "count.bin", count);
  save(dir, "run.bin", run);
  return 0;
}
