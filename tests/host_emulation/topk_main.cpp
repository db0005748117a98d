// Runs the row-wise top-k kernel of the library's source (made
// host-compilable by cuda_shim.h and the test's preprocessing) on files of
// inputs, one OS thread per CUDA thread, one row (CTA) at a time.  The shared
// block is allocated at exactly the kernel's size so AddressSanitizer sees its
// end.  Test infrastructure only.
//   DIR FORM R N k ld has_labels has_nvalid nv_offset label_base ld_out rows...
//   (a negative first "row" -G instead runs a grid of G blocks over all rows
//   with the row flags of flags.bin [R] i32: the flagged-launch form; with
//   outrow.bin [R] i32 present, row r's output goes to row out_row[r])
//   FORM 0: <256, 512, 2048>   1: <512, 1024, 8192>   2: <1024, 4096, 8192>
//   (scores.bin [R][ld] f32, labels.bin [R][ld] i32, nvalid.bin [R] i32)
//   -> idx.bin, val.bin [R][ld_out]
#include "topk_host.h"

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

template <int NT, int KMAX, int CAP>
static void run_rows(const lsi::TopkParams& p, const std::vector<int>& rows, int grid) {
  using SH = lsi::TopkShared<NT, KMAX, CAP>;
  blockDim = {static_cast<unsigned>(NT), 1, 1};
  gridDim = {static_cast<unsigned>(grid > 0 ? grid : p.R), 1, 1};
  std::vector<std::barrier<>*> wb;
  for (int w = 0; w < NT / 32; ++w) g_warp_bar[w] = new std::barrier<>(32);
  for (int r : rows) {
    std::barrier<> bar(NT);
    g_block_bar = &bar;
    // fresh shared block, filled with a pattern (shared memory starts undefined)
    unsigned char* smem = static_cast<unsigned char*>(std::malloc(sizeof(SH)));
    std::memset(smem, 0xA5, sizeof(SH));
    g_smem = smem;
    std::vector<std::thread> th;
    for (int t = 0; t < NT; ++t)
      th.emplace_back([&, t] {
        threadIdx = {static_cast<unsigned>(t), 0, 0};
        blockIdx = {static_cast<unsigned>(r), 0, 0};
        if (grid > 0) lsi::topk_kernel<NT, KMAX, CAP, true>(p);
        else lsi::topk_kernel<NT, KMAX, CAP, false>(p);
      });
    for (auto& x : th) x.join();
    std::free(smem);
  }
  for (int w = 0; w < NT / 32; ++w) delete g_warp_bar[w];
}

int main(int argc, char** argv) {
  if (argc < 12) return 2;
  const char* dir = argv[1];
  const int form = std::atoi(argv[2]);
  const int R = std::atoi(argv[3]), N = std::atoi(argv[4]), k = std::atoi(argv[5]);
  const long long ld = std::atoll(argv[6]);
  const int has_lab = std::atoi(argv[7]), has_nv = std::atoi(argv[8]);
  const int nv_offset = std::atoi(argv[9]), label_base = std::atoi(argv[10]);
  const long long ld_out = std::atoll(argv[11]);
  std::vector<int> rows;
  int grid = 0;
  for (int i = 12; i < argc; ++i) rows.push_back(std::atoi(argv[i]));
  if (!rows.empty() && rows[0] < 0) {
    grid = -rows[0];
    rows.clear();
    for (int b = 0; b < grid; ++b) rows.push_back(b);
  }
  // the inputs live in exactly-sized heap blocks, so reads past a row's end
  // or the array's end are reported
  auto sc = load<float>(dir, "scores.bin", static_cast<size_t>(R) * ld);
  std::vector<int32_t> lab, nv;
  if (has_lab) lab = load<int32_t>(dir, "labels.bin", static_cast<size_t>(R) * ld);
  if (has_nv) nv = load<int32_t>(dir, "nvalid.bin", static_cast<size_t>(R));
  std::vector<int32_t> idx(static_cast<size_t>(R) * ld_out, 777);
  std::vector<float> val(static_cast<size_t>(R) * ld_out, 777.f);
  lsi::TopkParams p;
  p.scores = sc.data();
  p.ld = ld;
  p.labels = has_lab ? lab.data() : nullptr;
  p.ld_labels = ld;
  p.n_valid = has_nv ? nv.data() : nullptr;
  p.nv_offset = nv_offset;
  p.label_base = label_base;
  p.R = R;
  p.N = N;
  p.k = k;
  p.idx_out = idx.data();
  p.val_out = val.data();
  p.ld_out = ld_out;
  // an out_row map [R] i32 when DIR/outrow.bin exists: row r's output goes to row out_row[r]
  std::vector<int32_t> outrow;
  {
    char path[1024];
    std::snprintf(path, sizeof path, "%s/outrow.bin", dir);
    if (FILE* f = std::fopen(path, "rb")) {
      std::fclose(f);
      outrow = load<int32_t>(dir, "outrow.bin", static_cast<size_t>(R));
      p.out_row = outrow.data();
    }
  }
  std::vector<int32_t> flags;
  if (grid > 0) {
    flags = load<int32_t>(dir, "flags.bin", static_cast<size_t>(R));
    p.row_flag = flags.data();
  }
  if (form == 0) run_rows<256, 512, 2048>(p, rows, grid);
  else if (form == 1) run_rows<512, 1024, 8192>(p, rows, grid);
  else run_rows<1024, 4096, 8192>(p, rows, grid);
  save(dir, "idx.bin", idx);
  save(dir, "val.bin", val);
  return 0;
}
