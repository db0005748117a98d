// Host stand-ins for the CUDA features the attention kernels use, so that
// their source compiles with g++ and runs on the CPU for the kernel-logic
// tests: one OS thread per CUDA thread of a block, std::barrier for
// __syncthreads and for the two halves of a warp shuffle, a mutex for atomics.
// Shared memory is a buffer of the launch's dynamic size (AddressSanitizer
// sees its end); a kernel's static __shared__ variables become static locals,
// shared by the threads of the one block that runs at a time.  Test
// infrastructure only.
#pragma once
#include <barrier>
#include <cmath>
#include <cstddef>
#include <cstdint>
#include <cstring>
#include <mutex>

#define __global__
#define __device__
#define __host__
#define __forceinline__ inline
#define __restrict__ __restrict
#define __launch_bounds__(...)
#define __shared__
#define __align__(x)

struct uint4 { uint32_t x, y, z, w; };
struct alignas(8) uint2 { uint32_t x, y; };
struct float2 { float x, y; };
struct alignas(16) float4 { float x, y, z, w; };
struct alignas(16) ulonglong2 { unsigned long long x, y; };
inline uint4 make_uint4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) { return {a, b, c, d}; }
inline float2 make_float2(float a, float b) { return {a, b}; }
inline float4 make_float4(float a, float b, float c, float d) { return {a, b, c, d}; }

struct Dim3 { unsigned x, y, z; };
extern thread_local Dim3 threadIdx, blockIdx;
extern Dim3 blockDim, gridDim;

struct alignas(16) int4 { int x, y, z, w; };
inline int4 make_int4(int a, int b, int c, int d) { return {a, b, c, d}; }

template <class T>
inline T __ldg(const T* p) { return *p; }
inline float __uint_as_float(uint32_t u) { float f; std::memcpy(&f, &u, 4); return f; }
inline uint32_t __float_as_uint(float f) { uint32_t u; std::memcpy(&u, &f, 4); return u; }
inline float __int_as_float(int i) { float f; std::memcpy(&f, &i, 4); return f; }
inline int __popc(uint32_t v) { return __builtin_popcount(v); }
inline int __clzll(long long v) { return v == 0 ? 64 : __builtin_clzll(static_cast<unsigned long long>(v)); }

extern std::barrier<>* g_block_bar;
extern std::barrier<>* g_warp_bar[32];
extern float g_xbuf[32][32];
extern std::mutex g_atomic_mu;
extern unsigned char* g_smem;

inline void __syncthreads() { g_block_bar->arrive_and_wait(); }
inline float __shfl_xor_sync(unsigned, float v, int o) {
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  g_xbuf[w][l] = v;
  g_warp_bar[w]->arrive_and_wait();
  const float r = g_xbuf[w][l ^ o];
  g_warp_bar[w]->arrive_and_wait();
  return r;
}
// Warp collectives beyond the float butterfly: every lane of the warp posts
// its 64-bit value, a barrier of the warp's 32 threads, then each lane reads.
inline uint64_t g_x64[32][32];
template <class F>
inline uint64_t warp_gather(uint64_t mine, F pick) {
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  g_x64[w][l] = mine;
  g_warp_bar[w]->arrive_and_wait();
  const uint64_t r = pick(g_x64[w], l);
  g_warp_bar[w]->arrive_and_wait();
  return r;
}
inline uint32_t __shfl_sync(unsigned, uint32_t v, int src) {
  return static_cast<uint32_t>(warp_gather(v, [&](const uint64_t* x, int) { return x[src & 31]; }));
}
inline uint32_t __shfl_up_sync(unsigned, uint32_t v, int d) {
  return static_cast<uint32_t>(warp_gather(v, [&](const uint64_t* x, int l) { return l >= d ? x[l - d] : x[l]; }));
}
inline unsigned long long __shfl_xor_sync(unsigned, unsigned long long v, int o) {
  return warp_gather(v, [&](const uint64_t* x, int l) { return x[l ^ o]; });
}
inline uint32_t __shfl_xor_sync(unsigned, uint32_t v, int o) {
  return static_cast<uint32_t>(warp_gather(v, [&](const uint64_t* x, int l) { return x[l ^ o]; }));
}
template <class T>
inline T min(T a, T b) { return b < a ? b : a; }
template <class T>
inline T max(T a, T b) { return a < b ? b : a; }
inline uint32_t __ballot_sync(unsigned, int pred) {
  return static_cast<uint32_t>(warp_gather(pred ? 1u : 0u, [&](const uint64_t* x, int) {
    uint32_t b = 0;
    for (int i = 0; i < 32; ++i) b |= static_cast<uint32_t>(x[i] & 1u) << i;
    return static_cast<uint64_t>(b);
  }));
}
inline int __any_sync(unsigned m, int pred) { return __ballot_sync(m, pred) != 0u; }
inline unsigned atomicAdd(unsigned* p, unsigned v) {
  std::lock_guard<std::mutex> g(g_atomic_mu);
  const unsigned old = *p;
  *p += v;
  return old;
}
inline int atomicMin(int* p, int v) {
  std::lock_guard<std::mutex> g(g_atomic_mu);
  const int old = *p;
  if (v < old) *p = v;
  return old;
}
inline int atomicOr(int* p, int v) {
  std::lock_guard<std::mutex> g(g_atomic_mu);
  const int old = *p;
  *p |= v;
  return old;
}
typedef int cudaError_t;

// fma.rn.f32x2: a correctly rounded fused multiply-add on each fp32 half
inline uint64_t host_fma2(uint64_t acc, uint64_t a, uint64_t b) {
  float c[2], x[2], y[2];
  std::memcpy(c, &acc, 8);
  std::memcpy(x, &a, 8);
  std::memcpy(y, &b, 8);
  c[0] = std::fma(x[0], y[0], c[0]);
  c[1] = std::fma(x[1], y[1], c[1]);
  std::memcpy(&acc, c, 8);
  return acc;
}

namespace lsi {
enum : int { FAULT_NONE = 0, FAULT_WAIT_TIMEOUT = 1, FAULT_BAD_INDEX = 2 };
extern int g_fault;
inline uint64_t pack_f32x2(float lo, float hi) {   // low half first, as mov.b64 {lo, hi}
  const float v[2] = {lo, hi};
  uint64_t r;
  std::memcpy(&r, v, 8);
  return r;
}
inline void unpack_f32x2(uint64_t r, float& lo, float& hi) {
  float v[2];
  std::memcpy(v, &r, 8);
  lo = v[0];
  hi = v[1];
}
}  // namespace lsi
