// Device helpers shared by every kernel of librope_attn.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace ra {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <class T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Device-side status word of this library (one per device that loads it): kernels that
// give up waiting set a nonzero code; rope_attn_last_error reads and clears it.  The whole
// library is one translation unit, so the definition lives here.
__device__ int g_status = 0;

enum DeviceStatus : int {
  kDevOk = 0,
  kDevTimeout = 1,
};

__device__ __forceinline__ void flag_error(int code) { atomicMax(&g_status, code); }

// ---- ordered accumulation (the backward's deterministic mode) ------------------------------
// A counter per accumulator tile says whose turn it is: contributor k adds its part once the
// counter reads k and passes the turn on afterwards, so the fp32 sums run in the order
// 0, 1, 2, ... on every run.  Contributors with a lower index are launched earlier (they are
// CTAs of lower linear index in the same grid), so each wait ends; it is bounded all the same.

// Wait (bounded by limit_ns of global time) until *turn == want; false after a timeout, which
// is also recorded in the status word.
__device__ __forceinline__ bool turn_wait(const unsigned* turn, unsigned want,
                                          unsigned long long limit_ns) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(turn) : "memory");
  if (v == want) return true;
  unsigned long long t0, t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  while (true) {
    __nanosleep(64);
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(turn) : "memory");
    if (v == want) return true;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    if (t - t0 > limit_ns) {
      flag_error(kDevTimeout);
      return false;
    }
  }
}

// Pass the turn on: everything this thread wrote (or saw written by the threads it
// synchronised with) before is visible to the next contributor.
__device__ __forceinline__ void turn_pass(unsigned* turn) {
  asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(turn) : "memory");
}

// Header at the start of every workspace: which problem's intermediates the workspace holds.
// The last kernel of a forward or backward call writes it; the backward's recomputation kernels
// read it on the device and skip their work when it already holds what they would write.
struct WsHeader {
  unsigned long long tag;  // tag of the problem (sizes, flags, RoPE base, input pointers)
  unsigned int magic;      // kWsMagic once written by the library
  unsigned int state;      // kWsValid | kWsDqZero
};
constexpr unsigned int kWsMagic = 0x53574152u;
constexpr unsigned int kWsValid = 1u;   // RoPE table, Q~, K~, V, l, delta and loss partials
constexpr unsigned int kWsDqZero = 2u;  // the dQ~ accumulator holds zeros

// A kernel given a gate skips its work when hdr holds `tag` with every bit of `need` set;
// with hdr == nullptr it always works.
struct WsGate {
  const WsHeader* hdr;
  unsigned long long tag;
  unsigned int need;
};

__device__ __forceinline__ bool gate_skip(const WsGate& g) {
  if (!g.hdr) return false;
  const unsigned long long tag = g.hdr->tag;
  const unsigned int magic = g.hdr->magic, state = g.hdr->state;
  return magic == kWsMagic && tag == g.tag && (state & g.need) == g.need;
}

// Row-major [rows][cols] float tile loader with a padded smem stride.
// Rows at or beyond `valid_rows` are filled with zeros.
template <class T>
__device__ __forceinline__ void load_tile_f32(float* dst, int ld_dst, const T* src, int rows,
                                              int cols, int valid_rows, int tid, int nthr) {
  for (int e = tid; e < rows * cols; e += nthr) {
    int r = e / cols, c = e - r * cols;
    dst[r * ld_dst + c] = (r < valid_rows) ? to_f(src[(size_t)r * cols + c]) : 0.f;
  }
}

}  // namespace ra
