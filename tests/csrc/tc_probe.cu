// Test harness for the sm_100a primitives of librope_attn (tests only).
//
// probe_mma: one CTA computes D = A * B with tcgen05 for one operand arrangement (A and B
//   each K-major or MN-major in 128-byte-swizzled shared memory, or A from TMEM), so each
//   descriptor form the library uses is checked in isolation against torch.
// probe_timeout: a kernel waits on an mbarrier that nothing arrives on; the bounded wait
//   must give up, record a timeout in the status word and return (no trap, no hang).
// probe_turn: the turn counters of the ordered (deterministic) accumulation: CTAs take turns
//   in a given order and log it, or one waits for a turn that never comes and gives up.
// probe_mma_rate: how long one tcgen05.mma (K = 16) of a given shape holds the tensor pipe
//   when one or two threads of a CTA issue them back to back, one CTA per SM (clock64 around
//   the issue loop and the completion; the operands are zeros).
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../loss_closed_form_b200/csrc/tc_ptx.cuh"

using namespace ra;
using namespace ra::tc;

namespace {

constexpr int kSmemA = 32768;   // up to 128 x 128 bf16
constexpr int kSmemB = 65536;   // up to 128 x 256 bf16
constexpr int kTmemCols = 512;

__global__ void __launch_bounds__(128)
probe_mma_kernel(const __nv_bfloat16* __restrict__ A, const __nv_bfloat16* __restrict__ B,
                 float* __restrict__ D, int M, int N, int K, int a_mn, int b_mn, int a_tmem,
                 unsigned long long limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kSmemA;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kSmemA + kSmemB);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 1);
  const uint32_t abort_flag = smem_u32(tslot + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // A into swizzled smem: 16-byte chunks of 8 consecutive elements along the major axis
  for (int e = tid; e < M * K / 8; e += 128) {
    uint32_t vals[4];
    __nv_bfloat16 tmp[8];
    uint32_t off;
    if (!a_mn) {  // rows = m, K contiguous
      const int m = e / (K / 8), k0 = (e % (K / 8)) * 8;
      for (int i = 0; i < 8; ++i) tmp[i] = A[(size_t)m * K + k0 + i];
      off = (k0 / 64) * (M * 128) + sw128_offset(m, (k0 % 64) / 8);
    } else {      // rows = k, M contiguous
      const int k = e / (M / 8), m0 = (e % (M / 8)) * 8;
      for (int i = 0; i < 8; ++i) tmp[i] = A[(size_t)(m0 + i) * K + k];
      off = (m0 / 64) * (K * 128) + sw128_offset(k, (m0 % 64) / 8);
    }
    for (int i = 0; i < 4; ++i)
      vals[i] = (uint32_t)__bfloat16_as_ushort(tmp[2 * i]) |
                ((uint32_t)__bfloat16_as_ushort(tmp[2 * i + 1]) << 16);
    st_shared_v4(smem_u32(sA) + off, vals[0], vals[1], vals[2], vals[3]);
  }
  for (int e = tid; e < K * N / 8; e += 128) {
    uint32_t vals[4];
    __nv_bfloat16 tmp[8];
    uint32_t off;
    if (!b_mn) {  // rows = n, K contiguous
      const int nn = e / (K / 8), k0 = (e % (K / 8)) * 8;
      for (int i = 0; i < 8; ++i) tmp[i] = B[(size_t)(k0 + i) * N + nn];
      off = (k0 / 64) * (N * 128) + sw128_offset(nn, (k0 % 64) / 8);
    } else {      // rows = k, N contiguous
      const int k = e / (N / 8), n0 = (e % (N / 8)) * 8;
      for (int i = 0; i < 8; ++i) tmp[i] = B[(size_t)k * N + n0 + i];
      off = (n0 / 64) * (K * 128) + sw128_offset(k, (n0 % 64) / 8);
    }
    for (int i = 0; i < 4; ++i)
      vals[i] = (uint32_t)__bfloat16_as_ushort(tmp[2 * i]) |
                ((uint32_t)__bfloat16_as_ushort(tmp[2 * i + 1]) << 16);
    st_shared_v4(smem_u32(sB) + off, vals[0], vals[1], vals[2], vals[3]);
  }
  if (tid == 0) {
    mbar_init(smem_u32(bar), 1);
    abort_set(abort_flag, 0);
    fence_barrier_init();
  }
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(smem_u32(tslot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t d_tmem = tmem;        // columns 0 .. N-1
  const uint32_t a_tm = tmem + 256;    // columns 256 .. 256 + K/2 - 1
  if (a_tmem) {  // M == 128: row `tid` of A into TMEM lane `tid`, two bf16 per column
    for (int c0 = 0; c0 < K / 2; c0 += 32) {
      uint32_t r[32];
      for (int c = 0; c < 32; ++c)
        r[c] = (uint32_t)__bfloat16_as_ushort(A[(size_t)tid * K + 2 * (c0 + c)]) |
               ((uint32_t)__bfloat16_as_ushort(A[(size_t)tid * K + 2 * (c0 + c) + 1]) << 16);
      tmem_st32(a_tm + ((uint32_t)(warp * 32) << 16) + c0, r);
    }
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid == 0) {
    const uint32_t idesc = idesc_bf16_f32(M, N, a_mn, b_mn);
    for (int kk = 0; kk < K / 16; ++kk) {
      uint64_t bd;
      if (!b_mn)
        bd = sw128_desc(smem_u32(sB) + (kk / 4) * (N * 128) + (kk % 4) * 32, 16, 1024);
      else
        bd = sw128_desc(smem_u32(sB) + kk * 2048, K * 128, 1024);
      if (a_tmem) {
        mma_ts(d_tmem, a_tm + kk * 8, bd, idesc, kk > 0);
      } else {
        uint64_t ad;
        if (!a_mn)
          ad = sw128_desc(smem_u32(sA) + (kk / 4) * (M * 128) + (kk % 4) * 32, 16, 1024);
        else
          ad = sw128_desc(smem_u32(sA) + kk * 2048, K * 128, 1024);
        mma_ss(d_tmem, ad, bd, idesc, kk > 0);
      }
    }
    mma_commit(smem_u32(bar));
  }
  __syncwarp();
  const bool ok = mbar_wait(smem_u32(bar), 0, abort_flag, limit_ns);
  tc_fence_after();
  if (ok) {
    // M = 128: row r in lane r.  M = 64: row r in lane (r % 16) + 32 * (r / 16).
    const int row = (M == 128) ? tid : (warp * 16 + lane);
    const bool has_row = (M == 128) || lane < 16;
    for (int c0 = 0; c0 < N; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(d_tmem + ((uint32_t)(warp * 32) << 16) + c0, r);
      tmem_wait_ld();
      if (has_row)
        for (int c = 0; c < 32; ++c) D[(size_t)row * N + c0 + c] = __uint_as_float(r[c]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

__global__ void probe_timeout_kernel(unsigned long long limit_ns, int* waited_ok) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_word;
  const uint32_t abort_flag = smem_u32(&abort_word);
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_set(abort_flag, 0);
    fence_barrier_init();
  }
  __syncthreads();
  // nothing ever arrives on `bar`: the wait must give up after limit_ns
  const bool ok = mbar_wait(smem_u32(&bar), 0, abort_flag, limit_ns);
  if (threadIdx.x == 0) *waited_ok = ok ? 1 : 0;
}

// CTA b takes turn b (or gridDim.x - 1 - b) and writes its index at that position of `log`.
__global__ void probe_turn_kernel(unsigned* counter, int* log, unsigned long long limit_ns,
                                  int reverse, int* all_ok) {
  if (threadIdx.x != 0) return;
  const unsigned me = reverse ? gridDim.x - 1 - blockIdx.x : blockIdx.x;
  if (!turn_wait(counter, me, limit_ns)) atomicExch(all_ok, 0);
  if (me < gridDim.x) log[me] = static_cast<int>(blockIdx.x);
  __threadfence();
  turn_pass(counter);
}

__global__ void probe_exp2_kernel(const float* __restrict__ x, float* __restrict__ poly,
                                  float* __restrict__ ref, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  poly[i] = exp2_poly(x[i]);
  ref[i] = exp2f(x[i]);
}


// One CTA per SM; warps w < nissuers each issue nmma products of shape M x N x 16 (A from
// shared memory, or from TMEM when a_tmem) into their own accumulator, then wait for them.
// cycles[cta] = clock64 from the first issue to the last completion seen by warp 0.
// The shape and the A source are template parameters: the issue loop then holds no branch
// and its descriptors stay in uniform registers, as in the library's kernels (with them as
// run-time values one thread issued at half the rate).
template <int M, int N, bool A_TMEM>
__global__ void __launch_bounds__(64, 1)
probe_mma_rate_kernel(int nissuers, int nmma, long long* cycles, int* ok,
                      unsigned long long limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  constexpr int kA = 16384, kB = 32768;  // 128 rows and 256 rows of 128 bytes
  const uint32_t sb = smem_u32(smem);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + kA + kB);
  const uint32_t bar0 = smem_u32(smem + kA + kB + 64), bar1 = bar0 + 8;
  const uint32_t flag = smem_u32(smem + kA + kB + 128);
  const int tid = threadIdx.x, warp = tid >> 5;
  for (int i = tid; i < (kA + kB) / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(smem)[i] = 0;
  if (tid == 0) {
    mbar_init(bar0, 1);
    mbar_init(bar1, 1);
    abort_set(flag, 0);
    fence_barrier_init();
  }
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(smem_u32(tslot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  long long t0 = clock64();
  if (warp < nissuers && (tid & 31) == 0) {
    constexpr uint32_t idesc = idesc_bf16_f32(M, N, false, false);
    const uint32_t a = sw128_lo(sb, 16), b = sw128_lo(sb + kA, 16);
    const uint32_t d = tmem + warp * 128, at = tmem + 384;
    const uint32_t bar = warp ? bar1 : bar0;
    t0 = clock64();
    for (int i = 0; i < nmma; ++i) {
      if constexpr (A_TMEM)
        mma_ts(d, at, sw128_at(b, (i & 3) * 32), idesc, i > 0);
      else
        mma_ss(d, sw128_at(a, (i & 3) * 32), sw128_at(b, (i & 3) * 32), idesc, i > 0);
    }
    mma_commit(bar);
    const bool done = mbar_wait(bar, 0, flag, limit_ns);
    const long long t1 = clock64();
    if (warp == 0) cycles[blockIdx.x] = t1 - t0;
    if (!done) atomicAnd(ok, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

extern "C" {

// exp2_poly and CUDA's exp2f on the same inputs (device buffers of n floats).
int probe_exp2(const float* x, float* poly, float* ref, int n) {
  probe_exp2_kernel<<<(n + 255) / 256, 256>>>(x, poly, ref, n);
  return (int)cudaGetLastError();
}

int probe_mma(const void* A, const void* B, float* D, int M, int N, int K, int a_mn, int b_mn,
              int a_tmem, void* stream) {
  if (!(M == 64 || M == 128) || !(N == 64 || N == 128 || N == 256) || !(K == 64 || K == 128) ||
      (a_tmem && (M != 128 || a_mn)))
    return -1;
  const int smem = kSmemA + kSmemB + 1024 + 64;
  cudaFuncSetAttribute(probe_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  probe_mma_kernel<<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(
      (const __nv_bfloat16*)A, (const __nv_bfloat16*)B, D, M, N, K, a_mn, b_mn, a_tmem,
      2000000000ull);
  return (int)cudaGetLastError();
}

// nblocks CTAs take turns on a counter starting at `start` (CTA b waits for turn b, or
// nblocks - 1 - b with reverse); log_host[k] gets the CTA that took turn k (nblocks ints),
// *ok_host whether every wait succeeded, *final_host the counter at the end.  Returns the
// status word (1 after a wait that gave up), or a negative value if a CUDA call failed.
int probe_turn(int nblocks, int reverse, unsigned start, unsigned long long limit_ns,
               int* log_host, int* ok_host, unsigned* final_host) {
  if (nblocks < 1 || nblocks > 128) return -1;
  unsigned* counter = nullptr;
  int* log = nullptr;
  int* ok = nullptr;
  if (cudaMalloc(&counter, sizeof(unsigned)) != cudaSuccess) return -2;
  if (cudaMalloc(&log, nblocks * sizeof(int)) != cudaSuccess) return -2;
  if (cudaMalloc(&ok, sizeof(int)) != cudaSuccess) return -2;
  const int one = 1, zero = 0;
  cudaMemcpy(counter, &start, sizeof(unsigned), cudaMemcpyHostToDevice);
  cudaMemset(log, 0xFF, nblocks * sizeof(int));
  cudaMemcpy(ok, &one, sizeof(int), cudaMemcpyHostToDevice);
  cudaMemcpyToSymbol(ra::g_status, &zero, sizeof(int));
  probe_turn_kernel<<<nblocks, 32>>>(counter, log, limit_ns, reverse, ok);
  if (cudaDeviceSynchronize() != cudaSuccess) return -3;
  int st = 0;
  cudaMemcpyFromSymbol(&st, ra::g_status, sizeof(int));
  cudaMemcpy(log_host, log, nblocks * sizeof(int), cudaMemcpyDeviceToHost);
  cudaMemcpy(ok_host, ok, sizeof(int), cudaMemcpyDeviceToHost);
  cudaMemcpy(final_host, counter, sizeof(unsigned), cudaMemcpyDeviceToHost);
  cudaFree(counter);
  cudaFree(log);
  cudaFree(ok);
  cudaMemcpyToSymbol(ra::g_status, &zero, sizeof(int));
  return st;
}

// Returns the status word after a wait that runs out: 1 (timeout) expected; also whether
// the wait reported success (must be 0).
int probe_timeout(unsigned long long limit_ns, int* waited_ok_host) {
  int* dflag = nullptr;
  if (cudaMalloc(&dflag, sizeof(int)) != cudaSuccess) return -1;
  int zero = 0;
  cudaMemcpyToSymbol(ra::g_status, &zero, sizeof(int));
  probe_timeout_kernel<<<1, 64>>>(limit_ns, dflag);
  if (cudaDeviceSynchronize() != cudaSuccess) return -2;
  int st = 0;
  cudaMemcpyFromSymbol(&st, ra::g_status, sizeof(int));
  cudaMemcpy(waited_ok_host, dflag, sizeof(int), cudaMemcpyDeviceToHost);
  cudaFree(dflag);
  cudaMemcpyToSymbol(ra::g_status, &zero, sizeof(int));
  return st;
}


// Average over one CTA per SM of the cycles per product of one SM (both issuers' products
// counted), after one unmeasured launch.  N = 256 needs one issuer; two issuers need
// N <= 128.  *ok_host = 1 if every wait completed.  Returns 0 or a CUDA error / -1.
int probe_mma_rate(int M, int N, int a_tmem, int nissuers, int nmma, double* cycles_per_mma,
                   int* ok_host) {
  if (!(M == 64 || M == 128) || !(N == 32 || N == 64 || N == 128 || N == 256) ||
      !(nissuers == 1 || nissuers == 2) || (nissuers == 2 && N > 128) || nmma < 1 ||
      (a_tmem && M != 128))
    return -1;
  int dev = 0, nsm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  long long* cyc = nullptr;
  int* ok = nullptr;
  if (cudaMalloc(&cyc, nsm * sizeof(long long)) != cudaSuccess) return -2;
  if (cudaMalloc(&ok, sizeof(int)) != cudaSuccess) return -2;
  const int one = 1;
  cudaMemcpy(ok, &one, sizeof(int), cudaMemcpyHostToDevice);
  const int smem = 16384 + 32768 + 1024 + 256;
  void (*k)(int, int, long long*, int*, unsigned long long) = nullptr;
#define RA_PROBE_SHAPE(m, n)                                                    \
  if (M == m && N == n)                                                         \
    k = a_tmem ? probe_mma_rate_kernel<m, n, true> : probe_mma_rate_kernel<m, n, false>;
  RA_PROBE_SHAPE(128, 32) RA_PROBE_SHAPE(128, 64) RA_PROBE_SHAPE(128, 128)
  RA_PROBE_SHAPE(128, 256) RA_PROBE_SHAPE(64, 32) RA_PROBE_SHAPE(64, 64)
  RA_PROBE_SHAPE(64, 128) RA_PROBE_SHAPE(64, 256)
#undef RA_PROBE_SHAPE
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  for (int rep = 0; rep < 2; ++rep)
    k<<<nsm, 64, smem>>>(nissuers, nmma, cyc, ok, 2000000000ull);
  int err = (int)cudaDeviceSynchronize();
  if (err == 0) {
    long long* h = new long long[nsm];
    cudaMemcpy(h, cyc, nsm * sizeof(long long), cudaMemcpyDeviceToHost);
    cudaMemcpy(ok_host, ok, sizeof(int), cudaMemcpyDeviceToHost);
    double sum = 0.0;
    for (int i = 0; i < nsm; ++i) sum += (double)h[i];
    *cycles_per_mma = sum / nsm / ((double)nmma * nissuers);
    delete[] h;
  }
  cudaFree(cyc);
  cudaFree(ok);
  return err;
}

}  // extern "C"
