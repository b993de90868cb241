// librope_attn: host side of the C ABI declared in include/rope_attn.h.
//
// Validates every argument before enqueuing anything, carves the caller's workspace,
// and launches the kernels on the caller's stream.  Never allocates, frees or
// synchronises (rope_attn_last_error excepted).
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>
#include <vector>

#include <cudaTypedefs.h>
#include <stdlib.h>

#include "../../include/rope_attn.h"
#include "common.cuh"
#include "simt_kernels.cuh"
#include "tc_attn_fwd.cuh"
#include "tc_attn_bwd.cuh"
#include "tc_proj_dw.cuh"
#include "approx_kernels.cuh"

namespace {

thread_local int64_t t_launches = 0;

// Kernel ids for launch counting and per-kernel event timing.
enum KernelId : int {
  K_ROPE_TABLE = 0,
  K_PROJ_SIMT,
  K_FWD_SIMT,
  K_BWD_PRE,
  K_BWD_SIMT,
  K_DW_PART_SIMT,
  K_DW_REDUCE,
  K_LOSS,
  K_FWD_TC,
  K_BWD_TC,
  K_PROJ_TC,
  K_DQ_UNROT,
  K_DW_TC,
  K_DA_TC,
  K_DA_SIMT,
  K_COMB_W,
  K_COMB_G,
  K_PROJ_SIMT_BWD,  // launches made by a backward call (skipped on the device when the
  K_PROJ_TC_BWD,    // workspace holds this problem's intermediates)
  K_APX_LOCAL,      // the approximate method's kernels
  K_APX_SCAN,
  K_APX_APPLY,
  K_APX_INTRA,
  K_APX_ROWS,
  K_COUNT
};
const char* const kKernelNames[K_COUNT] = {
    "rope_table", "proj_rope_simt", "attn_fwd_simt", "bwd_prep",
    "attn_bwd_simt", "dw_partial_simt", "dw_reduce", "loss_finalize",
    "attn_fwd_tc", "attn_bwd_tc", "proj_rope_tc", "dq_unrotate", "dw_tc",
    "input_grads_tc", "input_grads_simt", "combined_weights", "combined_grad",
    "proj_rope_simt_bwd", "proj_rope_tc_bwd", "approx_local_sum", "approx_scan", "approx_apply",
    "approx_intra", "approx_rows"};

struct ProfRecord {
  int id;
  cudaEvent_t start, stop;
};
struct Profiler {
  bool on = false;
  int only = -1;  // >= 0: only this kernel's launches get events
  std::vector<ProfRecord> recs;
  std::vector<cudaEvent_t> pool;
  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
  void recycle() {
    for (auto& r : recs) {
      pool.push_back(r.start);
      pool.push_back(r.stop);
    }
    recs.clear();
  }
};
thread_local Profiler t_prof;

// Brackets one kernel launch: counts it and, when profiling, records events around it.
struct Launch {
  cudaStream_t st;
  int slot = -1;
  Launch(KernelId id, cudaStream_t s) : st(s) {
    ++t_launches;
    if (t_prof.on && (t_prof.only < 0 || t_prof.only == id)) {
      ProfRecord r{id, t_prof.get(), t_prof.get()};
      cudaEventRecord(r.start, st);
      t_prof.recs.push_back(r);
      slot = (int)t_prof.recs.size() - 1;
    }
  }
  ~Launch() {
    if (slot >= 0) cudaEventRecord(t_prof.recs[slot].stop, st);
  }
};

constexpr size_t kAlignWs = 256;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace layout.  Offsets are bytes from the workspace base, each 256-byte aligned.
struct Layout {
  size_t hdr;        // ra::WsHeader: which problem's intermediates the workspace holds
  size_t rope;       // float2 [n][d/2]
  size_t qt, kt, v;  // intermediate [B][H][n][d] (element size `inter`)
  size_t ell;        // intermediate [B][H][n][d]
  size_t delta;      // float [B][H][n]
  size_t dqt;        // float [B][H][n][d]: gradient w.r.t. Q~ (accumulated)
  size_t dkt;        // float [B][H][n][d] (fp32 path): gradient w.r.t. K~
  size_t dv;         // float [B][H][n][d] (fp32 path)
  size_t dq16;       // bf16 [B][H][n][d] (bf16 path): rot^-1(dQ~)
  size_t dk16;       // bf16 [B][H][n][d] (bf16 path): rot^-1(dK~)
  size_t dv16;       // bf16 [B][H][n][d] (bf16 path)
  size_t dw_part;    // float [3][H][nsplit][d][d]
  size_t loss_part;  // double [nparts]
  size_t turn;       // unsigned [B][H][turn_stride]: turn counters of the deterministic mode
  size_t total;
  int inter;         // bytes per intermediate element
  int nsplit;        // weight-gradient row splits per head
  int chunk;         // rows per split (fp32 path) or 128-row tiles per split (bf16 path)
  int nparts;        // capacity of the loss partial sums
  int nparts_fwd;    // partial sums the forward writes
  int nparts_pre;    // partial sums the backward's own l = O - E pass writes
  int turn_stride;   // turn counters per instance: one per 32-row query tile
};

bool is_aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

ra_status check_problem(const ra_problem* p) {
  if (!p) return RA_ERR_INVALID_ARG;
  if (p->B < 1 || p->H < 1 || p->n < 1 || p->d < 1) return RA_ERR_INVALID_ARG;
  if (p->dtype != RA_F32 && p->dtype != RA_BF16) return RA_ERR_INVALID_ARG;
  if (p->causal != 0 && p->causal != 1) return RA_ERR_INVALID_ARG;
  if (p->deterministic != 0 && p->deterministic != 1) return RA_ERR_INVALID_ARG;
  if (!(p->rope_base > 0.0) || !isfinite(p->rope_base)) return RA_ERR_INVALID_ARG;
  if (!p->A1 || !p->A2 || !p->A3 || !p->WQ || !p->WK || !p->WV) return RA_ERR_INVALID_ARG;
  if (p->d != 64 && p->d != 128) return RA_ERR_UNSUPPORTED;
  // grid limits: B*H blocks in y, and sizes held in 32-bit ints inside the kernels
  if ((int64_t)p->B * p->H > 65535) return RA_ERR_UNSUPPORTED;
  if ((int64_t)p->n > (1 << 24)) return RA_ERR_UNSUPPORTED;
  // the tensor-core backward takes one CTA per 128-key tile in grid y (at most 65535)
  if (p->dtype == RA_BF16 && (int64_t)p->n > 65535LL * 128) return RA_ERR_UNSUPPORTED;
  const void* ptrs[] = {p->A1, p->A2, p->A3, p->WQ, p->WK, p->WV, p->E};
  for (const void* q : ptrs)
    if (q && !is_aligned(q, 16)) return RA_ERR_ALIGNMENT;
  if (p->pos && !is_aligned(p->pos, 4)) return RA_ERR_ALIGNMENT;
  return RA_OK;
}

// Tag of a problem: FNV-1a over its sizes, flags, RoPE base and input pointers.  The forward
// stamps it into the workspace header; the backward compares it on the device.
unsigned long long problem_tag(const ra_problem* p) {
  unsigned long long h = 1469598103934665603ull;
  auto mix = [&](unsigned long long v) {
    for (int i = 0; i < 8; ++i) {
      h ^= (v >> (8 * i)) & 0xFFu;
      h *= 1099511628211ull;
    }
  };
  mix((unsigned long long)(uint32_t)p->B);
  mix((unsigned long long)(uint32_t)p->H);
  mix((unsigned long long)(uint32_t)p->n);
  mix((unsigned long long)(uint32_t)p->d);
  mix((unsigned long long)(uint32_t)p->dtype);
  mix((unsigned long long)(uint32_t)p->causal);
  unsigned long long base_bits;
  memcpy(&base_bits, &p->rope_base, sizeof(base_bits));
  mix(base_bits);
  const void* ptrs[] = {p->pos, p->A1, p->A2, p->A3, p->WQ, p->WK, p->WV, p->E};
  for (const void* q : ptrs) mix((unsigned long long)(uintptr_t)q);
  return h;
}

Layout make_layout(const ra_problem* p) {
  Layout L{};
  const size_t B = p->B, H = p->H, n = p->n, d = p->d;
  L.inter = p->dtype == RA_BF16 ? 2 : 4;
  const size_t act = B * H * n * d;
  const long rows = (long)B * n;
  if (p->dtype == RA_BF16) {
    // tensor-core weight gradients: splits of whole 128-row tiles, about two CTAs per SM
    const long tiles = (long)B * ((n + 127) / 128);
    long ns = (2 * 148 + 3 * p->H - 1) / (3 * p->H);
    ns = ns < 1 ? 1 : (ns > tiles ? tiles : ns);
    const long per = (tiles + ns - 1) / ns;
    L.chunk = (int)per;                      // tiles per split
    L.nsplit = (int)((tiles + per - 1) / per);
  } else {
    long ns = (4 * 148 + 3 * p->H - 1) / (3 * p->H);
    ns = ns < 1 ? 1 : ns;
    long maxs = (rows + 63) / 64;
    if (ns > maxs) ns = maxs;
    L.nsplit = (int)ns;
    L.chunk = (int)((rows + ns - 1) / ns);
  }
  L.nparts_pre = (int)(((n + 31) / 32) * B * H);
  // the tensor-core forward writes four partial sums per 128-row query tile
  L.nparts_fwd = p->dtype == RA_BF16 ? (int)(((n + 127) / 128) * B * H * 4) : L.nparts_pre;
  L.nparts = L.nparts_pre > L.nparts_fwd ? L.nparts_pre : L.nparts_fwd;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, kAlignWs);
    return o;
  };
  L.hdr = take(sizeof(ra::WsHeader));
  L.rope = take(n * (d / 2) * sizeof(float2));
  L.qt = take(act * L.inter);
  L.kt = take(act * L.inter);
  L.v = take(act * L.inter);
  L.ell = take(act * L.inter);
  L.delta = take(B * H * n * sizeof(float));
  const bool tcp = p->dtype == RA_BF16;
  L.dqt = take(act * sizeof(float));
  L.dkt = take(tcp ? 0 : act * sizeof(float));
  L.dv = take(tcp ? 0 : act * sizeof(float));
  L.dq16 = take(tcp ? act * 2 : 0);
  L.dk16 = take(tcp ? act * 2 : 0);
  L.dv16 = take(tcp ? act * 2 : 0);
  L.dw_part = take(3 * H * (size_t)L.nsplit * d * d * sizeof(float));
  L.loss_part = take((size_t)L.nparts * sizeof(double));
  L.turn_stride = (int)((n + 31) / 32);
  L.turn = take(B * H * (size_t)L.turn_stride * sizeof(unsigned));
  L.total = off;
  return L;
}

template <class T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

// SM count of the current device (persistent grids take one CTA per SM).
int num_sms() {
  int dev = 0, v = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
    return 148;
  return v;
}

// Heads per scheduling group of the attention kernels: as many as keep the tensors that
// every CTA of a head re-reads (bytes_per_head) within about half of the 126 MB L2, at
// least one.
constexpr double kL2GroupBytes = 64.0 * 1024 * 1024;
int heads_per_l2_group(double bytes_per_head, int BH) {
  const int g = static_cast<int>(kL2GroupBytes / bytes_per_head);
  return g < 1 ? 1 : (g > BH ? BH : g);
}

ra_status launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

ra_status check_ws(const ra_problem* p, void* ws, size_t ws_bytes) {
  if (!ws) return RA_ERR_WORKSPACE;
  if (!is_aligned(ws, kAlignWs)) return RA_ERR_ALIGNMENT;
  if (ws_bytes < make_layout(p).total) return RA_ERR_WORKSPACE;
  return RA_OK;
}

// Bound on every on-chip wait inside the tensor-core kernels (RA_WAIT_LIMIT_MS, default 2 s).
unsigned long long wait_limit_ns() {
  static unsigned long long v = [] {
    const char* e = getenv("RA_WAIT_LIMIT_MS");
    long ms = e ? atol(e) : 2000;
    if (ms <= 0) ms = 2000;
    return (unsigned long long)ms * 1000000ull;
  }();
  return v;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (EncodeTiledFn) nullptr;
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

// 3-D map over bf16 rows [outer][rows][cols] with a box of 64 columns x box_rows rows and
// 128-byte swizzle; rows past `rows` of each outer index read as zero.
bool map_bf16_3d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows,
                 uint64_t outer, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {cols, rows, outer};
  cuuint64_t strides[2] = {cols * 2, rows * cols * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// 2-D map over fp32 rows [rows][cols] with boxes of 32 columns (128 bytes) x box_rows,
// 128-byte swizzle (the RoPE table rows of a tile, read back with swizzled shared loads).
bool map_f32_rows_sw128(CUtensorMap* m, void* base, uint64_t cols, uint64_t rows,
                        uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 4};
  cuuint32_t box[2] = {32, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over fp32 rows [outer][rows][cols] with boxes of 32 columns (128 bytes) x box_rows,
// 128-byte swizzle (the target of the d = 64 backward's bulk reductions, staged as swizzled
// rows so that one thread per row writes without bank conflicts).
bool map_f32_3d_sw128(CUtensorMap* m, void* base, uint64_t cols, uint64_t rows, uint64_t outer,
                      uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {cols, rows, outer};
  cuuint64_t strides[2] = {cols * 4, rows * cols * 4};
  cuuint32_t box[3] = {32, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over fp32 rows [outer][rows][cols] with a box of cols x box_rows, no swizzle
// (the target of bulk reductions).
bool map_f32_3d(CUtensorMap* m, void* base, uint64_t cols, uint64_t rows, uint64_t outer,
                uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {cols, rows, outer};
  cuuint64_t strides[2] = {cols * 4, rows * cols * 4};
  cuuint32_t box[3] = {(cuuint32_t)cols, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Last launch of every forward and backward call: the loss (when asked for) from the partial
// sums, then the workspace header (this problem's tag and `state`).  `count` partials belong to
// this call; when `gate` finds the recomputation skipped, the forward's partials are summed.
void finalize(const ra_problem* p, const Layout& L, void* ws, float* loss, int count,
              ra::WsGate gate, unsigned int state, cudaStream_t st) {
  Launch l(K_LOSS, st);
  ra::simt::loss_finalize_kernel<<<1, 1024, 0, st>>>(at<double>(ws, L.loss_part), count,
                                                    L.nparts_fwd, loss, gate,
                                                    at<ra::WsHeader>(ws, L.hdr), problem_tag(p),
                                                    state);
}

// theta_k = base^(-2k/d) for k < d/2, in double precision.
ra::simt::RopeTheta rope_theta(const ra_problem* p) {
  ra::simt::RopeTheta th{};
  const int half = p->d / 2;
  for (int k = 0; k < half && k < ra::simt::kMaxHalf; ++k)
    th.t[k] = std::pow(p->rope_base, -2.0 * (double)k / (double)p->d);
  return th;
}

// RoPE table of the forward (grid-stride, a few blocks per SM).
void rope_table(const ra_problem* p, const Layout& L, void* ws, cudaStream_t st) {
  const long long total = (long long)p->n * (p->d / 2);
  const long long want = (total + 255) / 256, cap = 8LL * num_sms();
  Launch l(K_ROPE_TABLE, st);
  ra::simt::rope_table_kernel<<<(unsigned)(want < cap ? want : cap), 256, 0, st>>>(
      at<float2>(ws, L.rope), p->pos, p->n, p->d / 2, rope_theta(p));
}

// Gates of the backward.  With ws_holds_fwd the device decides from the workspace header:
// the recomputation (RoPE table, projections, l and delta) is skipped when the header holds
// this problem's intermediates, the zeroing of dQ~ when it is zero already.  Without, both run.
struct BwdGates {
  ra::WsGate recompute, zero;
};
BwdGates bwd_gates(const ra_problem* p, const Layout& L, void* ws, int holds) {
  const ra::WsHeader* hdr = holds ? at<ra::WsHeader>(ws, L.hdr) : nullptr;
  const unsigned long long tag = problem_tag(p);
  return BwdGates{ra::WsGate{hdr, tag, ra::kWsValid},
                  ra::WsGate{hdr, tag, ra::kWsValid | ra::kWsDqZero}};
}

// The backward's preparation (one launch): unless the gates find the workspace ready, the
// RoPE table, l = O - E, delta and the loss partials, and the zeroing of dQ~.
template <class T, class TL>
void bwd_prep(const ra_problem* p, const Layout& L, const void* O, void* ws, const BwdGates& g,
              cudaStream_t st) {
  const long long BH = (long long)p->B * p->H;
  const long long vblocks = BH * ((p->n + ra::simt::kRows - 1) / ra::simt::kRows);
  const long long cap = 8LL * num_sms();
  Launch l(K_BWD_PRE, st);
  ra::simt::bwd_prep_kernel<T, TL><<<(unsigned)(vblocks < cap ? vblocks : cap),
                                     ra::simt::kThreads, 0, st>>>(
      (const T*)O, (const T*)p->E, at<TL>(ws, L.ell), at<float>(ws, L.delta),
      at<double>(ws, L.loss_part), p->n, p->d, (int)BH, at<float2>(ws, L.rope), p->pos,
      rope_theta(p), at<float4>(ws, L.dqt), BH * p->n * p->d / 4, g.recompute, g.zero,
      p->deterministic ? at<unsigned>(ws, L.turn) : nullptr, BH * L.turn_stride);
}

// ---------------------------------------------------------------------------------------
// fp32 CUDA-core path
// ---------------------------------------------------------------------------------------
// Projections + RoPE from the table in the workspace.  The gate (hdr == nullptr: none) lets
// the kernel skip the work on the device when the workspace already holds this problem's
// projections.
template <class T, class TX>
ra_status simt_project(const ra_problem* p, const Layout& L, void* ws, ra::WsGate gate,
                       bool in_bwd, cudaStream_t st) {
  using namespace ra::simt;
  const int n = p->n, d = p->d;
  float2* tab = at<float2>(ws, L.rope);
  {
    size_t smem = (size_t)(kRows * (d + 4) + d * d) * sizeof(float);
    auto k = proj_rope_kernel<T, TX>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    dim3 grid((n + kRows - 1) / kRows, p->B * p->H, 3);
    Launch l(in_bwd ? K_PROJ_SIMT_BWD : K_PROJ_SIMT, st);
    k<<<grid, kThreads, smem, st>>>(
        (const T*)p->A1, (const T*)p->A2, (const T*)p->A3, (const T*)p->WQ, (const T*)p->WK,
        (const T*)p->WV, tab, at<TX>(ws, L.qt), at<TX>(ws, L.kt), at<TX>(ws, L.v), p->H, n, d,
        gate);
  }
  return launch_status();
}

template <class T>
ra_status simt_fwd(const ra_problem* p, void* O, float* lse, float* loss, void* ws,
                   cudaStream_t st) {
  using namespace ra::simt;
  const Layout L = make_layout(p);
  rope_table(p, L, ws, st);
  ra_status s = simt_project<T, float>(p, L, ws, ra::WsGate{nullptr, 0, 0}, false, st);
  if (s != RA_OK) return s;
  const int n = p->n, d = p->d;
  const float scale = 1.0f / sqrtf((float)d);
  size_t smem = (size_t)(3 * kRows * (d + 4) + kRows * 33) * sizeof(float);
  auto k = attn_fwd_kernel<T, T>;
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  dim3 grid((n + kRows - 1) / kRows, p->B * p->H);
  {
    Launch l(K_FWD_SIMT, st);
    k<<<grid, kThreads, smem, st>>>(at<float>(ws, L.qt), at<float>(ws, L.kt), at<float>(ws, L.v),
                                    (const T*)p->E, (T*)O, lse, at<float>(ws, L.ell),
                                    at<float>(ws, L.delta), at<double>(ws, L.loss_part), n, d,
                                    p->causal, scale * ra::kLog2e);
  }
  // loss, then the header: with a target the workspace now holds l, delta and the partials
  finalize(p, L, ws, loss, L.nparts_fwd, ra::WsGate{nullptr, 0, 0}, p->E ? ra::kWsValid : 0u, st);
  return launch_status();
}

// ---------------------------------------------------------------------------------------
// bf16 tensor-core path
// ---------------------------------------------------------------------------------------
template <int D>
ra_status tc_project(const ra_problem* p, const Layout& L, void* ws, ra::WsGate gate,
                     bool in_bwd, cudaStream_t st) {
  using namespace ra::tc;
  using C = ProjCfg<D>;
  const int n = p->n, BH = p->B * p->H;
  float2* tab = at<float2>(ws, L.rope);
  CUtensorMap a1, a2, a3, w1, w2, w3, o1, o2, o3;
  if (!map_bf16_3d(&a1, p->A1, D, n, BH, C::BM) || !map_bf16_3d(&a2, p->A2, D, n, BH, C::BM) ||
      !map_bf16_3d(&a3, p->A3, D, n, BH, C::BM) || !map_bf16_3d(&w1, p->WQ, D, D, p->H, D) ||
      !map_bf16_3d(&w2, p->WK, D, D, p->H, D) || !map_bf16_3d(&w3, p->WV, D, D, p->H, D) ||
      !map_bf16_3d(&o1, at<void>(ws, L.qt), D, n, BH, C::BM) ||
      !map_bf16_3d(&o2, at<void>(ws, L.kt), D, n, BH, C::BM) ||
      !map_bf16_3d(&o3, at<void>(ws, L.v), D, n, BH, C::BM))
    return RA_ERR_CUDA;
  ProjParams pp;
  pp.tab = tab;
  pp.n = n;
  pp.B = p->B;
  pp.H = p->H;
  pp.nrt = (n + C::BM - 1) / C::BM;
  // persistent CTAs, one per SM, over the (row tile, z, head) tiles
  pp.tiles = (long long)p->B * pp.nrt * 3 * p->H;
  const long long sms = num_sms();
  const long long ctas = pp.tiles < sms ? pp.tiles : sms;
  pp.tiles_per_cta = (pp.tiles + ctas - 1) / ctas;
  const long long grid = (pp.tiles + pp.tiles_per_cta - 1) / pp.tiles_per_cta;
  pp.limit_ns = wait_limit_ns();
  pp.gate = gate;
  auto k = proj_rope_tc_kernel<D, false>;
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC);
  Launch l(in_bwd ? K_PROJ_TC_BWD : K_PROJ_TC, st);
  k<<<(unsigned)grid, C::THREADS, C::SMEM_ALLOC, st>>>(a1, a2, a3, w1, w2, w3, o1, o2, o3, pp);
  return launch_status();
}

// Input gradients dA_z = dX_z W_z^T from the bf16 dQ, dK, dV the backward left in the
// workspace (same persistent tcgen05 kernel as the projections, without rotation).
template <int D>
ra_status tc_input_grads(const ra_problem* p, const Layout& L, void* dA1, void* dA2, void* dA3,
                         void* ws, cudaStream_t st) {
  using namespace ra::tc;
  using C = ProjCfg<D>;
  const int n = p->n, BH = p->B * p->H;
  CUtensorMap a1, a2, a3, w1, w2, w3, o1, o2, o3;
  if (!map_bf16_3d(&a1, at<void>(ws, L.dq16), D, n, BH, C::BM) ||
      !map_bf16_3d(&a2, at<void>(ws, L.dk16), D, n, BH, C::BM) ||
      !map_bf16_3d(&a3, at<void>(ws, L.dv16), D, n, BH, C::BM) ||
      !map_bf16_3d(&w1, p->WQ, D, D, p->H, D) || !map_bf16_3d(&w2, p->WK, D, D, p->H, D) ||
      !map_bf16_3d(&w3, p->WV, D, D, p->H, D) || !map_bf16_3d(&o1, dA1, D, n, BH, C::BM) ||
      !map_bf16_3d(&o2, dA2, D, n, BH, C::BM) || !map_bf16_3d(&o3, dA3, D, n, BH, C::BM))
    return RA_ERR_CUDA;
  ProjParams pp;
  pp.tab = at<float2>(ws, L.rope);
  pp.n = n;
  pp.B = p->B;
  pp.H = p->H;
  pp.nrt = (n + C::BM - 1) / C::BM;
  pp.tiles = (long long)p->B * pp.nrt * 3 * p->H;
  const long long sms = num_sms();
  const long long ctas = pp.tiles < sms ? pp.tiles : sms;
  pp.tiles_per_cta = (pp.tiles + ctas - 1) / ctas;
  const long long grid = (pp.tiles + pp.tiles_per_cta - 1) / pp.tiles_per_cta;
  pp.limit_ns = wait_limit_ns();
  pp.gate = ra::WsGate{nullptr, 0, 0};
  auto k = proj_rope_tc_kernel<D, true>;
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC);
  Launch l(K_DA_TC, st);
  k<<<(unsigned)grid, C::THREADS, C::SMEM_ALLOC, st>>>(a1, a2, a3, w1, w2, w3, o1, o2, o3, pp);
  return launch_status();
}

// fp32 I/O: dA_z = rot^-1(dX~_z) W_z^T on the CUDA cores (dQ~, dK~ are kept rotated there).
ra_status simt_input_grads(const ra_problem* p, const Layout& L, void* dA1, void* dA2,
                           void* dA3, void* ws, cudaStream_t st) {
  const int n = p->n, d = p->d;
  dim3 grid((n + ra::simt::kDaRows - 1) / ra::simt::kDaRows, p->B * p->H, 3);
  const size_t smem = (size_t)(d * d + ra::simt::kDaRows * d) * sizeof(float);
  auto k = ra::simt::input_grad_kernel;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return RA_ERR_CUDA;
  Launch l(K_DA_SIMT, st);
  k<<<grid, ra::simt::kThreads, smem, st>>>(
      at<float>(ws, L.dqt), at<float>(ws, L.dkt), at<float>(ws, L.dv), at<float2>(ws, L.rope),
      (const float*)p->WQ, (const float*)p->WK, (const float*)p->WV, (float*)dA1, (float*)dA2,
      (float*)dA3, p->H, n, d);
  return launch_status();
}

template <int D>
ra_status tc_weight_grads(const ra_problem* p, const Layout& L, float* dWQ, float* dWK,
                          float* dWV, void* ws, ra::WsHeader* stamp,
                          const ra::simt::LossSum& ls, cudaStream_t st) {
  using namespace ra::tc;
  using C = DwCfg<D>;
  const int n = p->n, BH = p->B * p->H, half = D / 2;
  {
    const long long quads = (long long)BH * n * (half / 4);
    Launch l(K_DQ_UNROT, st);
    dq_unrotate_kernel<<<(unsigned)((quads + 255) / 256), 256, 0, st>>>(
        at<float4>(ws, L.dqt), at<float4>(ws, L.rope), at<uint4>(ws, L.dq16), quads, n, half,
        1.0f / sqrtf((float)D));
  }
  CUtensorMap a1, a2, a3, x1, x2, x3;
  if (!map_bf16_3d(&a1, p->A1, D, n, BH, C::BR) || !map_bf16_3d(&a2, p->A2, D, n, BH, C::BR) ||
      !map_bf16_3d(&a3, p->A3, D, n, BH, C::BR) ||
      !map_bf16_3d(&x1, at<void>(ws, L.dq16), D, n, BH, C::BR) ||
      !map_bf16_3d(&x2, at<void>(ws, L.dk16), D, n, BH, C::BR) ||
      !map_bf16_3d(&x3, at<void>(ws, L.dv16), D, n, BH, C::BR))
    return RA_ERR_CUDA;
  DwParams dp;
  dp.part = at<float>(ws, L.dw_part);
  dp.n = n;
  dp.B = p->B;
  dp.H = p->H;
  dp.nt = (n + C::BR - 1) / C::BR;
  dp.nsplit = L.nsplit;
  dp.tiles_per_split = L.chunk;
  dp.limit_ns = wait_limit_ns();
  auto k = dw_tc_kernel<D>;
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC);
  {
    dim3 grid(L.nsplit, 3, p->H);
    Launch l(K_DW_TC, st);
    k<<<grid, C::THREADS, C::SMEM_ALLOC, st>>>(a1, a2, a3, x1, x2, x3, dp);
  }
  {
    size_t total = (size_t)3 * p->H * D * D;
    Launch l(K_DW_REDUCE, st);
    // with a loss to sum, one more block sums it and writes the header (no loss_finalize)
    const unsigned blocks = (unsigned)((total + 255) / 256) + (ls.loss ? 1u : 0u);
    ra::simt::dw_reduce_kernel<<<blocks, 256, 0, st>>>(
        at<float>(ws, L.dw_part), dWQ, dWK, dWV, p->H, D, L.nsplit, stamp, problem_tag(p),
        ra::kWsValid, ls);
  }
  return launch_status();
}

template <int D>
ra_status tc_fwd_launch(const ra_problem* p, const Layout& L, void* O, float* lse, void* ws,
                        cudaStream_t st) {
  using namespace ra::tc;
  using C = FwdCfg<D>;
  const int n = p->n, BH = p->B * p->H;
  CUtensorMap mq, mk, mv, me, mo, mell;
  // without a target the E map is a placeholder over l (never read: the kernel checks p.E)
  if (!map_bf16_3d(&mq, at<void>(ws, L.qt), D, n, BH, 128) ||
      !map_bf16_3d(&mk, at<void>(ws, L.kt), D, n, BH, 128) ||
      !map_bf16_3d(&mv, at<void>(ws, L.v), D, n, BH, 128) ||
      !map_bf16_3d(&me, p->E ? const_cast<void*>(p->E) : at<void>(ws, L.ell), D, n, BH, 128) ||
      !map_bf16_3d(&mo, O, D, n, BH, 128) || !map_bf16_3d(&mell, at<void>(ws, L.ell), D, n, BH, 128))
    return RA_ERR_CUDA;
  FwdParams fp;
  fp.E = (const __nv_bfloat16*)p->E;
  fp.O = (__nv_bfloat16*)O;
  fp.lse = lse;
  fp.ell = at<__nv_bfloat16>(ws, L.ell);
  fp.delta = at<float>(ws, L.delta);
  fp.loss_part = at<double>(ws, L.loss_part);
  // with a target the backward will follow: zero its dQ~ accumulator on the forward's idle warps
  fp.dq_zero = p->E ? at<float>(ws, L.dqt) : nullptr;
  fp.n = n;
  fp.BH = BH;
  fp.nq = (n + C::BM - 1) / C::BM;
  fp.npair = (fp.nq + 1) / 2;
  fp.causal = p->causal;
  fp.hgroup = heads_per_l2_group(4.0 * n * D, BH);  // K~ and V, bf16
  fp.scale_log2 = ra::kLog2e / sqrtf((float)D);
  fp.limit_ns = wait_limit_ns();
  auto k = attn_fwd_tc_kernel<D>;
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC);
  dim3 grid(fp.hgroup, fp.npair, (BH + fp.hgroup - 1) / fp.hgroup);
  Launch l(K_FWD_TC, st);
  k<<<grid, C::THREADS, C::SMEM_ALLOC, st>>>(mq, mk, mv, me, mo, mell, fp);
  return RA_OK;
}

ra_status tc_fwd(const ra_problem* p, void* O, float* lse, float* loss, void* ws,
                 cudaStream_t st) {
  const Layout L = make_layout(p);
  const ra::WsGate none{nullptr, 0, 0};
  rope_table(p, L, ws, st);
  ra_status s = p->d == 128 ? tc_project<128>(p, L, ws, none, false, st)
                            : tc_project<64>(p, L, ws, none, false, st);
  if (s != RA_OK) return s;
  s = p->d == 128 ? tc_fwd_launch<128>(p, L, O, lse, ws, st)
                  : tc_fwd_launch<64>(p, L, O, lse, ws, st);
  if (s != RA_OK) return s;
  finalize(p, L, ws, loss, L.nparts_fwd, none, p->E ? (ra::kWsValid | ra::kWsDqZero) : 0u, st);
  return launch_status();
}

template <int D>
ra_status tc_bwd_launch(const ra_problem* p, const Layout& L, const float* lse, void* ws,
                        cudaStream_t st) {
  using namespace ra::tc;
  using C = BwdCfg<D>;
  const int n = p->n, BH = p->B * p->H;
  CUtensorMap mq, mk, mv, ml, mdq, mtab, mdk, mdv;
  if (!map_bf16_3d(&mq, at<void>(ws, L.qt), D, n, BH, C::BQ) ||
      !map_bf16_3d(&mk, at<void>(ws, L.kt), D, n, BH, C::BK) ||
      !map_bf16_3d(&mv, at<void>(ws, L.v), D, n, BH, C::BK) ||
      !map_bf16_3d(&ml, at<void>(ws, L.ell), D, n, BH, C::BQ) ||
      !(C::PAIR ? map_f32_3d_sw128(&mdq, at<void>(ws, L.dqt), D, n, BH, C::BQ)
                : map_f32_3d(&mdq, at<void>(ws, L.dqt), D, n, BH, C::BQ)) ||
      !map_f32_rows_sw128(&mtab, at<void>(ws, L.rope), D, n, C::BK) ||
      !map_bf16_3d(&mdk, at<void>(ws, L.dk16), D, n, BH, C::BK) ||
      !map_bf16_3d(&mdv, at<void>(ws, L.dv16), D, n, BH, C::BK))
    return RA_ERR_CUDA;
  BwdParams bp;
  bp.lse = lse;
  bp.delta = at<float>(ws, L.delta);
  bp.turn = p->deterministic ? at<unsigned>(ws, L.turn) : nullptr;
  bp.turn_stride = L.turn_stride;
  bp.n = n;
  bp.BH = BH;
  bp.nk = (n + C::BK - 1) / C::BK;
  bp.causal = p->causal;
  bp.hgroup = heads_per_l2_group(8.0 * n * D, BH);  // Q~, l (bf16) and dQ~ (fp32)
  bp.scale = 1.0f / sqrtf((float)D);
  bp.scale_log2 = ra::kLog2e / sqrtf((float)D);
  bp.limit_ns = wait_limit_ns();
  auto k = attn_bwd_tc_kernel<D>;
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC);
  dim3 grid(bp.hgroup, bp.nk, (BH + bp.hgroup - 1) / bp.hgroup);
  Launch l(K_BWD_TC, st);
  k<<<grid, C::THREADS, C::SMEM_ALLOC, st>>>(mq, mk, mv, ml, mdq, mtab, mdk, mdv, bp);
  return RA_OK;
}

// fp32 I/O: CUDA-core backward.
ra_status simt_bwd(const ra_problem* p, const void* O, const float* lse, float* loss,
                   float* dWQ, float* dWK, float* dWV, void* ws, int holds, cudaStream_t st) {
  using namespace ra::simt;
  const Layout L = make_layout(p);
  const int n = p->n, d = p->d;
  const BwdGates g = bwd_gates(p, L, ws, holds);
  bwd_prep<float, float>(p, L, O, ws, g, st);
  {
    ra_status s = simt_project<float, float>(p, L, ws, g.recompute, true, st);
    if (s != RA_OK) return s;
  }
  const float scale = 1.0f / sqrtf((float)d);
  {
    size_t smem = (size_t)(4 * kRows * (d + 4) + 2 * kRows * 33 + 2 * kRows) * sizeof(float);
    cudaFuncSetAttribute(attn_bwd_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    dim3 grid((n + kRows - 1) / kRows, p->B * p->H);
    Launch l(K_BWD_SIMT, st);
    attn_bwd_kernel<float><<<grid, kThreads, smem, st>>>(
        at<float>(ws, L.qt), at<float>(ws, L.kt), at<float>(ws, L.v), at<float>(ws, L.ell), lse,
        at<float>(ws, L.delta), at<float>(ws, L.dqt), at<float>(ws, L.dkt), at<float>(ws, L.dv),
        n, d, p->causal, scale, scale * ra::kLog2e,
        p->deterministic ? at<unsigned>(ws, L.turn) : nullptr, L.turn_stride, wait_limit_ns());
  }
  {
    size_t smem = (size_t)2 * 16 * d * sizeof(float);
    dim3 grid(L.nsplit, 3, p->H);
    {
      Launch l(K_DW_PART_SIMT, st);
      dw_partial_kernel<float, float><<<grid, kThreads, smem, st>>>(
          (const float*)p->A1, (const float*)p->A2, (const float*)p->A3, at<float>(ws, L.dqt),
          at<float>(ws, L.dkt), at<float>(ws, L.dv), at<float2>(ws, L.rope),
          at<float>(ws, L.dw_part), p->B, p->H, n, d, L.chunk);
    }
    size_t total = (size_t)3 * p->H * d * d;
    Launch l(K_DW_REDUCE, st);
    // the workspace now holds this problem's intermediates and dQ~ is no longer zero: the
    // header says so, written by the last launch of the call
    dw_reduce_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(
        at<float>(ws, L.dw_part), dWQ, dWK, dWV, p->H, d, L.nsplit,
        loss ? nullptr : at<ra::WsHeader>(ws, L.hdr), problem_tag(p), ra::kWsValid,
        ra::simt::LossSum{});
  }
  if (loss) finalize(p, L, ws, loss, L.nparts_pre, g.recompute, ra::kWsValid, st);
  return launch_status();
}

// bf16 I/O: tensor-core backward.
ra_status tc_bwd(const ra_problem* p, const void* O, const float* lse, float* loss, float* dWQ,
                 float* dWK, float* dWV, void* ws, int holds, cudaStream_t st) {
  const Layout L = make_layout(p);
  const int d = p->d;
  const BwdGates g = bwd_gates(p, L, ws, holds);
  bwd_prep<__nv_bfloat16, __nv_bfloat16>(p, L, O, ws, g, st);
  ra_status s = d == 128 ? tc_project<128>(p, L, ws, g.recompute, true, st)
                         : tc_project<64>(p, L, ws, g.recompute, true, st);
  if (s != RA_OK) return s;
  s = d == 128 ? tc_bwd_launch<128>(p, L, lse, ws, st) : tc_bwd_launch<64>(p, L, lse, ws, st);
  if (s != RA_OK) return s;
  // the workspace now holds this problem's intermediates and dQ~ is no longer zero: the header
  // says so, written by the last launch of the call, which also sums the loss
  ra::WsHeader* stamp = at<ra::WsHeader>(ws, L.hdr);
  const ra::simt::LossSum ls{at<double>(ws, L.loss_part), L.nparts_pre, L.nparts_fwd, loss,
                             g.recompute};
  s = d == 128 ? tc_weight_grads<128>(p, L, dWQ, dWK, dWV, ws, stamp, ls, st)
               : tc_weight_grads<64>(p, L, dWQ, dWK, dWV, ws, stamp, ls, st);
  if (s != RA_OK) return s;
  return launch_status();
}

// One step on the tensor-core path: the forward with its loss partials, then the backward on
// the same workspace.  The backward follows the forward inside the call, so its recomputation
// launches (preparation and projection, gated on the workspace header) are not made at all,
// and the loss is summed once, by the last launch, which also writes the header.
ra_status tc_step(const ra_problem* p, void* O, float* lse, float* loss, float* dWQ, float* dWK,
                  float* dWV, void* ws, cudaStream_t st) {
  const Layout L = make_layout(p);
  const ra::WsGate none{nullptr, 0, 0};
  const int d = p->d;
  rope_table(p, L, ws, st);
  ra_status s = d == 128 ? tc_project<128>(p, L, ws, none, false, st)
                         : tc_project<64>(p, L, ws, none, false, st);
  if (s != RA_OK) return s;
  // the forward also zeroes the backward's dQ~ accumulator (p->E is given)
  s = d == 128 ? tc_fwd_launch<128>(p, L, O, lse, ws, st)
               : tc_fwd_launch<64>(p, L, O, lse, ws, st);
  if (s != RA_OK) return s;
  if (p->deterministic &&
      cudaMemsetAsync(at<void>(ws, L.turn), 0,
                      (size_t)p->B * p->H * L.turn_stride * sizeof(unsigned), st) != cudaSuccess)
    return RA_ERR_CUDA;
  s = d == 128 ? tc_bwd_launch<128>(p, L, lse, ws, st) : tc_bwd_launch<64>(p, L, lse, ws, st);
  if (s != RA_OK) return s;
  // the last launch sums the loss (the forward's partials) and writes the header
  const ra::simt::LossSum ls{at<double>(ws, L.loss_part), L.nparts_fwd, L.nparts_fwd, loss,
                             none};
  s = d == 128 ? tc_weight_grads<128>(p, L, dWQ, dWK, dWV, ws, at<ra::WsHeader>(ws, L.hdr), ls,
                                      st)
               : tc_weight_grads<64>(p, L, dWQ, dWK, dWV, ws, at<ra::WsHeader>(ws, L.hdr), ls,
                                     st);
  if (s != RA_OK) return s;
  return launch_status();
}

// ---------------------------------------------------------------------------------------
// The near-linear approximate method (degree-1 polynomial, low-rank states; fp32 on the CUDA
// cores).  Workspace: RoPE table, fp32 Q~, K~, V and dQ~, dK~, dV of every instance, the loss
// partials, the weight-gradient partials, and per-instance buffers reused instance by instance
// (row vectors and the chunk states).
// ---------------------------------------------------------------------------------------
struct ApproxLayout {
  size_t rope, qt, kt, v, dqt, dkt, dv, loss_part, dw_part;
  size_t nd, ell, dn, delta, xq, xk, invd, sq, yv, small, big;
  size_t total;
  int nch, nrb, nsplit, chunk;
};

ApproxLayout make_approx_layout(const ra_problem* p) {
  ApproxLayout L{};
  const size_t B = p->B, H = p->H, n = p->n, d = p->d;
  const size_t act = B * H * n * d;
  L.nch = (int)((n + ra::approx::kChunk - 1) / ra::approx::kChunk);
  L.nrb = (int)((n + 31) / 32);
  const long rows = (long)B * p->n;
  long ns = (4 * 148 + 3 * p->H - 1) / (3 * p->H);
  ns = ns < 1 ? 1 : ns;
  const long maxs = (rows + 63) / 64;
  if (ns > maxs) ns = maxs;
  L.nsplit = (int)ns;
  L.chunk = (int)((rows + ns - 1) / ns);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, kAlignWs);
    return o;
  };
  L.rope = take(n * (d / 2) * sizeof(float2));
  L.qt = take(act * 4);
  L.kt = take(act * 4);
  L.v = take(act * 4);
  L.dqt = take(act * 4);
  L.dkt = take(act * 4);
  L.dv = take(act * 4);
  L.loss_part = take(B * H * (size_t)L.nrb * sizeof(double));
  L.dw_part = take(3 * H * (size_t)L.nsplit * d * d * 4);
  L.nd = take(n * (d + 1) * 4);
  L.ell = take(n * d * 4);
  L.dn = take(n * 4);
  L.delta = take(n * 4);
  L.xq = take(n * (d + 1) * 4);
  L.xk = take(n * (d + 1) * 4);
  L.invd = take(n * 4);
  L.sq = take(n * 4);
  L.yv = take(n * (d + 1) * 4);
  L.small = take((size_t)L.nch * (d + 1) * (d + 1) * 4);
  L.big = take((size_t)L.nch * (d + 1) * (d + 1) * d * 4);
  L.total = off;
  return L;
}

template <int D, bool KRON, int W>
void apx_state(const float* X, const float* x, const float* xs, const float* y, float* S, int n,
               int nch, int mode, cudaStream_t st) {
  using namespace ra::approx;
  const float c4 = powf((float)D, -0.25f);
  {
    Launch l(K_APX_LOCAL, st);
    local_sum_kernel<D, KRON, W><<<dim3(nch, 1, KRON ? D + 1 : 1), kThreads, 0, st>>>(
        X, x, xs, y, S, n, c4);
  }
  const long long size = (long long)(KRON ? D + 1 : 1) * (D + 1) * W;
  Launch l(K_APX_SCAN, st);
  state_scan_kernel<<<(unsigned)((size + 255) / 256), 256, 0, st>>>(S, size, nch, mode);
}

template <int D, bool KRON, int W>
void apx_apply(const float* X, const float* x, const float* ss, const float* S, float* out, int n,
               float scale, cudaStream_t st) {
  using namespace ra::approx;
  constexpr int NU = D + 1;
  const size_t smem = (size_t)(NU * kRowBlk * (KRON ? 2 : 1) + NU * kEBlk) * 4;
  auto k = apply_kernel<D, KRON, W>;
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  Launch l(K_APX_APPLY, st);
  k<<<dim3((n + kRowBlk - 1) / kRowBlk, (W + kEBlk - 1) / kEBlk), kThreads, smem, st>>>(
      X, x, ss, S, out, n, powf((float)D, -0.25f), scale);
}

template <int D, bool FWD>
void apx_intra(const float* Qt, const float* Kt, const float* V, const float* ell, const float* dn,
               const float* delta, float* nd, float* dqt, float* dkt, float* dv, int n, int nch,
               cudaStream_t st) {
  using namespace ra::approx;
  constexpr int NT = kChunk / kIT;
  const size_t smem = (size_t)(4 * kIT * (D + 1) + 2 * kIT * (kIT + 1)) * 4;
  auto k = intra_kernel<D, FWD>;
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  Launch l(K_APX_INTRA, st);
  k<<<dim3(NT * (NT + 1) / 2, nch), kThreads, smem, st>>>(Qt, Kt, V, ell, dn, delta, nd, dqt, dkt,
                                                         dv, n, 1.0f / sqrtf((float)D));
}

template <class T, int D>
ra_status approx_step(const ra_problem* p, void* O, float* loss, float* dWQ, float* dWK,
                      float* dWV, void* ws, cudaStream_t st) {
  using namespace ra::approx;
  const ApproxLayout L = make_approx_layout(p);
  const int n = p->n, BH = p->B * p->H;
  const size_t nd_ = (size_t)n * D;
  float2* tab = at<float2>(ws, L.rope);
  {
    const long long total = (long long)n * (D / 2);
    const long long want = (total + 255) / 256, cap = 8LL * num_sms();
    Launch l(K_ROPE_TABLE, st);
    ra::simt::rope_table_kernel<<<(unsigned)(want < cap ? want : cap), 256, 0, st>>>(
        tab, p->pos, n, D / 2, rope_theta(p));
  }
  {
    using namespace ra::simt;
    size_t smem = (size_t)(kRows * (D + 4) + D * D) * sizeof(float);
    auto k = proj_rope_kernel<T, float>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    dim3 grid((n + kRows - 1) / kRows, BH, 3);
    Launch l(K_PROJ_SIMT, st);
    k<<<grid, ra::simt::kThreads, smem, st>>>(
        (const T*)p->A1, (const T*)p->A2, (const T*)p->A3, (const T*)p->WQ, (const T*)p->WK,
        (const T*)p->WV, tab, at<float>(ws, L.qt), at<float>(ws, L.kt), at<float>(ws, L.v), p->H,
        n, D, ra::WsGate{nullptr, 0, 0});
  }
  const size_t act_bytes = (size_t)BH * nd_ * 4;
  if (cudaMemsetAsync(at<float>(ws, L.dqt), 0, act_bytes, st) != cudaSuccess ||
      cudaMemsetAsync(at<float>(ws, L.dkt), 0, act_bytes, st) != cudaSuccess ||
      cudaMemsetAsync(at<float>(ws, L.dv), 0, act_bytes, st) != cudaSuccess)
    return RA_ERR_CUDA;
  const int mode_pre = p->causal ? 0 : 2, mode_suf = p->causal ? 1 : 2;
  const float isd = 1.0f / sqrtf((float)D);
  float *nd = at<float>(ws, L.nd), *ell = at<float>(ws, L.ell), *dn = at<float>(ws, L.dn),
        *delta = at<float>(ws, L.delta), *xq = at<float>(ws, L.xq), *xk = at<float>(ws, L.xk),
        *invd = at<float>(ws, L.invd), *sq = at<float>(ws, L.sq), *yv = at<float>(ws, L.yv),
        *small = at<float>(ws, L.small), *big = at<float>(ws, L.big);
  for (int bh = 0; bh < BH; ++bh) {
    const float* Q = at<float>(ws, L.qt) + bh * nd_;
    const float* K = at<float>(ws, L.kt) + bh * nd_;
    const float* V = at<float>(ws, L.v) + bh * nd_;
    float* dQ = at<float>(ws, L.dqt) + bh * nd_;
    float* dK = at<float>(ws, L.dkt) + bh * nd_;
    float* dV = at<float>(ws, L.dv) + bh * nd_;
    {
      const long long e = (long long)n * (D + 1);
      Launch l(K_APX_ROWS, st);
      ext_rows_kernel<<<(unsigned)((e + 255) / 256), 256, 0, st>>>(V, yv, n, D);
    }
    // forward: [N_i, D_i] = U_i . sum_j F_j^T [v_j, 1] (keys before the chunk) + the chunk's pairs
    apx_state<D, false, D + 1>(K, nullptr, nullptr, yv, small, n, L.nch, mode_pre, st);
    if (cudaMemsetAsync(nd, 0, (size_t)n * (D + 1) * 4, st) != cudaSuccess) return RA_ERR_CUDA;
    apx_apply<D, false, D + 1>(Q, nullptr, nullptr, small, nd, n, 1.f, st);
    if (p->causal)
      apx_intra<D, true>(Q, K, V, nullptr, nullptr, nullptr, nd, nullptr, nullptr, nullptr, n,
                         L.nch, st);
    {
      Launch l(K_APX_ROWS, st);
      finish_fwd_kernel<T><<<L.nrb, kThreads, 0, st>>>(
          nd, (const T*)p->E + bh * nd_, (T*)O + bh * nd_, ell, dn, delta, xq, xk, invd, sq,
          at<double>(ws, L.loss_part) + (size_t)bh * L.nrb, n, D, isd);
    }
    // dQ~_i = (U_i (x) [l_i, -delta_i]) . sum_j (F_j (x) [v_j, 1])^T k~_j / (sqrt(d) D_i)
    apx_state<D, true, D>(K, yv, nullptr, K, big, n, L.nch, mode_pre, st);
    apx_apply<D, true, D>(Q, xq, sq, big, dQ, n, 1.f, st);
    // dK~_j = (F_j (x) [v_j, 1]) . sum_i (U_i (x) [l_i, -delta_i] / D_i)^T q~_i / sqrt(d)
    apx_state<D, true, D>(Q, xk, nullptr, Q, big, n, L.nch, mode_suf, st);
    apx_apply<D, true, D>(K, yv, nullptr, big, dK, n, isd, st);
    // dV_j = F_j . sum_i U_i^T l_i / D_i
    apx_state<D, false, D>(Q, nullptr, invd, ell, small, n, L.nch, mode_suf, st);
    apx_apply<D, false, D>(K, nullptr, nullptr, small, dV, n, 1.f, st);
    if (p->causal)
      apx_intra<D, false>(Q, K, V, ell, dn, delta, nullptr, dQ, dK, dV, n, L.nch, st);
  }
  {
    using namespace ra::simt;
    size_t smem = (size_t)2 * 16 * D * sizeof(float);
    dim3 grid(L.nsplit, 3, p->H);
    {
      Launch l(K_DW_PART_SIMT, st);
      dw_partial_kernel<T, float><<<grid, ra::simt::kThreads, smem, st>>>(
          (const T*)p->A1, (const T*)p->A2, (const T*)p->A3, at<float>(ws, L.dqt),
          at<float>(ws, L.dkt), at<float>(ws, L.dv), tab, at<float>(ws, L.dw_part), p->B, p->H,
          n, D, L.chunk);
    }
    size_t total = (size_t)3 * p->H * D * D;
    Launch l(K_DW_REDUCE, st);
    dw_reduce_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(
        at<float>(ws, L.dw_part), dWQ, dWK, dWV, p->H, D, L.nsplit, nullptr, 0, 0u,
        ra::simt::LossSum{});
  }
  if (loss) {
    Launch l(K_LOSS, st);
    ra::simt::loss_finalize_kernel<<<1, 1024, 0, st>>>(at<double>(ws, L.loss_part), BH * L.nrb,
                                                      0, loss, ra::WsGate{nullptr, 0, 0}, nullptr,
                                                      0, 0u);
  }
  return launch_status();
}

// ---------------------------------------------------------------------------------------
// Scratch for rope_attn_step_noalloc: lives in the library's device image, so every GPU that
// loads the library holds it until exit.  Host code must not use the symbol's name as a device
// address (it names a host-side shadow); the device address comes from cudaGetSymbolAddress.
// ---------------------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[RA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_addr[kMaxDevices] = {};
unsigned long long g_noalloc_ctx[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current CUDA context, 0 if there is none or the driver
// cannot tell.  A device reset destroys the context that held the scratch array; the context
// created after it has a new id, and the array may sit at a new address there.
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_cur = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    return (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
               ? reinterpret_cast<CtxGetCurrentFn>(f)
               : (CtxGetCurrentFn) nullptr;
  }();
  static CtxGetIdFn get_id = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    return (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
               ? reinterpret_cast<CtxGetIdFn>(f)
               : (CtxGetIdFn) nullptr;
  }();
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_cur || !get_id || get_cur(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the scratch array on the current device: looked up with the device
// current on its first use, and again whenever the device's context has changed since (after a
// device reset) or cannot be identified.
ra_status noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return RA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return RA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  const unsigned long long id = current_ctx_id();
  if (!g_noalloc_addr[dev] || id == 0 || id != g_noalloc_ctx[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return RA_ERR_CUDA;
    g_noalloc_addr[dev] = ptr;
    g_noalloc_ctx[dev] = current_ctx_id();  // the lookup made the primary context current
  }
  *out = g_noalloc_addr[dev];
  return RA_OK;
}

}  // namespace

extern "C" {

size_t rope_attn_workspace_bytes(const ra_problem* p) {
  if (check_problem(p) != RA_OK) return 0;
  return make_layout(p).total;
}

ra_status rope_attn_fwd(const ra_problem* p, void* O, float* lse, float* loss, void* ws,
                        size_t ws_bytes, void* stream) {
  ra_status s = check_problem(p);
  if (s != RA_OK) return s;
  if (!O || !lse) return RA_ERR_INVALID_ARG;
  if (loss && !p->E) return RA_ERR_INVALID_ARG;
  if (!is_aligned(O, 16) || !is_aligned(lse, 4) || (loss && !is_aligned(loss, 4)))
    return RA_ERR_ALIGNMENT;
  s = check_ws(p, ws, ws_bytes);
  if (s != RA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (p->dtype == RA_F32) return simt_fwd<float>(p, O, lse, loss, ws, st);
  return tc_fwd(p, O, lse, loss, ws, st);
}

ra_status rope_attn_loss_bwd(const ra_problem* p, const void* O, const float* lse, float* loss,
                             float* dWQ, float* dWK, float* dWV, void* ws, size_t ws_bytes,
                             int32_t ws_holds_fwd, void* stream) {
  ra_status s = check_problem(p);
  if (s != RA_OK) return s;
  if (!p->E || !O || !lse || !dWQ || !dWK || !dWV) return RA_ERR_INVALID_ARG;
  if (ws_holds_fwd != 0 && ws_holds_fwd != 1) return RA_ERR_INVALID_ARG;
  if (!is_aligned(O, 16) || !is_aligned(lse, 4) || (loss && !is_aligned(loss, 4)) ||
      !is_aligned(dWQ, 16) || !is_aligned(dWK, 16) || !is_aligned(dWV, 16))
    return RA_ERR_ALIGNMENT;
  s = check_ws(p, ws, ws_bytes);
  if (s != RA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (p->dtype == RA_F32)
    return simt_bwd(p, O, lse, loss, dWQ, dWK, dWV, ws, ws_holds_fwd, st);
  return tc_bwd(p, O, lse, loss, dWQ, dWK, dWV, ws, ws_holds_fwd, st);
}

ra_status rope_attn_loss_bwd_inputs(const ra_problem* p, const void* O, const float* lse,
                                    float* loss, float* dWQ, float* dWK, float* dWV, void* dA1,
                                    void* dA2, void* dA3, void* ws, size_t ws_bytes,
                                    int32_t ws_holds_fwd, void* stream) {
  if (!p || !dA1 || !dA2 || !dA3) return RA_ERR_INVALID_ARG;
  if (!is_aligned(dA1, 16) || !is_aligned(dA2, 16) || !is_aligned(dA3, 16))
    return RA_ERR_ALIGNMENT;
  ra_status s = rope_attn_loss_bwd(p, O, lse, loss, dWQ, dWK, dWV, ws, ws_bytes, ws_holds_fwd,
                                   stream);
  if (s != RA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Layout L = make_layout(p);
  if (p->dtype == RA_F32) return simt_input_grads(p, L, dA1, dA2, dA3, ws, st);
  return p->d == 128 ? tc_input_grads<128>(p, L, dA1, dA2, dA3, ws, st)
                     : tc_input_grads<64>(p, L, dA1, dA2, dA3, ws, st);
}

ra_status rope_attn_combined_weights(const void* X, int32_t H, int32_t d, int32_t dtype,
                                     void* WQ, void* WK, void* stream) {
  if (!X || !WQ || !WK || H < 1 || (d != 64 && d != 128)) return RA_ERR_INVALID_ARG;
  if (dtype != RA_F32 && dtype != RA_BF16) return RA_ERR_INVALID_ARG;
  if (!is_aligned(X, 16) || !is_aligned(WQ, 16) || !is_aligned(WK, 16)) return RA_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long total = (long long)H * d * d;
  const unsigned blocks = (unsigned)((total + 255) / 256);
  Launch l(K_COMB_W, st);
  if (dtype == RA_F32)
    ra::simt::combined_weights_kernel<float><<<blocks, 256, 0, st>>>(
        (const float*)X, (float*)WQ, (float*)WK, total, d);
  else
    ra::simt::combined_weights_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(
        (const __nv_bfloat16*)X, (__nv_bfloat16*)WQ, (__nv_bfloat16*)WK, total, d);
  return launch_status();
}

ra_status rope_attn_combined_grad(const float* dWK, int32_t H, int32_t d, float* dX,
                                  void* stream) {
  if (!dWK || !dX || H < 1 || (d != 64 && d != 128)) return RA_ERR_INVALID_ARG;
  if (!is_aligned(dWK, 16) || !is_aligned(dX, 16)) return RA_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long total = (long long)H * d * d;
  Launch l(K_COMB_G, st);
  ra::simt::transpose_heads_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(
      dWK, dX, total, d);
  return launch_status();
}

ra_status rope_attn_step(const ra_problem* p, void* O, float* lse, float* loss, float* dWQ,
                         float* dWK, float* dWV, void* ws, size_t ws_bytes, void* stream) {
  ra_status s = check_problem(p);
  if (s != RA_OK) return s;
  if (!p->E || !O || !lse || !dWQ || !dWK || !dWV) return RA_ERR_INVALID_ARG;
  if (!is_aligned(O, 16) || !is_aligned(lse, 4) || (loss && !is_aligned(loss, 4)) ||
      !is_aligned(dWQ, 16) || !is_aligned(dWK, 16) || !is_aligned(dWV, 16))
    return RA_ERR_ALIGNMENT;
  s = check_ws(p, ws, ws_bytes);
  if (s != RA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (p->dtype == RA_F32) {
    s = simt_fwd<float>(p, O, lse, loss, ws, st);
    if (s != RA_OK) return s;
    return simt_bwd(p, O, lse, nullptr, dWQ, dWK, dWV, ws, 1, st);
  }
  return tc_step(p, O, lse, loss, dWQ, dWK, dWV, ws, st);
}

ra_status rope_attn_step_noalloc(const ra_problem* p, void* O, float* lse, float* loss,
                                 float* dWQ, float* dWK, float* dWV, void* stream) {
  ra_status s = check_problem(p);
  if (s != RA_OK) return s;
  if (!p->E || !O || !lse || !dWQ || !dWK || !dWV) return RA_ERR_INVALID_ARG;
  if (!is_aligned(O, 16) || !is_aligned(lse, 4) || (loss && !is_aligned(loss, 4)) ||
      !is_aligned(dWQ, 16) || !is_aligned(dWK, 16) || !is_aligned(dWV, 16))
    return RA_ERR_ALIGNMENT;
  const size_t need = make_layout(p).total;
  if (need > RA_NOALLOC_SCRATCH_BYTES) return RA_ERR_WORKSPACE;
  void* ws = nullptr;
  s = noalloc_scratch(&ws);
  if (s != RA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the forward writes every intermediate the backward reads; the backward zeroes its dQ~
  // accumulator itself, so no state of an earlier call leaks into this one
  if (p->dtype == RA_F32) {
    s = simt_fwd<float>(p, O, lse, loss, ws, st);
    if (s != RA_OK) return s;
    return simt_bwd(p, O, lse, loss, dWQ, dWK, dWV, ws, 1, st);
  }
  s = tc_fwd(p, O, lse, loss, ws, st);
  if (s != RA_OK) return s;
  return tc_bwd(p, O, lse, loss, dWQ, dWK, dWV, ws, 1, st);
}

size_t rope_attn_approx_workspace_bytes(const ra_problem* p) {
  if (check_problem(p) != RA_OK) return 0;
  return make_approx_layout(p).total;
}

ra_status rope_attn_approx_step(const ra_problem* p, void* O, float* loss, float* dWQ, float* dWK,
                                float* dWV, void* ws, size_t ws_bytes, void* stream) {
  ra_status s = check_problem(p);
  if (s != RA_OK) return s;
  if (!p->E || !O || !dWQ || !dWK || !dWV) return RA_ERR_INVALID_ARG;
  if (!is_aligned(O, 16) || (loss && !is_aligned(loss, 4)) || !is_aligned(dWQ, 16) ||
      !is_aligned(dWK, 16) || !is_aligned(dWV, 16))
    return RA_ERR_ALIGNMENT;
  if (!ws) return RA_ERR_WORKSPACE;
  if (!is_aligned(ws, kAlignWs)) return RA_ERR_ALIGNMENT;
  if (ws_bytes < make_approx_layout(p).total) return RA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (p->dtype == RA_F32)
    return p->d == 128 ? approx_step<float, 128>(p, O, loss, dWQ, dWK, dWV, ws, st)
                       : approx_step<float, 64>(p, O, loss, dWQ, dWK, dWV, ws, st);
  return p->d == 128 ? approx_step<__nv_bfloat16, 128>(p, O, loss, dWQ, dWK, dWV, ws, st)
                     : approx_step<__nv_bfloat16, 64>(p, O, loss, dWQ, dWK, dWV, ws, st);
}

ra_status rope_attn_last_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return RA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, ra::g_status, sizeof(int)) != cudaSuccess) return RA_ERR_CUDA;
  if (v != 0) {
    int zero = 0;
    if (cudaMemcpyToSymbol(ra::g_status, &zero, sizeof(int)) != cudaSuccess) return RA_ERR_CUDA;
    return RA_ERR_TIMEOUT;
  }
  return RA_OK;
}

const char* rope_attn_status_string(ra_status s) {
  switch (s) {
    case RA_OK: return "RA_OK";
    case RA_ERR_INVALID_ARG: return "RA_ERR_INVALID_ARG: null pointer, bad size or flag";
    case RA_ERR_UNSUPPORTED: return "RA_ERR_UNSUPPORTED: head dimension or size not supported";
    case RA_ERR_ALIGNMENT: return "RA_ERR_ALIGNMENT: device pointer not aligned";
    case RA_ERR_WORKSPACE: return "RA_ERR_WORKSPACE: workspace missing or too small";
    case RA_ERR_CUDA: return "RA_ERR_CUDA: CUDA launch or runtime call failed";
    case RA_ERR_TIMEOUT: return "RA_ERR_TIMEOUT: a kernel gave up waiting on a barrier";
  }
  return "unknown ra_status";
}

int64_t rope_attn_launch_count(void) {
  int64_t v = t_launches;
  t_launches = 0;
  return v;
}

void rope_attn_profile_enable(int32_t on) {
  t_prof.on = on != 0;
  if (!t_prof.on) t_prof.recycle();
}

void rope_attn_profile_only(int32_t kernel_id) {
  t_prof.only = (kernel_id >= 0 && kernel_id < K_COUNT) ? kernel_id : -1;
}

int32_t rope_attn_profile_read(float* ms, int32_t* launches, int32_t max_kernels) {
  for (int k = 0; k < max_kernels && k < K_COUNT; ++k) {
    if (ms) ms[k] = 0.f;
    if (launches) launches[k] = 0;
  }
  int32_t ret = K_COUNT;
  for (auto& r : t_prof.recs) {
    float t = 0.f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess ||
        cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess) {
      ret = -1;
      continue;
    }
    if (r.id < max_kernels) {
      if (ms) ms[r.id] += t;
      if (launches) launches[r.id] += 1;
    }
  }
  t_prof.recycle();
  return ret;
}

const char* rope_attn_kernel_name(int32_t id) {
  return (id >= 0 && id < K_COUNT) ? kKernelNames[id] : nullptr;
}

}  // extern "C"
