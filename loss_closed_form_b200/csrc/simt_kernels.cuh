// fp32 CUDA-core kernels: the precision path for fp32 I/O.  Same math as the tensor-core
// path, all products and sums in fp32; intermediate Q~, K~, V, l kept in fp32.
//
// Definitions followed ("RoPE Attention kan bijna lineair worden getraind", Methodologie 1
// and 2): s = softmax of the scaled scores, l = O - E, beta = l V^T,
// gamma = diag(s) beta - s s^T beta evaluated row-wise as s_i o (beta_i - <l_i, O_i>).
#pragma once
#include "common.cuh"

namespace ra {
namespace simt {

constexpr int kRows = 32;      // query (or key) rows per block
constexpr int kThreads = 256;  // 8 threads per row

// ---------------------------------------------------------------------------------------
// RoPE table: tab[i][k] = (cos, sin)(pos_i * base^(-2k/d)), grid-stride over the n * half
// entries; the half <= 64 frequencies come from the host.
// ---------------------------------------------------------------------------------------
constexpr int kMaxHalf = 64;

// theta_k = base^(-2k/d), k < d/2, computed on the host in double precision.
struct RopeTheta {
  double t[kMaxHalf];
};

// (cos, sin) of pos_i theta_k for every row i and pair k.  The angle (up to about 1.3e5 rad at
// n = 131072) is formed and reduced to [-pi, pi] in double precision (2 pi as a double leaves
// an error of m * 2.4e-16 rad after m turns, far below what the fp32 table resolves); the sine
// and cosine of the reduced angle are then taken in single precision (sincosf), which on that
// range is accurate to a few fp32 ulps.
__device__ __forceinline__ void rope_table_fill(float2* __restrict__ tab,
                                                const int32_t* __restrict__ pos, int n, int half,
                                                const RopeTheta& th) {
  constexpr double kTwoPi = 6.283185307179586, kInvTwoPi = 0.15915494309189535;
  const long long total = (long long)n * half;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int i = (int)(idx / half), k = (int)(idx - (long long)i * half);
    const double p = pos ? (double)pos[i] : (double)i;
    const double a = p * th.t[k];
    const double r = a - rint(a * kInvTwoPi) * kTwoPi;
    float sn, cs;
    sincosf(static_cast<float>(r), &sn, &cs);
    tab[idx] = make_float2(cs, sn);
  }
}

__global__ void rope_table_kernel(float2* __restrict__ tab, const int32_t* __restrict__ pos,
                                  int n, int half, const RopeTheta th) {
  rope_table_fill(tab, pos, n, half, th);
}

// ---------------------------------------------------------------------------------------
// Projection + RoPE: out_z = rot(A_z W_z) for z = 0 (Q), 1 (K); out_2 = A3 WV (no rotation).
// grid (ceil(n/32), B*H, 3), 256 threads, dynamic smem (32*(d+4) + d*d) floats.
// ---------------------------------------------------------------------------------------
template <class TI, class TO>
__global__ void __launch_bounds__(kThreads)
proj_rope_kernel(const TI* __restrict__ A1, const TI* __restrict__ A2, const TI* __restrict__ A3,
                 const TI* __restrict__ WQ, const TI* __restrict__ WK, const TI* __restrict__ WV,
                 const float2* __restrict__ tab, TO* __restrict__ Qt, TO* __restrict__ Kt,
                 TO* __restrict__ Vo, int H, int n, int d, WsGate gate) {
  if (gate_skip(gate)) return;
  extern __shared__ float smem[];
  const int ld = d + 4;
  float* As = smem;             // [32][d+4]
  float* Ws = smem + kRows * ld;  // [d][d]
  const int z = blockIdx.z, bh = blockIdx.y, h = bh % H;
  const int i0 = blockIdx.x * kRows;
  const TI* A = (z == 0 ? A1 : z == 1 ? A2 : A3) + ((size_t)bh * n + i0) * d;
  const TI* W = (z == 0 ? WQ : z == 1 ? WK : WV) + (size_t)h * d * d;
  TO* out = (z == 0 ? Qt : z == 1 ? Kt : Vo) + ((size_t)bh * n + i0) * d;
  const int tid = threadIdx.x;
  load_tile_f32(As, ld, A, kRows, d, min(kRows, n - i0), tid, kThreads);
  for (int e = tid; e < d * d; e += kThreads) Ws[e] = to_f(W[e]);
  __syncthreads();
  const int r = tid >> 3, g = tid & 7;
  const int row = i0 + r;
  const int half = d >> 1;
  for (int pk = g; pk < half; pk += 8) {
    float a0 = 0.f, a1 = 0.f;
    for (int i = 0; i < d; ++i) {
      float a = As[r * ld + i];
      float2 w = *reinterpret_cast<const float2*>(&Ws[i * d + 2 * pk]);
      a0 = fmaf(a, w.x, a0);
      a1 = fmaf(a, w.y, a1);
    }
    if (row < n) {
      float o0 = a0, o1 = a1;
      if (z < 2) {
        float2 cs = tab[(size_t)row * half + pk];
        o0 = a0 * cs.x - a1 * cs.y;
        o1 = a0 * cs.y + a1 * cs.x;
      }
      out[(size_t)r * d + 2 * pk] = from_f<TO>(o0);
      out[(size_t)r * d + 2 * pk + 1] = from_f<TO>(o1);
    }
  }
}

// ---------------------------------------------------------------------------------------
// Forward: online softmax over key tiles of 32, O = s V, LSE; with a target E also
// l = O - E, delta_i = <l_i, O_i> and per-block partial sums of 1/2 l^2.
// grid (ceil(n/32), B*H), 256 threads; thread (r = tid/8, g = tid%8).
// ---------------------------------------------------------------------------------------
template <class TE, class TO>
__global__ void __launch_bounds__(kThreads)
attn_fwd_kernel(const float* __restrict__ Qt, const float* __restrict__ Kt,
                const float* __restrict__ V, const TE* __restrict__ E, TO* __restrict__ O,
                float* __restrict__ lse, float* __restrict__ ell, float* __restrict__ delta,
                double* __restrict__ loss_part, int n, int d, int causal, float scale_log2) {
  extern __shared__ float smem[];
  const int ld = d + 4;
  float* Qs = smem;
  float* Ks = Qs + kRows * ld;
  float* Vs = Ks + kRows * ld;
  float* Ps = Vs + kRows * ld;  // [32][33]
  __shared__ double red[kThreads / 32];
  const int bh = blockIdx.y, i0 = blockIdx.x * kRows, tid = threadIdx.x;
  const int r = tid >> 3, g = tid & 7;
  const int row = i0 + r;
  const size_t base = (size_t)bh * n * d;
  load_tile_f32(Qs, ld, Qt + base + (size_t)i0 * d, kRows, d, min(kRows, n - i0), tid, kThreads);
  float acc[16];
  const int ncol = d >> 3;  // columns g + 8u per thread
#pragma unroll
  for (int u = 0; u < 16; ++u) acc[u] = 0.f;
  float m = -INFINITY, l = 0.f;
  const int jend = causal ? min(n, i0 + kRows) : n;
  for (int j0 = 0; j0 < jend; j0 += kRows) {
    __syncthreads();
    load_tile_f32(Ks, ld, Kt + base + (size_t)j0 * d, kRows, d, min(kRows, n - j0), tid, kThreads);
    load_tile_f32(Vs, ld, V + base + (size_t)j0 * d, kRows, d, min(kRows, n - j0), tid, kThreads);
    __syncthreads();
    float s[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) s[q] = 0.f;
    for (int c = 0; c < d; c += 4) {
      float4 qv = *reinterpret_cast<const float4*>(&Qs[r * ld + c]);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float4 kv = *reinterpret_cast<const float4*>(&Ks[(g + 8 * q) * ld + c]);
        s[q] = fmaf(qv.x, kv.x, fmaf(qv.y, kv.y, fmaf(qv.z, kv.z, fmaf(qv.w, kv.w, s[q]))));
      }
    }
    float tmax = -INFINITY;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      int key = j0 + g + 8 * q;
      bool ok = key < n && (!causal || key <= row);
      s[q] = ok ? s[q] * scale_log2 : -INFINITY;
      tmax = fmaxf(tmax, s[q]);
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
    const float mnew = fmaxf(m, tmax);
    const float mref = (mnew == -INFINITY) ? 0.f : mnew;
    const float alpha = exp2f(m - mref);
    float psum = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float p = exp2f(s[q] - mref);
      psum += p;
      Ps[r * 33 + g + 8 * q] = p;
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
    l = l * alpha + psum;
    m = mnew;
    __syncthreads();
#pragma unroll
    for (int u = 0; u < 16; ++u) acc[u] *= alpha;
    for (int k = 0; k < kRows; ++k) {
      float p = Ps[r * 33 + k];
#pragma unroll
      for (int u = 0; u < 16; ++u)
        if (u < ncol) acc[u] = fmaf(p, Vs[k * ld + g + 8 * u], acc[u]);
    }
  }
  const float inv = 1.f / l;
  const bool vrow = row < n;
  const size_t ro = base + (size_t)row * d;
  float dl = 0.f, sq = 0.f;
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    if (u < ncol && vrow) {
      const int col = g + 8 * u;
      const float o = acc[u] * inv;
      O[ro + col] = from_f<TO>(o);
      if (E) {
        const float e = o - to_f(E[ro + col]);
        ell[ro + col] = e;
        dl = fmaf(e, o, dl);
        sq = fmaf(e, e, sq);
      }
    }
  }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {
    dl += __shfl_xor_sync(0xffffffffu, dl, o);
    sq += __shfl_xor_sync(0xffffffffu, sq, o);
  }
  if (vrow && g == 0) {
    lse[(size_t)bh * n + row] = (m + log2f(l)) * kLn2;
    if (E) delta[(size_t)bh * n + row] = dl;
  }
  double part = (vrow && g == 0) ? 0.5 * (double)sq : 0.0;
  if (E) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if ((tid & 31) == 0) red[tid >> 5] = part;
    __syncthreads();
    if (tid == 0) {
      double t = 0.0;
      for (int w = 0; w < kThreads / 32; ++w) t += red[w];
      loss_part[(size_t)blockIdx.y * gridDim.x + blockIdx.x] = t;
    }
  }
}

// ---------------------------------------------------------------------------------------
// l = O - E, delta_i = <l_i, O_i>, partial sums of 1/2 l^2, from a given O (I/O dtype), for
// the 32 rows of row block rb of instance bh (256 threads, 8 per row); the block's partial sum
// goes to loss_part[bh * nrb + rb].
// ---------------------------------------------------------------------------------------
template <class T, class TL>
__device__ __forceinline__ void bwd_pre_rows(const T* __restrict__ O, const T* __restrict__ E,
                                             TL* __restrict__ ell, float* __restrict__ delta,
                                             double* __restrict__ loss_part, int n, int d,
                                             int bh, int rb, int nrb, double* red) {
  const int tid = threadIdx.x, r = tid >> 3, g = tid & 7;
  const int row = rb * kRows + r;
  float dl = 0.f, sq = 0.f;
  if (row < n) {
    const size_t ro = ((size_t)bh * n + row) * d;
    for (int col = g; col < d; col += 8) {
      float o = to_f(O[ro + col]);
      float e = o - to_f(E[ro + col]);
      const TL er = from_f<TL>(e);
      ell[ro + col] = er;
      dl = fmaf(to_f(er), o, dl);  // delta from the stored l, which beta is built from
      sq = fmaf(e, e, sq);
    }
  }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {
    dl += __shfl_xor_sync(0xffffffffu, dl, o);
    sq += __shfl_xor_sync(0xffffffffu, sq, o);
  }
  if (row < n && g == 0) delta[(size_t)bh * n + row] = dl;
  double part = (row < n && g == 0) ? 0.5 * (double)sq : 0.0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if ((tid & 31) == 0) red[tid >> 5] = part;
  __syncthreads();
  if (tid == 0) {
    double t = 0.0;
    for (int w = 0; w < kThreads / 32; ++w) t += red[w];
    loss_part[(size_t)bh * nrb + rb] = t;
  }
  __syncthreads();  // red is reused by the block's next row block
}

// The backward's preparation in one launch (grid-stride, 256 threads per block):
//   unless `recompute` is skipped: the RoPE table and, for every 32-row block of every
//     instance, l = O - E, delta and the loss partial (nrb row blocks per instance);
//   unless `zero` is skipped: the dQ~ accumulator (n4 float4) is set to zero.
// Both gates read the workspace header; when it holds this problem's intermediates and a
// zeroed accumulator, the whole launch returns at once.
template <class T, class TL>
__global__ void __launch_bounds__(kThreads)
bwd_prep_kernel(const T* __restrict__ O, const T* __restrict__ E, TL* __restrict__ ell,
                float* __restrict__ delta, double* __restrict__ loss_part, int n, int d, int BH,
                float2* __restrict__ tab, const int32_t* __restrict__ pos, const RopeTheta th,
                float4* __restrict__ dq, long long n4, WsGate recompute, WsGate zero,
                unsigned* __restrict__ turn, long long nturn) {
  __shared__ double red[kThreads / 32];
  const bool rec = !gate_skip(recompute), zer = !gate_skip(zero);
  if (rec) {
    rope_table_fill(tab, pos, n, d / 2, th);
    const int nrb = (n + kRows - 1) / kRows;
    const long long nvb = (long long)nrb * BH;
    for (long long vb = blockIdx.x; vb < nvb; vb += gridDim.x)
      bwd_pre_rows<T, TL>(O, E, ell, delta, loss_part, n, d, (int)(vb / nrb), (int)(vb % nrb),
                          nrb, red);
  }
  if (zer)
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
         i += (long long)gridDim.x * blockDim.x)
      dq[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  // the deterministic mode's turn counters (not gated: every backward starts them at zero)
  if (turn)
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < nturn;
         i += (long long)gridDim.x * blockDim.x)
      turn[i] = 0u;
}

// ---------------------------------------------------------------------------------------
// Backward over one key tile of 32 rows, looping over query tiles of 32:
//   P^T = exp(S^T - lse), beta^T = V l^T, gamma^T = P^T o (beta^T - delta)
//   dV += P^T l,  dK~ += gamma^T Q~ / sqrt(d),  dQ~ += gamma K~ / sqrt(d) (atomic adds, or
//   with `turn` in the fixed key-tile order of the deterministic mode)
// grid (ceil(n/32), B*H), 256 threads, thread (r = tid/8, g = tid%8).
// ---------------------------------------------------------------------------------------
template <class TX>
__global__ void __launch_bounds__(kThreads)
attn_bwd_kernel(const TX* __restrict__ Qt, const TX* __restrict__ Kt,
                const TX* __restrict__ V, const TX* __restrict__ ell,
                const float* __restrict__ lse, const float* __restrict__ delta,
                float* __restrict__ dQt, float* __restrict__ dKt, float* __restrict__ dV,
                int n, int d, int causal, float scale, float scale_log2, unsigned* turn,
                int turn_stride, unsigned long long limit_ns) {
  extern __shared__ float smem[];
  const int ld = d + 4;
  float* Ks = smem;
  float* Vs = Ks + kRows * ld;
  float* Qs = Vs + kRows * ld;
  float* Ls = Qs + kRows * ld;
  float* PT = Ls + kRows * ld;   // [32][33]
  float* GT = PT + kRows * 33;   // [32][33]
  float* lse_s = GT + kRows * 33;
  float* del_s = lse_s + kRows;
  // deterministic mode: key tiles in reverse order (the shortest first when causal), each
  // taking its turn on a query tile after the higher key tiles that share it
  const int kt = turn ? static_cast<int>(gridDim.x - 1 - blockIdx.x) : static_cast<int>(blockIdx.x);
  const int bh = blockIdx.y, j0 = kt * kRows, tid = threadIdx.x;
  const int r = tid >> 3, g = tid & 7;
  const int key = j0 + r;
  const size_t base = (size_t)bh * n * d;
  const int ncol = d >> 3;
  load_tile_f32(Ks, ld, Kt + base + (size_t)j0 * d, kRows, d, min(kRows, n - j0), tid, kThreads);
  load_tile_f32(Vs, ld, V + base + (size_t)j0 * d, kRows, d, min(kRows, n - j0), tid, kThreads);
  float adk[16], adv[16];
#pragma unroll
  for (int u = 0; u < 16; ++u) adk[u] = adv[u] = 0.f;
  const int istart = causal ? j0 : 0;
  for (int i0 = istart; i0 < n; i0 += kRows) {
    __syncthreads();
    const int vr = min(kRows, n - i0);
    load_tile_f32(Qs, ld, Qt + base + (size_t)i0 * d, kRows, d, vr, tid, kThreads);
    load_tile_f32(Ls, ld, ell + base + (size_t)i0 * d, kRows, d, vr, tid, kThreads);
    if (tid < kRows) {
      lse_s[tid] = (tid < vr) ? lse[(size_t)bh * n + i0 + tid] * kLog2e : 0.f;
      del_s[tid] = (tid < vr) ? delta[(size_t)bh * n + i0 + tid] : 0.f;
    }
    __syncthreads();
    float s[4], b[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) s[q] = b[q] = 0.f;
    for (int c = 0; c < d; c += 4) {
      float4 kv = *reinterpret_cast<const float4*>(&Ks[r * ld + c]);
      float4 vv = *reinterpret_cast<const float4*>(&Vs[r * ld + c]);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float4 qv = *reinterpret_cast<const float4*>(&Qs[(g + 8 * q) * ld + c]);
        float4 lv = *reinterpret_cast<const float4*>(&Ls[(g + 8 * q) * ld + c]);
        s[q] = fmaf(kv.x, qv.x, fmaf(kv.y, qv.y, fmaf(kv.z, qv.z, fmaf(kv.w, qv.w, s[q]))));
        b[q] = fmaf(vv.x, lv.x, fmaf(vv.y, lv.y, fmaf(vv.z, lv.z, fmaf(vv.w, lv.w, b[q]))));
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int qi = g + 8 * q, qrow = i0 + qi;
      const bool ok = key < n && qrow < n && (!causal || key <= qrow);
      const float p = ok ? exp2f(s[q] * scale_log2 - lse_s[qi]) : 0.f;
      PT[r * 33 + qi] = p;
      GT[r * 33 + qi] = p * (b[q] - del_s[qi]);
    }
    __syncthreads();
    for (int k = 0; k < kRows; ++k) {
      const float p = PT[r * 33 + k], gm = GT[r * 33 + k];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        if (u < ncol) {
          adv[u] = fmaf(p, Ls[k * ld + g + 8 * u], adv[u]);
          adk[u] = fmaf(gm, Qs[k * ld + g + 8 * u], adk[u]);
        }
      }
    }
    // dQ~ rows of this query tile: thread (r -> query row, g -> columns)
    const int qrow = i0 + r;
    float aq[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) aq[u] = 0.f;
    if (qrow < n) {
      for (int k = 0; k < kRows; ++k) {
        const float gm = GT[k * 33 + r];
#pragma unroll
        for (int u = 0; u < 16; ++u)
          if (u < ncol) aq[u] = fmaf(gm, Ks[k * ld + g + 8 * u], aq[u]);
      }
    }
    float* dst = dQt + base + (size_t)qrow * d;
    if (turn) {
      // deterministic mode: query tile qt gets the parts of key tiles kmax, kmax - 1, ..., 0
      // in that order (all of them contribute to it), so this one adds its part once
      // kmax - kt others have (read-modify-write through L2)
      const int qt = i0 / kRows, nkt = static_cast<int>(gridDim.x);
      const int kmax = causal ? min(nkt - 1, qt) : nkt - 1;
      unsigned* tc = turn + (size_t)bh * turn_stride + qt;
      if (tid == 0) turn_wait(tc, static_cast<unsigned>(kmax - kt), limit_ns);
      __syncthreads();
      if (qrow < n) {
#pragma unroll
        for (int u = 0; u < 16; ++u)
          if (u < ncol) __stcg(dst + g + 8 * u, __ldcg(dst + g + 8 * u) + aq[u] * scale);
      }
      __threadfence();
      __syncthreads();
      if (tid == 0) turn_pass(tc);
    } else if (qrow < n) {
#pragma unroll
      for (int u = 0; u < 16; ++u)
        if (u < ncol) atomicAdd(dst + g + 8 * u, aq[u] * scale);
    }
  }
  if (key < n) {
    const size_t ro = base + (size_t)key * d;
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      if (u < ncol) {
        dKt[ro + g + 8 * u] = adk[u] * scale;
        dV[ro + g + 8 * u] = adv[u];
      }
    }
  }
}

// ---------------------------------------------------------------------------------------
// Weight-gradient partial sums over a chunk of the B*n rows of one head:
//   part[z][h][split] = sum_rows A_z[row]^T dX_z[row], dX_0 = rot^-1(dQ~), dX_1 = rot^-1(dK~),
//   dX_2 = dV.  grid (nsplit, 3, H), 256 threads, each an (d/16) x (d/16) sub-tile.
// ---------------------------------------------------------------------------------------
template <class TA, class TX>
__global__ void __launch_bounds__(kThreads)
dw_partial_kernel(const TA* __restrict__ A1, const TA* __restrict__ A2, const TA* __restrict__ A3,
                  const TX* __restrict__ dQt, const TX* __restrict__ dKt, const TX* __restrict__ dV,
                  const float2* __restrict__ tab, float* __restrict__ part, int B, int H, int n,
                  int d, int chunk) {
  constexpr int kR = 16;
  extern __shared__ float smem[];
  float* As = smem;            // [16][d]
  float* Xs = smem + kR * d;   // [16][d]
  const int split = blockIdx.x, z = blockIdx.y, h = blockIdx.z, nsplit = gridDim.x;
  const TA* A = z == 0 ? A1 : z == 1 ? A2 : A3;
  const TX* X = z == 0 ? dQt : z == 1 ? dKt : dV;
  const int tid = threadIdx.x, sub = d >> 4;
  const int ti = (tid >> 4) * sub, tj = (tid & 15) * sub;
  float acc[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[a][c] = 0.f;
  const long total = (long)B * n;
  const long r0 = (long)split * chunk, r1 = min(total, r0 + chunk);
  const int half = d >> 1;
  for (long rb = r0; rb < r1; rb += kR) {
    __syncthreads();
    for (int e = tid; e < kR * half; e += kThreads) {
      const int rr = e / half, pk = e - rr * half;
      const long gr = rb + rr;
      float a0 = 0.f, a1 = 0.f, x0 = 0.f, x1 = 0.f;
      if (gr < r1) {
        const int b = (int)(gr / n), i = (int)(gr - (long)b * n);
        const size_t off = (((size_t)b * H + h) * n + i) * d + 2 * pk;
        a0 = to_f(A[off]);
        a1 = to_f(A[off + 1]);
        float y0 = to_f(X[off]), y1 = to_f(X[off + 1]);
        if (z < 2) {
          // inverse rotation: angle -phi
          float2 cs = tab[(size_t)i * half + pk];
          x0 = y0 * cs.x + y1 * cs.y;
          x1 = -y0 * cs.y + y1 * cs.x;
        } else {
          x0 = y0;
          x1 = y1;
        }
      }
      As[rr * d + 2 * pk] = a0;
      As[rr * d + 2 * pk + 1] = a1;
      Xs[rr * d + 2 * pk] = x0;
      Xs[rr * d + 2 * pk + 1] = x1;
    }
    __syncthreads();
    for (int k = 0; k < kR; ++k) {
      float av[8], xv[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        av[a] = a < sub ? As[k * d + ti + a] : 0.f;
        xv[a] = a < sub ? Xs[k * d + tj + a] : 0.f;
      }
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[a][c] = fmaf(av[a], xv[c], acc[a][c]);
    }
  }
  float* dst = part + (((size_t)z * H + h) * nsplit + split) * d * d;
  for (int a = 0; a < sub; ++a)
    for (int c = 0; c < sub; ++c) dst[(size_t)(ti + a) * d + tj + c] = acc[a][c];
}

// Sum of the loss partials part[0 .. count) in a fixed order that does not depend on the block
// size: 1024 virtual lanes, lane v adding partials v, v + 1024, ... in four interleaved chains,
// then a pairwise tree over the lanes.  One block of blockDim.x threads (a divisor of 1024)
// computes it; red holds 1024 doubles of shared memory.  The result is red[0].
__device__ __forceinline__ void loss_sum_fixed(const double* __restrict__ part, int count,
                                               double* red) {
  constexpr int V = 1024;
  for (int v = threadIdx.x; v < V; v += blockDim.x) {
    double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
    int i = v;
    for (; i + 3 * V < count; i += 4 * V) {
      s0 += part[i];
      s1 += part[i + V];
      s2 += part[i + 2 * V];
      s3 += part[i + 3 * V];
    }
    for (; i < count; i += V) s0 += part[i];
    red[v] = (s0 + s1) + (s2 + s3);
  }
  __syncthreads();
  for (int w = V / 2; w > 0; w >>= 1) {
    for (int v = threadIdx.x; v < w; v += blockDim.x) red[v] += red[v + w];
    __syncthreads();
  }
}

// The loss of a call, summed by the last launch that needs it.  `count` partials belong to
// this call; when `gate` finds the backward's recomputation skipped, the forward's `count_kept`
// ones are summed.
struct LossSum {
  const double* part;
  int count, count_kept;
  float* loss;  // null: no loss to sum
  WsGate gate;
};

// dW_z[h] = sum over the nsplit row-range partials in a fixed order (fp64), one thread per
// output element.  With a loss to sum, one more block (block 0, so that it runs beside the
// others rather than after them) sums it and writes the workspace header; otherwise thread 0
// writes the header (stamp non-null).
__global__ void dw_reduce_kernel(const float* __restrict__ part, float* __restrict__ dWQ,
                                 float* __restrict__ dWK, float* __restrict__ dWV, int H, int d,
                                 int nsplit, WsHeader* stamp, unsigned long long stamp_tag,
                                 unsigned int stamp_state, LossSum ls) {
  if (ls.loss && blockIdx.x == 0) {
    __shared__ double red[1024];
    const int count = gate_skip(ls.gate) ? ls.count_kept : ls.count;
    __syncthreads();  // every thread has read the header before thread 0 rewrites it
    if (stamp && threadIdx.x == 0) {
      stamp->tag = stamp_tag;
      stamp->state = stamp_state;
      stamp->magic = kWsMagic;
    }
    loss_sum_fixed(ls.part, count, red);
    if (threadIdx.x == 0) *ls.loss = (float)red[0];
    return;
  }
  const size_t dd = (size_t)d * d;
  const size_t idx = (size_t)(blockIdx.x - (ls.loss ? 1 : 0)) * blockDim.x + threadIdx.x;
  if (stamp && !ls.loss && idx == 0) {
    stamp->tag = stamp_tag;
    stamp->state = stamp_state;
    stamp->magic = kWsMagic;
  }
  if (idx >= 3 * H * dd) return;
  const int z = (int)(idx / (H * dd));
  const size_t rem = idx - (size_t)z * H * dd;
  const int h = (int)(rem / dd);
  const size_t e = rem - (size_t)h * dd;
  const float* src = part + ((size_t)z * H + h) * nsplit * dd + e;
  double s = 0.0;
  for (int k = 0; k < nsplit; ++k) s += (double)src[(size_t)k * dd];
  float* dW = z == 0 ? dWQ : z == 1 ? dWK : dWV;
  dW[(size_t)h * dd + e] = (float)s;
}

// Last kernel of a forward or backward call (one block): loss = sum of the partials in a
// fixed order (fp64), when `loss` is given, then the workspace header is stamped with
// (stamp_tag, stamp_state).  The partials are the `count_kept` ones an earlier forward left
// when `gate` skipped the backward's recomputation, else the `count` ones of this call.
__global__ void loss_finalize_kernel(const double* __restrict__ part, int count, int count_kept,
                                     float* __restrict__ loss, WsGate gate, WsHeader* stamp,
                                     unsigned long long stamp_tag, unsigned int stamp_state) {
  // fixed summation order for a given count, whatever the block size (deterministic, and the
  // same as the loss block of dw_reduce_kernel)
  __shared__ double red[1024];
  if (gate_skip(gate)) count = count_kept;
  __syncthreads();  // every thread has read the header before thread 0 rewrites it
  if (stamp && threadIdx.x == 0) {
    stamp->tag = stamp_tag;
    stamp->state = stamp_state;
    stamp->magic = kWsMagic;
  }
  if (!loss) return;
  loss_sum_fixed(part, count, red);
  if (threadIdx.x == 0) *loss = (float)red[0];
}

// ---------------------------------------------------------------------------------------
// Input gradients (fp32 I/O): dA_z[b, h, i, :] = rot^-1(dX~_z[b, h, i, :]) W_z[h]^T, with
// z = 0 (dQ~, rotated), 1 (dK~, rotated), 2 (dV).  grid (row blocks, B * H, 3); W_z[h] is
// transposed into shared memory so the 16 threads of a row read consecutive words.
// ---------------------------------------------------------------------------------------
constexpr int kDaRows = 16;

__global__ void __launch_bounds__(kThreads)
input_grad_kernel(const float* __restrict__ dQt, const float* __restrict__ dKt,
                  const float* __restrict__ dV, const float2* __restrict__ tab,
                  const float* __restrict__ WQ, const float* __restrict__ WK,
                  const float* __restrict__ WV, float* __restrict__ dA1, float* __restrict__ dA2,
                  float* __restrict__ dA3, int H, int n, int d) {
  extern __shared__ float smem[];
  float* Wt = smem;          // [d][d]: Wt[o][a] = W[a][o]
  float* Xs = smem + d * d;  // [kDaRows][d]: un-rotated rows of dX
  const int z = blockIdx.z, bh = blockIdx.y, h = bh % H;
  const int r0 = blockIdx.x * kDaRows;
  const float* X = z == 0 ? dQt : z == 1 ? dKt : dV;
  const float* W = (z == 0 ? WQ : z == 1 ? WK : WV) + (size_t)h * d * d;
  float* dA = z == 0 ? dA1 : z == 1 ? dA2 : dA3;
  for (int e = threadIdx.x; e < d * d; e += blockDim.x) {
    const int a = e / d, o = e - a * d;
    Wt[o * d + a] = W[e];
  }
  const int half = d / 2;
  for (int e = threadIdx.x; e < kDaRows * half; e += blockDim.x) {
    const int rr = e / half, k = e - rr * half, i = r0 + rr;
    float x0 = 0.f, x1 = 0.f;
    if (i < n) {
      const size_t off = ((size_t)bh * n + i) * d + 2 * k;
      const float y0 = X[off], y1 = X[off + 1];
      if (z < 2) {
        const float2 cs = tab[(size_t)i * half + k];  // rotation by -phi
        x0 = y0 * cs.x + y1 * cs.y;
        x1 = -y0 * cs.y + y1 * cs.x;
      } else {
        x0 = y0;
        x1 = y1;
      }
    }
    Xs[rr * d + 2 * k] = x0;
    Xs[rr * d + 2 * k + 1] = x1;
  }
  __syncthreads();
  const int rr = threadIdx.x / 16, a0 = threadIdx.x % 16, i = r0 + rr;
  if (i >= n) return;
  for (int a = a0; a < d; a += 16) {
    float acc = 0.f;
    for (int o = 0; o < d; ++o) acc = fmaf(Xs[rr * d + o], Wt[o * d + a], acc);
    dA[((size_t)bh * n + i) * d + a] = acc;
  }
}

// ---------------------------------------------------------------------------------------
// One combined weight X per head: WQ = I and WK = X^T make the general problem's scores
// q~_i . k~_j = a1_i^T R_{j-i} X a2_j; its dWK is then dX^T.
// ---------------------------------------------------------------------------------------
template <class T>
__global__ void combined_weights_kernel(const T* __restrict__ X, T* __restrict__ WQ,
                                        T* __restrict__ WK, long long total, int d) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const long long hd = idx / ((long long)d * d);
  const int rc = (int)(idx - hd * d * d), r = rc / d, c = rc - r * d;
  WQ[idx] = from_f<T>(r == c ? 1.f : 0.f);
  WK[idx] = X[hd * d * d + (long long)c * d + r];
}

__global__ void transpose_heads_kernel(const float* __restrict__ in, float* __restrict__ out,
                                       long long total, int d) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const long long hd = idx / ((long long)d * d);
  const int rc = (int)(idx - hd * d * d), r = rc / d, c = rc - r * d;
  out[idx] = in[hd * d * d + (long long)c * d + r];
}

}  // namespace simt
}  // namespace ra
