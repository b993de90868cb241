// The near-linear approximate method ("RoPE Attention kan bijna lineair worden getraind",
// Methodologie 2 "Low-Rank Benaderingsstrategie" and Resultaten, Theorem 5.7) with the degree-1
// polynomial: on bounded scores exp(z) is replaced by 1 + z, which factors as
//   1 + q~_i . k~_j / sqrt(d) = U_i . F_j,   U_i = (1, d^-1/4 q~_i),  F_j = (1, d^-1/4 k~_j)
// (R = d + 1 features).  s~ = U F^T normalised per row stands for s (the low-rank U1 V1^T),
// l = s~ V - E, beta = l V^T, and gamma = s~ o (beta - delta) is never formed: every product with
// it is a contraction with low-rank states built once per chunk of rows,
//   gamma_1 (the s~ o beta part) through row-wise Kronecker products (U_i (x) [l_i, -delta_i]),
//   gamma_2 (the s~ delta part) through the precomputed delta_i = <l_i, O_i>,
// so the work is linear in n (states of (d + 1)^2 d floats per chunk) instead of quadratic.
// With a causal mask the states are exclusive prefix sums (keys before the chunk) or suffix sums
// (queries after it), and the pairs inside a chunk are evaluated directly.
//
// All arithmetic fp32 on the CUDA cores.  Rows are [n][d] fp32 of one (b, h) instance.
#pragma once
#include "common.cuh"

namespace ra {
namespace approx {

constexpr int kChunk = 256;   // rows per state chunk
constexpr int kThreads = 256;
constexpr int kTile = 32;     // rows staged per step in the local-sum kernel
constexpr int kRowBlk = 64;   // rows per apply CTA (8 per warp)
constexpr int kEBlk = 64;     // output columns per apply CTA (2 per lane)

// feature a (0 .. d) of the row x: 1 for a = 0, c4 * x[a - 1] otherwise (c4 = d^-1/4)
__device__ __forceinline__ float feat(const float* __restrict__ x, int a, float c4) {
  return a == 0 ? 1.f : c4 * x[a - 1];
}

// ---------------------------------------------------------------------------------------
// Local sums of one chunk of rows r (nr rows from r0):
//   KRON:  S[a][b][e] = sum_r f_ra x_rb y_re   (a = blockIdx.z, b in [0, D], e in [0, W))
//   !KRON: S[a][e]    = sum_r f_ra xs_r y_re    (a in [0, D], x a per-row scalar or 1)
// f_ra = feat(X[r], a).  Output for chunk ch at S + ch * state_size.
// grid (nch, 1, KRON ? D + 1 : 1), 256 threads as 16 (u) x 16 (e).
// ---------------------------------------------------------------------------------------
template <int D, bool KRON, int W>
__global__ void __launch_bounds__(kThreads)
local_sum_kernel(const float* __restrict__ X, const float* __restrict__ x, const float* __restrict__ xs,
                 const float* __restrict__ y, float* __restrict__ S, int n, float c4) {
  constexpr int NU = D + 1;
  constexpr int KU = (NU + 15) / 16, KE = (W + 15) / 16;
  constexpr int LDU = NU + 1, LDY = W + 1;
  __shared__ float cs[kTile * LDU];   // c_r(u) = f_ra x_ru (KRON) or f_ru xs_r
  __shared__ float ys[kTile * LDY];
  const int ch = blockIdx.x, a = blockIdx.z, tid = threadIdx.x;
  const int tu = tid >> 4, te = tid & 15;
  const int r0 = ch * kChunk, r1 = min(n, r0 + kChunk);
  float acc[KU][KE];
#pragma unroll
  for (int k = 0; k < KU; ++k)
#pragma unroll
    for (int m = 0; m < KE; ++m) acc[k][m] = 0.f;
  for (int rb = r0; rb < r1; rb += kTile) {
    const int nr = min(kTile, r1 - rb);
    __syncthreads();
    for (int e = tid; e < kTile * NU; e += kThreads) {
      const int rr = e / NU, u = e - rr * NU;
      float c = 0.f;
      if (rr < nr) {
        const int r = rb + rr;
        if (KRON) c = feat(X + (size_t)r * D, a, c4) * x[(size_t)r * NU + u];
        else c = feat(X + (size_t)r * D, u, c4) * (xs ? xs[r] : 1.f);
      }
      cs[rr * LDU + u] = c;
    }
    for (int e = tid; e < kTile * W; e += kThreads) {
      const int rr = e / W, c = e - rr * W;
      ys[rr * LDY + c] = rr < nr ? y[(size_t)(rb + rr) * W + c] : 0.f;
    }
    __syncthreads();
    for (int rr = 0; rr < nr; ++rr) {
      float cu[KU], ye[KE];
#pragma unroll
      for (int k = 0; k < KU; ++k) {
        const int u = tu + 16 * k;
        cu[k] = u < NU ? cs[rr * LDU + u] : 0.f;
      }
#pragma unroll
      for (int m = 0; m < KE; ++m) {
        const int e = te + 16 * m;
        ye[m] = e < W ? ys[rr * LDY + e] : 0.f;
      }
#pragma unroll
      for (int k = 0; k < KU; ++k)
#pragma unroll
        for (int m = 0; m < KE; ++m) acc[k][m] = fmaf(cu[k], ye[m], acc[k][m]);
    }
  }
  const size_t state = (size_t)(KRON ? NU : 1) * NU * W;
  float* out = S + ch * state + (KRON ? (size_t)a * NU * W : 0);
#pragma unroll
  for (int k = 0; k < KU; ++k)
#pragma unroll
    for (int m = 0; m < KE; ++m) {
      const int u = tu + 16 * k, e = te + 16 * m;
      if (u < NU && e < W) out[(size_t)u * W + e] = acc[k][m];
    }
}

// ---------------------------------------------------------------------------------------
// Scan of the per-chunk states along the chunks, in place, for every element:
//   mode 0: exclusive prefix (chunk ch gets the sum over chunks < ch)
//   mode 1: exclusive suffix (chunk ch gets the sum over chunks > ch)
//   mode 2: total (every chunk gets the sum over all chunks: no mask)
// ---------------------------------------------------------------------------------------
__global__ void state_scan_kernel(float* __restrict__ S, long long size, int nch, int mode) {
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= size) return;
  constexpr int U = 8;  // chunks loaded before any is written: eight loads in flight per thread
  float run = 0.f;
  if (mode == 2) {
    for (int c0 = 0; c0 < nch; c0 += U) {
      float v[U];
#pragma unroll
      for (int k = 0; k < U; ++k) v[k] = c0 + k < nch ? S[(size_t)(c0 + k) * size + e] : 0.f;
#pragma unroll
      for (int k = 0; k < U; ++k) run += v[k];
    }
    for (int c = 0; c < nch; ++c) S[(size_t)c * size + e] = run;
    return;
  }
  for (int k0 = 0; k0 < nch; k0 += U) {
    float v[U];
#pragma unroll
    for (int k = 0; k < U; ++k) {
      const int c = mode == 0 ? k0 + k : nch - 1 - (k0 + k);
      v[k] = k0 + k < nch ? S[(size_t)c * size + e] : 0.f;
    }
#pragma unroll
    for (int k = 0; k < U; ++k) {
      if (k0 + k >= nch) break;
      const int c = mode == 0 ? k0 + k : nch - 1 - (k0 + k);
      S[(size_t)c * size + e] = run;
      run += v[k];
    }
  }
}

// ---------------------------------------------------------------------------------------
// Apply the states to rows r (of the chunk each row lies in):
//   KRON:  out[r][e] += scale s_r sum_a f'_ra sum_b x'_rb S[a][b][e]
//   !KRON: out[r][e] += scale s_r sum_a f'_ra S[a][e]
// f'_ra = feat(X[r], a); s_r = ss[r] (or 1).  grid (ceil(n / 64), ceil(W / 64)), 256 threads:
// warp w takes rows 8 w .. 8 w + 7 of the block, its lane two output columns; the rows'
// coefficients are stored transposed so that each step over u reads them with two broadcast
// 16-byte loads and the state with one 8-byte load per lane (16 FMAs per three loads).
// ---------------------------------------------------------------------------------------
template <int D, bool KRON, int W>
__global__ void __launch_bounds__(kThreads)
apply_kernel(const float* __restrict__ X, const float* __restrict__ x, const float* __restrict__ ss,
             const float* __restrict__ S, float* __restrict__ out, int n, float c4, float scale) {
  constexpr int NU = D + 1;
  extern __shared__ __align__(16) float sm[];
  // [NU][64] per-row coefficients, transposed so that the 8 rows a warp handles are adjacent:
  // fT[a][r] = f'_ra (the features), xT[b][r] = x'_rb (KRON)
  float* fT = sm;
  float* xT = fT + NU * kRowBlk;
  float* St = xT + (KRON ? NU * kRowBlk : 0);   // [NU][64]: S[a][u][e0 ..] (KRON) or S[u][e0 ..]
  const int r0 = blockIdx.x * kRowBlk, e0 = blockIdx.y * kEBlk, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int nr = min(kRowBlk, n - r0);
  const int ch = r0 / kChunk;   // 64 divides kChunk: the block lies in one chunk
  const size_t state = (size_t)(KRON ? NU : 1) * NU * W;
  const float* Sc = S + ch * state;
  for (int e = tid; e < NU * kRowBlk; e += kThreads) {
    const int a = e / kRowBlk, rr = e - a * kRowBlk;
    fT[e] = rr < nr ? feat(X + (size_t)(r0 + rr) * D, a, c4) : 0.f;
    if (KRON) xT[e] = rr < nr ? x[(size_t)(r0 + rr) * NU + a] : 0.f;
  }
  // warp w: rows 8 w .. 8 w + 7; lane: output columns e0 + 2 lane, e0 + 2 lane + 1
  const int rb = 8 * warp;
  float acc[8][2];
#pragma unroll
  for (int k = 0; k < 8; ++k) acc[k][0] = acc[k][1] = 0.f;
  for (int a = 0; a < (KRON ? NU : 1); ++a) {
    __syncthreads();
    const float* src = Sc + (KRON ? (size_t)a * NU * W : 0);
    for (int e = tid; e < NU * kEBlk; e += kThreads) {
      const int u = e / kEBlk, c = e - u * kEBlk;
      St[e] = (e0 + c < W) ? src[(size_t)u * W + e0 + c] : 0.f;
    }
    __syncthreads();
    float dot[8][2];
#pragma unroll
    for (int k = 0; k < 8; ++k) dot[k][0] = dot[k][1] = 0.f;
    const float* cu = KRON ? xT : fT;   // KRON: sum over b of x'_rb S[a][b][e]; else over a
    for (int u = 0; u < NU; ++u) {
      const float4 c0 = *reinterpret_cast<const float4*>(cu + u * kRowBlk + rb);
      const float4 c1 = *reinterpret_cast<const float4*>(cu + u * kRowBlk + rb + 4);
      const float2 sv = *reinterpret_cast<const float2*>(St + u * kEBlk + 2 * lane);
      const float cr[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        dot[k][0] = fmaf(cr[k], sv.x, dot[k][0]);
        dot[k][1] = fmaf(cr[k], sv.y, dot[k][1]);
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float fa = KRON ? fT[a * kRowBlk + rb + k] : 1.f;
      acc[k][0] = fmaf(fa, dot[k][0], acc[k][0]);
      acc[k][1] = fmaf(fa, dot[k][1], acc[k][1]);
    }
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int rr = rb + k;
    if (rr >= nr) continue;
    const int r = r0 + rr;
    const float sr = scale * (ss ? ss[r] : 1.f);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int ecol = e0 + 2 * lane + q;
      if (ecol < W) out[(size_t)r * W + ecol] += sr * acc[k][q];
    }
  }
}

// ---------------------------------------------------------------------------------------
// Pairs inside a chunk (causal only), directly, over 64 x 64 tile pairs (query tile ti >= key
// tile tj of the same chunk; j <= i inside the diagonal tile pair):
//   a_ij = 1 + q~_i . k~_j / sqrt(d)
//   forward  (FWD):  nd[i] += sum_j a_ij [v_j, 1]                          (nd: [n][D + 1])
//   backward (!FWD): with g_ij = (a_ij / D_i) (l_i . v_j - delta_i)
//     dQ~_i += sum_j g_ij k~_j / sqrt(d),  dK~_j += sum_i g_ij q~_i / sqrt(d),
//     dV_j += sum_i (a_ij / D_i) l_i
// Several tile pairs add into the same rows: atomic adds.  grid (pairs per chunk, nch).
// ---------------------------------------------------------------------------------------
constexpr int kIT = 64;

template <int D, bool FWD>
__global__ void __launch_bounds__(kThreads)
intra_kernel(const float* __restrict__ Qt, const float* __restrict__ Kt, const float* __restrict__ V,
             const float* __restrict__ ell, const float* __restrict__ Dn,
             const float* __restrict__ delta, float* __restrict__ nd, float* __restrict__ dQt,
             float* __restrict__ dKt, float* __restrict__ dV, int n, float inv_sqrt_d) {
  constexpr int LD = D + 1, LDA = kIT + 1;
  extern __shared__ float sm[];
  float* Qs = sm;                    // [64][D + 1] q~_i
  float* Ls = Qs + kIT * LD;         // [64][D + 1] l_i (backward)
  float* Ks = Ls + kIT * LD;         // [64][D + 1] k~_j
  float* Vs = Ks + kIT * LD;         // [64][D + 1] v_j
  float* Am = Vs + kIT * LD;         // [64][65] a_ij, then g_ij
  float* Pm = Am + kIT * LDA;        // [64][65] a_ij / D_i (backward)
  // tile pair p of the chunk: ti >= tj, enumerated row by row
  constexpr int NT = kChunk / kIT;
  int p = blockIdx.x, ti = 0;
  while (p > ti) {
    p -= ti + 1;
    ++ti;
  }
  const int tj = p;
  const int c0 = blockIdx.y * kChunk;
  const int i0 = c0 + ti * kIT, j0 = c0 + tj * kIT;
  if (i0 >= n || ti >= NT) return;
  const int ni = min(kIT, n - i0), nj = min(kIT, n - j0);
  const int tid = threadIdx.x;
  for (int e = tid; e < kIT * D; e += kThreads) {
    const int rr = e / D, c = e - rr * D;
    Qs[rr * LD + c] = rr < ni ? Qt[(size_t)(i0 + rr) * D + c] : 0.f;
    Ks[rr * LD + c] = rr < nj ? Kt[(size_t)(j0 + rr) * D + c] : 0.f;
    Vs[rr * LD + c] = rr < nj ? V[(size_t)(j0 + rr) * D + c] : 0.f;
    if (!FWD) Ls[rr * LD + c] = rr < ni ? ell[(size_t)(i0 + rr) * D + c] : 0.f;
  }
  __syncthreads();
  // a_ij (and for the backward g_ij, a_ij / D_i), 16 pairs per thread
  for (int e = tid; e < kIT * kIT; e += kThreads) {
    const int ii = e / kIT, jj = e - ii * kIT;
    const bool valid = ii < ni && jj < nj && (ti != tj || jj <= ii);
    float aij = 0.f, gij = 0.f, pij = 0.f;
    if (valid) {
      float qk = 0.f, lv = 0.f;
      for (int c = 0; c < D; ++c) {
        qk = fmaf(Qs[ii * LD + c], Ks[jj * LD + c], qk);
        if (!FWD) lv = fmaf(Ls[ii * LD + c], Vs[jj * LD + c], lv);
      }
      aij = 1.f + qk * inv_sqrt_d;
      if (!FWD) {
        const float invd = 1.f / Dn[i0 + ii];
        pij = aij * invd;
        gij = pij * (lv - delta[i0 + ii]);
      }
    }
    Am[ii * LDA + jj] = FWD ? aij : gij;
    if (!FWD) Pm[ii * LDA + jj] = pij;
  }
  __syncthreads();
  if constexpr (FWD) {
    // nd[i][c] += sum_j a_ij v_j[c] (c < D), nd[i][D] += sum_j a_ij
    for (int e = tid; e < kIT * (D + 1); e += kThreads) {
      const int ii = e / (D + 1), c = e - ii * (D + 1);
      if (ii >= ni) continue;
      float s = 0.f;
      for (int jj = 0; jj < nj; ++jj) s = fmaf(Am[ii * LDA + jj], c < D ? Vs[jj * LD + c] : 1.f, s);
      atomicAdd(nd + (size_t)(i0 + ii) * (D + 1) + c, s);
    }
  } else {
  for (int e = tid; e < kIT * D; e += kThreads) {
    const int rr = e / D, c = e - rr * D;
    if (rr < ni) {  // dQ~_i
      float s = 0.f;
      for (int jj = 0; jj < nj; ++jj) s = fmaf(Am[rr * LDA + jj], Ks[jj * LD + c], s);
      atomicAdd(dQt + (size_t)(i0 + rr) * D + c, s * inv_sqrt_d);
    }
    if (rr < nj) {  // dK~_j and dV_j
      float sk = 0.f, sv = 0.f;
      for (int ii = 0; ii < ni; ++ii) {
        sk = fmaf(Am[ii * LDA + rr], Qs[ii * LD + c], sk);
        sv = fmaf(Pm[ii * LDA + rr], Ls[ii * LD + c], sv);
      }
      atomicAdd(dKt + (size_t)(j0 + rr) * D + c, sk * inv_sqrt_d);
      atomicAdd(dV + (size_t)(j0 + rr) * D + c, sv);
    }
  }
  }
}

// ---------------------------------------------------------------------------------------
// Row-wise helpers
// ---------------------------------------------------------------------------------------
// yv[r] = [v_r, 1]
__global__ void ext_rows_kernel(const float* __restrict__ V, float* __restrict__ yv, int n, int d) {
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (long long)n * (d + 1)) return;
  const long long r = e / (d + 1);
  const int c = (int)(e - r * (d + 1));
  yv[e] = c < d ? V[r * d + c] : 1.f;
}

// From nd = [N_i, D_i]: O_i = N_i / D_i (I/O dtype out), l_i = O_i - E_i, delta_i = <l_i, O_i>,
// the loss partial of the row block, and the row vectors the backward contracts with:
//   xq_i = [l_i, -delta_i],  xk_i = xq_i / D_i,  invD_i = 1 / D_i,  sq_i = 1 / (sqrt(d) D_i).
// grid (ceil(n / 32)), 256 threads (8 per row).
template <class T>
__global__ void __launch_bounds__(kThreads)
finish_fwd_kernel(const float* __restrict__ nd, const T* __restrict__ E, T* __restrict__ O,
                  float* __restrict__ ell, float* __restrict__ Dn, float* __restrict__ delta,
                  float* __restrict__ xq, float* __restrict__ xk, float* __restrict__ invD,
                  float* __restrict__ sq, double* __restrict__ loss_part, int n, int d,
                  float inv_sqrt_d) {
  __shared__ double red[kThreads / 32];
  const int tid = threadIdx.x, r = tid >> 3, g = tid & 7;
  const int row = blockIdx.x * 32 + r;
  float dl = 0.f, s2 = 0.f, Dv = 1.f;
  if (row < n) {
    Dv = nd[(size_t)row * (d + 1) + d];
    const float inv = 1.f / Dv;
    for (int c = g; c < d; c += 8) {
      const float o = nd[(size_t)row * (d + 1) + c] * inv;
      O[(size_t)row * d + c] = from_f<T>(o);
      const float e = o - to_f(E[(size_t)row * d + c]);
      ell[(size_t)row * d + c] = e;
      xq[(size_t)row * (d + 1) + c] = e;
      xk[(size_t)row * (d + 1) + c] = e * inv;
      dl = fmaf(e, o, dl);
      s2 = fmaf(e, e, s2);
    }
  }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {
    dl += __shfl_xor_sync(0xffffffffu, dl, o);
    s2 += __shfl_xor_sync(0xffffffffu, s2, o);
  }
  if (row < n && g == 0) {
    Dn[row] = Dv;
    delta[row] = dl;
    xq[(size_t)row * (d + 1) + d] = -dl;
    xk[(size_t)row * (d + 1) + d] = -dl / Dv;
    invD[row] = 1.f / Dv;
    sq[row] = inv_sqrt_d / Dv;
  }
  double part = (row < n && g == 0) ? 0.5 * (double)s2 : 0.0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if ((tid & 31) == 0) red[tid >> 5] = part;
  __syncthreads();
  if (tid == 0) {
    double t = 0.0;
    for (int w = 0; w < kThreads / 32; ++w) t += red[w];
    loss_part[blockIdx.x] = t;
  }
}

}  // namespace approx
}  // namespace ra
