// Tensor-core projections with RoPE, and the weight-gradient contractions.
//
//   proj_rope_tc: X = A_z W_z for a 128-row tile (tcgen05, A K-major, W as an MN-major B),
//                 then RoPE on (2k, 2k+1) pairs for Q and K in the epilogue, bf16 out.
//   dq_unrotate:  dQ = rot^-1(dQ~) (fp32 accumulator in, bf16 out).
//   dw_tc:        dW_z[h] partial = sum over a range of 128-row tiles of A_z^T dX_z
//                 (both operands MN-major; fp32 partials reduced in a fixed order later).
//
// The projections and the weight gradients are the outer steps of the problem of
// "RoPE Attention kan bijna lineair worden getraind" (Probleemdefinitie: the gradient of
// the loss with respect to the weight matrices).
#pragma once
#include "tc_ptx.cuh"

namespace ra {
namespace tc {

// ---------------------------------------------------------------------------------------
// projections + RoPE
// ---------------------------------------------------------------------------------------
template <int D>
struct ProjCfg {
  static constexpr int BM = 128;
  static constexpr int KB = D / 64;
  static constexpr int NS = 4;               // A-tile stages
  static constexpr int ATILE = BM * D * 2;
  static constexpr int WTILE = D * D * 2;
  static constexpr int ABLK = BM * 128;      // [128 rows][64 cols] block
  static constexpr int WBLK = D * 128;       // [D rows][64 cols] block
  static constexpr int W_OFF = 0;
  static constexpr int A_OFF = WTILE;
  static constexpr int BAR_OFF = A_OFF + NS * ATILE;
  // w_full, a_full[NS], a_empty[NS], acc_full[2], acc_empty[2], drain
  static constexpr int NBAR = 1 + 2 * NS + 4 + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM_ALLOC = MISC_OFF + 16 + 1024;
  static constexpr int THREADS = 192;        // warps 0-3 epilogue, 4 TMA, 5 MMA
  static constexpr uint32_t T_COLS = 2 * D;  // double-buffered accumulator
};

struct ProjParams {
  const float2* tab;       // [n][d/2] (cos, sin)
  __nv_bfloat16* out[3];   // Q~, K~, V: [BH][n][d]
  int n, B, H, nrt;        // nrt = 128-row tiles per instance
  int tiles_per_cta;
  unsigned long long limit_ns;
};

// grid (chunks, H, 3): the CTA (c, h, z) projects tiles t = b * nrt + rt in
// [c * tiles_per_cta, ...) of head h with W_z[h] loaded once; z = 0 (Q, rotated),
// 1 (K, rotated), 2 (V).
template <int D>
__global__ void __launch_bounds__(ProjCfg<D>::THREADS, 1)
proj_rope_tc_kernel(const __grid_constant__ CUtensorMap tm_a1, const __grid_constant__ CUtensorMap tm_a2,
                    const __grid_constant__ CUtensorMap tm_a3, const __grid_constant__ CUtensorMap tm_w1,
                    const __grid_constant__ CUtensorMap tm_w2, const __grid_constant__ CUtensorMap tm_w3,
                    const ProjParams p) {
  using C = ProjCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  const uint32_t abort_flag = smem_u32(smem + C::MISC_OFF + 4);
  const uint32_t b_w = smem_u32(&bars[0]);
  auto b_afull = [&](int s) { return smem_u32(&bars[1 + s]); };
  auto b_aempty = [&](int s) { return smem_u32(&bars[1 + C::NS + s]); };
  auto b_accfull = [&](int b) { return smem_u32(&bars[1 + 2 * C::NS + b]); };
  auto b_accempty = [&](int b) { return smem_u32(&bars[3 + 2 * C::NS + b]); };
  const uint32_t b_drain = smem_u32(&bars[5 + 2 * C::NS]);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y, z = blockIdx.z;
  const CUtensorMap* tma = z == 0 ? &tm_a1 : z == 1 ? &tm_a2 : &tm_a3;
  const CUtensorMap* tmw = z == 0 ? &tm_w1 : z == 1 ? &tm_w2 : &tm_w3;
  const int t0 = blockIdx.x * p.tiles_per_cta;
  const int NT = min(p.tiles_per_cta, p.B * p.nrt - t0);
  const uint64_t lim = p.limit_ns;
  if (tid == 0) {
    mbar_init(b_w, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(b_afull(s), 1);
      mbar_init(b_aempty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(b_accfull(b), 1);
      mbar_init(b_accempty(b), 128);
    }
    mbar_init(b_drain, 1);
    abort_set(abort_flag, 0);
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tslot), C::T_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  if (warp == 4) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_expect_tx(b_w, C::WTILE);
      for (int b = 0; b < C::KB; ++b)
        tma_load_3d(sbase + C::W_OFF + b * C::WBLK, tmw, b_w, 64 * b, 0, h);
      int last = -1;
      for (int t = 0; t < NT; ++t) {
        const int s = t % C::NS;
        if (!mbar_wait(b_aempty(s), ((t / C::NS) & 1) ^ 1, abort_flag, lim)) break;
        const int tt = t0 + t, b = tt / p.nrt, rt = tt - b * p.nrt;
        mbar_expect_tx(b_afull(s), C::ATILE);
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_3d(sbase + C::A_OFF + s * C::ATILE + kb * C::ABLK, tma, b_afull(s), 64 * kb,
                      rt * C::BM, b * p.H + h);
        last = t;
      }
      if (abort_get(abort_flag)) {
        mbar_drain(b_w, 0, lim);
        for (int t = (last - C::NS + 1 > 0 ? last - C::NS + 1 : 0); t <= last; ++t)
          mbar_drain(b_afull(t % C::NS), (t / C::NS) & 1, lim);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, D, false, true);
      bool ok = mbar_wait(b_w, 0, abort_flag, lim);
      for (int t = 0; ok && t < NT; ++t) {
        const int s = t % C::NS, ab = t & 1;
        if (!(ok = mbar_wait(b_afull(s), (t / C::NS) & 1, abort_flag, lim))) break;
        if (!(ok = mbar_wait(b_accempty(ab), ((t >> 1) & 1) ^ 1, abort_flag, lim))) break;
        tc_fence_after();
        const uint32_t a = sbase + C::A_OFF + s * C::ATILE;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + ab * D, sw128_desc(a + (kk >> 2) * C::ABLK + (kk & 3) * 32, 16, 1024),
                 sw128_desc(sbase + C::W_OFF + kk * 2048, C::WBLK, 1024), idesc, kk > 0);
        mma_commit(b_accfull(ab));
        mma_commit(b_aempty(s));
      }
      if (!ok) {
        mma_commit(b_drain);
        mbar_drain(b_drain, 0, lim);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue (warps 0-3)
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    __nv_bfloat16* out_base = p.out[z];
    for (int t = 0; t < NT; ++t) {
      const int ab = t & 1;
      if (!mbar_wait_warp(b_accfull(ab), (t >> 1) & 1, abort_flag, lim)) break;
      tc_fence_after();
      const int tt = t0 + t, b = tt / p.nrt, rt = tt - b * p.nrt;
      const int row = rt * C::BM + tid;
      const bool vrow = row < p.n;
      uint32_t r[D];
#pragma unroll
      for (int c = 0; c < D / 32; ++c)
        tmem_ld32(tmem + lane_base + ab * D + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * c]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(b_accempty(ab));
      if (vrow) {
        __nv_bfloat16* out = out_base + ((size_t)(b * p.H + h) * p.n + row) * D;
        const float4* tr = reinterpret_cast<const float4*>(p.tab + (size_t)row * (D / 2));
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {  // 8 columns = 4 pairs = one 16-byte store
          uint32_t w[4];
#pragma unroll
          for (int k2 = 0; k2 < 2; ++k2) {
            float x0 = __uint_as_float(r[8 * c + 4 * k2]), x1 = __uint_as_float(r[8 * c + 4 * k2 + 1]);
            float x2 = __uint_as_float(r[8 * c + 4 * k2 + 2]), x3 = __uint_as_float(r[8 * c + 4 * k2 + 3]);
            if (z < 2) {
              const float4 cs = tr[2 * c + k2];  // (cos, sin) of two consecutive pairs
              const float y0 = x0 * cs.x - x1 * cs.y, y1 = x0 * cs.y + x1 * cs.x;
              const float y2 = x2 * cs.z - x3 * cs.w, y3 = x2 * cs.w + x3 * cs.z;
              x0 = y0; x1 = y1; x2 = y2; x3 = y3;
            }
            w[2 * k2] = pack_bf16x2(x0, x1);
            w[2 * k2 + 1] = pack_bf16x2(x2, x3);
          }
          reinterpret_cast<uint4*>(out)[c] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::T_COLS);
  }
}

// ---------------------------------------------------------------------------------------
// dQ = rot^-1(dQ~): fp32 in, bf16 out; one thread per pair.
// ---------------------------------------------------------------------------------------
__global__ void dq_unrotate_kernel(const float2* __restrict__ dqt, const float2* __restrict__ tab,
                                   __nv_bfloat162* __restrict__ dq, long long pairs, int n,
                                   int half) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= pairs) return;
  const long long row = idx / half;
  const int k = (int)(idx - row * half);
  const int i = (int)(row % n);
  const float2 y = dqt[idx];
  const float2 cs = tab[(size_t)i * half + k];
  dq[idx] = __floats2bfloat162_rn(y.x * cs.x + y.y * cs.y, -y.x * cs.y + y.y * cs.x);
}

// ---------------------------------------------------------------------------------------
// weight-gradient partial sums
// ---------------------------------------------------------------------------------------
template <int D>
struct DwCfg {
  static constexpr int BR = 128;             // rows per step (the contraction dimension)
  static constexpr int NS = 3;               // pipeline stages
  static constexpr int TILE = BR * D * 2;    // one operand tile
  static constexpr int BLK = BR * 128;       // [128 rows][64 cols] block
  static constexpr int STAGE = 2 * TILE;     // A tile + dX tile
  static constexpr int BAR_OFF = NS * STAGE; // full[NS], empty[NS], done, drain
  static constexpr int MISC_OFF = BAR_OFF + (2 * NS + 2) * 8;
  static constexpr int SMEM_ALLOC = MISC_OFF + 16 + 1024;
  static constexpr int THREADS = 192;        // warps 0-3 epilogue, 4 TMA, 5 MMA
  static constexpr uint32_t T_COLS = D < 64 ? 64 : D;
};

struct DwParams {
  float* part;          // [3][H][nsplit][d][d]
  int n, B, H, nt, nsplit, tiles_per_split;
  unsigned long long limit_ns;
};

// grid (nsplit, 3, H).  Tiles t = b * nt + it cover rows it*128 .. of instance (b, h).
template <int D>
__global__ void __launch_bounds__(DwCfg<D>::THREADS, 1)
dw_tc_kernel(const __grid_constant__ CUtensorMap tm_a1, const __grid_constant__ CUtensorMap tm_a2,
             const __grid_constant__ CUtensorMap tm_a3, const __grid_constant__ CUtensorMap tm_x1,
             const __grid_constant__ CUtensorMap tm_x2, const __grid_constant__ CUtensorMap tm_x3,
             const DwParams p) {
  using C = DwCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  const uint32_t abort_flag = smem_u32(smem + C::MISC_OFF + 4);
  auto b_full = [&](int s) { return smem_u32(&bars[s]); };
  auto b_empty = [&](int s) { return smem_u32(&bars[C::NS + s]); };
  const uint32_t b_done = smem_u32(&bars[2 * C::NS]);
  const uint32_t b_drain = smem_u32(&bars[2 * C::NS + 1]);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, z = blockIdx.y, h = blockIdx.z;
  const CUtensorMap* tma = z == 0 ? &tm_a1 : z == 1 ? &tm_a2 : &tm_a3;
  const CUtensorMap* tmx = z == 0 ? &tm_x1 : z == 1 ? &tm_x2 : &tm_x3;
  const int t0 = split * p.tiles_per_split;
  const int t1 = min(p.B * p.nt, t0 + p.tiles_per_split);
  const int NT = t1 - t0;
  const uint64_t lim = p.limit_ns;
  if (tid == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(b_full(s), 1);
      mbar_init(b_empty(s), 1);
    }
    mbar_init(b_done, 1);
    mbar_init(b_drain, 1);
    abort_set(abort_flag, 0);
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tslot), C::T_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  if (warp == 4) {
    if (lane == 0) {
      int last = -1;
      for (int t = 0; t < NT; ++t) {
        const int s = t % C::NS;
        if (!mbar_wait(b_empty(s), ((t / C::NS) & 1) ^ 1, abort_flag, lim)) break;
        const int tt = t0 + t, b = tt / p.nt, it = tt - b * p.nt;
        const int bhz = b * p.H + h;
        mbar_expect_tx(b_full(s), C::STAGE);
        for (int k = 0; k < D / 64; ++k) {
          tma_load_3d(sbase + s * C::STAGE + k * C::BLK, tma, b_full(s), 64 * k, it * C::BR, bhz);
          tma_load_3d(sbase + s * C::STAGE + C::TILE + k * C::BLK, tmx, b_full(s), 64 * k,
                      it * C::BR, bhz);
        }
        last = t;
      }
      if (abort_get(abort_flag))
        for (int t = (last - C::NS + 1 > 0 ? last - C::NS + 1 : 0); t <= last; ++t)
          mbar_drain(b_full(t % C::NS), (t / C::NS) & 1, lim);
    }
  } else if (warp == 5) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(D, D, true, true);
      bool ok = true;
      for (int t = 0; t < NT; ++t) {
        const int s = t % C::NS;
        if (!(ok = mbar_wait(b_full(s), (t / C::NS) & 1, abort_flag, lim))) break;
        tc_fence_after();
        const uint32_t a = sbase + s * C::STAGE, x = a + C::TILE;
#pragma unroll
        for (int kk = 0; kk < C::BR / 16; ++kk)
          mma_ss(tmem, sw128_desc(a + kk * 2048, C::BLK, 1024),
                 sw128_desc(x + kk * 2048, C::BLK, 1024), idesc, (t > 0 || kk > 0));
        mma_commit(b_empty(s));
      }
      if (ok) {
        mma_commit(b_done);
      } else {
        mma_commit(b_drain);
        mbar_drain(b_drain, 0, lim);
      }
    }
  } else {
    // epilogue: accumulator row (input feature) r of M = D sits in lane r (D = 128) or in
    // lane (r % 16) + 32 (r / 16) (D = 64)
    const bool ok = NT > 0 && mbar_wait_warp(b_done, 0, abort_flag, lim);
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const int row = (D == 128) ? (warp * 32 + lane) : (warp * 16 + lane);
    const bool has_row = (D == 128) || lane < 16;
    float* dst = p.part + (((size_t)z * p.H + h) * p.nsplit + split) * D * D + (size_t)row * D;
    if (ok) {
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + 32 * c, r);
        tmem_wait_ld();
        if (has_row) {
          float4* o = reinterpret_cast<float4*>(dst + 32 * c);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            o[v] = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                               __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
        }
      }
    } else if (NT <= 0 && has_row) {
      for (int c = 0; c < D; ++c) dst[c] = 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::T_COLS);
  }
}

}  // namespace tc
}  // namespace ra
