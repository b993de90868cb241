// Tensor-core projections with RoPE, and the weight-gradient contractions.
//
//   proj_rope_tc: X = A_z W_z for a 128-row tile (tcgen05, A K-major, W as an MN-major B),
//                 then RoPE on (2k, 2k+1) pairs for Q and K in the epilogue, bf16 out.
//   dq_unrotate:  dQ = rot^-1(acc) / sqrt(d) (fp32 accumulator of gamma K~ in, bf16 out).
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
// Persistent kernel over 128-row tiles ordered (row tile, z, head) with the head fastest, so
// a CTA keeps one row tile's RoPE angles (cos, sin) in registers while it runs through the
// heads.  With IG (input gradients) the same kernel computes dA_z = dX_z W_z^T from the
// un-rotated dQ, dK, dV: W is then read as a K-major B operand and nothing is rotated.  Per tile: TMA loads A_z[b, h] rows and W_z[h]; one tcgen05 product into a
// double-buffered TMEM accumulator; the epilogue warps rotate, round to bf16 and write a
// 128-byte-swizzled staging tile that a TMA store sends to global memory (the staging is
// double-buffered, so the store of one tile overlaps the next tile's epilogue).
template <int D>
struct ProjCfg {
  static constexpr int BM = 128;
  static constexpr int KB = D / 64;
  static constexpr int NS = 2;               // (A, W) load stages
  static constexpr int ATILE = BM * D * 2;
  static constexpr int WTILE = D * D * 2;
  static constexpr int ABLK = BM * 128;      // [128 rows][64 cols] block
  static constexpr int WBLK = D * 128;       // [D rows][64 cols] block
  static constexpr int OTILE = BM * D * 2;   // bf16 output staging tile
  static constexpr int A_OFF = 0;
  static constexpr int W_OFF = A_OFF + NS * ATILE;
  static constexpr int O_OFF = W_OFF + NS * WTILE;
  static constexpr int BAR_OFF = O_OFF + 2 * OTILE;
  // ld_full[NS], ld_empty[NS], acc_full[2], acc_empty[2], o_full[2], o_free[2], drain
  static constexpr int NBAR = 2 * NS + 8 + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM_ALLOC = MISC_OFF + 16 + 1024;
  // warps 0-7 epilogue (warp w: TMEM lanes 32 (w % 4), columns D/2 (w / 4) ..), 8 TMA
  // loads, 9 MMA, 10 TMA stores
  static constexpr int THREADS = 352;
  static constexpr int W_LOAD = 8, W_MMA = 9, W_STORE = 10;
  static constexpr int CPT = D / 2;          // output columns per epilogue thread
  static constexpr uint32_t T_COLS = 2 * D;  // double-buffered accumulator
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

struct ProjParams {
  const float2* tab;       // [n][d/2] (cos, sin)
  int n, B, H, nrt;        // nrt = 128-row tiles per instance
  long long tiles;         // B * nrt * 3 * H
  long long tiles_per_cta;
  unsigned long long limit_ns;
  WsGate gate;             // skip everything when the workspace already holds the outputs
};

template <int D, bool IG>
__global__ void __launch_bounds__(ProjCfg<D>::THREADS, 1)
proj_rope_tc_kernel(const __grid_constant__ CUtensorMap tm_a1, const __grid_constant__ CUtensorMap tm_a2,
                    const __grid_constant__ CUtensorMap tm_a3, const __grid_constant__ CUtensorMap tm_w1,
                    const __grid_constant__ CUtensorMap tm_w2, const __grid_constant__ CUtensorMap tm_w3,
                    const __grid_constant__ CUtensorMap tm_o1, const __grid_constant__ CUtensorMap tm_o2,
                    const __grid_constant__ CUtensorMap tm_o3, const ProjParams p) {
  using C = ProjCfg<D>;
  if (gate_skip(p.gate)) return;  // uniform over the grid, before any barrier or TMEM use
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  const uint32_t abort_flag = smem_u32(smem + C::MISC_OFF + 4);
  auto b_ldfull = [&](int s) { return smem_u32(&bars[s]); };
  auto b_ldempty = [&](int s) { return smem_u32(&bars[C::NS + s]); };
  auto b_accfull = [&](int b) { return smem_u32(&bars[2 * C::NS + b]); };
  auto b_accempty = [&](int b) { return smem_u32(&bars[2 * C::NS + 2 + b]); };
  auto b_ofull = [&](int b) { return smem_u32(&bars[2 * C::NS + 4 + b]); };
  auto b_ofree = [&](int b) { return smem_u32(&bars[2 * C::NS + 6 + b]); };
  const uint32_t b_drain = smem_u32(&bars[2 * C::NS + 8]);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long t0 = (long long)blockIdx.x * p.tiles_per_cta;
  const int NT = (int)min(p.tiles_per_cta, p.tiles - t0);
  const uint64_t lim = p.limit_ns;
  // tile index -> (b, row tile, z, h): head fastest, then z, then row tile
  auto decode = [&](int t, int& b, int& rt, int& z, int& h) {
    long long q = t0 + t;
    h = (int)(q % p.H);
    q /= p.H;
    z = (int)(q % 3);
    q /= 3;
    rt = (int)(q % p.nrt);
    b = (int)(q / p.nrt);
  };
  if (tid == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(b_ldfull(s), 1);
      mbar_init(b_ldempty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(b_accfull(b), 1);
      mbar_init(b_accempty(b), 256);
      mbar_init(b_ofull(b), 256);
      mbar_init(b_ofree(b), 1);
    }
    mbar_init(b_drain, 1);
    abort_set(abort_flag, 0);
    fence_barrier_init();
  }
  if (warp == C::W_MMA) {
    tmem_alloc(smem_u32(tslot), C::T_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  if (warp == C::W_LOAD) {
    // ------------------------------------------------------------------ TMA loads
    if (lane == 0) {
      tma_prefetch(&tm_a1);
      tma_prefetch(&tm_a2);
      tma_prefetch(&tm_a3);
      int last = -1;
      for (int t = 0; t < NT; ++t) {
        const int s = t % C::NS;
        if (!mbar_wait(b_ldempty(s), ((t / C::NS) & 1) ^ 1, abort_flag, lim)) break;
        int b, rt, z, h;
        decode(t, b, rt, z, h);
        const CUtensorMap* tma = z == 0 ? &tm_a1 : z == 1 ? &tm_a2 : &tm_a3;
        const CUtensorMap* tmw = z == 0 ? &tm_w1 : z == 1 ? &tm_w2 : &tm_w3;
        mbar_expect_tx(b_ldfull(s), C::ATILE + C::WTILE);
        for (int kb = 0; kb < C::KB; ++kb) {
          tma_load_3d(sbase + C::A_OFF + s * C::ATILE + kb * C::ABLK, tma, b_ldfull(s), 64 * kb,
                      rt * C::BM, b * p.H + h);
          tma_load_3d(sbase + C::W_OFF + s * C::WTILE + kb * C::WBLK, tmw, b_ldfull(s), 64 * kb,
                      0, h);
        }
        last = t;
      }
      if (abort_get(abort_flag)) {
        for (int t = (last - C::NS + 1 > 0 ? last - C::NS + 1 : 0); t <= last; ++t)
          mbar_drain(b_ldfull(t % C::NS), (t / C::NS) & 1, lim);
      }
    }
  } else if (warp == C::W_MMA) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // X = A W: W[in][out] is the B operand (K = in, N = out contiguous: MN-major).
      // dA = dX W^T: B[k = out][n = in] = W[in][out] (K contiguous: K-major).
      constexpr uint32_t idesc = idesc_bf16_f32(128, D, false, !IG);
      bool ok = true;
      for (int t = 0; ok && t < NT; ++t) {
        const int s = t % C::NS, ab = t & 1;
        if (!(ok = mbar_wait(b_ldfull(s), (t / C::NS) & 1, abort_flag, lim))) break;
        if (!(ok = mbar_wait(b_accempty(ab), ((t >> 1) & 1) ^ 1, abort_flag, lim))) break;
        tc_fence_after();
        const uint32_t a = sbase + C::A_OFF + s * C::ATILE;
        const uint32_t w = sbase + C::W_OFF + s * C::WTILE;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t bdesc = IG ? sw128_desc(w + (kk >> 2) * C::WBLK + (kk & 3) * 32, 16, 1024)
                                    : sw128_desc(w + kk * 2048, C::WBLK, 1024);
          mma_ss(tmem + ab * D, sw128_desc(a + (kk >> 2) * C::ABLK + (kk & 3) * 32, 16, 1024),
                 bdesc, idesc, kk > 0);
        }
        mma_commit(b_accfull(ab));
        mma_commit(b_ldempty(s));
      }
      if (!ok) {
        mma_commit(b_drain);
        mbar_drain(b_drain, 0, lim);
      }
    }
  } else if (warp == C::W_STORE) {
    // ------------------------------------------------------------------ TMA stores
    if (lane == 0) {
      for (int t = 0; t < NT; ++t) {
        const int ob = t & 1;
        if (!mbar_wait(b_ofull(ob), (t >> 1) & 1, abort_flag, lim)) break;
        int b, rt, z, h;
        decode(t, b, rt, z, h);
        const CUtensorMap* tmo = z == 0 ? &tm_o1 : z == 1 ? &tm_o2 : &tm_o3;
        for (int kb = 0; kb < C::KB; ++kb)
          tma_store_3d(tmo, sbase + C::O_OFF + ob * C::OTILE + kb * C::ABLK, 64 * kb, rt * C::BM,
                       b * p.H + h);
        bulk_commit();
        bulk_wait_read0();
        mbar_arrive(b_ofree(ob));
      }
      bulk_wait0();  // the stores have landed before the CTA leaves
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ epilogue (warps 0-7)
    const int rl = 32 * (warp & 3) + lane;           // row within the tile = TMEM lane
    const int c0 = C::CPT * (warp >> 2);             // first output column of this thread
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    float2 cs[C::CPT / 2];                            // (cos, sin) of this row's pairs
    int key = -1;                                     // row tile the angles belong to
    for (int t = 0; t < NT; ++t) {
      const int ab = t & 1;
      int b, rt, z, h;
      decode(t, b, rt, z, h);
      const int row = rt * C::BM + rl;
      if (!IG && z < 2 && rt != key) {
        key = rt;
        const float4* tr = reinterpret_cast<const float4*>(p.tab + (size_t)(row < p.n ? row : 0) * (D / 2) + c0 / 2);
#pragma unroll
        for (int k = 0; k < C::CPT / 4; ++k) {
          const float4 v = tr[k];
          cs[2 * k] = make_float2(v.x, v.y);
          cs[2 * k + 1] = make_float2(v.z, v.w);
        }
      }
      if (!mbar_wait_warp(b_accfull(ab), (t >> 1) & 1, abort_flag, lim)) break;
      tc_fence_after();
      uint32_t r[C::CPT];
#pragma unroll
      for (int c = 0; c < C::CPT / 32; ++c)
        tmem_ld32(tmem + lane_base + ab * D + c0 + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * c]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(b_accempty(ab));
      // staging buffer ob is free once the store of tile t - 2 has read it
      const int ob = t & 1;
      if (t >= 2 && !mbar_wait_warp(b_ofree(ob), ((t - 2) >> 1) & 1, abort_flag, lim)) break;
      const uint32_t ost = sbase + C::O_OFF + ob * C::OTILE;
#pragma unroll
      for (int c = 0; c < C::CPT / 8; ++c) {  // 8 columns = 4 pairs = one 16-byte chunk
        uint32_t w[4];
#pragma unroll
        for (int k2 = 0; k2 < 4; ++k2) {
          float x0 = __uint_as_float(r[8 * c + 2 * k2]), x1 = __uint_as_float(r[8 * c + 2 * k2 + 1]);
          if (!IG && z < 2) {
            const float2 a = cs[4 * c + k2];
            const float y0 = x0 * a.x - x1 * a.y, y1 = x0 * a.y + x1 * a.x;
            x0 = y0;
            x1 = y1;
          }
          w[k2] = pack_bf16x2(x0, x1);
        }
        const int col = c0 + 8 * c;
        st_shared_v4(ost + (col >> 6) * C::ABLK + sw128_offset(rl, (col & 63) >> 3), w[0], w[1],
                     w[2], w[3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(b_ofull(ob));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == C::W_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, C::T_COLS);
  }
}

// ---------------------------------------------------------------------------------------
// dQ = rot^-1(acc) / sqrt(d): fp32 in, bf16 out; one thread per four pairs (d/2 is a multiple of 4,
// so the four pairs share a row): two 16-byte loads of dQ~ and of (cos, sin), one 16-byte
// store.
// ---------------------------------------------------------------------------------------
__global__ void dq_unrotate_kernel(const float4* __restrict__ dqt, const float4* __restrict__ tab,
                                   uint4* __restrict__ dq, long long quads, int n, int half,
                                   float scale) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= quads) return;
  const int qpr = half / 4;  // quads per row
  const long long row = idx / qpr;
  const int k = (int)(idx - row * qpr);
  const int i = (int)(row % n);
  const float4 y0 = dqt[2 * idx], y1 = dqt[2 * idx + 1];
  const float4* tr = tab + ((size_t)i * half) / 2 + 2 * k;
  const float4 c0 = tr[0], c1 = tr[1];
  // the accumulator holds gamma K~ summed over key tiles: scale by 1/sqrt(d), rotate by -phi
  auto rot = [scale](float x, float y, float c, float sn) {
    return pack_bf16x2((x * c + y * sn) * scale, (-x * sn + y * c) * scale);
  };
  dq[idx] = make_uint4(rot(y0.x, y0.y, c0.x, c0.y), rot(y0.z, y0.w, c0.z, c0.w),
                       rot(y1.x, y1.y, c1.x, c1.y), rot(y1.z, y1.w, c1.z, c1.w));
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
