// Tensor-core forward: one CTA per 128-row query tile of one (b, h) instance.
//
//   S_j = Q~ K~_j^T                 (tcgen05, K-major x K-major, fp32 in TMEM, double-buffered)
//   online softmax over key tiles    (one query row per thread; rows = TMEM lanes)
//   P_j -> TMEM as bf16, O += P_j V_j (tcgen05 with A read from TMEM, V as an MN-major B)
//   epilogue: O = acc / l, lse, l = O - E, delta_i = <l_i, O_i>, partial 1/2 sum l^2
//
// Definitions: s = softmax(Q~ K~^T / sqrt(d)) and O = s V are exact attention D^-1 A V
// ("HyperAttention" article, section 方法の概要); l = O - E is the error term l(x) of
// "RoPE Attention kan bijna lineair worden getraind" (Methodologie 1).
//
// Rescaling of the accumulator is deferred while a row's running maximum grows by at most
// 2^8 (log2 units): O and l keep one common reference, so the final O / l is unchanged and
// P stays <= 256 in bf16.
//
// Warp roles (320 threads): warps 0-7 softmax + epilogue (two warpgroups over the same 128
// query rows, each taking 64 of the 128 key columns of a tile; the row maximum, row sum and
// <l, O> are combined through shared memory), warp 8 TMA producer, warp 9 MMA issuer and
// TMEM owner.
#pragma once
#include "tc_ptx.cuh"

namespace ra {
namespace tc {

template <int D>
struct FwdCfg {
  static constexpr int BM = 128;               // query rows per tile
  static constexpr int BN = 128;               // keys per tile
  static constexpr int NS = 2;                 // K / V pipeline stages
  static constexpr int KB = D / 64;            // 128-byte swizzle blocks per row
  static constexpr int TILE = 128 * D * 2;     // bytes of a 128 x D bf16 tile
  static constexpr int BLK = 128 * 128;        // bytes of one 128-row swizzle block
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + TILE;
  static constexpr int V_OFF = K_OFF + NS * TILE;
  static constexpr int BAR_OFF = V_OFF + NS * TILE;
  // barriers: q_full, k_full[NS], k_empty[NS], v_full[NS], v_empty[NS], s_full[2],
  //           p_full[2], pv_done[2], drain, xch[2], ep1, ep2
  static constexpr int NBAR = 1 + 4 * NS + 6 + 1 + 4;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;  // tmem slot, abort flag, 8 partial sums
  static constexpr int XCH_OFF = MISC_OFF + 64;        // float [2 buffers][2 halves][128 rows]
  static constexpr int EPL_OFF = XCH_OFF + 2 * 2 * 128 * 4;  // float [2 halves][128]: row sums
  static constexpr int EPD_OFF = EPL_OFF + 2 * 128 * 4;      // float [128]: <l, O> of half 1
  static constexpr int SMEM_USED = EPD_OFF + 128 * 4;
  // at least half of the SM's shared memory: one CTA per SM, so the 512-column TMEM
  // allocation never waits on another CTA
  static constexpr int SMEM_ALLOC = (SMEM_USED + 1024 > 120 * 1024) ? SMEM_USED + 1024 : 120 * 1024;
  static constexpr int THREADS = 320;
  static constexpr int W_PROD = 8, W_MMA = 9;
  // TMEM columns
  static constexpr uint32_t T_S0 = 0, T_S1 = 128, T_O = 256, T_P0 = 384, T_P1 = 448;
  static constexpr uint32_t T_COLS = 512;
};

struct FwdParams {
  const __nv_bfloat16* E;  // [BH][n][d] or null
  __nv_bfloat16* O;        // [BH][n][d]
  float* lse;              // [BH][n]
  __nv_bfloat16* ell;      // [BH][n][d] (with E)
  float* delta;            // [BH][n] (with E)
  double* loss_part;       // [BH * nq] (with E)
  int n, BH, nq, causal;
  float scale_log2;        // log2(e) / sqrt(d)
  unsigned long long limit_ns;
};

template <int D>
__global__ void __launch_bounds__(FwdCfg<D>::THREADS, 1)
attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  const uint32_t abort_flag = smem_u32(smem + C::MISC_OFF + 4);
  const uint32_t red = sbase + C::MISC_OFF + 16;  // 8 partial sums of 1/2 l^2

  const uint32_t b_q = smem_u32(&bars[0]);
  auto b_kfull = [&](int s) { return smem_u32(&bars[1 + s]); };
  auto b_kempty = [&](int s) { return smem_u32(&bars[1 + C::NS + s]); };
  auto b_vfull = [&](int s) { return smem_u32(&bars[1 + 2 * C::NS + s]); };
  auto b_vempty = [&](int s) { return smem_u32(&bars[1 + 3 * C::NS + s]); };
  auto b_sfull = [&](int b) { return smem_u32(&bars[1 + 4 * C::NS + b]); };
  auto b_pfull = [&](int b) { return smem_u32(&bars[3 + 4 * C::NS + b]); };
  auto b_pvdone = [&](int b) { return smem_u32(&bars[5 + 4 * C::NS + b]); };
  const uint32_t b_drain = smem_u32(&bars[7 + 4 * C::NS]);
  auto b_xch = [&](int b) { return smem_u32(&bars[8 + 4 * C::NS + b]); };
  const uint32_t b_ep1 = smem_u32(&bars[10 + 4 * C::NS]);
  const uint32_t b_ep2 = smem_u32(&bars[11 + 4 * C::NS]);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // head-major order: the query tiles of one (b, h) run side by side and share its K~, V in
  // L2; within a head the longest causal tiles go first
  const int bh = blockIdx.y;
  const int qt = p.nq - 1 - blockIdx.x;
  const int n = p.n;
  const int T = p.causal ? qt + 1 : (n + C::BN - 1) / C::BN;
  const uint64_t lim = p.limit_ns;

  if (tid == 0) {
    mbar_init(b_q, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(b_kfull(s), 1);
      mbar_init(b_kempty(s), 1);
      mbar_init(b_vfull(s), 1);
      mbar_init(b_vempty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(b_sfull(b), 1);
      mbar_init(b_pfull(b), 256);
      mbar_init(b_pvdone(b), 1);
      mbar_init(b_xch(b), 256);
    }
    mbar_init(b_drain, 1);
    mbar_init(b_ep1, 256);
    mbar_init(b_ep2, 256);
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

  if (warp == C::W_PROD) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch(&tm_q);
      tma_prefetch(&tm_k);
      tma_prefetch(&tm_v);
      mbar_expect_tx(b_q, C::TILE);
      for (int b = 0; b < C::KB; ++b)
        tma_load_3d(sbase + C::Q_OFF + b * C::BLK, &tm_q, b_q, 64 * b, qt * C::BM, bh);
      int last_k = -1, last_v = -1;
      for (int j = 0; j < T; ++j) {
        const int s = j % C::NS;
        const uint32_t ph = (j / C::NS) & 1;
        if (!mbar_wait(b_kempty(s), ph ^ 1, abort_flag, lim)) break;
        mbar_expect_tx(b_kfull(s), C::TILE);
        for (int b = 0; b < C::KB; ++b)
          tma_load_3d(sbase + C::K_OFF + s * C::TILE + b * C::BLK, &tm_k, b_kfull(s), 64 * b,
                      j * C::BN, bh);
        last_k = j;
        if (!mbar_wait(b_vempty(s), ph ^ 1, abort_flag, lim)) break;
        mbar_expect_tx(b_vfull(s), C::TILE);
        for (int b = 0; b < C::KB; ++b)
          tma_load_3d(sbase + C::V_OFF + s * C::TILE + b * C::BLK, &tm_v, b_vfull(s), 64 * b,
                      j * C::BN, bh);
        last_v = j;
      }
      if (abort_get(abort_flag)) {
        // let the copies already issued land before the CTA leaves (at most one pending
        // phase per stage: a stage is refilled only after its previous contents were used)
        mbar_drain(b_q, 0, lim);
        for (int j = (last_k - C::NS + 1 > 0 ? last_k - C::NS + 1 : 0); j <= last_k; ++j)
          mbar_drain(b_kfull(j % C::NS), (j / C::NS) & 1, lim);
        for (int j = (last_v - C::NS + 1 > 0 ? last_v - C::NS + 1 : 0); j <= last_v; ++j)
          mbar_drain(b_vfull(j % C::NS), (j / C::NS) & 1, lim);
      }
    }
  } else if (warp == C::W_MMA) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
      bool ok = mbar_wait(b_q, 0, abort_flag, lim);
      tc_fence_after();
      for (int j = 0; ok && j <= T; ++j) {
        if (j < T) {
          const int s = j % C::NS;
          if (!(ok = mbar_wait(b_kfull(s), (j / C::NS) & 1, abort_flag, lim))) break;
          tc_fence_after();
          const uint32_t d_s = tmem + ((j & 1) ? C::T_S1 : C::T_S0);
          const uint32_t qa = sbase + C::Q_OFF, kb = sbase + C::K_OFF + s * C::TILE;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::BLK + (kk & 3) * 32;
            mma_ss(d_s, sw128_desc(qa + off, 16, 1024), sw128_desc(kb + off, 16, 1024), idesc_s,
                   kk > 0);
          }
          mma_commit(b_sfull(j & 1));
          mma_commit(b_kempty(s));
        }
        if (j >= 1) {
          const int jj = j - 1, s = jj % C::NS, sb = jj & 1;
          if (!(ok = mbar_wait(b_pfull(sb), (jj >> 1) & 1, abort_flag, lim))) break;
          if (!(ok = mbar_wait(b_vfull(s), (jj / C::NS) & 1, abort_flag, lim))) break;
          tc_fence_after();
          const uint32_t pa = tmem + (sb ? C::T_P1 : C::T_P0);
          const uint32_t vb = sbase + C::V_OFF + s * C::TILE;
#pragma unroll
          for (int kk = 0; kk < C::BN / 16; ++kk)
            mma_ts(tmem + C::T_O, pa + kk * 8, sw128_desc(vb + kk * 2048, C::BLK, 1024), idesc_pv,
                   (jj > 0 || kk > 0));
          mma_commit(b_pvdone(sb));
          mma_commit(b_vempty(s));
        }
      }
      if (!ok) {
        // wait (bounded) for every MMA issued so far before TMEM is released
        mma_commit(b_drain);
        mbar_drain(b_drain, 0, lim);
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax warps 0-7
    // warp w reaches TMEM lanes 32 (w % 4) ...; warpgroup `half` takes key columns
    // 64 half .. 64 half + 63 of each tile and head-dimension columns D/2 half .. of O
    const int r = tid & 127, half = warp >> 2;
    const int row = qt * C::BM + r;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t xch = sbase + C::XCH_OFF;
    constexpr int OH = D / 2;  // O columns per warpgroup
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      const int sb = j & 1;
      if (!(ok = mbar_wait_warp(b_sfull(sb), (j >> 1) & 1, abort_flag, lim))) break;
      tc_fence_after();
      float x[64];
      {
        const uint32_t s_addr = tmem + lane_base + (sb ? C::T_S1 : C::T_S0) + 64 * half;
        uint32_t r0[32], r1[32];
        tmem_ld32(s_addr, r0);
        tmem_ld32(s_addr + 32, r1);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          x[i] = __uint_as_float(r0[i]);
          x[32 + i] = __uint_as_float(r1[i]);
        }
      }
      // raw scores: the scale log2(e)/sqrt(d) > 0 is applied to the row maximum and folded
      // into the exponent's argument
      const int key0 = j * C::BN + 64 * half;
      if (j * C::BN + C::BN > n || (p.causal && j == qt)) {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const int key = key0 + i;
          if (key >= n || (p.causal && key > row)) x[i] = -INFINITY;
        }
      }
      float mt = x[0];
#pragma unroll
      for (int i = 1; i < 64; ++i) mt = fmaxf(mt, x[i]);
      // the other half of the row's maximum
      st_shared_f32(xch + ((sb * 2 + half) * 128 + r) * 4, mt);
      mbar_arrive(b_xch(sb));
      if (!(ok = mbar_wait_warp(b_xch(sb), (j >> 1) & 1, abort_flag, lim))) break;
      const float mo = ld_shared_f32(xch + ((sb * 2 + (half ^ 1)) * 128 + r) * 4);
      const float mnew = fmaxf(m, fmaxf(mt, mo) * p.scale_log2);
      if (j == 0) {
        m = mnew;
      } else {
        // both halves of a row take the same decision (same m, same mnew), and warps w and
        // w + 4 hold the same rows, so the vote agrees across the two warpgroups
        const bool need = mnew > m + 8.f;
        if (__any_sync(0xffffffffu, need)) {
          // O holds P_0..P_{j-1} V: wait for the last product, then rescale in TMEM
          if (!(ok = mbar_wait_warp(b_pvdone((j - 1) & 1), ((j - 1) >> 1) & 1, abort_flag, lim)))
            break;
          tc_fence_after();
          const float alpha = need ? ex2(m - mnew) : 1.f;
          if (need) {
            l *= alpha;
            m = mnew;
          }
#pragma unroll
          for (int c = 0; c < OH / 32; ++c) {
            uint32_t rr[32];
            const uint32_t oa = tmem + lane_base + C::T_O + OH * half + 32 * c;
            tmem_ld32(oa, rr);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
            tmem_st32(oa, rr);
          }
          tmem_wait_st();
        }
      }
      if (j >= 2) {  // P buffer sb was read by the product of tile j - 2
        if (!(ok = mbar_wait_warp(b_pvdone(sb), ((j - 2) >> 1) & 1, abort_flag, lim))) break;
        tc_fence_after();
      }
      float psum = 0.f;
      uint32_t pk[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float p0 = ex2(fmaf(x[2 * i], p.scale_log2, -m));
        const float p1 = ex2(fmaf(x[2 * i + 1], p.scale_log2, -m));
        psum += p0 + p1;
        pk[i] = pack_bf16x2(p0, p1);
      }
      tmem_st32(tmem + lane_base + (sb ? C::T_P1 : C::T_P0) + 32 * half, pk);
      l += psum;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(b_pfull(sb));
    }
    // ---- epilogue: each warpgroup finishes its D/2 columns of O
    float sq = 0.f, dl = 0.f;
    if (ok) ok = mbar_wait_warp(b_pvdone((T - 1) & 1), ((T - 1) >> 1) & 1, abort_flag, lim);
    st_shared_f32(sbase + C::EPL_OFF + (half * 128 + r) * 4, l);
    mbar_arrive(b_ep1);
    const bool ok1 = mbar_wait_warp(b_ep1, 0, abort_flag, lim);
    const bool vrow = row < n;
    float l_row = 1.f;
    if (ok && ok1) {
      tc_fence_after();
      l_row = ld_shared_f32(sbase + C::EPL_OFF + r * 4) +
              ld_shared_f32(sbase + C::EPL_OFF + (128 + r) * 4);
      const float inv_l = 1.f / l_row;
      const size_t ro = ((size_t)bh * n + row) * D + OH * half;
#pragma unroll
      for (int c = 0; c < OH / 32; ++c) {
        uint32_t rr[32];
        tmem_ld32(tmem + lane_base + C::T_O + OH * half + 32 * c, rr);
        tmem_wait_ld();
        if (vrow) {
          float o[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __uint_as_float(rr[i]) * inv_l;
          uint4* Og = reinterpret_cast<uint4*>(p.O + ro + 32 * c);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            Og[v] = make_uint4(pack_bf16x2(o[8 * v], o[8 * v + 1]), pack_bf16x2(o[8 * v + 2], o[8 * v + 3]),
                               pack_bf16x2(o[8 * v + 4], o[8 * v + 5]), pack_bf16x2(o[8 * v + 6], o[8 * v + 7]));
          if (p.E) {
            const uint4* Eg = reinterpret_cast<const uint4*>(p.E + ro + 32 * c);
            uint4* Lg = reinterpret_cast<uint4*>(p.ell + ro + 32 * c);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const uint4 ev = Eg[v];
              const uint32_t ew[4] = {ev.x, ev.y, ev.z, ev.w};
              uint32_t lw[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const __nv_bfloat162 e2 = *reinterpret_cast<const __nv_bfloat162*>(&ew[q]);
                const float e0 = o[8 * v + 2 * q] - __low2float(e2);
                const float e1 = o[8 * v + 2 * q + 1] - __high2float(e2);
                dl = fmaf(e0, o[8 * v + 2 * q], fmaf(e1, o[8 * v + 2 * q + 1], dl));
                sq = fmaf(e0, e0, fmaf(e1, e1, sq));
                lw[q] = pack_bf16x2(e0, e1);
              }
              Lg[v] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
          }
        }
      }
    }
    // combine <l, O> of the two halves and the per-warp sums of l^2
    if (half == 1) st_shared_f32(sbase + C::EPD_OFF + r * 4, dl);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if (lane == 0) st_shared_f32(red + warp * 4, sq);
    mbar_arrive(b_ep2);
    const bool ok2 = mbar_wait_warp(b_ep2, 0, abort_flag, lim);
    if (ok && ok1 && ok2) {
      if (half == 0 && vrow) {
        p.lse[(size_t)bh * n + row] = (m + log2f(l_row)) * kLn2;
        if (p.E) p.delta[(size_t)bh * n + row] = dl + ld_shared_f32(sbase + C::EPD_OFF + r * 4);
      }
      if (p.E && tid == 0) {
        double t = 0.0;
        for (int w = 0; w < 8; ++w) t += (double)ld_shared_f32(red + w * 4);
        p.loss_part[(size_t)blockIdx.y * gridDim.x + blockIdx.x] = 0.5 * t;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == C::W_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, C::T_COLS);
  }
}

}  // namespace tc
}  // namespace ra
