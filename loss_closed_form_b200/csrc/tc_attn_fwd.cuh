// Tensor-core forward: one CTA per pair of 128-row query tiles of one (b, h) instance.
//
//   S_t,j = Q~_t K~_j^T               (tcgen05, K-major x K-major, fp32 in TMEM)
//   online softmax over key tiles     (one query row per thread; rows = TMEM lanes)
//   P_t,j -> TMEM as bf16 over S_t,j, O_t += P_t,j V_j (tcgen05, A read from TMEM)
//   epilogue: O = acc / l, lse, l = O - E, delta_i = <l_i, O_i>, partial 1/2 sum l^2
//
// Definitions: s = softmax(Q~ K~^T / sqrt(d)) and O = s V are exact attention D^-1 A V
// ("HyperAttention" article, section 方法の概要); l = O - E is the error term l(x) of
// "RoPE Attention kan bijna lineair worden getraind" (Methodologie 1).
//
// The two query tiles t = 0, 1 share every K~ / V tile and alternate on the tensor cores:
// while warpgroup t turns S_t,j into P_t,j, the MMA warp runs the other tile's products, so
// the exponentials of one tile overlap the matrix products of the other.  TMEM holds S_0,
// S_1, O_0, O_1 (4 x 128 columns); P_t,j is written over the first 64 columns of S_t,j, and
// S_t,j+1 is issued only once the product that reads P_t,j has completed.
//
// Rescaling of the accumulator is deferred while a row's running maximum grows by at most
// 2^8 (log2 units): O and l keep one common reference, so the final O / l is unchanged and
// P stays <= 256 in bf16.  The row maximum is taken on raw scores; the scale
// log2(e)/sqrt(d) > 0 is applied to it and folded into each exponent's FFMA.
//
// Warp roles (384 threads): warps 0-3 softmax + epilogue of query tile 0, warps 4-7 of
// query tile 1, warp 8 TMA producer, warp 9 MMA issuer and TMEM owner, warps 10-11 zero the
// pair's rows of the backward's dQ~ accumulator (when asked to) and are otherwise idle.
// The third warpgroup hands registers to the two softmax warpgroups (setmaxnreg): a thread
// there holds a whole 128-column row of scores.
#pragma once
#include "tc_ptx.cuh"


namespace ra {
namespace tc {

template <int D>
struct FwdCfg {
  static constexpr int BM = 128;               // query rows per tile
  static constexpr int BN = 128;               // keys per tile
  static constexpr int NS = D == 64 ? 4 : 2;   // K / V pipeline stages
  static constexpr int KB = D / 64;            // 128-byte swizzle blocks per row
  static constexpr int TILE = 128 * D * 2;     // bytes of a 128 x D bf16 tile
  static constexpr int BLK = 128 * 128;        // bytes of one 128-row swizzle block
  static constexpr int Q_OFF = 0;              // two query tiles
  static constexpr int K_OFF = Q_OFF + 2 * TILE;
  static constexpr int V_OFF = K_OFF + NS * TILE;
  static constexpr int BAR_OFF = V_OFF + NS * TILE;
  // barriers: q_full, k_full[NS], k_empty[NS], v_full[NS], v_empty[NS], s_full[2],
  //           p_full[2], pv_done[2], drain, e_full[2], s_free[2]
  static constexpr int NBAR = 1 + 4 * NS + 6 + 1 + 2 + 2;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;  // tmem slot, abort flag
  static constexpr int SMEM_USED = MISC_OFF + 16;
  // at least half of the SM's shared memory: one CTA per SM, so the 512-column TMEM
  // allocation never waits on another CTA
  static constexpr int SMEM_ALLOC = (SMEM_USED + 1024 > 120 * 1024) ? SMEM_USED + 1024 : 120 * 1024;
  static constexpr int THREADS = 384;
  static constexpr int W_PROD = 8, W_MMA = 9;
  // registers per thread after the hand-over: 256 x REG_SOFTMAX + 128 x REG_OTHER must not
  // exceed the 384 x 168 the CTA is launched with
  static constexpr int REG_SOFTMAX = 216, REG_OTHER = 64;
  static_assert(256 * REG_SOFTMAX + 128 * REG_OTHER <= 384 * 168, "register hand-over");
  // TMEM columns: S_t at 128 t, O_t at 256 + O_STRIDE t.  With D = 128 the four take all 512
  // columns and P_t is written over the first 64 columns of S_t; with D = 64 each O_t takes 64
  // columns and P_t gets its own 64 at 384 + 64 t (SEP_P), so S_t,j+1 need not wait for the
  // product that reads P_t,j
  static constexpr bool SEP_P = D == 64;
  static constexpr uint32_t O_STRIDE = SEP_P ? D : 128;
  static constexpr uint32_t T_S0 = 0, T_O0 = 256, T_P0 = 384, T_COLS = 512;
  static_assert(!SEP_P || T_O0 + 2 * O_STRIDE <= T_P0, "TMEM plan");
  // loss partial sums written per query tile (one per softmax warp)
  static constexpr int LOSS_PARTS = 4;
};

struct FwdParams {
  const __nv_bfloat16* E;  // [BH][n][d] or null
  __nv_bfloat16* O;        // [BH][n][d]
  float* lse;              // [BH][n]
  __nv_bfloat16* ell;      // [BH][n][d] (with E)
  float* delta;            // [BH][n] (with E)
  double* loss_part;       // [BH][nq][4] (with E)
  float* dq_zero;          // [BH][n][d] fp32 accumulator of the backward, zeroed here, or null
  int n, BH, nq, npair, causal;
  int hgroup;              // heads per scheduling group (their K~, V fit in L2 together)
  float scale_log2;        // log2(e) / sqrt(d)
  unsigned long long limit_ns;
};

template <int D>
__global__ void __launch_bounds__(FwdCfg<D>::THREADS, 1)
attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_e,
                   const __grid_constant__ CUtensorMap tm_o,
                   const __grid_constant__ CUtensorMap tm_ell, const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  const uint32_t abort_flag = smem_u32(smem + C::MISC_OFF + 4);

  const uint32_t b_q = smem_u32(&bars[0]);
  auto b_kfull = [&](int s) { return smem_u32(&bars[1 + s]); };
  auto b_kempty = [&](int s) { return smem_u32(&bars[1 + C::NS + s]); };
  auto b_vfull = [&](int s) { return smem_u32(&bars[1 + 2 * C::NS + s]); };
  auto b_vempty = [&](int s) { return smem_u32(&bars[1 + 3 * C::NS + s]); };
  auto b_sfull = [&](int t) { return smem_u32(&bars[1 + 4 * C::NS + t]); };
  auto b_pfull = [&](int t) { return smem_u32(&bars[3 + 4 * C::NS + t]); };
  auto b_pvdone = [&](int t) { return smem_u32(&bars[5 + 4 * C::NS + t]); };
  const uint32_t b_drain = smem_u32(&bars[7 + 4 * C::NS]);
  auto b_efull = [&](int t) { return smem_u32(&bars[8 + 4 * C::NS + t]); };  // E tile landed
  auto b_sfree = [&](int t) { return smem_u32(&bars[10 + 4 * C::NS + t]); };  // S_t read (SEP_P)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // grid (heads of a group, pair rank, group): the CTAs are dispatched x fastest, so each
  // group of p.hgroup heads, whose K~ and V stay in L2 together, runs its longest causal
  // pairs first across all of its heads and the grid ends on short CTAs
  const int bh = blockIdx.z * gridDim.x + blockIdx.x;  // gridDim.x = p.hgroup
  const int qp = p.npair - 1 - blockIdx.y;
  if (bh >= p.BH) return;  // the last group may hold fewer heads
  const int n = p.n;
  const int nk = (n + C::BN - 1) / C::BN;
  // key tiles visited by query tile t = 2 qp + t (tile 1 may lie past n: its rows are
  // computed on zero-filled queries and never stored)
  const int T0 = p.causal ? 2 * qp + 1 : nk;
  const int T1 = p.causal ? 2 * qp + 2 : nk;
  const uint64_t lim = p.limit_ns;

  if (tid == 0) {
    mbar_init(b_q, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(b_kfull(s), 1);
      mbar_init(b_kempty(s), 1);
      mbar_init(b_vfull(s), 1);
      mbar_init(b_vempty(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(b_sfull(t), 1);
      mbar_init(b_pfull(t), 4);  // one arrival per softmax warp
      mbar_init(b_pvdone(t), 1);
      mbar_init(b_sfree(t), 4);  // one arrival per softmax warp
    }
    mbar_init(b_drain, 1);
    mbar_init(b_efull(0), 1);
    mbar_init(b_efull(1), 1);
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

  if (warp >= 8) regs_dec<C::REG_OTHER>();

  if (warp == C::W_PROD) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch(&tm_q);
      tma_prefetch(&tm_k);
      tma_prefetch(&tm_v);
      mbar_expect_tx(b_q, 2 * C::TILE);
      for (int t = 0; t < 2; ++t)
        for (int b = 0; b < C::KB; ++b)
          tma_load_3d(sbase + C::Q_OFF + t * C::TILE + b * C::BLK, &tm_q, b_q, 64 * b,
                      (2 * qp + t) * C::BM, bh);
      int last_k = -1, last_v = -1;
      for (int j = 0; j < T1; ++j) {
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
    // issue order per key tile j: PV_0,j, S_0,j+1, PV_1,j, S_1,j+1
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
      const uint32_t qa0 = sbase + C::Q_OFF;
      // descriptor low words per buffer (sw128_lo), offsets added per K step (sw128_at)
      auto issue_s = [&](int t, int j) {
        const uint32_t qa = sw128_lo(qa0 + t * C::TILE, 16);
        const uint32_t kb = sw128_lo(sbase + C::K_OFF + (j % C::NS) * C::TILE, 16);
        const uint32_t d_s = tmem + C::T_S0 + 128 * t;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::BLK + (kk & 3) * 32;
          mma_ss(d_s, sw128_at(qa, off), sw128_at(kb, off), idesc_s, kk > 0);
        }
        mma_commit(b_sfull(t));
      };
      auto issue_pv = [&](int t, int j) {
        const uint32_t pa = tmem + (C::SEP_P ? C::T_P0 + 64 * t : C::T_S0 + 128 * t);
        const uint32_t vb = sw128_lo(sbase + C::V_OFF + (j % C::NS) * C::TILE, C::BLK);
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk)
          mma_ts(tmem + C::T_O0 + C::O_STRIDE * t, pa + kk * 8, sw128_at(vb, kk * 2048),
                 idesc_pv, (j > 0 || kk > 0));
        mma_commit(b_pvdone(t));
      };
      bool ok = mbar_wait(b_q, 0, abort_flag, lim);
      if (ok) ok = mbar_wait(b_kfull(0), 0, abort_flag, lim);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
        mma_commit(b_kempty(0));
      }
      if constexpr (C::SEP_P) {
        // per key tile j: S_t,j+1 as soon as softmax t has read S_t,j, then P_t,j V_j once
        // softmax t has written P_t,j (its own columns: no wait on the previous product)
        for (int j = 0; ok && j < T1; ++j) {
          if (j + 1 < T1) {
            const int s1 = (j + 1) % C::NS;
            if (!(ok = mbar_wait(b_kfull(s1), ((j + 1) / C::NS) & 1, abort_flag, lim))) break;
            for (int t = 0; ok && t < 2; ++t) {
              if (j + 1 >= (t ? T1 : T0)) continue;
              if (!(ok = mbar_wait(b_sfree(t), j & 1, abort_flag, lim))) break;
              tc_fence_after();
              issue_s(t, j + 1);
            }
            if (!ok) break;
            mma_commit(b_kempty(s1));
          }
          const int s = j % C::NS;
          if (!(ok = mbar_wait(b_vfull(s), (j / C::NS) & 1, abort_flag, lim))) break;
          for (int t = 0; ok && t < 2; ++t) {
            if (j >= (t ? T1 : T0)) continue;
            if (!(ok = mbar_wait(b_pfull(t), j & 1, abort_flag, lim))) break;
            tc_fence_after();
            issue_pv(t, j);
          }
          if (!ok) break;
          mma_commit(b_vempty(s));
        }
      } else {
        for (int j = 0; ok && j < T1; ++j) {
          const int s = j % C::NS;
          const bool next0 = j + 1 < T0, next1 = j + 1 < T1;
          if (!(ok = mbar_wait(b_vfull(s), (j / C::NS) & 1, abort_flag, lim))) break;
          if (j < T0) {
            if (!(ok = mbar_wait(b_pfull(0), j & 1, abort_flag, lim))) break;
            tc_fence_after();
            issue_pv(0, j);
          }
          if (next1) {
            const int s1 = (j + 1) % C::NS;
            if (!(ok = mbar_wait(b_kfull(s1), ((j + 1) / C::NS) & 1, abort_flag, lim))) break;
          }
          if (next0) {
            // S_0,j+1 overwrites P_0,j: wait until the product reading it has completed
            if (!(ok = mbar_wait(b_pvdone(0), j & 1, abort_flag, lim))) break;
            tc_fence_after();
            issue_s(0, j + 1);
          }
          if (!(ok = mbar_wait(b_pfull(1), j & 1, abort_flag, lim))) break;
          tc_fence_after();
          issue_pv(1, j);
          mma_commit(b_vempty(s));
          if (next1) {
            if (!(ok = mbar_wait(b_pvdone(1), j & 1, abort_flag, lim))) break;
            tc_fence_after();
            issue_s(1, j + 1);
            mma_commit(b_kempty((j + 1) % C::NS));
          }
        }
      }
      if (!ok) {
        // wait (bounded) for every MMA issued so far before TMEM is released
        mma_commit(b_drain);
        mbar_drain(b_drain, 0, lim);
      }
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ softmax warps 0-7
    // warpgroup t = warp / 4 owns query tile 2 qp + t; warp w reaches TMEM lanes 32 (w % 4)
    regs_inc<C::REG_SOFTMAX>();
    const int t = warp >> 2, r = tid & 127;
    const int qt = 2 * qp + t;
    const int row = qt * C::BM + r;
    const int Tt = t ? T1 : T0;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t s_col = tmem + lane_base + C::T_S0 + 128 * t;
    const uint32_t o_col = tmem + lane_base + C::T_O0 + C::O_STRIDE * t;
    // P_t: over the first 64 columns of S_t, or its own columns (SEP_P)
    const uint32_t p_col = C::SEP_P ? tmem + lane_base + C::T_P0 + 64 * t : s_col;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < Tt; ++j) {
      if (!(ok = mbar_wait_warp(b_sfull(t), j & 1, abort_flag, lim))) break;
      tc_fence_after();
      // the four 32-column loads share one wait
      uint32_t xr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(s_col + 32 * c, xr[c]);
      tmem_wait_ld();
      float x[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        reg_fence32(xr[c]);
#pragma unroll
        for (int i = 0; i < 32; ++i) x[32 * c + i] = __uint_as_float(xr[c][i]);
      }
      if constexpr (C::SEP_P) {
        // S_t is in registers: the MMA warp may compute S_t,j+1 into its columns now
        tc_fence_before();
        mbar_arrive_warp(b_sfree(t));
      }
      const int key0 = j * C::BN;
      if (key0 + C::BN > n || (p.causal && j == qt)) {
#pragma unroll
        for (int i = 0; i < 128; ++i) {
          const int key = key0 + i;
          if (key >= n || (p.causal && key > row)) x[i] = -INFINITY;
        }
      }
      // row maximum: four chains of three-input max (elements k, k + 4, k + 8, ...)
      float mt[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) mt[k] = fmax3f(x[k], x[k + 4], x[k + 8]);
#pragma unroll
      for (int i = 12; i < 124; i += 8) {
#pragma unroll
        for (int k = 0; k < 4; ++k) mt[k] = fmax3f(mt[k], x[i + k], x[i + 4 + k]);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) mt[k] = fmaxf(mt[k], x[124 + k]);
      const float mnew = fmaxf(m, fmax3f(mt[0], mt[1], fmaxf(mt[2], mt[3])) * p.scale_log2);
      if constexpr (C::SEP_P) {
        // the product P_t,j-1 V_j-1 has completed before P_t,j is written over P_t,j-1 and O_t
        // may be rescaled (S_t,j no longer implies it)
        if (j > 0) {
          if (!(ok = mbar_wait_warp(b_pvdone(t), (j - 1) & 1, abort_flag, lim))) break;
          tc_fence_after();
        }
      }
      if (j == 0) {
        m = mnew;
      } else {
        const bool need = mnew > m + 8.f;
        if (__any_sync(0xffffffffu, need)) {
          // O_t is final for tiles < j (D = 128: S_t,j was issued after the product of tile
          // j - 1 completed and its commit covers that product; SEP_P: waited for above) and
          // can be rescaled in place
          const float alpha = need ? ex2(m - mnew) : 1.f;
          if (need) {
            l *= alpha;
            m = mnew;
          }
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t rr[32];
            tmem_ld32(o_col + 32 * c, rr);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
            tmem_st32(o_col + 32 * c, rr);
          }
        }
      }
      // exponent arguments and row sums two columns per packed FFMA / FADD
      const uint64_t sc2 = f32x2(p.scale_log2, p.scale_log2), nm2 = f32x2(-m, -m);
      uint64_t ps2a = f32x2(0.f, 0.f), ps2b = f32x2(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 y =
              unpack_f32x2(ffma2(f32x2(x[32 * c + 2 * i], x[32 * c + 2 * i + 1]), sc2, nm2));
          const float p0 = ex2(y.x), p1 = ex2(y.y);
          if (i & 1)
            ps2b = fadd2(ps2b, f32x2(p0, p1));
          else
            ps2a = fadd2(ps2a, f32x2(p0, p1));
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st16(p_col + 16 * c, pk);
      }
      const float2 ps = unpack_f32x2(fadd2(ps2a, ps2b));
      l += ps.x + ps.y;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive_warp(b_pfull(t));
    }
    // ---- epilogue: one full row of O per thread.  The tile's query buffer is free (every
    //      S_t has completed): E_t comes in there by TMA, each thread overwrites its own row
    //      of E with its row of O (128-byte swizzle), one TMA store sends O out, then l = O - E
    //      follows the same way.  Rows are private to their thread, so only the hand-overs to
    //      the storing thread need a barrier (named barrier 1 + t over the warpgroup's 128
    //      threads, reached the same number of times by every thread).
    float sq = 0.f, dl = 0.f;
    if (ok) ok = mbar_wait_warp(b_pvdone(t), (Tt - 1) & 1, abort_flag, lim);
    const bool vrow = row < n;
    const uint32_t stg = sbase + C::Q_OFF + t * C::TILE;
    const bool has_e = p.E != nullptr;
    const bool e_issued = ok && r == 0 && has_e;
    if (e_issued) {
      mbar_expect_tx(b_efull(t), C::TILE);
      for (int b = 0; b < C::KB; ++b)
        tma_load_3d(stg + b * C::BLK, &tm_e, b_efull(t), 64 * b, qt * C::BM, bh);
    }
    if (ok && has_e) ok = mbar_wait_warp(b_efull(t), 0, abort_flag, lim);
    // after an abort, the copy this thread issued lands before the CTA leaves
    if (e_issued && !ok) mbar_drain(b_efull(t), 0, lim);
    uint32_t lw[D / 2];  // l = O - E of this row, bf16 pairs
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t rr[32];
        tmem_ld32(o_col + 32 * c, rr);
        tmem_wait_ld();
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint32_t a = stg + (c >> 1) * C::BLK + sw128_offset(r, 4 * (c & 1) + v);
          float o[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) o[i] = __uint_as_float(rr[8 * v + i]) * inv_l;
          if (has_e) {
            const float4 ev = ld_shared_v4f(a);
            const uint32_t ew[4] = {__float_as_uint(ev.x), __float_as_uint(ev.y),
                                    __float_as_uint(ev.z), __float_as_uint(ev.w)};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const __nv_bfloat162 e2 = *reinterpret_cast<const __nv_bfloat162*>(&ew[q]);
              const float e0 = o[2 * q] - __low2float(e2);
              const float e1 = o[2 * q + 1] - __high2float(e2);
              const uint32_t lr = pack_bf16x2(e0, e1);
              lw[16 * c + 4 * v + q] = lr;
              if (vrow) {
                // delta from the stored (bf16) l, the l the backward's beta = l V^T is built
                // from: then sum_j s_ij (beta_ij - delta_i) = 0 holds for the rounded l too, and
                // rows with one key (s = 1) get gamma = 0 exactly; the loss keeps the fp32 l
                const __nv_bfloat162 l2 = *reinterpret_cast<const __nv_bfloat162*>(&lr);
                dl = fmaf(__low2float(l2), o[2 * q], fmaf(__high2float(l2), o[2 * q + 1], dl));
                sq = fmaf(e0, e0, fmaf(e1, e1, sq));
              }
            }
          }
          st_shared_v4(a, pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]),
                       pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
        }
      }
      if (vrow) {
        p.lse[(size_t)bh * n + row] = (m + log2f(l)) * kLn2;
        if (has_e) p.delta[(size_t)bh * n + row] = dl;
      }
    }
    fence_proxy_async_smem();
    named_bar_sync(1 + t, 128);
    if (ok && r == 0) {
      for (int b = 0; b < C::KB; ++b)
        tma_store_3d(&tm_o, stg + b * C::BLK, 64 * b, qt * C::BM, bh);
      bulk_commit();
      bulk_wait_read0();
    }
    if (has_e) {
      named_bar_sync(1 + t, 128);  // the O store has read the staging
      if (ok) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c)
#pragma unroll
          for (int v = 0; v < 4; ++v)
            st_shared_v4(stg + (c >> 1) * C::BLK + sw128_offset(r, 4 * (c & 1) + v),
                         lw[16 * c + 4 * v], lw[16 * c + 4 * v + 1], lw[16 * c + 4 * v + 2],
                         lw[16 * c + 4 * v + 3]);
      }
      fence_proxy_async_smem();
      named_bar_sync(1 + t, 128);
      if (ok && r == 0) {
        for (int b = 0; b < C::KB; ++b)
          tma_store_3d(&tm_ell, stg + b * C::BLK, 64 * b, qt * C::BM, bh);
        bulk_commit();
      }
    }
    // the stores have read the staging before the CTA leaves (their writes complete with the
    // kernel)
    if (ok && r == 0) bulk_wait_read0();
    // per-warp partial of 1/2 sum l^2 (fixed order: deterministic)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if (p.E && ok && lane == 0 && qt < p.nq)
      p.loss_part[((size_t)bh * p.nq + qt) * C::LOSS_PARTS + (warp & 3)] = 0.5 * (double)sq;
  } else if (p.dq_zero) {
    // ------------------------------------------------------------------ warps 10-11
    // zero rows 2 qp * 128 .. of this instance's dQ~ accumulator (the pair's two query tiles,
    // clipped to n): every row of every instance belongs to exactly one pair
    const int r0 = 2 * qp * C::BM;
    const int r1 = min(n, r0 + 2 * C::BM);
    if (r1 > r0) {
      float4* dst = reinterpret_cast<float4*>(p.dq_zero + ((size_t)bh * n + r0) * D);
      const int cnt = (r1 - r0) * (D / 4);
      for (int i = tid - 32 * (C::W_MMA + 1); i < cnt; i += 64)
        dst[i] = make_float4(0.f, 0.f, 0.f, 0.f);
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
