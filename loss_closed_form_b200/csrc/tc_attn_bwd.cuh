// Tensor-core closed-form backward: one CTA per 128-key tile of one (b, h) instance, looping
// over the 64-row query tiles that see those keys.
//
// Per query tile i (all products tcgen05, bf16 operands, fp32 accumulators in TMEM):
//   S^T    = K~ Q~_i^T                  scores, keys on TMEM lanes
//   beta^T = V l_i^T                    beta(x) = l V^T, transposed
//   P^T    = exp(S^T / sqrt(d) - lse_i)  recomputed softmax s(x) from the stored log-sum-exp
//   gamma^T = P^T o (beta^T - delta_i)   gamma = diag(s) beta - s s^T beta, with the row sums
//                                        s_i^T beta_i = <l_i, O_i> = delta_i
//   (P^T and gamma^T are written to TMEM over the columns S^T occupied, where they are the A
//    operands of the next two products; gamma^T also goes to shared memory as the B operand
//    of dQ~^T, which is accumulated over the columns beta^T occupied)
//   dV    += P^T l_i                   (accumulated in TMEM over all query tiles)
//   dK~   += gamma^T Q~_i              (scaled by 1/sqrt(d) and un-rotated at the end)
//   dQ~_i^T = K~^T gamma^T             (d on TMEM lanes; staged in shared memory and added to
//                                        the global fp32 accumulator by one TMA bulk
//                                        reduce-add; the 1/sqrt(d) is applied when the
//                                        accumulator is un-rotated, which keeps the drain warps'
//                                        per-element work to a load and a store)
//   at d = 64 instead, once per pair of query tiles i, i + 1:
//   dQ~_i,i+1 = [gamma_i; gamma_i+1] K~  (the 128 queries on TMEM lanes, in columns of its own:
//                                        a product with M = d = 64 holds the tensor pipe as
//                                        long as one with M = 128)
// so no n x n matrix ever leaves the chip.
//
// Definitions: "RoPE Attention kan bijna lineair worden getraind", Methodologie 1 (s, l,
// beta, gamma) and 2 (gamma_1 = diag(s) beta, gamma_2 = s s^T beta).
//
// TMEM holds two step buffers of 128 columns, [S^T | beta^T] for query tiles i and i + 1
// (i even in buffer 0), then dK~ and dV (and at d = 64 two 64-column buffers for the pair
// products' dQ~): while the softmax warps turn one buffer into P^T and gamma^T, the tensor
// cores run the other buffer's products, and the next-but-one step's S^T and beta^T are issued
// as soon as a buffer's products have completed and (d = 128) its dQ~^T has been read out.
//
// Warp roles (480 threads): warps 0-7 softmax / gamma (two warpgroups over the same 128 key
// rows, each taking half of the 64 query columns) and the epilogue (warps 0-3 dK, 4-7 dV),
// warps 8-11 drain dQ~ from TMEM into the staging tile (thread 256 issues the bulk
// reduction), warp 12 TMA producer (it also stages the query tile's lse and delta), warp 13
// issues the gradient products and owns TMEM, warp 14 issues S^T and beta^T.
#pragma once
#include "tc_ptx.cuh"

namespace ra {
namespace tc {

template <int D>
struct BwdCfg {
  static constexpr int BK = 128;              // keys per CTA
  static constexpr int BQ = 64;               // query rows per step
  static constexpr int NSQ = 3;               // query-tile pipeline stages
  static constexpr int KB = D / 64;           // 128-byte swizzle blocks per row
  static constexpr int KTILE = BK * D * 2;    // K~ or V tile bytes
  static constexpr int QTILE = BQ * D * 2;    // Q~_i or l_i tile bytes
  static constexpr int KBLK = BK * 128;       // one swizzle block of a 128-row tile
  static constexpr int QBLK = BQ * 128;       // one swizzle block of a 64-row tile
  static constexpr int PG = BK * BQ * 2;      // gamma^T buffer bytes (one swizzle block)
  // d = 64: dQ~ of two consecutive query tiles in one product, dQ~ = gamma K~ with the 128
  // queries on TMEM lanes (M = 128; the transposed product would have M = d = 64, which
  // takes a tensor-core instruction as long as M = 128 does), accumulated in TMEM columns of
  // its own.  d = 128 has no free columns and keeps one dQ~^T = K~^T gamma^T per tile.
  static constexpr bool PAIR = (D == 64);
  static constexpr int NG = PAIR ? 4 : 2;     // gamma^T slots
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + KTILE;
  static constexpr int Q_OFF = V_OFF + KTILE;            // NSQ stages
  static constexpr int L_OFF = Q_OFF + NSQ * QTILE;      // NSQ stages
  static constexpr int G_OFF = L_OFF + NSQ * QTILE;      // gamma^T [NG], an operand of dQ~
  // fp32 dQ~ staging: [BQ][D] row-major (d = 128), or per pair two halves (one per query
  // tile) of two [64 rows][32 columns] boxes in the 128-byte swizzle (d = 64)
  static constexpr int DQS_OFF = G_OFF + NG * PG;
  static constexpr int DQS = (PAIR ? 2 : 1) * BQ * D * 4;
  static constexpr int DQ_HALF = BQ * D * 4, DQ_BOX = BQ * 32 * 4;
  // float [NSQ][BQ / 2][4]: (-lse * log2(e) of rows 2i, 2i + 1, delta of rows 2i, 2i + 1)
  static constexpr int LD_OFF = DQS_OFF + DQS;
  static constexpr int BAR_OFF = LD_OFF + NSQ * BQ * 8;
  // kv_full, q_full[NSQ], q_empty[NSQ], s_full[2], pg_full[2], pg_done[2], dq_full[2],
  // dq_free[2], acc_done, drain, dqs_full, dqs_free, tab_full, ep_full, drain2
  static constexpr int NBAR = 1 + 2 * NSQ + 10 + 7;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM_USED = MISC_OFF + 64;
  static constexpr int SMEM_ALLOC =
      (SMEM_USED + 1024 > 120 * 1024) ? SMEM_USED + 1024 : 120 * 1024;
  // epilogue: the (cos, sin) rows of the key tile as D / 32 boxes of [128 rows][128 bytes]
  // (128-byte swizzle) over K~ / V, and dK / dV staged over the query-tile stages
  static constexpr int TBLK = BK * 128;
  static constexpr int TABT = BK * D * 4;
  static_assert(TABT <= 2 * KTILE && 2 * KTILE <= 2 * NSQ * QTILE, "epilogue staging");
  static constexpr int THREADS = 480;
  static constexpr int W_DRAIN = 8, W_PROD = 12, W_MMA = 13, W_MMA2 = 14;
  // deterministic mode: steps between a query tile's reduction and passing its turn on
  static constexpr int TURN_LAG = 1;
  // TMEM columns: step buffer b at 128 b holds S^T (columns 0-63) and beta^T (64-127); the
  // softmax warpgroup h then writes P^T at 32 h and gamma^T at 32 h + 16 (16 columns each, two
  // bf16 per column) and dQ~^T is accumulated at 64
  static constexpr uint32_t T_BUF = 128, T_B = 64, T_DQ = 64, T_GT = 16, T_DK = 256,
                            T_DV = 256 + D;
  // d = 64: the pair products' dQ~ (128 query lanes x 64 columns) in two buffers
  static constexpr uint32_t T_DQP = 256 + 2 * D;
  static constexpr uint32_t T_COLS = 512;
  static_assert(!PAIR || T_DQP + 2 * D <= T_COLS, "TMEM budget");
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

struct BwdParams {
  const float* lse;     // [BH][n]
  const float* delta;   // [BH][n]
  // deterministic mode: [BH][turn_stride] turn counters, one per 64-row query tile, zero at
  // launch (null: the dQ~ tiles are added in whatever order the key tiles get there)
  unsigned* turn;
  int turn_stride;
  int n, BH, nk, causal;
  int hgroup;          // heads per scheduling group (their Q~, l, dQ~ fit in L2 together)
  float scale;         // 1 / sqrt(d)
  float scale_log2;    // log2(e) / sqrt(d)
  unsigned long long limit_ns;
};

template <int D>
__global__ void __launch_bounds__(BwdCfg<D>::THREADS, 1)
attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_l,
                   const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ CUtensorMap tm_tab,
                   const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                   const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  const uint32_t abort_flag = smem_u32(smem + C::MISC_OFF + 4);

  const uint32_t b_kv = smem_u32(&bars[0]);
  auto b_qfull = [&](int s) { return smem_u32(&bars[1 + s]); };
  auto b_qempty = [&](int s) { return smem_u32(&bars[1 + C::NSQ + s]); };
  auto b_sfull = [&](int b) { return smem_u32(&bars[1 + 2 * C::NSQ + b]); };   // S, beta in
  auto b_pgfull = [&](int b) { return smem_u32(&bars[3 + 2 * C::NSQ + b]); };  // P, gamma out
  auto b_pgdone = [&](int b) { return smem_u32(&bars[5 + 2 * C::NSQ + b]); };  // products done
  auto b_dqfull = [&](int b) { return smem_u32(&bars[7 + 2 * C::NSQ + b]); };  // dQ~^T in
  auto b_dqfree = [&](int b) { return smem_u32(&bars[9 + 2 * C::NSQ + b]); };  // dQ~^T read
  const uint32_t b_acc = smem_u32(&bars[11 + 2 * C::NSQ]);
  const uint32_t b_drain = smem_u32(&bars[12 + 2 * C::NSQ]);
  const uint32_t b_dqsfull = smem_u32(&bars[13 + 2 * C::NSQ]);
  const uint32_t b_dqsfree = smem_u32(&bars[14 + 2 * C::NSQ]);
  const uint32_t b_tab = smem_u32(&bars[15 + 2 * C::NSQ]);  // RoPE rows of the key tile landed
  const uint32_t b_ep = smem_u32(&bars[16 + 2 * C::NSQ]);   // dK / dV staging written
  const uint32_t b_drain2 = smem_u32(&bars[17 + 2 * C::NSQ]);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // grid (heads of a group, key tile, group): the CTAs are dispatched x fastest, so each
  // group of p.hgroup heads, whose Q~, l and dQ~ stay in L2 together, runs its longest key
  // tiles first (key tile 0 sees the most query tiles when causal) across all of its heads
  // and the grid ends on short CTAs
  // deterministic mode: the shortest key tiles (highest index when causal) are dispatched
  // first, and take their turn first on every query tile (see the drain)
  const int kt = p.turn ? p.nk - 1 - static_cast<int>(blockIdx.y) : static_cast<int>(blockIdx.y);
  const int bh = blockIdx.z * gridDim.x + blockIdx.x;  // gridDim.x = p.hgroup
  if (bh >= p.BH) return;  // the last group may hold fewer heads
  const int n = p.n;
  const int nqt = (n + C::BQ - 1) / C::BQ;
  const int i_start = p.causal ? (kt * C::BK) / C::BQ : 0;
  const int NI = nqt - i_start;
  const uint64_t lim = p.limit_ns;

  if (tid == 0) {
    mbar_init(b_kv, 1);
    for (int s = 0; s < C::NSQ; ++s) {
      mbar_init(b_qfull(s), 2);  // TMA bytes + the staged lse / delta
      mbar_init(b_qempty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(b_sfull(b), 1);
      mbar_init(b_pgfull(b), 256);
      mbar_init(b_pgdone(b), 1);
      mbar_init(b_dqfull(b), 1);
      mbar_init(b_dqfree(b), 128);
    }
    mbar_init(b_acc, 1);
    mbar_init(b_drain, 1);
    mbar_init(b_drain2, 1);
    mbar_init(b_dqsfull, 128);
    mbar_init(b_dqsfree, 1);
    mbar_init(b_tab, 1);
    mbar_init(b_ep, 256);
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
      tma_prefetch(&tm_l);
      tma_prefetch(&tm_dq);
      mbar_expect_tx(b_kv, 2 * C::KTILE);
      for (int b = 0; b < C::KB; ++b) {
        tma_load_3d(sbase + C::K_OFF + b * C::KBLK, &tm_k, b_kv, 64 * b, kt * C::BK, bh);
        tma_load_3d(sbase + C::V_OFF + b * C::KBLK, &tm_v, b_kv, 64 * b, kt * C::BK, bh);
      }
    }
    __syncwarp();
    int last = -1;
    for (int ii = 0; ii < NI; ++ii) {
      const int s = ii % C::NSQ;
      if (!mbar_wait_warp(b_qempty(s), ((ii / C::NSQ) & 1) ^ 1, abort_flag, lim)) break;
      const int q0 = (i_start + ii) * C::BQ;
      if (lane == 0) {
        mbar_expect_tx(b_qfull(s), 2 * C::QTILE);
        for (int b = 0; b < C::KB; ++b) {
          tma_load_3d(sbase + C::Q_OFF + s * C::QTILE + b * C::QBLK, &tm_q, b_qfull(s), 64 * b,
                      q0, bh);
          tma_load_3d(sbase + C::L_OFF + s * C::QTILE + b * C::QBLK, &tm_l, b_qfull(s), 64 * b,
                      q0, bh);
        }
      }
#pragma unroll
      for (int h = 0; h < C::BQ / 32; ++h) {
        const int c = lane + 32 * h, q = q0 + c;
        const float nl = q < n ? -(p.lse[(size_t)bh * n + q] * kLog2e) : 0.f;
        const float dz = q < n ? p.delta[(size_t)bh * n + q] : 0.f;
        // per column pair: (-lse_c log2 e, -lse_c+1 log2 e, delta_c, delta_c+1)
        const uint32_t pr = sbase + C::LD_OFF + (s * C::BQ + (c & ~1)) * 8 + (c & 1) * 4;
        st_shared_f32(pr, nl);
        st_shared_f32(pr + 8, dz);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(b_qfull(s));
      last = ii;
    }
    if (lane == 0 && abort_get(abort_flag)) {
      mbar_drain(b_kv, 0, lim);
      for (int ii = (last - C::NSQ + 1 > 0 ? last - C::NSQ + 1 : 0); ii <= last; ++ii)
        mbar_drain(b_qfull(ii % C::NSQ), (ii / C::NSQ) & 1, lim);
    }
  } else if (warp == C::W_MMA || warp == C::W_MMA2) {
    // ------------------------------------------------------------------ MMA issuers
    // Two issuing threads: warp W_MMA2 issues S^T and beta^T of every step, warp W_MMA the
    // gradient products.  A thread that issues tcgen05.mma is held at each issue until the
    // tensor pipe takes the product, so with one thread a wait for one chain (the drain
    // freeing beta^T's columns) also held the other (the next step's products).
    //   step i, buffer b = i % 2:  S^T_i once dV and dK of step i - 2 have read P^T, gamma^T
    //   over its columns; beta^T_i (d = 128) once the drain has read dQ~^T_i-2 over its
    //   columns; dV, dK (P^T, gamma^T from TMEM) then dQ~^T_i (over the beta^T columns, which
    //   the softmax warps have read) once P^T_i, gamma^T_i are written.  At d = 64 the pair
    //   products' dQ~ has columns of its own, so beta^T_i waits only for its query tile.
    // Both poll their barriers: a suspended wait resumes a few hundred cycles after the phase
    // completes, on the chain every step waits for.
    if (lane == 0) {
      constexpr uint32_t idesc_sb = idesc_bf16_f32(128, C::BQ, false, false);
      constexpr uint32_t idesc_kv = idesc_bf16_f32(128, D, false, true);
      constexpr uint32_t idesc_dq = idesc_bf16_f32(D, C::BQ, true, true);
      // descriptor low words per buffer (sw128_lo), offsets added per K step (sw128_at)
      const uint32_t ka_k = sw128_lo(sbase + C::K_OFF, 16), va_k = sw128_lo(sbase + C::V_OFF, 16);
      const uint32_t ka_mn = sw128_lo(sbase + C::K_OFF, C::KBLK);
      bool ok = mbar_wait_poll(b_kv, 0, abort_flag, lim);
      tc_fence_after();
      if (warp == C::W_MMA2) {
        // S^T (z = 0) or beta^T (z = 1) of step ii into its buffer
        auto issue_sb = [&](int ii, int z) {
          const int s = ii % C::NSQ;
          const uint32_t ab = z ? va_k : ka_k;
          const uint32_t bb = sw128_lo(sbase + (z ? C::L_OFF : C::Q_OFF) + s * C::QTILE, 16);
          const uint32_t d_acc = tmem + (ii & 1) * C::T_BUF + (z ? C::T_B : 0);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t ko = (kk >> 2) * C::KBLK + (kk & 3) * 32;
            const uint32_t qo = (kk >> 2) * C::QBLK + (kk & 3) * 32;
            mma_ss(d_acc, sw128_at(ab, ko), sw128_at(bb, qo), idesc_sb, kk > 0);
          }
        };
        for (int ii = 0; ok && ii < NI; ++ii) {
          const int b = ii & 1;
          const uint32_t pph = ((ii - 2) >> 1) & 1;  // phase of step ii - 2 in buffer b
          const int s = ii % C::NSQ;
          if (!(ok = mbar_wait_poll(b_qfull(s), (ii / C::NSQ) & 1, abort_flag, lim))) break;
          if (ii >= 2 && !(ok = mbar_wait_poll(b_pgdone(b), pph, abort_flag, lim))) break;
          tc_fence_after();
          issue_sb(ii, 0);
          if (!C::PAIR && ii >= 2 && !(ok = mbar_wait_poll(b_dqfree(b), pph, abort_flag, lim)))
            break;
          tc_fence_after();
          issue_sb(ii, 1);
          mma_commit(b_sfull(b));
        }
        if (!ok) {
          mma_commit(b_drain2);
          mbar_drain(b_drain2, 0, lim);
        }
      } else {
        for (int ii = 0; ok && ii < NI; ++ii) {
          const int s = ii % C::NSQ, b = ii & 1;
          if (!(ok = mbar_wait_poll(b_pgfull(b), (ii >> 1) & 1, abort_flag, lim))) break;
          tc_fence_after();
          const uint32_t buf = tmem + b * C::T_BUF;
          // dV += P^T l_i, dK += gamma^T Q~_i: M = 128 keys, N = D, K = 64 queries, with P^T
          // and gamma^T read from TMEM (two bf16 per column, 8 columns per K step of 16
          // queries: queries 16 kk .. of warpgroup kk / 2 at 32 (kk / 2) + 8 (kk % 2))
          const uint32_t qb_mn = sw128_lo(sbase + C::Q_OFF + s * C::QTILE, C::QBLK);
          const uint32_t lb_mn = sw128_lo(sbase + C::L_OFF + s * C::QTILE, C::QBLK);
#pragma unroll
          for (int kk = 0; kk < C::BQ / 16; ++kk) {
            const uint32_t pa = buf + 32 * (kk >> 1) + 8 * (kk & 1);
            mma_ts(tmem + C::T_DV, pa, sw128_at(lb_mn, kk * 2048), idesc_kv, (ii > 0 || kk > 0));
            mma_ts(tmem + C::T_DK, pa + C::T_GT, sw128_at(qb_mn, kk * 2048), idesc_kv,
                   (ii > 0 || kk > 0));
          }
          mma_commit(b_pgdone(b));
          mma_commit(b_qempty(s));
          if constexpr (!C::PAIR) {
            // dQ~_i^T = K~^T gamma^T (M = D, N = 64 queries, K = 128 keys) over the columns
            // beta^T held
            const uint32_t gt_mn = sw128_lo(sbase + C::G_OFF + b * C::PG, C::KBLK);
#pragma unroll
            for (int kk = 0; kk < C::BK / 16; ++kk)
              mma_ss(buf + C::T_DQ, sw128_at(ka_mn, kk * 2048), sw128_at(gt_mn, kk * 2048),
                     idesc_dq, kk > 0);
            mma_commit(b_dqfull(b));
          } else if ((ii & 1) || ii == NI - 1) {
            // dQ~ of query tiles 2 pr and 2 pr + 1 = gamma K~: M = 128 queries (A: the two
            // gamma^T slots, query-contiguous, 64 queries apart by PG), N = D, K = 128 keys
            // (B: K~, d-contiguous).  When NI is odd, the last product's rows 64-127 read a
            // stale slot and are not reduced.  Its buffer is free once the drain has read
            // pair pr - 2.
            constexpr uint32_t idesc_dqp = idesc_bf16_f32(128, D, true, true);
            const int pr = ii >> 1, pb = pr & 1;
            if (pr >= 2 && !(ok = mbar_wait_poll(b_dqfree(pb), ((pr - 2) >> 1) & 1, abort_flag,
                                                 lim)))
              break;
            tc_fence_after();
            const uint32_t ga = sw128_lo(sbase + C::G_OFF + ((2 * pr) % C::NG) * C::PG, C::PG);
#pragma unroll
            for (int kk = 0; kk < C::BK / 16; ++kk)
              mma_ss(tmem + C::T_DQP + pb * D, sw128_at(ga, kk * 2048),
                     sw128_at(ka_mn, kk * 2048), idesc_dqp, kk > 0);
            mma_commit(b_dqfull(pb));
          }
        }
        if (ok) {
          mma_commit(b_acc);
        } else {
          mma_commit(b_drain);
          mbar_drain(b_drain, 0, lim);
        }
      }
    }
  } else if (warp < C::W_DRAIN) {
    // ------------------------------------------------------------------ P^T, gamma^T
    // warp w reaches TMEM lanes 32 (w % 4) ...; warpgroup `half` takes query columns
    // 32 half .. 32 half + 31 of the 64
    const int row = tid & 127, half = warp >> 2;
    const int key = kt * C::BK + row;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    bool ok = true;
    for (int ii = 0; ii < NI; ++ii) {
      const int q0 = (i_start + ii) * C::BQ;
      const int stg = ii % C::NSQ, b = ii & 1;
      // the stage's lse / delta (and S^T, beta^T below) for this query tile
      if (!(ok = mbar_wait_warp(b_qfull(stg), (ii / C::NSQ) & 1, abort_flag, lim))) break;
      if (!(ok = mbar_wait_warp(b_sfull(b), (ii >> 1) & 1, abort_flag, lim))) break;
      tc_fence_after();
      // this warpgroup's 32 query columns of S^T and beta^T in step buffer b
      const uint32_t buf = tmem + lane_base + b * C::T_BUF + 32 * half;
      uint32_t sr[32], br[32];
      tmem_ld32(buf, sr);
      tmem_ld32(buf + C::T_B, br);
      tmem_wait_ld();
      const uint32_t ld_row = sbase + C::LD_OFF + (stg * C::BQ + 32 * half) * 8;
      const int qh = q0 + 32 * half;
      const bool full = key < n && qh + 32 <= n && (!p.causal || key <= qh);
      uint32_t pw[16], gw[16];
      const uint64_t sc2 = f32x2(p.scale_log2, p.scale_log2);
#pragma unroll
      for (int h = 0; h < 16; ++h) {
        const int c = 2 * h;
        // (-lse_c log2 e, -lse_c+1 log2 e, delta_c, delta_c+1): two columns per packed op
        const float4 lz = ld_shared_v4f(ld_row + h * 16);
        const float2 y = unpack_f32x2(
            ffma2(f32x2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sc2,
                  f32x2(lz.x, lz.y)));
        const float p0 = ex2(y.x), p1 = ex2(y.y);
        const float2 g = unpack_f32x2(
            fmul2(f32x2(p0, p1), fsub2(f32x2(__uint_as_float(br[c]), __uint_as_float(br[c + 1])),
                                       f32x2(lz.z, lz.w))));
        pw[h] = pack_bf16x2(p0, p1);
        gw[h] = pack_bf16x2(g.x, g.y);
      }
      // Pairs past n or above the causal diagonal (only warps that reach the diagonal or
      // the ragged end): their P and gamma become +0, whatever was computed there
      if (!__all_sync(0xffffffffu, full)) {
#pragma unroll
        for (int h = 0; h < 16; ++h) {
          const int q = qh + 2 * h;
          const bool v0 = key < n && q < n && (!p.causal || key <= q);
          const bool v1 = key < n && q + 1 < n && (!p.causal || key <= q + 1);
          const uint32_t keep = (v0 ? 0x0000FFFFu : 0u) | (v1 ? 0xFFFF0000u : 0u);
          pw[h] &= keep;
          gw[h] &= keep;
        }
      }
      // P^T and gamma^T over the S^T columns this warpgroup has just read (the products of
      // step i - 2, which read this buffer and gamma^T slot i % NG, completed before S^T of
      // step i was issued; at d = 64 the pair product that read the slot was issued before
      // dV and dK of step i - 2, whose completion S^T of step i waits for)
      tmem_st16(buf, pw);
      tmem_st16(buf + C::T_GT, gw);
      const uint32_t gsm = sbase + C::G_OFF + (ii % C::NG) * C::PG;
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8)
        st_shared_v4(gsm + sw128_offset(row, 4 * half + c8), gw[4 * c8], gw[4 * c8 + 1],
                     gw[4 * c8 + 2], gw[4 * c8 + 3]);
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(b_pgfull(b));
    }
    // ---- dK = rot^-1(scale * sum gamma^T Q~) (warps 0-3), dV = sum P^T l (warps 4-7):
    //      one key row per thread.  Once every product has completed, K~, V and the query
    //      stages are free: the RoPE (cos, sin) rows of this key tile come in by TMA over
    //      K~ / V, and dK, dV are staged (128-byte swizzle) over the query stages and leave by
    //      TMA stores (per-thread rows of 16-byte accesses would be uncoalesced).
    if (ok) ok = mbar_wait_warp(b_acc, 0, abort_flag, lim);
    const uint32_t tab_s = sbase + C::K_OFF;
    const uint32_t stg = sbase + C::Q_OFF + half * C::KTILE;
    const bool tab_issued = ok && tid == 0;
    if (tab_issued) {
      mbar_expect_tx(b_tab, C::TABT);
      for (int b = 0; b < D / 32; ++b)
        tma_load_2d(tab_s + b * C::TBLK, &tm_tab, b_tab, 32 * b, kt * C::BK);
    }
    if (ok && half == 0) ok = mbar_wait_warp(b_tab, 0, abort_flag, lim);
    // after an abort, the copy this thread issued lands before the CTA leaves
    if (tab_issued && !ok) mbar_drain(b_tab, 0, lim);
    if (ok) {
      tc_fence_after();
      const uint32_t src = tmem + lane_base + (half == 0 ? C::T_DK : C::T_DV);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(src + 32 * c, r);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int k = 0; k < 16; k += 2) {
          const float x0 = __uint_as_float(r[2 * k]), x1 = __uint_as_float(r[2 * k + 1]);
          const float x2 = __uint_as_float(r[2 * k + 2]), x3 = __uint_as_float(r[2 * k + 3]);
          if (half == 0) {
            // pairs 16 c + k, 16 c + k + 1: (cos, sin, cos, sin), rotation by -phi
            const float4 cs = ld_shared_v4f(tab_s + c * C::TBLK + sw128_offset(row, k >> 1));
            const float y0 = x0 * p.scale, y1 = x1 * p.scale, y2 = x2 * p.scale, y3 = x3 * p.scale;
            w[k] = pack_bf16x2(y0 * cs.x + y1 * cs.y, -y0 * cs.y + y1 * cs.x);
            w[k + 1] = pack_bf16x2(y2 * cs.z + y3 * cs.w, -y2 * cs.w + y3 * cs.z);
          } else {
            w[k] = pack_bf16x2(x0, x1);
            w[k + 1] = pack_bf16x2(x2, x3);
          }
        }
        // output columns 32 c .. 32 c + 31: 64-column box c / 2, 16-byte chunks 4 (c % 2) ..
#pragma unroll
        for (int v = 0; v < 4; ++v)
          st_shared_v4(stg + (c >> 1) * C::KBLK + sw128_offset(row, 4 * (c & 1) + v), w[4 * v],
                       w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
      }
    }
    fence_proxy_async_smem();
    mbar_arrive(b_ep);
    if (tid == 0 && ok && mbar_wait(b_ep, 0, abort_flag, lim)) {
      for (int b = 0; b < D / 64; ++b) {
        tma_store_3d(&tm_dk, sbase + C::Q_OFF + b * C::KBLK, 64 * b, kt * C::BK, bh);
        tma_store_3d(&tm_dv, sbase + C::Q_OFF + C::KTILE + b * C::KBLK, 64 * b, kt * C::BK, bh);
      }
      bulk_commit();
      // the stores have read the staging before the CTA leaves (their writes complete with
      // the kernel)
      bulk_wait_read0();
    }
  } else {
    // ------------------------------------------------------------------ dQ~ drain (warps 8-11)
    const int wq = warp - C::W_DRAIN;
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t stage = sbase + C::DQS_OFF;
    const bool issuer = tid == 32 * C::W_DRAIN;
    int passed = 0;  // query tiles whose turn this key tile has passed on (deterministic mode)
    if constexpr (!C::PAIR) {
      // accumulator row (head-dimension index) held by this lane: M = 128 puts row r in lane
      // r, M = 64 puts row r in lane (r % 16) + 32 (r / 16)
      const int drow = (D == 128) ? (wq * 32 + lane) : (wq * 16 + lane);
      const bool has_row = (D == 128) || lane < 16;
      for (int ii = 0; ii < NI; ++ii) {
        const int b = ii & 1;
        // polled: the MMA issuer waits for this drain before it can issue beta^T two steps on
        if (!mbar_wait_warp_poll(b_dqfull(b), (ii >> 1) & 1, abort_flag, lim)) break;
        tc_fence_after();
        uint32_t r0[32], r1[32];
        const uint32_t dq = tmem + lane_base + b * C::T_BUF + C::T_DQ;
        tmem_ld32(dq, r0);
        tmem_ld32(dq + 32, r1);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(b_dqfree(b));
        // the staging tile is free once the previous bulk reduction has read it
        if (!mbar_wait_warp(b_dqsfree, (ii & 1) ^ 1, abort_flag, lim)) break;
        if (has_row) {
          // row-major [q][d] fp32: for one q the lanes write consecutive d
  #pragma unroll
          for (int c = 0; c < 32; ++c) {
            st_shared_f32(stage + (c * D + drow) * 4, __uint_as_float(r0[c]));
            st_shared_f32(stage + ((32 + c) * D + drow) * 4, __uint_as_float(r1[c]));
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(b_dqsfull);
        bool iok = true;
        if (issuer) {
          iok = mbar_wait(b_dqsfull, ii & 1, abort_flag, lim);
          if (iok && p.turn) {
            // deterministic mode: query tile q gets the parts of key tiles kmax(q), kmax(q) - 1,
            // ..., 0 in that order (all of them contribute to it), so key tile kt adds its part
            // once kmax(q) - kt others have.  Those others were dispatched before this CTA and
            // reach q two query tiles sooner.  The turn of a tile passes on once its reduction
            // has landed, checked TURN_LAG steps later (when at most the TURN_LAG newer ones are
            // in flight: the key tile after this one in the order reaches q later still).
            const int q = i_start + ii;
            const int kmax = p.causal ? min(p.nk - 1, (q * C::BQ + C::BQ - 1) / C::BK) : p.nk - 1;
            unsigned* tc = p.turn + (size_t)bh * p.turn_stride + q;
            if (turn_wait(tc, static_cast<unsigned>(kmax - kt), lim)) {
              fence_proxy_async_global();
              tma_reduce_add_3d(&tm_dq, stage, 0, (i_start + ii) * C::BQ, bh);
              bulk_commit();
              bulk_wait_read0();
              mbar_arrive(b_dqsfree);
              if (passed <= ii - C::TURN_LAG) {
                bulk_wait_n<C::TURN_LAG>();
                fence_proxy_async_global();
                turn_pass(tc - (ii - passed));
                ++passed;
              }
            } else {
              abort_set(abort_flag, 1);  // given up: the turns still pass, the status says so
              iok = false;
              mbar_arrive(b_dqsfree);
            }
          } else if (iok) {
            tma_reduce_add_3d(&tm_dq, stage, 0, (i_start + ii) * C::BQ, bh);
            bulk_commit();
            bulk_wait_read0();
            mbar_arrive(b_dqsfree);
          }
        }
        if (!__all_sync(0xffffffffu, iok)) break;  // leave the loop together
      }
    } else {
      // d = 64: one pair of query tiles per product, lanes = queries 0-127 of the pair (tiles
      // 2 pr, 2 pr + 1), 64 columns = d.  Each lane writes its row as 16-byte chunks in the
      // 128-byte swizzle (chunk j of row q at j ^ (q % 8)), so a warp's stores spread over
      // all banks; each query tile then leaves as two [64 rows][32 columns] reductions.
      int issued = 0;  // query tiles whose reduction has been issued
      const int NP = (NI + 1) / 2;
      const int q = wq * 32 + lane;
      const uint32_t qrow = stage + (q >> 6) * C::DQ_HALF + (q & 63) * 128;
      const uint32_t sw = static_cast<uint32_t>(q & 7);
      for (int pr = 0; pr < NP; ++pr) {
        const int pb = pr & 1;
        // suspended, not polled: no product waits for this drain except the pair product two
        // pairs on, and polling took issue slots from the softmax warps (0.7 % at d = 64)
        if (!mbar_wait_warp(b_dqfull(pb), (pr >> 1) & 1, abort_flag, lim)) break;
        tc_fence_after();
        uint32_t r0[32], r1[32];
        const uint32_t dq = tmem + lane_base + C::T_DQP + pb * D;
        tmem_ld32(dq, r0);
        tmem_ld32(dq + 32, r1);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(b_dqfree(pb));
        // the staging tile is free once the previous bulk reductions have read it
        if (!mbar_wait_warp(b_dqsfree, (pr & 1) ^ 1, abort_flag, lim)) break;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t off = (static_cast<uint32_t>(j) ^ sw) << 4;
          st_shared_v4(qrow + off, r0[4 * j], r0[4 * j + 1], r0[4 * j + 2], r0[4 * j + 3]);
          st_shared_v4(qrow + C::DQ_BOX + off, r1[4 * j], r1[4 * j + 1], r1[4 * j + 2],
                       r1[4 * j + 3]);
        }
        fence_proxy_async_smem();
        mbar_arrive(b_dqsfull);
        bool iok = true;
        if (issuer) {
          iok = mbar_wait(b_dqsfull, pr & 1, abort_flag, lim);
          for (int h = 0; iok && h < 2 && 2 * pr + h < NI; ++h) {
            const int qt = i_start + 2 * pr + h;
            if (p.turn) {
              // deterministic mode: as for d = 128 above, per query tile
              const int kmax = p.causal ? min(p.nk - 1, (qt * C::BQ + C::BQ - 1) / C::BK)
                                        : p.nk - 1;
              unsigned* tc = p.turn + (size_t)bh * p.turn_stride + qt;
              if (!turn_wait(tc, static_cast<unsigned>(kmax - kt), lim)) {
                abort_set(abort_flag, 1);  // given up: the turns still pass, the status says so
                iok = false;
                break;
              }
              fence_proxy_async_global();
            }
            const uint32_t src = stage + h * C::DQ_HALF;
            tma_reduce_add_3d(&tm_dq, src, 0, qt * C::BQ, bh);
            tma_reduce_add_3d(&tm_dq, src + C::DQ_BOX, 32, qt * C::BQ, bh);
            bulk_commit();
            ++issued;
            while (p.turn && passed + C::TURN_LAG < issued) {
              bulk_wait_n<C::TURN_LAG>();
              fence_proxy_async_global();
              turn_pass(p.turn + (size_t)bh * p.turn_stride + i_start + passed);
              ++passed;
            }
          }
          bulk_wait_read0();
          mbar_arrive(b_dqsfree);
        }
        if (!__all_sync(0xffffffffu, iok)) break;  // leave the loop together
      }
    }
    if (issuer) bulk_wait_read0();  // the reductions have read the staging tile
    if (issuer && p.turn) {
      // the last tile's reduction has landed; after an abort, the query tiles this key tile
      // has not added to pass their turn all the same, so the key tiles after it do not wait
      // out their limit
      bulk_wait0();
      fence_proxy_async_global();
      for (int q = passed; q < NI; ++q) turn_pass(p.turn + (size_t)bh * p.turn_stride + i_start + q);
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
