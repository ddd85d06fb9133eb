// fa_bwd_dkdv_sm100.cuh -- dK and dV of the attention backward on sm_100a, for the backward
// that takes dQ from the query-stationary kernel (fa_bwd_dq_sm100.cuh) instead of atomics.
//
// Derivative of O = softmax(S) V ("Attention optimisation: FlashAttention and sparse
// attention", mdooai Ch.04, core formula), in the recompute form:
//   P_ij  = 2^(s_ij * scale2 - lse_i * log2 e)            (0 for masked keys)
//   dV_j  = sum_i P_ij dO_i
//   dP_ij = dO_i . v_j
//   dS_ij = P_ij (dP_ij - Dvec_i),  Dvec_i = dO_i . O_i
//   dK_j  = scale * sum_i dS_ij q_i
//
// One CTA owns 128 keys (K and V stay in shared memory) and walks the query tiles that can see
// them, for every query head that reads its K/V head.  Per query tile t of 128 rows:
//   S^T(t)  = K Q^T   (M=128 keys, N=128, K=D)  smem x smem -> TMEM S[t%SB]
//   dP^T(t) = V dO^T  (M=128, N=128, K=D)       smem x smem -> TMEM dP
//   compute warpgroups (two, each owning 64 of the query columns): P^T in bf16 over the front
//     half of its own S^T columns, dS^T in bf16 over the front half of its dP^T columns
//   dV += P^T dO      (M=128, N=D, K=128)       TMEM x smem -> TMEM
//   dK += dS^T Q      (M=128, N=D, K=128)       TMEM x smem -> TMEM
// Without a dQ accumulator in TMEM every MMA has N = 128 (the smem operands stream at the
// tensor pipe's rate; N = 64 smem x smem MMAs are bound by shared-memory bandwidth).
// MMA order per tile t: dV(t) [P(t) ready], then the next scores into S (after dV(t) has read
// P(t) there -- MMAs of one thread execute in issue order), dK(t) [dS(t) ready], then dP(t+1)
// into dP (after dK(t)).  At d = 64 S is double-buffered (SB = 2) and S(t+2) follows dV(t).
//
// TMEM (512 columns): d = 128: S [0,128) dP [128,256) dV [256,384) dK [384,512); d = 64: S0
// [0,128) S1 [128,256) dP [256,384) dV [384,448) dK [448,512).
// CTA: 320 threads.  warps 0-7 compute, warp 8 TMA producer, warp 9 MMA issuer.
#pragma once
#include "fa_bwd_sm100.cuh"
#include "ptx.cuh"

namespace fa {

template <int D>
struct BwdDkdvLayout {
  static constexpr int BN = 128;                  // keys per CTA
  static constexpr int BM = 128;                  // query rows per step
  static constexpr int SB = D == 64 ? 2 : 1;      // S buffers
  // Q/dO/lse/Dvec stages: the scores of step t+SB are issued at step t, so stage (t+SB)%QST
  // must have been released (after dK(t+SB-QST)) and reloaded by then
  static constexpr int QST = D == 64 ? 4 : 2;
  static constexpr int DPB = 1;                   // dP buffers
  static constexpr int SUB = D / 64;
  static constexpr int KV_SUBTILE = 128 * 128;
  static constexpr int Q_SUBTILE = BM * 128;
  static constexpr int KV_TILE = 128 * D * 2;
  static constexpr int Q_TILE = BM * D * 2;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_TILE;
  static constexpr int OFF_Q = OFF_V + KV_TILE;
  static constexpr int OFF_DO = OFF_Q + QST * Q_TILE;
  static constexpr int OFF_LSE = OFF_DO + QST * Q_TILE;
  static constexpr int OFF_DVEC = OFF_LSE + QST * BM * 4;
  static constexpr int OFF_BAR = OFF_DVEC + QST * BM * 4;
  // kv, q_full[QST], q_empty[QST], s_full[SB], dp_full[DPB], p_full[2], ds_full[2], done, fin
  static constexpr int NBAR = 1 + 2 * QST + SB + DPB + 2 + 2 + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = BYTES + 1024;
  static constexpr int THREADS = 320;
  static constexpr int HALF = BM / 2;               // query columns per compute warpgroup
  static constexpr int NCH = HALF / 32;             // 32-column chunks per compute warpgroup
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t DP_COL0 = SB * BM;
  static constexpr uint32_t DV_COL = SB * BM + DPB * BM;
  static constexpr uint32_t DK_COL = DV_COL + D;
  __device__ static constexpr uint32_t s_col(int t) { return static_cast<uint32_t>(t % SB) * BM; }
  __device__ static constexpr uint32_t dp_col(int t) {
    return DP_COL0 + static_cast<uint32_t>(t % DPB) * BM;
  }
  static_assert(DK_COL + D <= TMEM_COLS, "TMEM budget");
};

enum : int {
  SITE_DKDV_LOAD_EMPTY = 61, SITE_DKDV_LOAD_DRAIN = 62, SITE_DKDV_MMA_KV = 63,
  SITE_DKDV_MMA_Q = 64, SITE_DKDV_MMA_P = 65, SITE_DKDV_MMA_DS = 66, SITE_DKDV_MMA_FIN = 67,
  SITE_DKDV_C_Q = 68, SITE_DKDV_C_S = 69, SITE_DKDV_C_DP = 70, SITE_DKDV_C_DONE = 71
};

template <int D>
__global__ void __launch_bounds__(320, 1)
fa_bwd_dkdv_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_do,
                         const __grid_constant__ CUtensorMap tm_dk,
                         const __grid_constant__ CUtensorMap tm_dv, const BwdParams p) {
  using L = BwdDkdvLayout<D>;
  constexpr int BM = L::BM;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* bar_kv = bars;
  uint64_t* bar_qf = bars + 1;
  uint64_t* bar_qe = bar_qf + L::QST;
  uint64_t* bar_s = bar_qe + L::QST;     // [SB]: S^T(t) in buffer t%SB
  uint64_t* bar_dp = bar_s + L::SB;      // [DPB]: dP^T(t) in buffer t%DPB
  uint64_t* bar_p = bar_dp + L::DPB;     // [2]: P^T(t) in TMEM, by t%2 (P(t+1) can be ready
                                         // before the MMA warp has waited for P(t))
  uint64_t* bar_ds = bar_p + 2;          // [2]: dS^T(t) in TMEM, by t%2
  uint64_t* bar_done = bar_ds + 2;
  uint64_t* bar_fin = bar_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
  const float* s_lse = reinterpret_cast<const float*>(smem + L::OFF_LSE);
  const float* s_dvec = reinterpret_cast<const float*>(smem + L::OFF_DVEC);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = p.H / p.H_kv;                          // query heads per K/V head
  const int BHkv = p.B * p.H_kv;
  // CTA order: groups of p.hgroup K/V heads in turn (a group's Q and dO fit in half of L2, so
  // the re-reads of Q and dO by the KV tiles of a head hit L2), and inside a group the KV tiles
  // with the most query tiles (small jt) first.
  const int per_group = p.hgroup * p.n_ktiles;
  const int grp = static_cast<int>(blockIdx.x) / per_group;
  const int g0 = grp * p.hgroup;
  const int gn = min(p.hgroup, BHkv - g0);              // heads in this group (the last may have fewer)
  const int rr = static_cast<int>(blockIdx.x) - grp * per_group;
  const int jt = rr / gn;                               // KV tile
  const int bhk = g0 + rr % gn;                         // (b, K/V head)
  const int b = bhk / p.H_kv;
  const int bhq0 = b * p.H + (bhk % p.H_kv) * G;       // first query head of the group
  const int N = p.N;
  const int k0 = jt * 128;
  int kvlen = N;
  if (p.kv_len != nullptr) kvlen = min(max(p.kv_len[b], 0), N);
  const int nb = (N + 127) / 128;
  const int n_qt = (N + BM - 1) / BM;
  const bool kv_live = k0 < kvlen;

  // query tile `it` (rows it*BM ..) has at least one (row, key) pair with this KV tile
  auto q_active = [&](int it) -> bool {
    if (!kv_live) return false;
    const int i0 = it * BM;
    if (p.causal && i0 + BM - 1 < k0) return false;
    if (p.block_mask != nullptr && !p.block_mask[static_cast<size_t>(i0 >> 7) * nb + jt])
      return false;
    return true;
  };
  // Work item w: query head g = w / span, query tile it_first + w % span.
  const int it_first = p.causal ? k0 / BM : 0;
  const int span = n_qt - it_first;
  int n_steps = 0;
  if (p.block_mask == nullptr) n_steps = kv_live ? span : 0;
  else for (int it = it_first; it < n_qt; ++it) n_steps += q_active(it) ? 1 : 0;
  n_steps *= G;

  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    for (int s = 0; s < L::QST; ++s) {
      mbar_init(&bar_qf[s], 1);
      mbar_init(&bar_qe[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_p[i], 256);
      mbar_init(&bar_ds[i], 256);
    }
    for (int i = 0; i < L::SB; ++i) mbar_init(&bar_s[i], 1);
    for (int i = 0; i < L::DPB; ++i) mbar_init(&bar_dp[i], 1);
    mbar_init(bar_done, 1);
    mbar_init(bar_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && n_steps > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(bar_kv, 2 * L::KV_TILE);
      for (int s = 0; s < L::SUB; ++s) {
        tma_load_3d(smem + L::OFF_K + s * L::KV_SUBTILE, &tm_k, bar_kv, s * 64, k0, bhk);
        tma_load_3d(smem + L::OFF_V + s * L::KV_SUBTILE, &tm_v, bar_kv, s * 64, k0, bhk);
      }
      int t = 0;
      for (int w = 0; w < G * span; ++w) {
        const int g = w / span;
        const int it = it_first + (w - g * span);
        if (!q_active(it)) continue;
        const int bh = bhq0 + g;
        const int st = t % L::QST;
        if (t >= L::QST &&
            !mbar_wait(&bar_qe[st], ((t / L::QST) - 1) & 1, abort_flag, SITE_DKDV_LOAD_EMPTY))
          break;
        const int i0 = it * BM;
        mbar_arrive_expect_tx(&bar_qf[st], 2 * L::Q_TILE + 2 * BM * 4);
        for (int s = 0; s < L::SUB; ++s) {
          tma_load_3d(smem + L::OFF_Q + st * L::Q_TILE + s * L::Q_SUBTILE, &tm_q, &bar_qf[st],
                      s * 64, i0, bh);
          tma_load_3d(smem + L::OFF_DO + st * L::Q_TILE + s * L::Q_SUBTILE, &tm_do, &bar_qf[st],
                      s * 64, i0, bh);
        }
        const size_t off = static_cast<size_t>(bh) * p.N_pad + i0;
        bulk_load(smem + L::OFF_LSE + st * BM * 4, p.lse2 + off, BM * 4, &bar_qf[st]);
        bulk_load(smem + L::OFF_DVEC + st * BM * 4, p.dvec + off, BM * 4, &bar_qf[st]);
        ++t;
      }
      mbar_wait(bar_kv, 0, abort_flag, SITE_DKDV_LOAD_DRAIN);
      for (int r = max(0, t - L::QST); r < t; ++r)
        mbar_wait(&bar_qf[r % L::QST], (r / L::QST) & 1, abort_flag, SITE_DKDV_LOAD_DRAIN);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA issuer
    // The whole warp walks the loop (descriptors stay warp-uniform); one elected lane issues
    // the MMAs four at a time.
    if (n_steps > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, BM, false, false);
      constexpr uint32_t idesc_g = idesc_bf16_f32(128, D, false, true);
      const uint32_t k_addr = smem_u32(smem + L::OFF_K);
      const uint32_t v_addr = smem_u32(smem + L::OFF_V);
      const uint32_t q_addr = smem_u32(smem + L::OFF_Q);
      const uint32_t do_addr = smem_u32(smem + L::OFF_DO);
      const uint64_t k_kd = sdesc_sw128(k_addr, 16, 1024);
      const uint64_t v_kd = sdesc_sw128(v_addr, 16, 1024);
      const uint64_t q_kd = sdesc_sw128(q_addr, 16, 1024);
      const uint64_t do_kd = sdesc_sw128(do_addr, 16, 1024);
      const uint64_t q_mn = sdesc_sw128(q_addr, L::Q_SUBTILE, 1024);
      const uint64_t do_mn = sdesc_sw128(do_addr, L::Q_SUBTILE, 1024);
      auto off16 = [](int bytes) -> uint64_t { return static_cast<uint64_t>(bytes >> 4); };
      // X^T = A B^T over D: A = K or V (128 rows), B = Q or dO of stage st (BM rows), K-major.
      auto mma_scores = [&](uint64_t a_desc, uint64_t b_desc, int st, uint32_t d_col) {
        const uint64_t bst = b_desc + off16(st * L::Q_TILE);
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb) {
          uint64_t a[4], bb[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int k = 4 * kb + i;
            a[i] = a_desc + off16((k >> 2) * L::KV_SUBTILE + (k & 3) * 32);
            bb[i] = bst + off16((k >> 2) * L::Q_SUBTILE + (k & 3) * 32);
          }
          mma_ss_x4(tmem + d_col, a, bb, idesc_s, kb > 0 ? 1u : 0u);
        }
      };
      // G += X^T(TMEM, bf16) B over BM rows: B = dO or Q of stage st, MN-major.  Query columns
      // [16k, 16k+16) of X^T were written by compute warpgroup h = 16k / HALF into the front
      // half of its own columns.
      auto mma_grad = [&](uint32_t a_col, uint64_t b_desc, int st, uint32_t d_col, bool acc) {
        const uint64_t bst = b_desc + off16(st * L::Q_TILE);
#pragma unroll
        for (int kb = 0; kb < BM / 64; ++kb) {
          uint32_t a[4];
          uint64_t bb[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int k = 4 * kb + i;
            const uint32_t h = static_cast<uint32_t>((16 * k) / L::HALF);
            a[i] = tmem + a_col + 8u * k + h * (L::HALF / 2);
            bb[i] = bst + off16(k * 2048);
          }
          mma_ts_x4(tmem + d_col, a, bb, idesc_g, (acc || kb > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait_w(bar_kv, 0, abort_flag, SITE_DKDV_MMA_KV);
      ok = ok && mbar_wait_w(&bar_qf[0], 0, abort_flag, SITE_DKDV_MMA_Q);
      tc_fence_after();
      if (ok) {
        mma_scores(k_kd, q_kd, 0, L::s_col(0));
        mma_commit_w(&bar_s[0]);
        mma_scores(v_kd, do_kd, 0, L::dp_col(0));
        mma_commit_w(&bar_dp[0]);
        if (L::SB == 2 && n_steps > 1) {
          ok = mbar_wait_w(&bar_qf[1], 0, abort_flag, SITE_DKDV_MMA_Q);
          tc_fence_after();
          if (ok) {
            mma_scores(k_kd, q_kd, 1, L::s_col(1));
            mma_commit_w(&bar_s[1 % L::SB]);
          }
        }
      }
      for (int t = 0; ok && t < n_steps; ++t) {
        const int st = t % L::QST;
        const int pb = t & 1;
        if (!mbar_wait_w(&bar_p[pb], (t >> 1) & 1, abort_flag, SITE_DKDV_MMA_P)) { ok = false; break; }
        tc_fence_after();
        mma_grad(L::s_col(t), do_mn, st, L::DV_COL, t > 0);
        const int ts = t + L::SB;       // the scores issued now, into the buffer dV(t) just read
        if (ts < n_steps) {
          const int sts = ts % L::QST;
          if (!mbar_wait_w(&bar_qf[sts], (ts / L::QST) & 1, abort_flag, SITE_DKDV_MMA_Q)) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_scores(k_kd, q_kd, sts, L::s_col(ts));
          mma_commit_w(&bar_s[ts % L::SB]);
        }
        if (!mbar_wait_w(&bar_ds[pb], (t >> 1) & 1, abort_flag, SITE_DKDV_MMA_DS)) { ok = false; break; }
        tc_fence_after();
        mma_grad(L::dp_col(t), q_mn, st, L::DK_COL, t > 0);
        mma_commit_w(&bar_qe[st]);  // Q(t), dO(t), lse(t), Dvec(t) are no longer read after dK(t)
        if (t + 1 < n_steps) {        // dP(t+1) after dK(t) has read dS(t) from dP
          mma_scores(v_kd, do_kd, (t + 1) % L::QST, L::dp_col(t + 1));
          mma_commit_w(&bar_dp[(t + 1) % L::DPB]);
        }
      }
      mma_commit_w(bar_done);
      mma_commit_w(bar_fin);
      mbar_wait_w(bar_fin, 0, abort_flag, SITE_DKDV_MMA_FIN);
    }
  } else {
    // ------------------------------------------------------------------ compute warpgroups
    const int h = warp >> 2;                  // which half of the query columns
    const int qw = warp & 3;
    const int jl = 32 * qw + lane;            // key row within the tile (= TMEM lane)
    const int kj = k0 + jl;                   // key index
    const uint32_t t_lane = static_cast<uint32_t>(32 * qw) << 16;
    const float scale2 = p.scale2;
    bool ok = true;
    int t = 0;
    for (int w = 0; w < G * span; ++w) {
      const int g = w / span;
      const int it = it_first + (w - g * span);
      if (!q_active(it)) continue;
      const int st = t % L::QST;
      const int pb = t & 1;
      const int i0 = it * BM;
      const int c0 = h * L::HALF;             // first query column of this warpgroup
      const uint32_t s_cols = tmem + t_lane + L::s_col(t) + c0;      // my S^T columns
      const uint32_t dp_cols = tmem + t_lane + L::dp_col(t) + c0;   // my dP^T columns
      bool got = mbar_wait(&bar_qf[st], (t / L::QST) & 1, abort_flag, SITE_DKDV_C_Q);
      got = got && mbar_wait(&bar_s[t % L::SB], (t / L::SB) & 1, abort_flag, SITE_DKDV_C_S);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
      const float4* lse4 = reinterpret_cast<const float4*>(s_lse + st * BM + c0);
      const float4* dv4 = reinterpret_cast<const float4*>(s_dvec + st * BM + c0);
      const bool edge = (k0 + 128 > kvlen) || (p.causal && k0 + 32 * qw + 31 > i0 + c0);
      // ---- P = 2^(s*scale2 - lse2): bf16 into TMEM for dV, fp32 kept for dS
      float pf[L::NCH * 32];
#pragma unroll
      for (int c = 0; c < L::NCH; ++c) {
        uint32_t sr[32];
        tmem_ld32(s_cols + 32 * c, sr);
        tmem_ld_wait();
        reg_fence(sr);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float4 l4 = lse4[8 * c + u];
          float x[4];
          ffma2(x[0], x[1], __uint_as_float(sr[4 * u]), __uint_as_float(sr[4 * u + 1]), scale2,
                scale2, -l4.x, -l4.y);
          ffma2(x[2], x[3], __uint_as_float(sr[4 * u + 2]), __uint_as_float(sr[4 * u + 3]),
                scale2, scale2, -l4.z, -l4.w);
#pragma unroll
          for (int e = 0; e < 4; ++e) pf[32 * c + 4 * u + e] = ex2_approx(x[e]);
        }
        if (edge) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int qi = i0 + c0 + 32 * c + i;
            if (kj >= kvlen || (p.causal && kj > qi)) pf[32 * c + i] = 0.f;
          }
        }
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(pf[32 * c + 2 * i], pf[32 * c + 2 * i + 1]);
        tmem_st16(s_cols + 16 * c, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bar_p[pb]);
      // ---- dS = P (dP - Dvec): bf16 into TMEM over my dP^T columns
      got = mbar_wait(&bar_dp[t % L::DPB], (t / L::DPB) & 1, abort_flag, SITE_DKDV_C_DP);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < L::NCH; ++c) {
        uint32_t dr[32];
        tmem_ld32(dp_cols + 32 * c, dr);
        tmem_ld_wait();
        reg_fence(dr);
        uint32_t dd[16];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float4 d4 = dv4[8 * c + u];
          const int i = 32 * c + 4 * u;
          dd[2 * u] = pack_bf16x2(pf[i] * (__uint_as_float(dr[4 * u]) - d4.x),
                                  pf[i + 1] * (__uint_as_float(dr[4 * u + 1]) - d4.y));
          dd[2 * u + 1] = pack_bf16x2(pf[i + 2] * (__uint_as_float(dr[4 * u + 2]) - d4.z),
                                      pf[i + 3] * (__uint_as_float(dr[4 * u + 3]) - d4.w));
        }
        tmem_st16(dp_cols + 16 * c, dd);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bar_ds[pb]);
      ++t;
    }
    // ---------------------------------------------------------------- epilogue: dK, dV
    // warpgroup 0 writes dV, warpgroup 1 writes dK (x scale)
    if (ok && n_steps > 0) {
      const bool got = mbar_wait(bar_done, 0, abort_flag, SITE_DKDV_C_DONE);
      ok = __all_sync(0xffffffffu, got);
      tc_fence_after();
    }
    if (ok) {
      // This warp's 32 key rows are staged as D/64 [32 rows][64 d] bf16 boxes with the 128-byte
      // swizzle (16-byte chunk c of row r at chunk c ^ (r & 7)) in the Q ring, which no MMA or
      // load touches any more (bar_done follows the last MMA), and written by one TMA store per
      // box (rows past N are not written) instead of one memory transaction per lane and store.
      const uint32_t col0 = h == 0 ? L::DV_COL : L::DK_COL;
      const float mul = h == 0 ? 1.0f : p.scale;
      uint8_t* stg = smem + L::OFF_Q + warp * (D / 64) * 4096;
      static_assert(8 * (D / 64) * 4096 <= L::QST * L::Q_TILE, "dK/dV staging fits the Q ring");
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t gr[32];
        if (n_steps > 0) {
          tmem_ld32(tmem + t_lane + col0 + 32 * c, gr);
          tmem_ld_wait();
          reg_fence(gr);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) gr[i] = 0u;
        }
        uint32_t hv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          hv[i] = pack_bf16x2(__uint_as_float(gr[2 * i]) * mul, __uint_as_float(gr[2 * i + 1]) * mul);
        uint8_t* box = stg + (c >> 1) * 4096 + lane * 128;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int q = (c & 1) * 4 + i;  // 16-byte chunk of the 128-byte row
          *reinterpret_cast<uint4*>(box + ((q ^ (lane & 7)) * 16)) =
              make_uint4(hv[4 * i], hv[4 * i + 1], hv[4 * i + 2], hv[4 * i + 3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
#pragma unroll
        for (int s = 0; s < D / 64; ++s)
          tma_store_3d(h == 0 ? &tm_dv : &tm_dk, stg + s * 4096, 64 * s, k0 + 32 * qw, bhk);
        bulk_commit_group();
        bulk_wait_read_all();  // the boxes have been read before the CTA ends
      }
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

}  // namespace fa
