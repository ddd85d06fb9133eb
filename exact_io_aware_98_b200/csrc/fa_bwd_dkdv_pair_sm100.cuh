// fa_bwd_dkdv_pair_sm100.cuh -- dK and dV of the deterministic attention backward at d = 128 on
// pairs of CTAs whose tensor cores act as one (tcgen05 cta_group::2, M = 256).
//
// The arithmetic is that of fa_bwd_dkdv_sm100.cuh (derivative of O = softmax(S) V, "Attention
// optimisation: FlashAttention and sparse attention", mdooai Ch.04, core formula, recompute
// form):
//   P_ij  = 2^(s_ij * scale2 - lse_i * log2 e)            (0 for masked keys)
//   dV_j  = sum_i P_ij dO_i,   dS_ij = P_ij (dP_ij - Dvec_i),   dK_j = scale * sum_i dS_ij q_i
// and the summation order of every dK/dV element is the same, so the results are bit-identical
// to that kernel's.  What changes is how the MMAs are fed.
//
// A cluster of two CTAs owns 256 consecutive keys: CTA r holds keys k0 + 128 r .. +127 (its K
// and V tiles) and the TMEM rows of those keys.  Per query tile of 128 rows, the even CTA issues
// for the pair
//   S^T  = K Q^T    M = 256 keys, N = 128 query rows, K = d   (smem x smem)
//   dP^T = V dO^T   same shape
//   dV  += P^T dO   M = 256, N = d = 128, K = 128 query rows  (A from TMEM)
//   dK  += dS^T Q   same shape
// A 2-CTA MMA takes rows [128 r, 128 r + 128) of A and rows [N/2 r, N/2 r + N/2) of B from CTA
// r, so the B operand -- Q or dO -- is split two ways: along query rows for S^T and dP^T (CTA
// r loads query rows i0 + 64 r .. +63, all of d, K-major) and along d for dV and dK (CTA r
// loads d columns 64 r .. 64 r + 63 of all 128 query rows, MN-major).  Each CTA's tensor core
// then reads half of B from its own shared memory per instruction, instead of all of it, while
// each CTA still loads its Q/dO halves with plain (non-multicast) TMA tiles from this GPU's
// memory: 64 KB per stage, as in the single-CTA kernel.
//
// Hand-offs between the two CTAs:
//   * Q/dO and K/V loads of both CTAs complete their bytes on the even CTA's barriers (TMA with
//     .cta_group::2); lse and Dvec go to each CTA's own barrier (its compute warps read them);
//   * the even CTA commits MMA completion (S^T, dP^T ready; stage free; all done) to the
//     barriers of both CTAs;
//   * the compute warps of both CTAs report P^T and dS^T ready to the even CTA, one arrival per
//     warp, released at cluster scope;
//   * at the end, each CTA arrives on the other's exit barrier and waits for the other's
//     arrival (bounded), so neither leaves while the other's MMAs or arrivals may still reach
//     it; then both release the TMEM they allocated together.
//
// CTA: 320 threads.  warps 0-7 compute (warpgroup h owns query columns 64 h .. 64 h + 63 of
// its CTA's S^T / dP^T), warp 8 TMA producer, warp 9 MMA issuer (even CTA) / idle (odd CTA).
// TMEM per CTA (512 columns): S^T [0,128) dP^T [128,256) dV [256,384) dK [384,512).
#pragma once
#include "fa_bwd_sm100.cuh"
#include "ptx.cuh"

namespace fa {

struct BwdPairLayout {
  static constexpr int D = 128;
  static constexpr int BN = 128;                  // keys per CTA (256 per pair)
  static constexpr int BM = 128;                  // query rows per step
  static constexpr int HM = BM / 2;               // query rows per CTA in the row split
  static constexpr int QST = 2;                   // Q/dO/lse/Dvec stages
  static constexpr int KV_SUBTILE = 128 * 128;    // 128 rows x 64 d (128-byte rows)
  static constexpr int KV_TILE = 128 * D * 2;
  static constexpr int ROWS_SUBTILE = HM * 128;   // 64 query rows x 64 d
  static constexpr int ROWS_TILE = HM * D * 2;    // 64 query rows x all d (two sub-tiles)
  static constexpr int COLS_TILE = BM * 64 * 2;   // 128 query rows x this CTA's 64 d
  static constexpr int QR = 0, DOR = ROWS_TILE, QC = 2 * ROWS_TILE, DOC = 2 * ROWS_TILE + COLS_TILE;
  static constexpr int STAGE = 2 * ROWS_TILE + 2 * COLS_TILE;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_TILE;
  static constexpr int OFF_ST = OFF_V + KV_TILE;  // stage s at OFF_ST + s * STAGE
  static constexpr int OFF_LSE = OFF_ST + QST * STAGE;
  static constexpr int OFF_DVEC = OFF_LSE + QST * BM * 4;
  static constexpr int OFF_BAR = OFF_DVEC + QST * BM * 4;
  // kv, q_full[QST], l_full[QST], q_empty[QST], s_full, dp_full, p_full[2], ds_full[2], done,
  // fin, exit
  static constexpr int NBAR = 1 + 3 * QST + 2 + 2 + 2 + 3;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = BYTES + 1024;
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
  static constexpr int HALF = BM / 2;             // query columns per compute warpgroup
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t S_COL = 0, DP_COL = 128, DV_COL = 256, DK_COL = 384;
  static constexpr uint32_t PAIR_WARPS = 16;      // compute warps of both CTAs
};

enum : int {
  SITE_PAIR_LOAD_EMPTY = 81, SITE_PAIR_LOAD_DRAIN = 82, SITE_PAIR_MMA_KV = 83,
  SITE_PAIR_MMA_Q = 84, SITE_PAIR_MMA_P = 85, SITE_PAIR_MMA_DS = 86, SITE_PAIR_MMA_FIN = 87,
  SITE_PAIR_C_L = 88, SITE_PAIR_C_S = 89, SITE_PAIR_C_DP = 90, SITE_PAIR_C_DONE = 91,
  SITE_PAIR_EXIT = 92
};

// tm_q, tm_do: boxes of 64 columns x 64 rows; tm_k, tm_v: boxes of 64 columns x 128 rows.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(320, 1)
fa_bwd_dkdv_pair_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                              const __grid_constant__ CUtensorMap tm_k,
                              const __grid_constant__ CUtensorMap tm_v,
                              const __grid_constant__ CUtensorMap tm_do, const BwdParams p) {
  using L = BwdPairLayout;
  constexpr int D = L::D, BM = L::BM;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* bar_kv = bars;                    // even CTA: K/V of both CTAs loaded
  uint64_t* bar_qf = bars + 1;                // even CTA: Q/dO stage of both CTAs loaded
  uint64_t* bar_lf = bar_qf + L::QST;         // each CTA: its lse/Dvec stage loaded
  uint64_t* bar_qe = bar_lf + L::QST;         // each CTA: stage read by the MMAs (free)
  uint64_t* bar_s = bar_qe + L::QST;          // each CTA: S^T in TMEM
  uint64_t* bar_dp = bar_s + 1;               // each CTA: dP^T in TMEM
  uint64_t* bar_p = bar_dp + 1;               // even CTA [2]: P^T of both CTAs in TMEM
  uint64_t* bar_ds = bar_p + 2;               // even CTA [2]: dS^T of both CTAs in TMEM
  uint64_t* bar_done = bar_ds + 2;            // each CTA: every MMA finished
  uint64_t* bar_fin = bar_done + 1;           // even CTA: MMA warp's own completion wait
  uint64_t* bar_exit = bar_fin + 1;           // each CTA: the other CTA is done with this one
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
  const float* s_lse = reinterpret_cast<const float*>(smem + L::OFF_LSE);
  const float* s_dvec = reinterpret_cast<const float*>(smem + L::OFF_DVEC);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();    // 0: the even CTA, which issues the MMAs
  const uint32_t peer = rank ^ 1u;
  const int G = p.H / p.H_kv;                 // query heads per K/V head
  const int BHkv = p.B * p.H_kv;
  const int n_pairs = (p.n_ktiles + 1) / 2;
  // CTA-pair order: groups of p.hgroup K/V heads in turn (a group's Q and dO fit in half of
  // L2), and inside a group the key pairs with the most query tiles first.
  const int pair = static_cast<int>(blockIdx.x) >> 1;
  const int per_group = p.hgroup * n_pairs;
  const int grp = pair / per_group;
  const int g0 = grp * p.hgroup;
  const int gn = min(p.hgroup, BHkv - g0);
  const int rr = pair - grp * per_group;
  const int jp = rr / gn;                     // key pair: KV tiles 2 jp and 2 jp + 1
  const int bhk = g0 + rr % gn;               // (b, K/V head)
  const int b = bhk / p.H_kv;
  const int bhq0 = b * p.H + (bhk % p.H_kv) * G;
  const int N = p.N;
  const int kp0 = jp * 256;                   // first key of the pair
  const int k0 = kp0 + 128 * static_cast<int>(rank);  // first key of this CTA
  int kvlen = N;
  if (p.kv_len != nullptr) kvlen = min(max(p.kv_len[b], 0), N);
  const int nb = (N + 127) / 128;
  const int n_qt = (N + BM - 1) / BM;
  const bool pair_live = kp0 < kvlen;

  // query tile `it` has at least one (row, key) pair with one of the pair's 256 keys; both
  // CTAs walk the same tiles (the MMAs are shared)
  auto q_active = [&](int it) -> bool {
    if (!pair_live) return false;
    const int i0 = it * BM;
    if (p.causal && i0 + BM - 1 < kp0) return false;
    if (p.block_mask != nullptr) {
      const uint8_t* row = p.block_mask + static_cast<size_t>(i0 >> 7) * nb;
      const int j0 = 2 * jp;
      if (!row[j0] && !(j0 + 1 < nb && row[j0 + 1])) return false;
    }
    return true;
  };
  const int it_first = p.causal ? kp0 / BM : 0;
  const int span = n_qt - it_first;
  int n_steps = 0;
  if (p.block_mask == nullptr) n_steps = pair_live ? span : 0;
  else for (int it = it_first; it < n_qt; ++it) n_steps += q_active(it) ? 1 : 0;
  n_steps *= G;

  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    for (int s = 0; s < L::QST; ++s) {
      mbar_init(&bar_qf[s], 1);
      mbar_init(&bar_lf[s], 1);
      mbar_init(&bar_qe[s], 1);
    }
    mbar_init(bar_s, 1);
    mbar_init(bar_dp, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_p[i], L::PAIR_WARPS);
      mbar_init(&bar_ds[i], L::PAIR_WARPS);
    }
    mbar_init(bar_done, 1);
    mbar_init(bar_fin, 1);
    mbar_init(bar_exit, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc_pair(tmem_slot, L::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the even CTA's barriers, as seen from this CTA
  const uint32_t lead_kv = cluster_addr(bar_kv, 0);

  if (warp == 8) {
    // ------------------------------------------------------------------ TMA producer (both)
    if (lane == 0 && n_steps > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      if (rank == 0) mbar_arrive_expect_tx(bar_kv, 2 * 2 * L::KV_TILE);
      for (int s = 0; s < 2; ++s) {
        tma_load_3d_pair(smem + L::OFF_K + s * L::KV_SUBTILE, &tm_k, lead_kv, s * 64, k0, bhk);
        tma_load_3d_pair(smem + L::OFF_V + s * L::KV_SUBTILE, &tm_v, lead_kv, s * 64, k0, bhk);
      }
      int t = 0;
      for (int w = 0; w < G * span; ++w) {
        const int g = w / span;
        const int it = it_first + (w - g * span);
        if (!q_active(it)) continue;
        const int bh = bhq0 + g;
        const int st = t % L::QST;
        if (t >= L::QST &&
            !mbar_wait_cl(&bar_qe[st], ((t / L::QST) - 1) & 1, abort_flag, SITE_PAIR_LOAD_EMPTY))
          break;
        const int i0 = it * BM;
        uint8_t* stage = smem + L::OFF_ST + st * L::STAGE;
        const uint32_t lead_qf = cluster_addr(&bar_qf[st], 0);
        if (rank == 0) mbar_arrive_expect_tx(&bar_qf[st], 2 * L::STAGE);
        // rows split: query rows i0 + 64 rank .. +63, all of d (two 64-column sub-tiles)
        for (int s = 0; s < 2; ++s) {
          tma_load_3d_pair(stage + L::QR + s * L::ROWS_SUBTILE, &tm_q, lead_qf, s * 64,
                           i0 + 64 * static_cast<int>(rank), bh);
          tma_load_3d_pair(stage + L::DOR + s * L::ROWS_SUBTILE, &tm_do, lead_qf, s * 64,
                           i0 + 64 * static_cast<int>(rank), bh);
        }
        // columns split: d columns 64 rank .. +63 of query rows i0 .. i0+127 (two 64-row boxes)
        for (int hb = 0; hb < 2; ++hb) {
          tma_load_3d_pair(stage + L::QC + hb * L::ROWS_SUBTILE, &tm_q, lead_qf,
                           64 * static_cast<int>(rank), i0 + 64 * hb, bh);
          tma_load_3d_pair(stage + L::DOC + hb * L::ROWS_SUBTILE, &tm_do, lead_qf,
                           64 * static_cast<int>(rank), i0 + 64 * hb, bh);
        }
        mbar_arrive_expect_tx(&bar_lf[st], 2 * BM * 4);
        const size_t off = static_cast<size_t>(bh) * p.N_pad + i0;
        bulk_load(smem + L::OFF_LSE + st * BM * 4, p.lse2 + off, BM * 4, &bar_lf[st]);
        bulk_load(smem + L::OFF_DVEC + st * BM * 4, p.dvec + off, BM * 4, &bar_lf[st]);
        ++t;
      }
      // Never leave with a copy in flight.  lse/Dvec complete here; the tiles complete on the
      // even CTA's barriers, which its producer drains (its MMA warp has normally consumed
      // them all), and the exit handshake below keeps this CTA alive until then.
      for (int r = max(0, t - L::QST); r < t; ++r)
        mbar_wait_drain(&bar_lf[r % L::QST], (r / L::QST) & 1, SITE_PAIR_LOAD_DRAIN);
      if (rank == 0) {
        mbar_wait_drain(bar_kv, 0, SITE_PAIR_LOAD_DRAIN);
        for (int r = max(0, t - L::QST); r < t; ++r)
          mbar_wait_drain(&bar_qf[r % L::QST], (r / L::QST) & 1, SITE_PAIR_LOAD_DRAIN);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA issuer (even CTA)
    if (rank == 0 && n_steps > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(256, BM, false, false);
      constexpr uint32_t idesc_g = idesc_bf16_f32(256, D, false, true);
      const uint64_t k_kd = sdesc_sw128(smem_u32(smem + L::OFF_K), 16, 1024);
      const uint64_t v_kd = sdesc_sw128(smem_u32(smem + L::OFF_V), 16, 1024);
      const uint32_t st0 = smem_u32(smem + L::OFF_ST);
      const uint64_t qr_kd = sdesc_sw128(st0 + L::QR, 16, 1024);
      const uint64_t dor_kd = sdesc_sw128(st0 + L::DOR, 16, 1024);
      const uint64_t qc_mn = sdesc_sw128(st0 + L::QC, L::COLS_TILE, 1024);
      const uint64_t doc_mn = sdesc_sw128(st0 + L::DOC, L::COLS_TILE, 1024);
      // barriers of both CTAs the MMA completions are reported to
      const uint32_t s_me = cluster_addr(bar_s, 0), s_peer = cluster_addr(bar_s, 1);
      const uint32_t dp_me = cluster_addr(bar_dp, 0), dp_peer = cluster_addr(bar_dp, 1);
      const uint32_t done_me = cluster_addr(bar_done, 0), done_peer = cluster_addr(bar_done, 1);
      auto off16 = [](int bytes) -> uint64_t { return static_cast<uint64_t>(bytes >> 4); };
      // X^T = A B^T over d: A = K or V (this CTA's 128 keys; the other CTA's are rows 128-255),
      // B = the stage's Q or dO rows half (64 query rows per CTA), K-major.
      auto mma_scores = [&](uint64_t a_desc, uint64_t b_desc, int st, uint32_t d_col) {
        const uint64_t bst = b_desc + off16(st * L::STAGE);
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb) {
          uint64_t a[4], bb[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int k = 4 * kb + i;
            a[i] = a_desc + off16((k >> 2) * L::KV_SUBTILE + (k & 3) * 32);
            bb[i] = bst + off16((k >> 2) * L::ROWS_SUBTILE + (k & 3) * 32);
          }
          mma2_ss_x4(tmem + d_col, a, bb, idesc_s, kb > 0 ? 1u : 0u);
        }
      };
      // G += X^T(TMEM, bf16) B over the 128 query rows: B = the stage's dO or Q columns half
      // (this CTA's 64 d; the other CTA's are d 64-127), MN-major.  Query columns
      // [16k, 16k+16) of X^T were written by compute warpgroup h = 16k / HALF of each CTA into
      // the front half of its own columns.
      auto mma_grad = [&](uint32_t a_col, uint64_t b_desc, int st, uint32_t d_col, bool acc) {
        const uint64_t bst = b_desc + off16(st * L::STAGE);
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
          mma2_ts_x4(tmem + d_col, a, bb, idesc_g, (acc || kb > 0) ? 1u : 0u);
        }
      };
      auto commit_both = [&](uint32_t me, uint32_t other) {
        mma2_commit_w(me);
        mma2_commit_w(other);
      };
      bool ok = mbar_wait_w(bar_kv, 0, abort_flag, SITE_PAIR_MMA_KV);
      ok = ok && mbar_wait_w(&bar_qf[0], 0, abort_flag, SITE_PAIR_MMA_Q);
      tc_fence_after();
      if (ok) {
        mma_scores(k_kd, qr_kd, 0, L::S_COL);
        commit_both(s_me, s_peer);
        mma_scores(v_kd, dor_kd, 0, L::DP_COL);
        commit_both(dp_me, dp_peer);
      }
      for (int t = 0; ok && t < n_steps; ++t) {
        const int st = t % L::QST;
        const int pb = t & 1;
        if (!mbar_wait_cl(&bar_p[pb], (t >> 1) & 1, abort_flag, SITE_PAIR_MMA_P)) { ok = false; break; }
        tc_fence_after();
        mma_grad(L::S_COL, doc_mn, st, L::DV_COL, t > 0);
        if (t + 1 < n_steps) {  // the next scores, into the S^T columns dV(t) just read
          const int st1 = (t + 1) % L::QST;
          if (!mbar_wait_w(&bar_qf[st1], ((t + 1) / L::QST) & 1, abort_flag, SITE_PAIR_MMA_Q)) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_scores(k_kd, qr_kd, st1, L::S_COL);
          commit_both(s_me, s_peer);
        }
        if (!mbar_wait_cl(&bar_ds[pb], (t >> 1) & 1, abort_flag, SITE_PAIR_MMA_DS)) { ok = false; break; }
        tc_fence_after();
        mma_grad(L::DP_COL, qc_mn, st, L::DK_COL, t > 0);
        // Q/dO(t) and lse/Dvec(t) are no longer read after dK(t)
        commit_both(cluster_addr(&bar_qe[st], 0), cluster_addr(&bar_qe[st], 1));
        if (t + 1 < n_steps) {  // dP(t+1) after dK(t) has read dS(t) from the dP^T columns
          mma_scores(v_kd, dor_kd, (t + 1) % L::QST, L::DP_COL);
          commit_both(dp_me, dp_peer);
        }
      }
      commit_both(done_me, done_peer);
      mma2_commit_w(cluster_addr(bar_fin, 0));  // every tcgen05 op here uses cta_group::2
      mbar_wait_w(bar_fin, 0, abort_flag, SITE_PAIR_MMA_FIN);
    }
  } else {
    // ------------------------------------------------------------------ compute warpgroups
    const int h = warp >> 2;                  // which half of the query columns
    const int qw = warp & 3;
    const int jl = 32 * qw + lane;            // key row within this CTA's tile (= TMEM lane)
    const int kj = k0 + jl;                   // key index
    const uint32_t t_lane = static_cast<uint32_t>(32 * qw) << 16;
    const float scale2 = p.scale2;
    const uint32_t lead_p[2] = {cluster_addr(&bar_p[0], 0), cluster_addr(&bar_p[1], 0)};
    const uint32_t lead_ds[2] = {cluster_addr(&bar_ds[0], 0), cluster_addr(&bar_ds[1], 0)};
    // this warp's TMEM writes are complete and ordered before the even CTA's MMAs read them
    auto report = [&](uint32_t lead_bar) {
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(lead_bar);
    };
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
      const uint32_t s_cols = tmem + t_lane + L::S_COL + c0;
      const uint32_t dp_cols = tmem + t_lane + L::DP_COL + c0;
      bool got = mbar_wait(&bar_lf[st], (t / L::QST) & 1, abort_flag, SITE_PAIR_C_L);
      got = got && mbar_wait_cl(bar_s, t & 1, abort_flag, SITE_PAIR_C_S);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
      const float4* lse4 = reinterpret_cast<const float4*>(s_lse + st * BM + c0);
      const float4* dv4 = reinterpret_cast<const float4*>(s_dvec + st * BM + c0);
      const bool edge = (k0 + 128 > kvlen) || (p.causal && k0 + 32 * qw + 31 > i0 + c0);
      // The pair walks the query tiles that see either CTA's keys; where the block mask hides
      // this CTA's key tile from this query tile (or this CTA's keys lie past N), P is 0.
      const bool hidden = p.block_mask != nullptr &&
                          ((k0 >> 7) >= nb || !p.block_mask[static_cast<size_t>(i0 >> 7) * nb + (k0 >> 7)]);
      // ---- P = 2^(s*scale2 - lse2): bf16 into TMEM for dV, fp32 kept for dS
      float pf[32 * (L::HALF / 32)];
#pragma unroll
      for (int c = 0; c < L::HALF / 32; ++c) {
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
        if (hidden) {
#pragma unroll
          for (int i = 0; i < 32; ++i) pf[32 * c + i] = 0.f;
        } else if (edge) {
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
      report(lead_p[pb]);
      // ---- dS = P (dP - Dvec): bf16 into TMEM over my dP^T columns
      got = mbar_wait_cl(bar_dp, t & 1, abort_flag, SITE_PAIR_C_DP);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < L::HALF / 32; ++c) {
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
      report(lead_ds[pb]);
      ++t;
    }
    // ---------------------------------------------------------------- epilogue: dK, dV
    // warpgroup 0 writes dV, warpgroup 1 writes dK (x scale), each for this CTA's 128 keys
    if (ok && n_steps > 0) {
      const bool got = mbar_wait_cl(bar_done, 0, abort_flag, SITE_PAIR_C_DONE);
      ok = __all_sync(0xffffffffu, got);
      tc_fence_after();
    }
    if (ok) {
      const uint32_t col0 = h == 0 ? L::DV_COL : L::DK_COL;
      const float mul = h == 0 ? 1.0f : p.scale;
      __nv_bfloat16* dst_row = (h == 0 ? p.dv : p.dk) + (static_cast<size_t>(bhk) * N + kj) * D;
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
        if (kj < N) {
          uint4* dst = reinterpret_cast<uint4*>(dst_row + 32 * c);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(hv[4 * i], hv[4 * i + 1], hv[4 * i + 2], hv[4 * i + 3]);
        }
      }
    }
  }

  // ------------------------------------------------------------------ teardown
  // A wait that gave up in this CTA stops the other CTA's waits too.
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    if (*abort_flag) st_cluster_u32(cluster_addr(const_cast<int*>(abort_flag), peer), 1u);
    // this CTA is done with the other one (its arrivals sent, its tiles loaded, and -- in the
    // even CTA -- its MMAs complete); wait until the other CTA is done with this one
    mbar_arrive_cluster(cluster_addr(bar_exit, peer));
    mbar_wait_drain_cl(bar_exit, 0, SITE_PAIR_EXIT);
  }
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, L::TMEM_COLS);
  }
}

}  // namespace fa
