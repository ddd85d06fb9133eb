// fa_bwd_dq_sm100.cuh -- dQ of the attention backward without atomics, on sm_100a.
//
// The main backward kernel (fa_bwd_sm100.cuh) owns a KV tile per CTA, so its dQ contributions
// from different KV tiles meet in global memory through fp32 atomics whose order, and so whose
// last bits, vary from run to run.  For the deterministic backward the main kernel computes dK
// and dV only and this kernel computes dQ with the query tile as the stationary operand: one
// CTA owns 128 query rows and walks the KV tiles that those rows can see, in increasing order,
// accumulating dQ in TMEM.  Every sum then runs in a fixed order.  The price is the recompute
// of S and dP here (three MMAs per tile pair instead of one), 14 d FLOP per (row, key) pair in
// total instead of 10 d.
//
// Derivative of O = softmax(S) V ("Attention optimisation: FlashAttention and sparse
// attention", mdooai Ch.04, core formula), in the recompute form of the main kernel:
//   P_ij  = 2^(s_ij * scale2 - lse_i * log2 e)     (0 for masked keys)
//   dP_ij = dO_i . v_j
//   dS_ij = P_ij (dP_ij - Dvec_i),  Dvec_i = dO_i . O_i
//   dQ_i  = scale * sum_j dS_ij k_j
//
// Per KV tile t (128 keys):
//   S(t)  = Q K_t^T   (M=128 rows, N=128 keys, K=D)   smem x smem -> TMEM S[t%2]
//   dP(t) = dO V_t^T  (M=128, N=128, K=D)             smem x smem -> TMEM dP
//   compute warpgroups (two; warpgroup h owns key columns 64h .. 64h+63): P from S(t) in
//     registers, dS = P (dP - Dvec) in bf16 written back over the front half of its own S(t)
//     columns
//   dQ   += dS K_t    (M=128, N=D, K=128 keys)        TMEM x smem -> TMEM dQ
// MMA order per tile: dP(t+1) as soon as the compute warpgroups have read dP(t); dQ(t) once
// dS(t) is in TMEM; then S(t+2) into S[t%2] (after dQ(t) in issue order, so it cannot overwrite
// dS(t) before dQ(t) has read it -- tcgen05 MMAs of one thread execute in order).
//
// TMEM (512 columns): S0 [0,128), S1 [128,256), dP [256,384), dQ [384,384+D).
// CTA: 320 threads.  warps 0-7 compute, warp 8 TMA producer, warp 9 MMA issuer.
#pragma once
#include "ptx.cuh"

namespace fa {

struct BwdDqParams {
  const uint8_t* block_mask;  // [nb][nb] or nullptr
  const int32_t* kv_len;      // [B] or nullptr
  const float* lse2;          // [B*H][N_pad] lse*log2(e); +inf for rows with no key / padding
  const float* dvec;          // [B*H][N_pad]
  __nv_bfloat16* dq;          // [B*H][N][D]
  int B, H, H_kv, N, N_pad;
  int n_mtiles;               // ceil(N / 128)
  int hgroup;                 // query heads per CTA-order group (>= 1; B*H: one group)
  float scale, scale2;
  int causal;
};

template <int D>
struct BwdDqLayout {
  static constexpr int BM = 128;                  // query rows per CTA
  static constexpr int BN = 128;                  // keys per KV tile
  static constexpr int KST = D == 64 ? 4 : 3;     // K ring depth
  static constexpr int VST = D == 64 ? 4 : 2;     // V ring depth
  static constexpr int SUB = D / 64;              // 64-column (128-byte) sub-tiles
  static constexpr int SUBTILE = 128 * 128;       // bytes of one 128-row x 64-column sub-tile
  static constexpr int TILE = 128 * D * 2;        // bytes of one 128-row tile
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = OFF_Q + TILE;
  static constexpr int OFF_K = OFF_DO + TILE;
  static constexpr int OFF_V = OFF_K + KST * TILE;
  static constexpr int OFF_BAR = OFF_V + VST * TILE;
  // q, k_full[KST], k_empty[KST], v_full[VST], v_empty[VST], s_full[2], dp_full, dp_free,
  // ds_full, dq_done
  static constexpr int NBAR = 1 + 2 * KST + 2 * VST + 2 + 4;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = BYTES + 1024;  // slack for 1024-byte alignment
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t DP_COL = 256;
  static constexpr uint32_t DQ_COL = 384;
  __device__ static constexpr uint32_t s_col(int buf) { return static_cast<uint32_t>(buf) * 128u; }
  static_assert(DQ_COL + D <= TMEM_COLS, "TMEM budget");
};

enum : int {
  SITE_DQ_LOAD_EMPTY = 41, SITE_DQ_LOAD_DRAIN = 42, SITE_DQ_MMA_Q = 43, SITE_DQ_MMA_K = 44,
  SITE_DQ_MMA_V = 45, SITE_DQ_MMA_DPF = 46, SITE_DQ_MMA_DS = 47, SITE_DQ_MMA_FIN = 48,
  SITE_DQ_C_S = 49, SITE_DQ_C_DP = 50, SITE_DQ_C_DONE = 51
};

template <int D>
__global__ void __launch_bounds__(320, 1)
fa_bwd_dq_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_do, const BwdDqParams p) {
  using L = BwdDqLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* bar_q = bars;
  uint64_t* bar_kf = bars + 1;
  uint64_t* bar_ke = bar_kf + L::KST;
  uint64_t* bar_vf = bar_ke + L::KST;
  uint64_t* bar_ve = bar_vf + L::VST;
  uint64_t* bar_sf = bar_ve + L::VST;    // [2]: S(t) in buffer t%2
  uint64_t* bar_dpf = bar_sf + 2;        // dP(t) in TMEM
  uint64_t* bar_dpe = bar_dpf + 1;       // dP(t) read by the compute warpgroups
  uint64_t* bar_dsf = bar_dpe + 1;       // dS(t) in TMEM
  uint64_t* bar_done = bar_dsf + 1;      // every MMA finished: dQ final
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int BH = p.B * p.H;
  // CTA order: groups of p.hgroup query heads in turn (the K and V the group reads fit in half
  // of L2, so the query tiles of a head re-read them from L2), and inside a group the heaviest
  // query tiles (the last rows under a causal mask) first.
  const int per_group = p.hgroup * p.n_mtiles;
  const int grp = static_cast<int>(blockIdx.x) / per_group;
  const int g0 = grp * p.hgroup;
  const int gn = min(p.hgroup, BH - g0);                // heads in this group (the last may have fewer)
  const int rr = static_cast<int>(blockIdx.x) - grp * per_group;
  const int mt = p.n_mtiles - 1 - rr / gn;
  const int bh = g0 + rr % gn;
  const int b = bh / p.H;
  const int bh_kv = b * p.H_kv + (bh % p.H) / (p.H / p.H_kv);  // K/V head of this query head
  const int N = p.N;
  const int m0 = mt * L::BM;
  int kvlen = N;
  if (p.kv_len != nullptr) kvlen = min(max(p.kv_len[b], 0), N);
  const int nb = (N + 127) / 128;
  int j_end = (kvlen + 127) / 128;
  if (p.causal) j_end = min(j_end, (min(m0 + L::BM, N) - 1) / 128 + 1);
  // KV tile j holds at least one key that a row of this query tile may attend to
  auto visible = [&](int j) -> bool {
    return p.block_mask == nullptr || p.block_mask[static_cast<size_t>(m0 >> 7) * nb + j] != 0;
  };
  int n_tiles = 0;
  if (p.block_mask == nullptr) n_tiles = j_end;
  else for (int j = 0; j < j_end; ++j) n_tiles += visible(j) ? 1 : 0;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < L::KST; ++s) {
      mbar_init(&bar_kf[s], 1);
      mbar_init(&bar_ke[s], 1);
    }
    for (int s = 0; s < L::VST; ++s) {
      mbar_init(&bar_vf[s], 1);
      mbar_init(&bar_ve[s], 1);
    }
    mbar_init(&bar_sf[0], 1);
    mbar_init(&bar_sf[1], 1);
    mbar_init(bar_dpf, 1);
    mbar_init(bar_dpe, 256);
    mbar_init(bar_dsf, 256);
    mbar_init(bar_done, 1);
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
    if (lane == 0 && n_tiles > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(bar_q, 2 * L::TILE);
      for (int s = 0; s < L::SUB; ++s) {
        tma_load_3d(smem + L::OFF_Q + s * L::SUBTILE, &tm_q, bar_q, s * 64, m0, bh);
        tma_load_3d(smem + L::OFF_DO + s * L::SUBTILE, &tm_do, bar_q, s * 64, m0, bh);
      }
      // K(t) and V(t) in separate rings: V(t) frees after dP(t), K(t) only after dQ(t)
      int t = 0;
      for (int j = 0; j < j_end; ++j) {
        if (!visible(j)) continue;
        const int ks = t % L::KST, vs = t % L::VST;
        if (t >= L::KST &&
            !mbar_wait(&bar_ke[ks], ((t / L::KST) - 1) & 1, abort_flag, SITE_DQ_LOAD_EMPTY))
          break;
        mbar_arrive_expect_tx(&bar_kf[ks], L::TILE);
        for (int s = 0; s < L::SUB; ++s)
          tma_load_3d(smem + L::OFF_K + ks * L::TILE + s * L::SUBTILE, &tm_k, &bar_kf[ks], s * 64,
                      j * 128, bh_kv);
        if (t >= L::VST &&
            !mbar_wait(&bar_ve[vs], ((t / L::VST) - 1) & 1, abort_flag, SITE_DQ_LOAD_EMPTY))
          break;
        mbar_arrive_expect_tx(&bar_vf[vs], L::TILE);
        for (int s = 0; s < L::SUB; ++s)
          tma_load_3d(smem + L::OFF_V + vs * L::TILE + s * L::SUBTILE, &tm_v, &bar_vf[vs], s * 64,
                      j * 128, bh_kv);
        ++t;
      }
      // never leave the CTA with a copy in flight
      mbar_wait(bar_q, 0, abort_flag, SITE_DQ_LOAD_DRAIN);
      for (int r = max(0, t - L::KST); r < t; ++r)
        mbar_wait(&bar_kf[r % L::KST], (r / L::KST) & 1, abort_flag, SITE_DQ_LOAD_DRAIN);
      for (int r = max(0, t - L::VST); r < t; ++r)
        mbar_wait(&bar_vf[r % L::VST], (r / L::VST) & 1, abort_flag, SITE_DQ_LOAD_DRAIN);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA issuer
    // The whole warp walks the loop (descriptors stay warp-uniform); one elected lane issues
    // the MMAs four at a time.
    if (n_tiles > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_q = idesc_bf16_f32(128, D, false, true);
      // Q, dO, K, V: K-major for the score MMAs; K MN-major (d contiguous) for dQ = dS K.
      const uint64_t q_kd = sdesc_sw128(smem_u32(smem + L::OFF_Q), 16, 1024);
      const uint64_t do_kd = sdesc_sw128(smem_u32(smem + L::OFF_DO), 16, 1024);
      const uint64_t k_kd = sdesc_sw128(smem_u32(smem + L::OFF_K), 16, 1024);
      const uint64_t v_kd = sdesc_sw128(smem_u32(smem + L::OFF_V), 16, 1024);
      const uint64_t k_mn = sdesc_sw128(smem_u32(smem + L::OFF_K), L::SUBTILE, 1024);
      auto koff = [](int k) -> uint64_t {  // K-step k of a K-major operand, in 16-byte units
        return static_cast<uint64_t>(((k >> 2) * L::SUBTILE + (k & 3) * 32) >> 4);
      };
      // X = A B^T over D into TMEM column d_col: A = Q or dO, B = K or V of ring stage st
      auto mma_scores = [&](uint64_t a_desc, uint64_t b_desc, int st, uint32_t d_col) {
        const uint64_t bst = b_desc + static_cast<uint64_t>((st * L::TILE) >> 4);
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb) {
          uint64_t a[4], bb[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            a[i] = a_desc + koff(4 * kb + i);
            bb[i] = bst + koff(4 * kb + i);
          }
          mma_ss_x4(tmem + d_col, a, bb, idesc_s, kb > 0 ? 1u : 0u);
        }
      };
      // dQ += dS K(st): dS from TMEM (key columns 16k .. 16k+15 were written by warpgroup
      // h = k / 4 over the front half of its own S columns), K MN-major.
      auto mma_dq = [&](int buf, int st, bool acc) {
        const uint64_t kst = k_mn + static_cast<uint64_t>((st * L::TILE) >> 4);
#pragma unroll
        for (int kb = 0; kb < L::BN / 64; ++kb) {
          uint32_t a[4];
          uint64_t bb[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int k = 4 * kb + i;
            a[i] = tmem + L::s_col(buf) + 8u * k + 32u * static_cast<uint32_t>(k >> 2);
            bb[i] = kst + static_cast<uint64_t>((k * 2048) >> 4);
          }
          mma_ts_x4(tmem + L::DQ_COL, a, bb, idesc_q, (acc || kb > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait_w(bar_q, 0, abort_flag, SITE_DQ_MMA_Q);
      ok = ok && mbar_wait_w(&bar_kf[0], 0, abort_flag, SITE_DQ_MMA_K);
      ok = ok && mbar_wait_w(&bar_vf[0], 0, abort_flag, SITE_DQ_MMA_V);
      tc_fence_after();
      if (ok) {
        mma_scores(q_kd, k_kd, 0, L::s_col(0));
        mma_commit_w(&bar_sf[0]);
        mma_scores(do_kd, v_kd, 0, L::DP_COL);
        mma_commit_w(bar_dpf);
        mma_commit_w(&bar_ve[0]);  // V(0) read by dP(0)
        if (n_tiles > 1) {
          ok = mbar_wait_w(&bar_kf[1 % L::KST], (1 / L::KST) & 1, abort_flag, SITE_DQ_MMA_K);
          tc_fence_after();
          if (ok) {
            mma_scores(q_kd, k_kd, 1 % L::KST, L::s_col(1));
            mma_commit_w(&bar_sf[1]);
          }
        }
      }
      for (int t = 0; ok && t < n_tiles; ++t) {
        const int buf = t & 1;
        const int ks = t % L::KST;
        if (t + 1 < n_tiles) {
          // dP(t+1) as soon as the compute warpgroups have read dP(t)
          const int vs1 = (t + 1) % L::VST;
          if (!mbar_wait_w(bar_dpe, t & 1, abort_flag, SITE_DQ_MMA_DPF) ||
              !mbar_wait_w(&bar_vf[vs1], ((t + 1) / L::VST) & 1, abort_flag, SITE_DQ_MMA_V)) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_scores(do_kd, v_kd, vs1, L::DP_COL);
          mma_commit_w(bar_dpf);
          mma_commit_w(&bar_ve[vs1]);  // V(t+1) read by dP(t+1)
        }
        if (!mbar_wait_w(bar_dsf, t & 1, abort_flag, SITE_DQ_MMA_DS)) { ok = false; break; }
        tc_fence_after();
        mma_dq(buf, ks, t > 0);
        mma_commit_w(&bar_ke[ks]);     // K(t) read by S(t) and dQ(t)
        if (t + 2 < n_tiles) {
          // S(t+2) into S[t%2]: issued after dQ(t), which reads dS(t) from those columns
          const int ks2 = (t + 2) % L::KST;
          if (!mbar_wait_w(&bar_kf[ks2], ((t + 2) / L::KST) & 1, abort_flag, SITE_DQ_MMA_K)) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_scores(q_kd, k_kd, ks2, L::s_col(buf));
          mma_commit_w(&bar_sf[buf]);
        }
      }
      // all MMAs issued by this warp have completed: dQ is final and TMEM may be released
      mma_commit_w(bar_done);
      mbar_wait_w(bar_done, 0, abort_flag, SITE_DQ_MMA_FIN);
    }
  } else {
    // ------------------------------------------------------------------ compute warpgroups
    const int h = warp >> 2;                  // key columns 64h .. 64h+63 of every tile
    const int qw = warp & 3;
    const int rl = 32 * qw + lane;            // query row within the tile (= TMEM lane)
    const int qi = m0 + rl;                   // query index
    const uint32_t t_lane = static_cast<uint32_t>(32 * qw) << 16;
    const float scale2 = p.scale2;
    const size_t prow = static_cast<size_t>(bh) * p.N_pad + m0 + rl;  // < N_pad: m0 + 127 < N_pad
    const float lse2 = p.lse2[prow];          // +inf for padding rows and rows with no key
    const float dvec = p.dvec[prow];
    bool ok = true;
    int t = 0;
    for (int j = 0; j < j_end; ++j) {
      if (!visible(j)) continue;
      const int buf = t & 1;
      const int k0 = j * 128;
      const uint32_t s_cols = tmem + t_lane + L::s_col(buf) + 64 * h;
      const uint32_t dp_cols = tmem + t_lane + L::DP_COL + 64 * h;
      bool got = mbar_wait(&bar_sf[buf], (t >> 1) & 1, abort_flag, SITE_DQ_C_S);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
      // ---- P = 2^(s*scale2 - lse2) for my 64 keys
      const bool edge = (k0 + 128 > kvlen) || (p.causal && k0 + 64 * h + 63 > m0 + 32 * qw);
      float pv[64];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t sr[32];
        tmem_ld32(s_cols + 32 * c, sr);
        tmem_ld_wait();
        reg_fence(sr);
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float x0, x1;
          ffma2(x0, x1, __uint_as_float(sr[i]), __uint_as_float(sr[i + 1]), scale2, scale2,
                -lse2, -lse2);
          pv[32 * c + i] = ex2_approx(x0);
          pv[32 * c + i + 1] = ex2_approx(x1);
        }
      }
      if (edge) {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const int kj = k0 + 64 * h + i;
          if (kj >= kvlen || (p.causal && kj > qi)) pv[i] = 0.f;
        }
      }
      // ---- dS = P (dP - Dvec) in bf16 over the front half of my S(t) columns
      got = mbar_wait(bar_dpf, t & 1, abort_flag, SITE_DQ_C_DP);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
      uint32_t dr[2][32];
      tmem_ld32(dp_cols, dr[0]);
      tmem_ld32(dp_cols + 32, dr[1]);
      tmem_ld_wait();
      reg_fence(dr[0]);
      reg_fence(dr[1]);
      tc_fence_before();
      mbar_arrive(bar_dpe);                   // dP(t) is in registers: dP(t+1) may overwrite it
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t dd[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float d0 = pv[32 * c + 2 * i] * (__uint_as_float(dr[c][2 * i]) - dvec);
          const float d1 = pv[32 * c + 2 * i + 1] * (__uint_as_float(dr[c][2 * i + 1]) - dvec);
          dd[i] = pack_bf16x2(d0, d1);
        }
        tmem_st16(s_cols + 16 * c, dd);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_dsf);
      ++t;
    }
    // ---------------------------------------------------------------- epilogue: dQ
    // warpgroup h writes dQ columns h*D/2 .. h*D/2 + D/2 - 1 of its rows (x scale)
    if (ok && n_tiles > 0) {
      const bool got = mbar_wait(bar_done, 0, abort_flag, SITE_DQ_C_DONE);
      ok = __all_sync(0xffffffffu, got);
      tc_fence_after();
    }
    if (ok) {  // warp-uniform: tcgen05.ld is collective; the stores check qi < N
      __nv_bfloat16* dst_row = p.dq + (static_cast<size_t>(bh) * N + qi) * D + h * (D / 2);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t g[32];
        if (n_tiles > 0) {
          tmem_ld32(tmem + t_lane + L::DQ_COL + h * (D / 2) + 32 * c, g);
          tmem_ld_wait();
          reg_fence(g);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) g[i] = 0u;
        }
        uint32_t hv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          hv[i] = pack_bf16x2(__uint_as_float(g[2 * i]) * p.scale,
                              __uint_as_float(g[2 * i + 1]) * p.scale);
        if (qi < N) {
          uint4* dst = reinterpret_cast<uint4*>(dst_row + 32 * c);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(hv[4 * i], hv[4 * i + 1], hv[4 * i + 2], hv[4 * i + 3]);
        }
      }
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
