// fa_bwd_sm100.cuh -- exact attention backward on sm_100a, recomputing the scores from Q, K
// and the forward's per-row log-sum-exp (no N x N matrix is stored).
//
// Derivative of O = softmax(S) V with S = scale * Q K^T (the formula of "Attention
// optimisation: FlashAttention and sparse attention", mdooai Ch.04), written with
// Dvec_i = sum_c dO_ic O_ic, which equals sum_k A_ik dA_ik because O = A V:
//   P_ij  = 2^(s_ij * scale2 - lse_i * log2 e)            (= A_ij; 0 for masked keys)
//   dV_j  = sum_i P_ij dO_i
//   dP_ij = dO_i . v_j
//   dS_ij = P_ij (dP_ij - Dvec_i)
//   dK_j  = scale * sum_i dS_ij q_i
//   dQ_i  = scale * sum_j dS_ij k_j
//
// One CTA owns 128 keys (K and V stay in shared memory) and walks the query tiles that can
// see them (causal, key padding and block mask skip whole tiles).  Per query tile of BM rows:
//   S^T  = K Q^T     (M=128 keys, N=BM, K=D)      smem x smem  -> TMEM
//   dP^T = V dO^T    (M=128, N=BM, K=D)           smem x smem  -> TMEM (D=64)
//                                                 TMEM x smem  -> TMEM (D=128: V copied
//                                                 into TMEM once per CTA)
//   compute warpgroups (two, each owning half of the BM query columns): P^T and dS^T in bf16
//   back into TMEM (each over the front half of its own S^T / dP^T columns) and dS^T to smem
//   dV  += P^T dO    (M=128, N=D, K=BM)           TMEM x smem  -> TMEM
//   dK  += dS^T Q    (M=128, N=D, K=BM)           TMEM x smem  -> TMEM
//   D=64 : dQ   = dS K     (M=BM=128, N=64,  K=128) smem x smem -> TMEM (row per lane)
//   D=128: dQ^T = K^T dS^T (M=128,    N=BM=64, K=128) smem x smem -> TMEM (column per lane)
//   dQ warpgroup: TMEM -> the fp32 dQ workspace by TMA reduce-adds of boxes staged in shared
//   memory: at D=128 one per warp of a [64 rows][32 d] box in the V tile's shared memory (free
//   once V is in TMEM); at D=64 two per warp of [32 rows][32 d] boxes (128-byte swizzled) in the
//   dS^T buffer the step's dQ MMA has just finished reading, handed back to the compute
//   warpgroups once the reduce-adds have read it.
// Hand-offs per step: P ready (-> dV(t), then S(t+1)) and dS ready (-> dK(t), then dP(t+1),
// then dQ(t)).  In-order MMA execution lets S(t+1) reuse the TMEM that dV(t) read P^T(t) from,
// and dP(t+1) the TMEM of dS^T(t); the compute warpgroups compute dS(t) while dV(t) and S(t+1)
// run, and P(t+1) while dK(t), dP(t+1) and dQ(t) run.
//
// CTA: 448 threads. warps 0-7 compute (two warpgroups), warp 8 TMA producer, warp 9 MMA
// issuer, warps 10-13 dQ.
#pragma once
#include "ptx.cuh"

namespace fa {

struct BwdParams {
  const uint8_t* block_mask;  // [nb][nb] or nullptr
  const int32_t* kv_len;      // [B] or nullptr
  const float* lse2;          // [B*H][N_pad] lse*log2(e); +inf for rows with no key / padding
  const float* dvec;          // [B*H][N_pad]
  float* dq_acc;              // [B*H][N][D] fp32, zeroed by the preprocess kernel
  __nv_bfloat16* dk;          // [B*H][N][D]
  __nv_bfloat16* dv;          // [B*H][N][D]
  int B, H, N, N_pad;
  int H_kv;                   // K/V heads: query heads G*j .. G*j+G-1 (G = H / H_kv) read head j
  int n_ktiles;               // ceil(N / 128)
  int hgroup;                 // K/V heads per CTA-order group (>= 1; B*H_kv: one group)
  float scale, scale2;
  int causal;
};

template <int D>
struct BwdLayout {
  static constexpr int BN = 128;                  // keys per CTA
  static constexpr int BM = D == 64 ? 128 : 64;   // query rows per step
  static constexpr int QST = D == 128 ? 4 : 3;    // Q/dO/lse/Dvec stages
  static constexpr int SUB = D / 64;
  static constexpr int KV_SUBTILE = 128 * 128;
  static constexpr int Q_SUBTILE = BM * 128;
  static constexpr int KV_TILE = 128 * D * 2;
  static constexpr int Q_TILE = BM * D * 2;
  static constexpr int DS_TILE = BN * BM * 2;     // dS^T rows j, 64-column i-blocks
  static constexpr int DS_IBLK = BN * 128;        // bytes between i-blocks of dS^T
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_TILE;
  static constexpr int OFF_Q = OFF_V + KV_TILE;
  static constexpr int OFF_DO = OFF_Q + QST * Q_TILE;
  static constexpr int OFF_DS = OFF_DO + QST * Q_TILE;
  static constexpr int OFF_LSE = OFF_DS + 2 * DS_TILE;
  static constexpr int OFF_DVEC = OFF_LSE + QST * BM * 4;
  static constexpr int OFF_BAR = OFF_DVEC + QST * BM * 4;
  // kv, q_full[QST], q_empty[QST], s_full, dp_full, p_full, ds_full, dq_full[2], dq_empty[2],
  // kv_done, fin, v_tmem, ds_free[2], dv_done
  static constexpr int NBAR = 1 + 2 * QST + 4 + 2 + 2 + 1 + 1 + 1 + 2 + 1;
  static constexpr int THREADS = 448;
  static constexpr int HALF = BM / 2;               // query columns per compute warpgroup
  static constexpr int NCH = HALF / 32;             // 32-column chunks per compute warpgroup
  static constexpr int EMU_EVERY = 0;               // one P pair in EMU_EVERY exponentiated on FMA (0: none)
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  // Dynamic shared memory starts 1024-byte aligned on sm_100 (the kernel checks), so no slack
  // is allocated: at d = 128 the fourth Q/dO stage fits only without it.
  static constexpr int SMEM_ALLOC = BYTES;
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
  static constexpr uint32_t TMEM_COLS = 512;
  // d = 128: V moves into TMEM (the A operand of dP^T) once per CTA, and its shared-memory tile
  // then stages dQ^T for TMA reduce-adds into the fp32 accumulator (no per-element atomics).
  // The 64 TMEM columns come from holding one dQ^T buffer instead of two.
  static constexpr bool V_IN_TMEM = D == 128;
  // d = 64: warpgroup 0 writes dV as soon as the last dV MMA has finished (before the last dK
  // and dQ MMAs), staging it in the dS^T buffer the last two steps no longer use.  At d = 128 a
  // dS^T buffer (16 KB) cannot hold dV (32 KB).
  static constexpr bool EARLY_DV = !V_IN_TMEM;
  // d = 64: launched to overlap the preprocess kernel (programmatic dependent launch).  Its calls
  // are short, so the launch gaps and the set-up are a visible share of them; at d = 128 they are
  // not, and the kernel keeps a plain launch.
  static constexpr bool OVERLAP_PREV = D == 64;
  static constexpr int DQB = V_IN_TMEM ? 1 : 2;         // dQ buffers of 64 columns
  static constexpr uint32_t S_COL = 0;
  static constexpr uint32_t DP_COL = BM;
  static constexpr uint32_t DQ_COL = 2 * BM;
  static constexpr uint32_t VT_COL = DQ_COL + DQB * 64;  // V, d = 128 only
  static constexpr uint32_t DV_COL = 2 * BM + 128;
  static constexpr uint32_t DK_COL = 2 * BM + 128 + D;
  static_assert(!V_IN_TMEM || VT_COL + D / 2 <= DV_COL, "TMEM: V overlaps dV");
  static constexpr int DQ_STAGE = 64 * 32 * 4;         // one dQ warp's [64 rows][32 d] fp32 box
  static_assert(!V_IN_TMEM || 4 * DQ_STAGE <= KV_TILE, "dQ staging fits in the V tile");
  // d = 64: one dQ warp's [32 rows][64 d] fp32 box, staged as two swizzled [32][32] halves
  static constexpr int DQ64_STAGE = 32 * 64 * 4;
  static_assert(V_IN_TMEM || 4 * DQ64_STAGE <= DS_TILE, "dQ staging fits in a dS^T buffer");
  static_assert(DK_COL + D <= TMEM_COLS, "TMEM budget");
};

enum : int {
  SITE_BWD_LOAD_EMPTY = 21, SITE_BWD_LOAD_DRAIN = 22, SITE_BWD_MMA_KV = 23, SITE_BWD_MMA_Q = 24,
  SITE_BWD_MMA_DS = 25, SITE_BWD_MMA_DQE = 26, SITE_BWD_MMA_FIN = 27, SITE_BWD_C_Q = 28,
  SITE_BWD_C_S = 29, SITE_BWD_C_DQ = 30, SITE_BWD_C_DONE = 31, SITE_BWD_DQ = 32,
  SITE_BWD_MMA_P = 33, SITE_BWD_C_DP = 34, SITE_BWD_SMEM_ALIGN = 35, SITE_BWD_MMA_VT = 36,
  SITE_BWD_C_KV = 37
};

template <int D>
// 14 warps: some SM sub-partitions hold four of them, which caps registers at 128 per thread.
// tm_dq: the fp32 dQ accumulator [B*H][N][D], boxes of 32 columns x 64 rows (d = 128) or of
// 32 columns x 32 rows with the 128-byte swizzle (d = 64).
__global__ void __launch_bounds__(448, 1)
fa_bwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dq,
                    const __grid_constant__ CUtensorMap tm_dk,
                    const __grid_constant__ CUtensorMap tm_dv, const BwdParams p) {
  using L = BwdLayout<D>;
  constexpr int BM = L::BM;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 128-byte-swizzled TMA tiles need 1024-byte alignment; without slack in the allocation a
  // misaligned base is reported (status word) and the CTA returns before touching anything.
  if ((smem_u32(smem_raw) & 1023u) != 0u) {
    if (threadIdx.x == 0)
      atomicCAS(&g_status, 0u, (static_cast<unsigned>(SITE_BWD_SMEM_ALIGN) << 16) | (blockIdx.x & 0xffffu));
    return;
  }
  uint8_t* smem = smem_raw;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* bar_kv = bars;
  uint64_t* bar_qf = bars + 1;
  uint64_t* bar_qe = bar_qf + L::QST;
  uint64_t* bar_s = bar_qe + L::QST;
  uint64_t* bar_dp = bar_s + 1;
  uint64_t* bar_p = bar_dp + 1;
  uint64_t* bar_ds = bar_p + 1;
  uint64_t* bar_dqf = bar_ds + 1;
  uint64_t* bar_dqe = bar_dqf + 2;
  uint64_t* bar_done = bar_dqe + 2;
  uint64_t* bar_fin = bar_done + 1;
  uint64_t* bar_vt = bar_fin + 1;        // V copied into TMEM (d = 128)
  uint64_t* bar_dsf = bar_vt + 1;        // [2] d = 64: dS^T buffer free again (dQ staged out)
  uint64_t* bar_dvd = bar_dsf + 2;       // EARLY_DV: the last dV MMA has finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
  const float* s_lse = reinterpret_cast<const float*>(smem + L::OFF_LSE);
  const float* s_dvec = reinterpret_cast<const float*>(smem + L::OFF_DVEC);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = p.H / p.H_kv;                         // query heads per K/V head
  const int BHkv = p.B * p.H_kv;
  // CTA order: groups of p.hgroup K/V heads in turn, and inside a group the KV tiles with the
  // most query tiles (small jt) first.  A group's fp32 dQ accumulator, Q and dO fit in L2, so
  // the dQ reductions of the CTAs in flight hit L2 instead of missing to HBM.
  const int per_group = p.hgroup * p.n_ktiles;
  const int grp = static_cast<int>(blockIdx.x) / per_group;
  const int g0 = grp * p.hgroup;
  const int gn = min(p.hgroup, BHkv - g0);             // heads in this group (the last may have fewer)
  const int r = static_cast<int>(blockIdx.x) - grp * per_group;
  const int jt = r / gn;                               // KV tile
  const int bhk = g0 + r % gn;                         // (b, K/V head)
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
  // The CTA walks the query tiles it_first .. n_qt-1 of each of the G query heads of its group
  // (work item w: head g = w / span, tile it_first + w % span); dK and dV of the shared K/V
  // head accumulate over all of them.  Steps: a closed form unless a block mask decides tile by
  // tile (a loop over all query tiles in every thread costs thousands of cycles at N = 16384).
  const int it_first = p.causal ? k0 / BM : 0;  // query tiles before it_first see no key here
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
    mbar_init(bar_s, 1);
    mbar_init(bar_dp, 1);
    mbar_init(bar_p, 256);
    mbar_init(bar_ds, 256);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_dqf[i], 1);
      mbar_init(&bar_dqe[i], 128);
    }
    mbar_init(bar_done, 1);
    mbar_init(bar_fin, 1);
    mbar_init(bar_vt, 128);
    mbar_init(&bar_dsf[0], 4);
    mbar_init(&bar_dsf[1], 4);
    mbar_init(bar_dvd, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, L::TMEM_COLS);
    tmem_relinquish();
  }
  // OVERLAP_PREV: set-up, the K/V loads and the first Q/dO loads run under the preprocess
  // kernel's tail; lse2, Dvec and the zeroed dQ accumulator are touched only after grid_dep_wait.
  // The dQ convert after this kernel may launch now.
  if constexpr (L::OVERLAP_PREV) grid_dep_launch();
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
        const int bh = bhq0 + g;              // query head of this step
        const int st = t % L::QST;
        if (t >= L::QST &&
            !mbar_wait(&bar_qe[st], ((t / L::QST) - 1) & 1, abort_flag, SITE_BWD_LOAD_EMPTY))
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
        if (L::OVERLAP_PREV && t == 0) grid_dep_wait();  // lse2 and Dvec: preprocess kernel
        bulk_load(smem + L::OFF_LSE + st * BM * 4, p.lse2 + off, BM * 4, &bar_qf[st]);
        bulk_load(smem + L::OFF_DVEC + st * BM * 4, p.dvec + off, BM * 4, &bar_qf[st]);
        ++t;
      }
      mbar_wait(bar_kv, 0, abort_flag, SITE_BWD_LOAD_DRAIN);
      for (int r = max(0, t - L::QST); r < t; ++r)
        mbar_wait(&bar_qf[r % L::QST], (r / L::QST) & 1, abort_flag, SITE_BWD_LOAD_DRAIN);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA issuer
    // The whole warp walks the loop (descriptors stay warp-uniform); one elected lane issues
    // the MMAs four at a time.
    if (n_steps > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, BM, false, false);
      constexpr uint32_t idesc_g = idesc_bf16_f32(128, D, false, true);
      constexpr uint32_t idesc_q = idesc_bf16_f32(128, 64, true, true);
      const uint32_t k_addr = smem_u32(smem + L::OFF_K);
      const uint32_t v_addr = smem_u32(smem + L::OFF_V);
      const uint32_t q_addr = smem_u32(smem + L::OFF_Q);
      const uint32_t do_addr = smem_u32(smem + L::OFF_DO);
      const uint32_t ds_addr = smem_u32(smem + L::OFF_DS);
      // K-major views (scores), MN-major views (gradients and dQ).
      const uint64_t k_kd = sdesc_sw128(k_addr, 16, 1024);
      const uint64_t v_kd = sdesc_sw128(v_addr, 16, 1024);
      const uint64_t q_kd = sdesc_sw128(q_addr, 16, 1024);
      const uint64_t do_kd = sdesc_sw128(do_addr, 16, 1024);
      const uint64_t q_mn = sdesc_sw128(q_addr, L::Q_SUBTILE, 1024);
      const uint64_t do_mn = sdesc_sw128(do_addr, L::Q_SUBTILE, 1024);
      const uint64_t k_mn = sdesc_sw128(k_addr, L::KV_SUBTILE, 1024);
      const uint64_t ds_mn = sdesc_sw128(ds_addr, L::DS_IBLK, 1024);
      auto off16 = [](int bytes) -> uint64_t { return static_cast<uint64_t>(bytes >> 4); };
      // X^T = A B^T over D: A = K or V (128 rows), B = Q or dO of stage st (BM rows), K-major.
      // a_tmem: A is V in TMEM (16 elements of d per K-step = 8 columns).
      auto mma_scores = [&](uint64_t a_desc, bool a_tmem, uint64_t b_desc, int st, uint32_t d_col) {
        const uint64_t bst = b_desc + off16(st * L::Q_TILE);
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb) {
          uint64_t b[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int k = 4 * kb + i;
            b[i] = bst + off16((k >> 2) * L::Q_SUBTILE + (k & 3) * 32);
          }
          if (a_tmem) {
            uint32_t a[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = tmem + L::VT_COL + 8u * (4 * kb + i);
            mma_ts_x4(tmem + d_col, a, b, idesc_s, kb > 0 ? 1u : 0u);
          } else {
            uint64_t a[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int k = 4 * kb + i;
              a[i] = a_desc + off16((k >> 2) * L::KV_SUBTILE + (k & 3) * 32);
            }
            mma_ss_x4(tmem + d_col, a, b, idesc_s, kb > 0 ? 1u : 0u);
          }
        }
      };
      // G += X^T(TMEM, bf16) B over BM rows: B = dO or Q of stage st, MN-major.  Query columns
      // [16k, 16k+16) of X^T were written by compute warpgroup h = 16k / HALF into the front
      // half of its own columns, hence the per-step TMEM column.
      auto mma_grad = [&](uint32_t a_col, uint64_t b_desc, int st, uint32_t d_col, bool acc) {
        const uint64_t bst = b_desc + off16(st * L::Q_TILE);
#pragma unroll
        for (int kb = 0; kb < BM / 64; ++kb) {
          uint32_t a[4];
          uint64_t b[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int k = 4 * kb + i;
            const uint32_t h = static_cast<uint32_t>((16 * k) / L::HALF);
            a[i] = tmem + a_col + 8u * k + h * (L::HALF / 2);
            b[i] = bst + off16(k * 2048);
          }
          mma_ts_x4(tmem + d_col, a, b, idesc_g, (acc || kb > 0) ? 1u : 0u);
        }
      };
      auto mma_dq = [&](int buf) {
        const uint64_t ds = ds_mn + off16(buf * L::DS_TILE);
#pragma unroll
        for (int kb = 0; kb < L::BN / 64; ++kb) {
          uint64_t a[4], b[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int k = 4 * kb + i;
            if constexpr (D == 64) {  // dQ = dS K: A = dS (i contiguous), B = K (d contiguous)
              a[i] = ds + off16(k * 2048);
              b[i] = k_mn + off16(k * 2048);
            } else {                  // dQ^T = K^T dS^T: A = K^T (d contiguous), B = dS^T
              a[i] = k_mn + off16(k * 2048);
              b[i] = ds + off16(k * 2048);
            }
          }
          mma_ss_x4(tmem + L::DQ_COL + (buf % L::DQB) * 64, a, b, idesc_q, kb > 0 ? 1u : 0u);
        }
      };
      bool ok = mbar_wait_w(bar_kv, 0, abort_flag, SITE_BWD_MMA_KV);
      ok = ok && mbar_wait_w(&bar_qf[0], 0, abort_flag, SITE_BWD_MMA_Q);
      tc_fence_after();
      if (ok) {
        mma_scores(k_kd, false, q_kd, 0, L::S_COL);
        mma_commit_w(bar_s);
        if (L::V_IN_TMEM) {
          ok = mbar_wait_w(bar_vt, 0, abort_flag, SITE_BWD_MMA_VT);
          tc_fence_after();
        }
      }
      if (ok) {
        mma_scores(v_kd, L::V_IN_TMEM, do_kd, 0, L::DP_COL);
        mma_commit_w(bar_dp);
      }
      for (int t = 0; ok && t < n_steps; ++t) {
        const int st = t % L::QST;
        const int buf = t & 1;
        const bool next = t + 1 < n_steps;
        const int st1 = (t + 1) % L::QST;
        if (!mbar_wait_w(bar_p, t & 1, abort_flag, SITE_BWD_MMA_P)) { ok = false; break; }
        tc_fence_after();
        mma_grad(L::S_COL, do_mn, st, L::DV_COL, t > 0);
        if (L::EARLY_DV && !next) mma_commit_w(bar_dvd);
        if (next) {
          if (!mbar_wait_w(&bar_qf[st1], ((t + 1) / L::QST) & 1, abort_flag, SITE_BWD_MMA_Q)) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_scores(k_kd, false, q_kd, st1, L::S_COL);
          mma_commit_w(bar_s);
        }
        if (!mbar_wait_w(bar_ds, t & 1, abort_flag, SITE_BWD_MMA_DS)) { ok = false; break; }
        tc_fence_after();
        mma_grad(L::DP_COL, q_mn, st, L::DK_COL, t > 0);
        mma_commit_w(&bar_qe[st]);  // Q(t), dO(t), lse(t), Dvec(t) are no longer read after dK(t)
        if (next) {
          mma_scores(v_kd, L::V_IN_TMEM, do_kd, st1, L::DP_COL);
          mma_commit_w(bar_dp);
        }
        // dQ(t) into TMEM buffer t % DQB once dQ(t - DQB) has been read out of it
        if (t >= L::DQB && !mbar_wait_w(&bar_dqe[(t - L::DQB) & 1], ((t - L::DQB) >> 1) & 1,
                                        abort_flag, SITE_BWD_MMA_DQE)) {
          ok = false;
          break;
        }
        tc_fence_after();
        mma_dq(buf);
        mma_commit_w(&bar_dqf[buf]);
      }
      mma_commit_w(bar_done);
      mma_commit_w(bar_fin);
      mbar_wait_w(bar_fin, 0, abort_flag, SITE_BWD_MMA_FIN);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ compute warpgroups
    const int h = warp >> 2;                  // which half of the query columns
    const int qw = warp & 3;
    const int jl = 32 * qw + lane;            // key row within the tile (= TMEM lane)
    const int kj = k0 + jl;                   // key index
    const uint32_t t_lane = static_cast<uint32_t>(32 * qw) << 16;
    const uint32_t s_cols = tmem + t_lane + L::S_COL + h * L::HALF;    // my S^T columns
    const uint32_t dp_cols = tmem + t_lane + L::DP_COL + h * L::HALF;  // my dP^T columns
    const float scale2 = p.scale2;
    bool ok = true;
    if (L::V_IN_TMEM && h == 0 && n_steps > 0) {
      // V row jl into TMEM as the A operand of dP^T: 16-byte chunk c of sub-tile s holds
      // d = 64s + 8c .. +7 at swizzled position c ^ (jl & 7); a column holds a pair of d.
      const bool got = mbar_wait(bar_kv, 0, abort_flag, SITE_BWD_C_KV);
      ok = __all_sync(0xffffffffu, got);
      if (ok) {
#pragma unroll
        for (int s = 0; s < L::SUB; ++s) {
          uint32_t vr[32];
          const uint8_t* vrow = smem + L::OFF_V + s * L::KV_SUBTILE + jl * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 v4 = *reinterpret_cast<const uint4*>(vrow + ((c ^ (jl & 7)) * 16));
            vr[4 * c] = v4.x;
            vr[4 * c + 1] = v4.y;
            vr[4 * c + 2] = v4.z;
            vr[4 * c + 3] = v4.w;
          }
          tmem_st32(tmem + t_lane + L::VT_COL + 32 * s, vr);
        }
        tmem_st_wait();
        tc_fence_before();
      }
      mbar_arrive(bar_vt);
    }
    int t = 0;
    for (int w = 0; ok && w < G * span; ++w) {
      const int g = w / span;
      const int it = it_first + (w - g * span);
      if (!q_active(it)) continue;
      const int st = t % L::QST;
      const int buf = t & 1;
      const int i0 = it * BM;
      const int c0 = h * L::HALF;             // first query column of this warpgroup
      bool got = mbar_wait(&bar_qf[st], (t / L::QST) & 1, abort_flag, SITE_BWD_C_Q);
      got = got && mbar_wait(bar_s, t & 1, abort_flag, SITE_BWD_C_S);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
      const float4* lse4 = reinterpret_cast<const float4*>(s_lse + st * BM + c0);
      const float4* dv4 = reinterpret_cast<const float4*>(s_dvec + st * BM + c0);
      const bool edge = (k0 + 128 > kvlen) || (p.causal && k0 + 32 * qw + 31 > i0 + c0);
      // ---- P = 2^(s*scale2 - lse2), written to TMEM in bf16.  For dS it is kept in fp32 when
      // one 32-column chunk per thread fits the register budget (d = 128), else as the same
      // bf16 pairs that feed the dV MMA (d = 64).
      constexpr bool kP32 = L::NCH == 1;
      float pf[kP32 ? 32 : 1];
      uint32_t pk[L::NCH][16];
#pragma unroll
      for (int c = 0; c < L::NCH; ++c) {
        uint32_t sr[32];
        tmem_ld32(s_cols + 32 * c, sr);
        tmem_ld_wait();
        reg_fence(sr);
        float pv[32];
        // x = s*scale2 - lse2 in packed pairs; on tiles without masked keys one pair in
        // L::EMU_EVERY takes 2^x on the FMA pipe, the rest on MUFU
        auto p_chunk = [&](bool masked) {
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const float4 l4 = lse4[8 * c + u];
            float x[4];
            ffma2(x[0], x[1], __uint_as_float(sr[4 * u]), __uint_as_float(sr[4 * u + 1]), scale2,
                  scale2, -l4.x, -l4.y);
            ffma2(x[2], x[3], __uint_as_float(sr[4 * u + 2]), __uint_as_float(sr[4 * u + 3]), scale2,
                  scale2, -l4.z, -l4.w);
#pragma unroll
            for (int hp = 0; hp < 2; ++hp) {
              const int i = 4 * u + 2 * hp;
              float p0, p1;
              if (!masked && L::EMU_EVERY > 0 && ((i >> 1) % (L::EMU_EVERY > 0 ? L::EMU_EVERY : 1)) == L::EMU_EVERY - 1) {
                exp2_fma2(p0, p1, x[2 * hp], x[2 * hp + 1]);
              } else {
                p0 = ex2_approx(x[2 * hp]);
                p1 = ex2_approx(x[2 * hp + 1]);
              }
              if (masked) {
                const int qi = i0 + c0 + 32 * c + i;
                if (kj >= kvlen || (p.causal && kj > qi)) p0 = 0.f;
                if (kj >= kvlen || (p.causal && kj > qi + 1)) p1 = 0.f;
              }
              pv[i] = p0;
              pv[i + 1] = p1;
            }
          }
        };
        if (edge) p_chunk(true);
        else p_chunk(false);
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[c][i] = pack_bf16x2(pv[2 * i], pv[2 * i + 1]);
        if constexpr (kP32) {
#pragma unroll
          for (int i = 0; i < 32; ++i) pf[i] = pv[i];
        }
        tmem_st16(s_cols + 16 * c, pk[c]);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_p);
      // ---- dS = P (dP - Dvec): bf16 into TMEM (over my dP^T) and into smem for the dQ MMA
      got = mbar_wait(bar_dp, t & 1, abort_flag, SITE_BWD_C_DP);
      // dS^T buffer buf was read by dQ(t-2) and, at d = 64, then held dQ(t-2)'s staged boxes
      if (t >= 2) {
        if constexpr (L::V_IN_TMEM)
          got = got && mbar_wait(&bar_dqf[buf], ((t - 2) >> 1) & 1, abort_flag, SITE_BWD_C_DQ);
        else
          got = got && mbar_wait(&bar_dsf[buf], ((t - 2) >> 1) & 1, abort_flag, SITE_BWD_C_DQ);
      }
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
      uint8_t* ds_row = smem + L::OFF_DS + buf * L::DS_TILE + jl * 128;
#pragma unroll
      for (int c = 0; c < L::NCH; ++c) {
        uint32_t dr[32];
        tmem_ld32(dp_cols + 32 * c, dr);
        tmem_ld_wait();
        reg_fence(dr);
        float dsv[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float4 d4 = dv4[8 * c + u];
          const float dvv[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = 4 * u + e;
            float pe;
            if constexpr (kP32) {
              pe = pf[i];
            } else {
              const uint32_t w = pk[c][i >> 1];
              pe = __uint_as_float((i & 1) ? (w & 0xffff0000u) : (w << 16));
            }
            dsv[i] = pe * (__uint_as_float(dr[i]) - dvv[e]);
          }
        }
        uint32_t dd[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) dd[i] = pack_bf16x2(dsv[2 * i], dsv[2 * i + 1]);
        tmem_st16(dp_cols + 16 * c, dd);
        // dS^T row jl, query columns c0+32c .. +31 -> 4 swizzled 16-byte chunks
        const int col = c0 + 32 * c;
        const int iblk = col >> 6;
        const int chunk0 = (col & 63) >> 3;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int pos = (chunk0 + u) ^ (jl & 7);
          *reinterpret_cast<uint4*>(ds_row + iblk * L::DS_IBLK + pos * 16) =
              make_uint4(dd[4 * u], dd[4 * u + 1], dd[4 * u + 2], dd[4 * u + 3]);
        }
      }
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar_ds);
      ++t;
    }
    // ---------------------------------------------------------------- epilogue: dK, dV
    // warpgroup 0 writes dV, warpgroup 1 writes dK (x scale)
    const bool early = L::EARLY_DV && h == 0 && n_steps > 0;
    if (ok && n_steps > 0) {
      // early dV: its staging buffer held dS(t-2), last read by dQ(t-2) (finished before the
      // last dV) and by the dQ warps' boxes of that step
      bool got = mbar_wait(early ? bar_dvd : bar_done, 0, abort_flag, SITE_BWD_C_DONE);
      if (early && t >= 2)
        got = got && mbar_wait(&bar_dsf[t & 1], ((t - 2) >> 1) & 1, abort_flag, SITE_BWD_C_DQ);
      ok = __all_sync(0xffffffffu, got);
      tc_fence_after();
    }
    if (ok) {
      // This warp's 32 key rows are staged as D/64 [32 rows][64 d] bf16 boxes with the 128-byte
      // swizzle (16-byte chunk c of row r at chunk c ^ (r & 7), so the 32 lanes' stores spread
      // over all banks) in the Q ring, which no MMA or load touches any more (bar_done follows
      // the last MMA), and written by one TMA store per box (rows past N are not written).
      // Per-lane 16-byte stores to rows 2D bytes apart cost one memory transaction per lane.
      const uint32_t col0 = h == 0 ? L::DV_COL : L::DK_COL;
      const float mul = h == 0 ? 1.0f : p.scale;
      uint8_t* stg = early ? smem + L::OFF_DS + (t & 1) * L::DS_TILE + warp * (D / 64) * 4096
                           : smem + L::OFF_Q + warp * (D / 64) * 4096;
      static_assert(8 * (D / 64) * 4096 <= L::QST * L::Q_TILE, "dK/dV staging fits the Q ring");
      static_assert(!L::EARLY_DV || 4 * (D / 64) * 4096 <= L::DS_TILE, "dV staging fits a dS^T buffer");
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t g[32];
        if (n_steps > 0) {
          tmem_ld32(tmem + t_lane + col0 + 32 * c, g);
          tmem_ld_wait();
          reg_fence(g);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) g[i] = 0u;
        }
        uint32_t hv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          hv[i] = pack_bf16x2(__uint_as_float(g[2 * i]) * mul, __uint_as_float(g[2 * i + 1]) * mul);
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
  } else {
    // ------------------------------------------------------------------ dQ warpgroup
    if constexpr (L::OVERLAP_PREV) grid_dep_wait();  // the preprocess zeroes the accumulator
    const int qw = warp & 3;
    const uint32_t t_lane = static_cast<uint32_t>(32 * qw) << 16;
    int t = 0;
    for (int w = 0; w < G * span; ++w) {
      const int g = w / span;
      const int it = it_first + (w - g * span);
      if (!q_active(it)) continue;
      const int bh = bhq0 + g;                // query head of this step
      const int buf = t & 1;
      const int i0 = it * BM;
      const bool got = mbar_wait(&bar_dqf[buf], (t >> 1) & 1, abort_flag, SITE_BWD_DQ);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      uint32_t v[2][32];
      tmem_ld32(tmem + t_lane + L::DQ_COL + (buf % L::DQB) * 64, v[0]);
      tmem_ld32(tmem + t_lane + L::DQ_COL + (buf % L::DQB) * 64 + 32, v[1]);
      tmem_ld_wait();
      reg_fence(v[0]);
      reg_fence(v[1]);
      tc_fence_before();
      mbar_arrive(&bar_dqe[buf]);
      if constexpr (D == 64) {
        // lane = query row i0 + 32qw + lane, 64 columns of dQ: staged as this warp's [32 rows]
        // [64 d] box in dS^T buffer buf (dQ(t), the last reader of that buffer, has completed),
        // as two [32 rows][32 d] halves with the 128-byte swizzle (16-byte chunk c of row r at
        // chunk c ^ (r & 7): the 32 lanes' stores spread over all banks), and added to the
        // accumulator by two TMA reduce-adds (rows >= N are skipped).  Once the reduce-adds have
        // read the box, the buffer goes back to the compute warpgroups.
        uint8_t* stg = smem + L::OFF_DS + buf * L::DS_TILE + qw * L::DQ64_STAGE;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<float4*>(stg + hh * 4096 + lane * 128 + ((c ^ (lane & 7)) * 16)) =
                make_float4(__uint_as_float(v[hh][4 * c]), __uint_as_float(v[hh][4 * c + 1]),
                            __uint_as_float(v[hh][4 * c + 2]), __uint_as_float(v[hh][4 * c + 3]));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_3d(&tm_dq, stg, 0, i0 + 32 * qw, bh);
          tma_reduce_add_3d(&tm_dq, stg + 4096, 32, i0 + 32 * qw, bh);
          bulk_commit_group();
          bulk_wait_read_all();
          mbar_arrive(&bar_dsf[buf]);
        }
        __syncwarp();
      } else {
        // lane = head dimension 32qw + lane, columns = query rows i0 .. i0+63: staged as this
        // warp's [64][32] fp32 box in the V tile (V lives in TMEM by now: dQ(0) follows the
        // copy) and added to the accumulator by one TMA reduce (rows >= N are skipped).
        float* stg = reinterpret_cast<float*>(smem + L::OFF_V + qw * L::DQ_STAGE);
        if (t > 0) {
          if (lane == 0) bulk_wait_read_all();  // the previous box has been read
          __syncwarp();
        }
#pragma unroll
        for (int i = 0; i < 64; ++i) stg[i * 32 + lane] = __uint_as_float(v[i >> 5][i & 31]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_3d(&tm_dq, stg, 32 * qw, i0, bh);
          bulk_commit_group();
        }
      }
      ++t;
    }
    if (lane == 0) bulk_wait_all();  // the reductions are complete before the CTA ends
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

}  // namespace fa
