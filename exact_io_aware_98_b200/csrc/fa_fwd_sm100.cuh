// fa_fwd_sm100.cuh -- exact attention forward on sm_100a: TMA-fed tiles, tcgen05 MMAs with
// TMEM accumulators, online softmax in warp-specialised warpgroups.
//
// Computes, per (b, h): S = scale * Q K^T with masked keys at -inf, A = row softmax of S,
// O = A V, and the per-row log-sum-exp of S ("Attention optimisation: FlashAttention and
// sparse attention", mdooai Ch.04, core formula and the sparse-masking paragraph), without
// ever writing S or A to HBM: the five stages of "What is FlashAttention? Why smarter memory
// use speeds up transformers" (tile Q/K/V; load small blocks on chip; local scores with a
// running normalisation; accumulate the output without materialising the full matrix;
// schedule for the target accelerator).
//
// CTA layout (320 threads):
//   warps 0-3  softmax warpgroup for Q tile 0 (rows m0 .. m0+127), one thread per row
//   warps 4-7  softmax warpgroup for Q tile 1 (rows m0+128 .. m0+255)
//   warp  8    TMA producer: Q once, then K and V tiles of BN keys through separate rings
//              (a K stage frees as soon as both S MMAs of its tile finish, a V stage after
//              both PV MMAs, so K runs further ahead than a shared ring would allow)
//   warp  9    MMA issuer (whole warp, one elected lane issues): S_w = Q_w K^T into TMEM,
//              O_w += P_w V with P taken from TMEM
// TMEM: S_0 [0,BN), S_1 [BN,2BN), O_0 [2BN,2BN+D), O_1 [2BN+D,2BN+2D).  P_w (bf16, two per
// 32-bit column) overwrites columns [0,BN/2) of S_w after the softmax warpgroup has read S_w
// into registers.
// Key-tile width BN: 128 at d = 128 (one CTA per SM, all 512 TMEM columns).  At d = 64 it is
// 64, which halves TMEM (256 columns) and shared memory (~100 KB) per CTA so that two CTAs share
// an SM: the head dimension is small, the softmax (one exponential per score whatever d is)
// dominates, and one CTA's set-up, first loads and epilogue -- about 5 us between consecutive
// CTAs on an SM, measured -- then overlap the other CTA's loop, while four softmax warpgroups
// per SM keep the exponential units busy during each other's MMA round trips.
//
// Per KV tile the MMA thread issues, for w = 0 then 1: PV_w of the previous tile, then S_w of
// this tile.  tcgen05 MMAs from one thread execute in issue order, so S_w(t+1) cannot overwrite
// P_w(t) before PV_w(t) has read it, and the commit that signals S_w(t+1) also certifies that
// PV_w(t) has finished -- which is what lets a softmax warpgroup rescale O_w right after it
// sees S_w(t+1), with no extra barrier.
//
// Online softmax (log2 domain, scale2 = scale*log2 e): the running reference m is raised only
// when a tile's maximum exceeds it by more than 8 (a factor 256); O and l are then multiplied
// by 2^(m_old - m_new).  P = 2^(s*scale2 - m) <= 256 and l accumulate exactly as with an
// always-updated maximum, and the final O/l and lse = (m + log2 l) ln 2 use the same m, so the
// result is the same softmax.
#pragma once
#include "ptx.cuh"

namespace fa {

struct FwdParams {
  const uint8_t* block_mask;  // [nb][nb] (nb = ceil(N/128)) or nullptr
  const int32_t* kv_len;      // [B] or nullptr
  __nv_bfloat16* o;           // [B*H][N][D]
  float* o32;                 // [B*H][N][D] fp32 O/l, written instead of o by the O32 variant
  float* lse;                 // [B*H][N]
  int B, H, N;
  int H_kv;                   // K/V heads; query head h reads K/V head h / (H / H_kv)
  int n_mtiles;               // ceil(N / 256)
  int hgroup;                 // query heads per CTA-order group (>= 1; B*H: one group)
  float scale2;               // scale * log2(e)
  int causal;
};

// Key-tile width: fwd_bn<D> keys per KV tile in the library's forward; the deviation study
// also runs d = 64 with 128-key tiles.
template <int D>
constexpr int fwd_bn() { return D == 64 ? 64 : 128; }

template <int D, int BN_ = fwd_bn<D>()>
struct FwdLayout {
  static constexpr int BM = 128;                    // query rows per Q tile
  static constexpr int BN = BN_;                    // keys per KV tile
  static constexpr int CTAS_PER_SM = BN == 64 ? 2 : 1;
  static constexpr int KST = BN == 64 ? 4 : (D == 64 ? 5 : 3);  // K ring depth
  static constexpr int VST = BN == 64 ? 4 : (D == 64 ? 4 : 2);  // V ring depth
  static constexpr int SUB = D / 64;                // 64-column (128-byte) sub-tiles
  static constexpr int SUBTILE = 128 * 128;         // bytes of one 128-row x 64-col Q sub-tile
  static constexpr int TILE = 128 * D * 2;          // bytes of one 128-row Q tile
  static constexpr int KV_SUBTILE = BN * 128;       // bytes of one BN-row x 64-col K/V sub-tile
  static constexpr int KV_TILE = BN * D * 2;        // bytes of one K or V tile
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * TILE;
  static constexpr int OFF_V = OFF_K + KST * KV_TILE;
  static constexpr int OFF_BAR = OFF_V + VST * KV_TILE;
  // q, k_full[KST], k_empty[KST], v_full[VST], v_empty[VST], s_full[2], p_full[2], o_done[2], fin
  // P in two key halves (128-key tiles): the MMA warp issues P.V over keys 0-63 as soon as that
  // half of P is in TMEM, while the softmax warpgroup computes the exponentials of keys 64-127
  static constexpr bool SPLIT_P = BN == 128;
  // q, k_full[KST], k_empty[KST], v_full[VST], v_empty[VST], s_full[2], p_full[2], o_done[2],
  // p2_full[2], fin
  static constexpr int NBAR = 1 + 2 * KST + 2 * VST + 6 + 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  // block-mask CTA order (d = 64): per Q tile its unmasked blocks, then the Q tiles by that count
  static constexpr int OFF_ORD = OFF_MISC + 16;
  static constexpr int BYTES = OFF_ORD + 2 * 64 * 4;          // 2 x FWD_RANK_TILES ints
  static constexpr int SMEM_ALLOC = BYTES + 1024;   // slack for 1024-byte alignment
  static_assert(CTAS_PER_SM * (SMEM_ALLOC + 1024) <= 233472, "shared memory per SM");
  static constexpr uint32_t TMEM_COLS = 2 * BN + 2 * D <= 256 ? 256 : 512;
  static constexpr uint32_t O_COL0 = 2 * BN;
  static_assert(O_COL0 + 2 * D <= TMEM_COLS, "TMEM budget");
  // one P pair in EMU_EVERY is exponentiated on the FMA pipe (0 = all on MUFU)
  static constexpr int EMU_EVERY = 4;
  __device__ static constexpr uint32_t s_col(int w) { return static_cast<uint32_t>(w) * BN; }
};

// Block-mask CTA order: the Q tile (256 rows) of rank `rank` when the Q tiles are ordered by
// their number of unmasked 128 x 128 blocks (causal: on or below the diagonal), most first, ties
// to the later Q tile.  Every thread of the CTA calls it (three barriers); s_wt and s_ord are
// FWD_RANK_TILES ints each of shared memory.
constexpr int FWD_RANK_TILES = 64;  // Q tiles ranked (N <= 16384)
__device__ __noinline__ int fwd_ranked_qtile(const uint8_t* __restrict__ block_mask, int N,
                                             int n_mtiles, int causal, int rank, int* s_wt,
                                             int* s_ord) {
  if (static_cast<int>(threadIdx.x) < n_mtiles) s_wt[threadIdx.x] = 0;
  __syncthreads();
  const int nbm = (N + 127) / 128;
  for (int e = threadIdx.x; e < nbm * nbm; e += blockDim.x) {
    const int r = e / nbm, c = e - r * nbm;  // query block r, key block c
    if (block_mask[e] && (!causal || c <= r)) atomicAdd(&s_wt[r >> 1], 1);
  }
  __syncthreads();
  if (static_cast<int>(threadIdx.x) < n_mtiles) {
    const int i = threadIdx.x, wi = s_wt[i];
    int rk = 0;
    for (int j = 0; j < n_mtiles; ++j) {
      const int wj = s_wt[j];
      rk += (wj > wi || (wj == wi && j > i)) ? 1 : 0;
    }
    s_ord[rk] = i;
  }
  __syncthreads();
  return s_ord[rank];
}

// Wait-site codes recorded in the status word on a timeout.
enum : int {
  SITE_FWD_LOAD_EMPTY = 1, SITE_FWD_LOAD_DRAIN = 2, SITE_FWD_MMA_Q = 3, SITE_FWD_MMA_K = 4,
  SITE_FWD_MMA_V = 5, SITE_FWD_MMA_P = 6, SITE_FWD_MMA_FIN = 7, SITE_FWD_SM_S = 8,
  SITE_FWD_SM_O = 9
};

// O32: write the fp32 O/l to p.o32 instead of bf16 O to p.o (the deviation study's view of the
// output before its bf16 rounding).
// RANKED: the CTA order ranks the Q tiles by their unmasked blocks (block-masked calls; a
// separate instantiation, since the ranking changes the register allocation of the loop).
template <int D, int BN_ = fwd_bn<D>(), bool O32 = false, bool RANKED = false>
__global__ void __launch_bounds__(320, FwdLayout<D, BN_>::CTAS_PER_SM)
fa_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_o, const FwdParams p) {
  using L = FwdLayout<D, BN_>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* bar_q = bars;
  uint64_t* bar_kf = bars + 1;
  uint64_t* bar_ke = bar_kf + L::KST;
  uint64_t* bar_vf = bar_ke + L::KST;
  uint64_t* bar_ve = bar_vf + L::VST;
  uint64_t* bar_sf = bar_ve + L::VST;
  uint64_t* bar_pf = bar_sf + 2;
  uint64_t* bar_od = bar_pf + 2;
  uint64_t* bar_p2 = bar_od + 2;          // [2] second half of P_w in TMEM (SPLIT_P)
  uint64_t* bar_fin = bar_p2 + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int BH = p.B * p.H;
  // CTA order: groups of p.hgroup heads in turn (a group's Q, K, V and O fit in L2), and
  // inside a group the heaviest Q tiles first: the last rows under a causal mask, or, RANKED
  // (block masks), the Q tiles with the most unmasked blocks, counted by every CTA from the
  // mask, so that the longest CTAs do not start last.
  const int per_group = p.hgroup * p.n_mtiles;
  const int grp = static_cast<int>(blockIdx.x) / per_group;
  const int g0 = grp * p.hgroup;
  const int gn = min(p.hgroup, BH - g0);               // heads in this group (the last may have fewer)
  const int slot = static_cast<int>(blockIdx.x) - grp * per_group;
  const int mt = RANKED ? fwd_ranked_qtile(p.block_mask, p.N, p.n_mtiles, p.causal, slot / gn,
                                           reinterpret_cast<int*>(smem + L::OFF_ORD),
                                           reinterpret_cast<int*>(smem + L::OFF_ORD) + FWD_RANK_TILES)
                        : p.n_mtiles - 1 - slot / gn;
  const int bh = g0 + slot % gn;
  const int b = bh / p.H;
  const int bh_kv = b * p.H_kv + (bh % p.H) / (p.H / p.H_kv);  // K/V head of this query head
  const int N = p.N;
  const int m0 = mt * 256;
  int kvlen = N;
  if (p.kv_len != nullptr) kvlen = min(max(p.kv_len[b], 0), N);
  constexpr int BN = L::BN;
  const int nb = (N + 127) / 128;                      // 128 x 128 blocks of the block mask
  const int n_kv = (kvlen + BN - 1) / BN;
  int j_end = n_kv;
  if (p.causal) j_end = min(j_end, (min(m0 + 256, N) - 1) / BN + 1);

  // bit w set: KV tile j holds at least one key that Q tile w may attend to
  auto flags_of = [&](int j) -> int {
    int f = 0;
    const int k0 = j * BN;
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      const int q0 = m0 + 128 * w;
      if (q0 >= N) continue;
      const int q1 = min(q0 + 127, N - 1);
      if (p.causal && k0 > q1) continue;
      if (p.block_mask != nullptr && !p.block_mask[static_cast<size_t>(q0 >> 7) * nb + (k0 >> 7)])
        continue;
      f |= 1 << w;
    }
    return f;
  };

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
    for (int w = 0; w < 2; ++w) {
      mbar_init(&bar_sf[w], 1);
      mbar_init(&bar_pf[w], 128);
      mbar_init(&bar_p2[w], 128);
      mbar_init(&bar_od[w], 1);
    }
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
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const int nq = (m0 + 128 < N) ? 2 : 1;
      mbar_arrive_expect_tx(bar_q, nq * L::TILE);
      for (int w = 0; w < nq; ++w)
        for (int s = 0; s < L::SUB; ++s)
          tma_load_3d(smem + L::OFF_Q + w * L::TILE + s * L::SUBTILE, &tm_q, bar_q, s * 64,
                      m0 + 128 * w, bh);
      int kn = 0, vn = 0;  // K and V tiles issued so far
      for (int j = 0; j < j_end; ++j) {
        if (flags_of(j) == 0) continue;
        const int ks = kn % L::KST, vs = vn % L::VST;
        if (kn >= L::KST &&
            !mbar_wait(&bar_ke[ks], ((kn / L::KST) - 1) & 1, abort_flag, SITE_FWD_LOAD_EMPTY))
          break;
        mbar_arrive_expect_tx(&bar_kf[ks], L::KV_TILE);
        for (int s = 0; s < L::SUB; ++s)
          tma_load_3d(smem + L::OFF_K + ks * L::KV_TILE + s * L::KV_SUBTILE, &tm_k, &bar_kf[ks],
                      s * 64, j * BN, bh_kv);
        ++kn;
        if (vn >= L::VST &&
            !mbar_wait(&bar_ve[vs], ((vn / L::VST) - 1) & 1, abort_flag, SITE_FWD_LOAD_EMPTY))
          break;
        mbar_arrive_expect_tx(&bar_vf[vs], L::KV_TILE);
        for (int s = 0; s < L::SUB; ++s)
          tma_load_3d(smem + L::OFF_V + vs * L::KV_TILE + s * L::KV_SUBTILE, &tm_v, &bar_vf[vs],
                      s * 64, j * BN, bh_kv);
        ++vn;
      }
      // Never leave the CTA with a copy in flight: wait for the last loads of every stage
      // (immediate in the normal path, where the MMA thread consumed them).
      mbar_wait(bar_q, 0, abort_flag, SITE_FWD_LOAD_DRAIN);
      for (int r = max(0, kn - L::KST); r < kn; ++r)
        mbar_wait(&bar_kf[r % L::KST], (r / L::KST) & 1, abort_flag, SITE_FWD_LOAD_DRAIN);
      for (int r = max(0, vn - L::VST); r < vn; ++r)
        mbar_wait(&bar_vf[r % L::VST], (r / L::VST) & 1, abort_flag, SITE_FWD_LOAD_DRAIN);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA issuer
    // The whole warp walks the loop (descriptors stay warp-uniform); one elected lane issues.
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, BN, false, false);
    constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, false, true);
    // Base descriptors; stage, sub-tile and K-step offsets are added to the start-address
    // field (16-byte units).  Q/K: K-major, 128-byte rows, 8-row groups 1 KB apart.
    // V: MN-major, 64-column blocks one sub-tile apart.
    const uint64_t q_desc = sdesc_sw128(smem_u32(smem + L::OFF_Q), 16, 1024);
    const uint64_t k_desc = sdesc_sw128(smem_u32(smem + L::OFF_K), 16, 1024);
    const uint64_t v_desc = sdesc_sw128(smem_u32(smem + L::OFF_V), L::KV_SUBTILE, 1024);
    // K-step k of a K-major operand whose 64-column sub-tiles are `sub` bytes apart, in
    // 16-byte units
    auto koff = [](int k, int sub) -> uint64_t {
      return static_cast<uint64_t>(((k >> 2) * sub + (k & 3) * 32) >> 4);
    };
    bool ok = mbar_wait_w(bar_q, 0, abort_flag, SITE_FWD_MMA_Q);
    tc_fence_after();
    int it = 0;
    int cnt0 = 0, cnt1 = 0;
    int prev_flags = 0, prev_vs = 0;
    // O_w += P_w V(vs): P_w from TMEM (bf16 pairs over S_w), V MN-major.
    // With SPLIT_P the second batch of four K-steps (keys 64-127) waits for the second half of P.
    auto issue_pv = [&](int w, int vs, int& cnt) -> bool {
      if (!mbar_wait_w(&bar_pf[w], cnt & 1, abort_flag, SITE_FWD_MMA_P)) return false;
      tc_fence_after();
      const uint32_t a_tmem = tmem + L::s_col(w);
      const uint32_t d_tmem = tmem + L::O_COL0 + w * D;
      const uint64_t vb = v_desc + static_cast<uint64_t>((vs * L::KV_TILE) >> 4);
#pragma unroll
      for (int kb = 0; kb < L::BN / 64; ++kb) {
        if (L::SPLIT_P && kb == 1) {
          if (!mbar_wait_w(&bar_p2[w], cnt & 1, abort_flag, SITE_FWD_MMA_P)) return false;
          tc_fence_after();
        }
        uint32_t a[4];
        uint64_t b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int k = 4 * kb + i;
          a[i] = a_tmem + 8 * k;
          b[i] = vb + static_cast<uint64_t>((k * 2048) >> 4);
        }
        mma_ts_x4(d_tmem, a, b, idesc_o, (cnt > 0 || kb > 0) ? 1u : 0u);
      }
      mma_commit_w(&bar_od[w]);
      ++cnt;
      return true;
    };
    // S_w = Q_w K(ks)^T
    auto issue_s = [&](int w, int ks) {
      const uint64_t qa = q_desc + static_cast<uint64_t>((w * L::TILE) >> 4);
      const uint64_t kb0 = k_desc + static_cast<uint64_t>((ks * L::KV_TILE) >> 4);
#pragma unroll
      for (int kb = 0; kb < D / 64; ++kb) {
        uint64_t a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          a[i] = qa + koff(4 * kb + i, L::SUBTILE);
          b[i] = kb0 + koff(4 * kb + i, L::KV_SUBTILE);
        }
        mma_ss_x4(tmem + L::s_col(w), a, b, idesc_s, kb > 0 ? 1u : 0u);
      }
      mma_commit_w(&bar_sf[w]);
    };
    for (int j = 0; ok && j < j_end; ++j) {
      const int f = flags_of(j);
      if (f == 0) continue;
      const int ks = it % L::KST, vs = it % L::VST;
      if (!mbar_wait_w(&bar_kf[ks], (it / L::KST) & 1, abort_flag, SITE_FWD_MMA_K)) { ok = false; break; }
      if (prev_flags != 0 &&
          !mbar_wait_w(&bar_vf[prev_vs], ((it - 1) / L::VST) & 1, abort_flag, SITE_FWD_MMA_V)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // for w = 0 then 1: PV_w of the previous tile, then S_w of this tile
      if (prev_flags & 1) ok = ok && issue_pv(0, prev_vs, cnt0);
      if (ok && (f & 1)) issue_s(0, ks);
      if (ok && (prev_flags & 2)) ok = issue_pv(1, prev_vs, cnt1);
      if (ok && (f & 2)) issue_s(1, ks);
      if (!ok) break;
      mma_commit_w(&bar_ke[ks]);                          // K(j) read by both S MMAs
      if (prev_flags != 0) mma_commit_w(&bar_ve[prev_vs]);  // V(prev) read by both PV MMAs
      prev_flags = f;
      prev_vs = vs;
      ++it;
    }
    if (ok && prev_flags != 0) {
      if (mbar_wait_w(&bar_vf[prev_vs], ((it - 1) / L::VST) & 1, abort_flag, SITE_FWD_MMA_V)) {
        tc_fence_after();
        if (prev_flags & 1) ok = issue_pv(0, prev_vs, cnt0);
        if (ok && (prev_flags & 2)) ok = issue_pv(1, prev_vs, cnt1);
        mma_commit_w(&bar_ve[prev_vs]);
      }
    }
    // all MMAs issued by this warp have completed before TMEM is released
    mma_commit_w(bar_fin);
    mbar_wait_w(bar_fin, 0, abort_flag, SITE_FWD_MMA_FIN);
  } else {
    // ------------------------------------------------------------------ softmax warpgroups
    const int w = warp >> 2;
    const int qw = warp & 3;
    const int row_in_tile = 32 * qw + lane;
    const int q0 = m0 + 128 * w;
    const int row = q0 + row_in_tile;
    const uint32_t t_lane = static_cast<uint32_t>(32 * qw) << 16;
    const uint32_t t_s = tmem + t_lane + L::s_col(w);
    const uint32_t t_o = tmem + t_lane + L::O_COL0 + w * D;
    const float scale2 = p.scale2;
    float m_ref = -INFINITY;  // running reference maximum (log2 domain, scaled)
    float l = 0.f;            // running row sum of P
    int cnt = 0;
    bool ok = true;
    for (int j = 0; j < j_end; ++j) {
      if (!((flags_of(j) >> w) & 1)) continue;
      const bool got = mbar_wait(&bar_sf[w], cnt & 1, abort_flag, SITE_FWD_SM_S);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
      constexpr int NC = BN / 32;  // 32-column chunks of S_w
      uint32_t r[NC][32];
#pragma unroll
      for (int c = 0; c < NC; ++c) tmem_ld32(t_s + 32 * c, r[c]);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < NC; ++c) reg_fence(r[c]);
      const int k0 = j * BN;
      const bool edge = (k0 + BN > kvlen) || (p.causal && k0 + BN - 1 > q0 + 32 * qw);
      if (edge) {
#pragma unroll
        for (int c = 0; c < NC; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int col = k0 + 32 * c + i;
            if (col >= kvlen || (p.causal && col > row)) r[c][i] = __float_as_uint(-INFINITY);
          }
      }
      // row maximum: eight independent chains of 3-input max
      float mc[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mc[u] = -INFINITY;
#pragma unroll
      for (int k = 0; k < BN; k += 2)
        mc[(k >> 1) & 7] = fmax3(mc[(k >> 1) & 7], __uint_as_float(r[k >> 5][k & 31]),
                                 __uint_as_float(r[k >> 5][(k & 31) + 1]));
      const float mx = fmax3(fmax3(mc[0], mc[1], mc[2]), fmax3(mc[3], mc[4], mc[5]),
                             fmaxf(mc[6], mc[7]));
      const float tmax = mx * scale2;
      float m_new = m_ref;
      if (tmax > m_ref + 8.0f) m_new = tmax;  // also taken when m_ref is still -inf
      const float alpha = (m_new == m_ref) ? 1.0f : ex2_approx(m_ref - m_new);
      const float neg_base = (m_new == -INFINITY) ? 0.0f : -m_new;
      const bool rescale = (cnt > 0) && (m_new != m_ref);
      m_ref = m_new;
      // P = 2^(s*scale2 - m) in pairs: packed fp32x2 scale-and-shift and row sums (four
      // independent accumulator pairs).  On tiles without masked elements, one pair in
      // L::EMU_EVERY takes 2^x on the FMA pipe instead of MUFU, which the other pairs keep busy.
      // P goes to TMEM (bf16 over the front of S_w) and is handed to the MMA warp in halves of
      // the key tile with SPLIT_P, else at once.
      float ra[4] = {0.f, 0.f, 0.f, 0.f}, rb[4] = {0.f, 0.f, 0.f, 0.f};
      // chunk c (32 keys) of P; called with compile-time c so that r[c] stays in registers
      auto exp_chunk = [&](bool use_fma, int c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int q = 16 * c + i;
          float x0, x1, p0, p1;
          ffma2(x0, x1, __uint_as_float(r[c][2 * i]), __uint_as_float(r[c][2 * i + 1]), scale2,
                scale2, neg_base, neg_base);
          if (use_fma && L::EMU_EVERY > 0 && (q % (L::EMU_EVERY > 0 ? L::EMU_EVERY : 1)) == L::EMU_EVERY - 1) {
            exp2_fma2(p0, p1, x0, x1);
          } else {
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
          }
          fadd2(ra[q & 3], rb[q & 3], ra[q & 3], rb[q & 3], p0, p1);
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st16(t_s + 16 * c, pk);
      };
      auto hand_over = [&](uint64_t* bar) {
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar);
      };
      // O rescale (rare: the reference maximum moved by more than 8), before the first P of
      // this tile is handed over so that it precedes this tile's P.V; PV_w of the previous tile
      // has finished (S_w of this tile was issued after it).  It runs after the first
      // hand-over's exponentials, whose scores no longer occupy registers.
      auto rescale_o = [&]() {
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(t_o + 32 * c, o);
            tmem_ld_wait();
            reg_fence(o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(t_o + 32 * c, o);
          }
        }
      };
      // masked elements are -inf: MUFU gives exact zeros, so edge tiles take no FMA-pipe 2^x
      constexpr int C1 = L::SPLIT_P ? NC / 2 : NC;  // chunks of the first hand-over
      if (edge) {
#pragma unroll
        for (int c = 0; c < C1; ++c) exp_chunk(false, c);
      } else {
#pragma unroll
        for (int c = 0; c < C1; ++c) exp_chunk(true, c);
      }
      rescale_o();
      hand_over(&bar_pf[w]);
      if constexpr (L::SPLIT_P) {
        if (edge) {
#pragma unroll
          for (int c = C1; c < NC; ++c) exp_chunk(false, c);
        } else {
#pragma unroll
          for (int c = C1; c < NC; ++c) exp_chunk(true, c);
        }
        hand_over(&bar_p2[w]);
      }
      l = alpha * l + ((ra[0] + ra[1]) + (ra[2] + ra[3]) + ((rb[0] + rb[1]) + (rb[2] + rb[3])));
      ++cnt;
    }
    // ---------------------------------------------------------------- epilogue: O / l, lse
    if (ok && q0 < N) {
      if (cnt > 0) {
        const bool got = mbar_wait(&bar_od[w], (cnt - 1) & 1, abort_flag, SITE_FWD_SM_O);
        ok = __all_sync(0xffffffffu, got);
        tc_fence_after();
      }
      // bf16 O at d = 64: this warp's 32 rows staged as a [32 rows][64 d] box with the 128-byte
      // swizzle (16-byte chunk c of row r at chunk c ^ (r & 7)) in its own Q tile, which no MMA
      // reads any more (the last P.V of this Q tile has finished, and every S MMA before it), then
      // one TMA store (rows past N are not written).  Per-lane 16-byte stores to rows 2D bytes
      // apart cost one memory transaction per lane, which two CTAs per SM feel in every CTA's
      // turnaround; at d = 128 (one CTA per SM) those stores drain after the CTA has gone,
      // while the TMA store's read of the staging box would sit on the CTA's exit.
      constexpr bool TMA_O = !O32 && D == 64;
      if constexpr (TMA_O) {
        // no key tile for this Q tile (no keys, or its block-mask row is empty): the Q load the
        // staging area belongs to may still be in flight
        if (cnt == 0) ok = __all_sync(0xffffffffu, mbar_wait(bar_q, 0, abort_flag, SITE_FWD_SM_O));
      }
      const float inv = (l > 0.f) ? 1.0f / l : 0.0f;
      float* orow32 = p.o32 + (static_cast<size_t>(bh) * N + row) * D;
      uint8_t* stg = smem + L::OFF_Q + w * L::TILE + qw * (D / 64) * 4096;
      __nv_bfloat16* orow = p.o + (static_cast<size_t>(bh) * N + row) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        if (cnt > 0 && ok) {
          tmem_ld32(t_o + 32 * c, o);
          tmem_ld_wait();
          reg_fence(o);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        if constexpr (O32) {
          if (row < N) {
            float4* dst = reinterpret_cast<float4*>(orow32 + 32 * c);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(o[4 * i]) * inv, __uint_as_float(o[4 * i + 1]) * inv,
                                   __uint_as_float(o[4 * i + 2]) * inv, __uint_as_float(o[4 * i + 3]) * inv);
          }
        } else {
          uint32_t h[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            h[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
          if constexpr (TMA_O) {
            uint8_t* box = stg + (c >> 1) * 4096 + lane * 128;
            if (ok) {
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int q = (c & 1) * 4 + i;  // 16-byte chunk of the 128-byte row
                *reinterpret_cast<uint4*>(box + ((q ^ (lane & 7)) * 16)) =
                    make_uint4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]);
              }
            }
          } else if (row < N) {
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]);
          }
        }
      }
      if (TMA_O && ok) {
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
#pragma unroll
          for (int s = 0; s < D / 64; ++s) tma_store_3d(&tm_o, stg + s * 4096, 64 * s, q0 + 32 * qw, bh);
          bulk_commit_group();
          bulk_wait_read_all();  // the boxes have been read before the CTA ends
        }
        __syncwarp();
      }
      if (row < N)
        p.lse[static_cast<size_t>(bh) * N + row] =
            (l > 0.f) ? (m_ref + __log2f(l)) * 0.69314718055994531f : -INFINITY;
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
