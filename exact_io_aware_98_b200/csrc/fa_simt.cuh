// fa_simt.cuh -- CUDA-core kernels around the tensor-core path:
//   * fa_fwd_rowwarp_kernel: online-softmax forward with one warp per query row, used as
//       - the FP32 path (fp32 inputs, fp32 FMA, exact exp; tensor cores cannot meet the fp32
//         tolerance, and fp32-only use of the method is the hard case the FlashAttention-2
//         article calls out under "fp16/bf16 support"), and
//       - the tile-width reference for the numeric-deviation sweep of "Is Flash Attention
//         Stable?" (aibr.jp summary, section 3): bf16 inputs, the running maximum is updated
//         at every Bc-key tile (no lazy threshold) and P is rounded to bf16 before P.V.  Two
//         more axes of that study are flags: the order in which the key tiles are visited
//         (first to last, or last to first), and whether the normaliser l sums the fp32 P or
//         the bf16-rounded P that enters P.V.
//   * naive_* kernels: the materialised "Baseline Attention" of the same study -- S written to
//     HBM in bf16, row softmax from it with P written back in bf16, then P.V.
//   * bwd_preprocess_kernel / dq_convert_kernel: the elementwise steps around the tensor-core
//     backward (Dvec_i = dO_i . O_i, lse in log2 units, zeroing and converting the dQ
//     accumulator).
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace fa {

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ bool key_allowed(int i, int j, int kvlen, int causal,
                                            const uint8_t* bm, int nb) {
  if (j >= kvlen) return false;
  if (causal && j > i) return false;
  if (bm != nullptr && !bm[static_cast<size_t>(i >> 7) * nb + (j >> 7)]) return false;
  return true;
}

// One warp per query row.  Keys are processed in tiles of `bc` (a multiple of 32, <= 256);
// lane l holds the scores of keys tile0 + 32*u + l.  Output column c = 32*u + lane.
// flags: kTileReverse visits the key tiles last to first; kTileLRounded sums l over the
// rounded P (only meaningful with ROUND_P).  o32 != nullptr: the fp32 O/l goes there instead of
// the rounded O to o.
constexpr int kTileReverse = 1;
constexpr int kTileLRounded = 2;
template <typename T, bool ROUND_P>
__global__ void __launch_bounds__(256)
fa_fwd_rowwarp_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                      T* __restrict__ o, float* __restrict__ lse, const uint8_t* block_mask,
                      const int32_t* kv_len, int B, int H, int N, int d, float scale, int causal,
                      int bc, int flags, int H_kv, float* __restrict__ o32) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row_g = static_cast<long long>(blockIdx.x) * 8 + warp;  // flat bh*N + i
  if (row_g >= static_cast<long long>(B) * H * N) return;
  const int i = static_cast<int>(row_g % N);
  const int bh = static_cast<int>(row_g / N);
  const int b = bh / H;
  int kvlen = N;
  if (kv_len != nullptr) kvlen = min(max(kv_len[b], 0), N);
  const int nb = (N + 127) / 128;
  const T* qi = q + row_g * d;
  const int bh_kv = b * H_kv + (bh % H) / (H / H_kv);  // K/V head of query head bh
  const T* kh = k + static_cast<size_t>(bh_kv) * N * d;
  const T* vh = v + static_cast<size_t>(bh_kv) * N * d;
  const int ncol = (d + 31) / 32;  // <= 4
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  float m = -INFINITY, l = 0.f;
  const int n_tiles = (N + bc - 1) / bc;
  const bool l_rounded = ROUND_P && (flags & kTileLRounded) != 0;
  for (int tt = 0; tt < n_tiles; ++tt) {
    const int t0 = ((flags & kTileReverse) ? n_tiles - 1 - tt : tt) * bc;
    float sc[8];
    float tmax = -INFINITY;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      sc[u] = -INFINITY;
      const int j = t0 + 32 * u + lane;
      if (32 * u < bc && j < N && key_allowed(i, j, kvlen, causal, block_mask, nb)) {
        const T* kj = kh + static_cast<size_t>(j) * d;
        float dot = 0.f;
        for (int c = 0; c < d; ++c) dot = fmaf(to_f(qi[c]), to_f(kj[c]), dot);
        sc[u] = dot * scale;
        tmax = fmaxf(tmax, sc[u]);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
    if (tmax == -INFINITY) continue;  // every key of this tile is masked for this row
    const float m_new = fmaxf(m, tmax);
    const float alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
    float psum = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float pe = (sc[u] == -INFINITY) ? 0.f : expf(sc[u] - m_new);
      const float pr = ROUND_P ? __bfloat162float(__float2bfloat16_rn(pe)) : pe;
      psum += l_rounded ? pr : pe;
      sc[u] = pr;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
    l = alpha * l + psum;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) acc[cc] *= alpha;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (32 * u >= bc) break;
      for (int src = 0; src < 32; ++src) {
        const float pe = __shfl_sync(0xffffffffu, sc[u], src);
        const int j = t0 + 32 * u + src;
        if (pe == 0.f || j >= N) continue;
        const T* vj = vh + static_cast<size_t>(j) * d;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int c = 32 * cc + lane;
          if (cc < ncol && c < d) acc[cc] = fmaf(pe, to_f(vj[c]), acc[cc]);
        }
      }
    }
    m = m_new;
  }
  const float inv = (l > 0.f) ? 1.0f / l : 0.f;
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    const int c = 32 * cc + lane;
    if (cc < ncol && c < d) {
      if (o32 != nullptr) o32[row_g * d + c] = acc[cc] * inv;  // fp32 O/l before any rounding
      else o[row_g * d + c] = from_f<T>(acc[cc] * inv);
    }
  }
  if (lane == 0) lse[row_g] = (l > 0.f) ? m + logf(l) : -INFINITY;
}

// ---------------------------------------------------------------------------- naive baseline
// S[bh][i][j] = bf16(scale * q_i . k_j) (fp32 accumulation), -inf where masked.
__global__ void __launch_bounds__(256)
naive_scores_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                    __nv_bfloat16* __restrict__ s, const uint8_t* block_mask,
                    const int32_t* kv_len, int H, int N, int d, float scale, int causal) {
  __shared__ float qs[16][129];
  __shared__ float ks[16][129];
  const int bh = blockIdx.z, b = bh / H;
  const int i0 = blockIdx.y * 16, j0 = blockIdx.x * 16;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const __nv_bfloat16* qh = q + static_cast<size_t>(bh) * N * d;
  const __nv_bfloat16* kh = k + static_cast<size_t>(bh) * N * d;
  for (int e = threadIdx.x; e < 16 * d; e += 256) {
    const int r = e / d, c = e % d;
    qs[r][c] = (i0 + r < N) ? __bfloat162float(qh[static_cast<size_t>(i0 + r) * d + c]) : 0.f;
    ks[r][c] = (j0 + r < N) ? __bfloat162float(kh[static_cast<size_t>(j0 + r) * d + c]) : 0.f;
  }
  __syncthreads();
  const int i = i0 + ty, j = j0 + tx;
  if (i >= N || j >= N) return;
  int kvlen = N;
  if (kv_len != nullptr) kvlen = min(max(kv_len[b], 0), N);
  float dot = 0.f;
  for (int c = 0; c < d; ++c) dot = fmaf(qs[ty][c], ks[tx][c], dot);
  const float val = key_allowed(i, j, kvlen, causal, block_mask, (N + 127) / 128) ? dot * scale
                                                                                  : -INFINITY;
  s[(static_cast<size_t>(bh) * N + i) * N + j] = __float2bfloat16_rn(val);
}

// Row softmax in place: bf16 S -> bf16 P (fp32 arithmetic); lse in fp32.
__global__ void __launch_bounds__(256)
naive_softmax_kernel(__nv_bfloat16* __restrict__ s, float* __restrict__ lse, long long rows,
                     int N) {
  const long long r = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  __nv_bfloat16* row = s + r * N;
  float mx = -INFINITY;
  for (int j = lane; j < N; j += 32) mx = fmaxf(mx, __bfloat162float(row[j]));
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  float sum = 0.f;
  if (mx != -INFINITY)
    for (int j = lane; j < N; j += 32) sum += expf(__bfloat162float(row[j]) - mx);
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  const float inv = sum > 0.f ? 1.0f / sum : 0.f;
  for (int j = lane; j < N; j += 32) {
    const float e = (mx == -INFINITY) ? 0.f : expf(__bfloat162float(row[j]) - mx);
    row[j] = __float2bfloat16_rn(e * inv);
  }
  if (lane == 0) lse[r] = sum > 0.f ? mx + logf(sum) : -INFINITY;
}

// O[bh][i][c] = bf16(sum_j P_ij V_jc), fp32 accumulation.
__global__ void __launch_bounds__(256)
naive_pv_kernel(const __nv_bfloat16* __restrict__ pm, const __nv_bfloat16* __restrict__ v,
                __nv_bfloat16* __restrict__ o, int N, int d) {
  __shared__ float ps[16][17];
  __shared__ float vs[16][129];
  const int bh = blockIdx.z;
  const int i0 = blockIdx.y * 16;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const __nv_bfloat16* ph = pm + static_cast<size_t>(bh) * N * N;
  const __nv_bfloat16* vh = v + static_cast<size_t>(bh) * N * d;
  const int ncc = (d + 15) / 16;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int j0 = 0; j0 < N; j0 += 16) {
    {
      const int i = i0 + ty, j = j0 + tx;
      ps[ty][tx] = (i < N && j < N) ? __bfloat162float(ph[static_cast<size_t>(i) * N + j]) : 0.f;
    }
    for (int e = threadIdx.x; e < 16 * d; e += 256) {
      const int r = e / d, c = e % d;
      vs[r][c] = (j0 + r < N) ? __bfloat162float(vh[static_cast<size_t>(j0 + r) * d + c]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
      const int c = 16 * cc + tx;
      if (cc < ncc && c < d)
        for (int jj = 0; jj < 16; ++jj) acc[cc] = fmaf(ps[ty][jj], vs[jj][c], acc[cc]);
    }
    __syncthreads();
  }
  const int i = i0 + ty;
  if (i >= N) return;
#pragma unroll
  for (int cc = 0; cc < 8; ++cc) {
    const int c = 16 * cc + tx;
    if (cc < ncc && c < d) o[(static_cast<size_t>(bh) * N + i) * d + c] = __float2bfloat16_rn(acc[cc]);
  }
}

// ---------------------------------------------------------------------------- backward helpers
// Dvec_i = sum_c dO_ic O_ic (fp32); lse2_i = lse_i * log2(e) (+inf for rows with no key and for
// the padding rows N..N_pad-1); zeroes the fp32 dQ accumulator unless dq_acc is null (the
// deterministic backward has none).  HBM-bound: each thread takes 8 consecutive elements of a
// row (16-byte loads of O and dO, 32-byte stores of zeros), D/8 threads per row, the row's dot
// product reduced over those lanes.  D is 64 or 128.
template <int D>
__global__ void __launch_bounds__(256)
bwd_preprocess_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dO,
                      const float* __restrict__ lse, float* __restrict__ lse2,
                      float* __restrict__ dvec, float* __restrict__ dq_acc, int BH, int N,
                      int N_pad) {
  constexpr int T = D / 8;  // threads per row
  grid_dep_launch();          // the main backward kernel may start its set-up now
  const long long r = (static_cast<long long>(blockIdx.x) * 256 + threadIdx.x) / T;
  const int part = threadIdx.x % T;
  if (r >= static_cast<long long>(BH) * N_pad) return;  // whole row groups leave together
  const int bh = static_cast<int>(r / N_pad), i = static_cast<int>(r % N_pad);
  if (i >= N) {
    if (part == 0) {
      lse2[r] = INFINITY;
      dvec[r] = 0.f;
    }
    return;
  }
  const size_t off = (static_cast<size_t>(bh) * N + i) * D + part * 8;
  const uint4 a = *reinterpret_cast<const uint4*>(o + off);
  const uint4 g = *reinterpret_cast<const uint4*>(dO + off);
  const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, gw[4] = {g.x, g.y, g.z, g.w};
  float acc = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    acc = fmaf(__uint_as_float(gw[e] << 16), __uint_as_float(aw[e] << 16), acc);
    acc = fmaf(__uint_as_float(gw[e] & 0xffff0000u), __uint_as_float(aw[e] & 0xffff0000u), acc);
  }
  // the T lanes of this row (aligned within the warp; other rows' lanes may have returned)
  const unsigned lane = threadIdx.x & 31u;
  const unsigned group = ((T == 32) ? 0xffffffffu : ((1u << T) - 1u)) << (lane & ~(T - 1u));
#pragma unroll
  for (int offs = T / 2; offs > 0; offs >>= 1) acc += __shfl_xor_sync(group, acc, offs);
  if (dq_acc != nullptr) {
    float4* z = reinterpret_cast<float4*>(dq_acc + off);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (part == 0) {
    const float ls = lse[static_cast<size_t>(bh) * N + i];
    lse2[r] = (ls == -INFINITY) ? INFINITY : ls * 1.4426950408889634f;
    dvec[r] = acc;
  }
}

// dQ = bf16(scale * dQacc), 8 elements per thread.
__global__ void __launch_bounds__(256)
dq_convert_kernel(const float* __restrict__ dq_acc, __nv_bfloat16* __restrict__ dq, long long n,
                  float scale) {
  grid_dep_wait();  // may be launched to overlap the kernel that completes the accumulator
  const long long e = (static_cast<long long>(blockIdx.x) * 256 + threadIdx.x) * 8;
  if (e + 8 <= n) {
    const float4 a = *reinterpret_cast<const float4*>(dq_acc + e);
    const float4 c = *reinterpret_cast<const float4*>(dq_acc + e + 4);
    __nv_bfloat162 h0 = __floats2bfloat162_rn(a.x * scale, a.y * scale);
    __nv_bfloat162 h1 = __floats2bfloat162_rn(a.z * scale, a.w * scale);
    __nv_bfloat162 h2 = __floats2bfloat162_rn(c.x * scale, c.y * scale);
    __nv_bfloat162 h3 = __floats2bfloat162_rn(c.z * scale, c.w * scale);
    uint4 u;
    u.x = *reinterpret_cast<uint32_t*>(&h0);
    u.y = *reinterpret_cast<uint32_t*>(&h1);
    u.z = *reinterpret_cast<uint32_t*>(&h2);
    u.w = *reinterpret_cast<uint32_t*>(&h3);
    *reinterpret_cast<uint4*>(dq + e) = u;
  } else {
    for (long long x = e; x < n; ++x) dq[x] = __float2bfloat16_rn(dq_acc[x] * scale);
  }
}

// ---------------------------------------------------------------------------- fp32 backward
// The backward of the fp32 path on CUDA cores, with the recompute form of the tensor-core
// backward: P_ij = exp(s_ij - lse_i), dS_ij = P_ij (dO_i . v_j - Dvec_i), Dvec_i = dO_i . O_i.
// Two kernels, each owning its output rows, so every sum runs in a fixed order (no atomics):
// the gradients are deterministic.  Query head h reads K/V head h / (H / H_kv).

// Dvec_i = sum_c dO_ic O_ic in fp32.  One warp per query row.
__global__ void __launch_bounds__(256)
bwd_dvec_f32_kernel(const float* __restrict__ o, const float* __restrict__ dO,
                    float* __restrict__ dvec, long long rows, int d) {
  const long long r = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  float acc = 0.f;
  for (int c = lane; c < d; c += 32) acc = fmaf(dO[r * d + c], o[r * d + c], acc);
  for (int offs = 16; offs > 0; offs >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, offs);
  if (lane == 0) dvec[r] = acc;
}

__device__ __forceinline__ float dot_f32(const float* __restrict__ a, const float* __restrict__ b,
                                         int d) {
  float s = 0.f;
  for (int c = 0; c < d; ++c) s = fmaf(a[c], b[c], s);
  return s;
}

// dQ_i = scale sum_j dS_ij k_j.  One warp per query row; lane l takes keys t0 + 32u + l of each
// 256-key tile, then the warp accumulates output column 32cc + lane over the tile's keys.
__global__ void __launch_bounds__(256)
fa_bwd_f32_dq_kernel(const float* __restrict__ q, const float* __restrict__ k,
                     const float* __restrict__ v, const float* __restrict__ dO,
                     const float* __restrict__ lse, const float* __restrict__ dvec,
                     float* __restrict__ dq, const uint8_t* block_mask, const int32_t* kv_len,
                     int B, int H, int H_kv, int N, int d, float scale, int causal) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row_g = static_cast<long long>(blockIdx.x) * 8 + warp;  // flat bh*N + i
  if (row_g >= static_cast<long long>(B) * H * N) return;
  const int i = static_cast<int>(row_g % N);
  const int bh = static_cast<int>(row_g / N);
  const int b = bh / H;
  const int bh_kv = b * H_kv + (bh % H) / (H / H_kv);
  int kvlen = N;
  if (kv_len != nullptr) kvlen = min(max(kv_len[b], 0), N);
  const int nb = (N + 127) / 128;
  const float* qi = q + row_g * d;
  const float* doi = dO + row_g * d;
  const float* kh = k + static_cast<size_t>(bh_kv) * N * d;
  const float* vh = v + static_cast<size_t>(bh_kv) * N * d;
  const float lse_i = lse[row_g];
  const float dv_i = dvec[row_g];
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  if (lse_i != -INFINITY) {  // a row with no key has P = 0 everywhere
    for (int t0 = 0; t0 < N; t0 += 256) {
      float ds[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        ds[u] = 0.f;
        const int j = t0 + 32 * u + lane;
        if (j < N && key_allowed(i, j, kvlen, causal, block_mask, nb)) {
          const float p = expf(dot_f32(qi, kh + static_cast<size_t>(j) * d, d) * scale - lse_i);
          ds[u] = p * (dot_f32(doi, vh + static_cast<size_t>(j) * d, d) - dv_i);
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        for (int src = 0; src < 32; ++src) {
          const float w = __shfl_sync(0xffffffffu, ds[u], src);
          const int j = t0 + 32 * u + src;
          if (w == 0.f || j >= N) continue;
          const float* kj = kh + static_cast<size_t>(j) * d;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const int c = 32 * cc + lane;
            if (c < d) acc[cc] = fmaf(w, kj[c], acc[cc]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    const int c = 32 * cc + lane;
    if (c < d) dq[row_g * d + c] = acc[cc] * scale;
  }
}

// dV_j = sum_i P_ij dO_i and dK_j = scale sum_i dS_ij q_i over every query head of the K/V
// head's group.  One warp per key row; lane l takes queries t0 + 32u + l of each 256-row tile.
__global__ void __launch_bounds__(256)
fa_bwd_f32_dkdv_kernel(const float* __restrict__ q, const float* __restrict__ k,
                       const float* __restrict__ v, const float* __restrict__ dO,
                       const float* __restrict__ lse, const float* __restrict__ dvec,
                       float* __restrict__ dk, float* __restrict__ dv, const uint8_t* block_mask,
                       const int32_t* kv_len, int B, int H, int H_kv, int N, int d, float scale,
                       int causal) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row_g = static_cast<long long>(blockIdx.x) * 8 + warp;  // flat bh_kv*N + j
  if (row_g >= static_cast<long long>(B) * H_kv * N) return;
  const int j = static_cast<int>(row_g % N);
  const int bh_kv = static_cast<int>(row_g / N);
  const int b = bh_kv / H_kv;
  const int G = H / H_kv;
  int kvlen = N;
  if (kv_len != nullptr) kvlen = min(max(kv_len[b], 0), N);
  const int nb = (N + 127) / 128;
  const float* kj = k + row_g * d;
  const float* vj = v + row_g * d;
  float acc_k[4] = {0.f, 0.f, 0.f, 0.f}, acc_v[4] = {0.f, 0.f, 0.f, 0.f};
  for (int g = 0; g < G && j < kvlen; ++g) {
    const int bh = b * H + (bh_kv % H_kv) * G + g;  // query head of the group
    const float* qh = q + static_cast<size_t>(bh) * N * d;
    const float* doh = dO + static_cast<size_t>(bh) * N * d;
    for (int t0 = 0; t0 < N; t0 += 256) {
      float pv[8], ds[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        pv[u] = 0.f;
        ds[u] = 0.f;
        const int i = t0 + 32 * u + lane;
        if (i < N && key_allowed(i, j, kvlen, causal, block_mask, nb)) {
          const size_t r = static_cast<size_t>(bh) * N + i;
          const float p = expf(dot_f32(qh + static_cast<size_t>(i) * d, kj, d) * scale - lse[r]);
          pv[u] = p;
          ds[u] = p * (dot_f32(doh + static_cast<size_t>(i) * d, vj, d) - dvec[r]);
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        for (int src = 0; src < 32; ++src) {
          const float wp = __shfl_sync(0xffffffffu, pv[u], src);
          const float ws = __shfl_sync(0xffffffffu, ds[u], src);
          const int i = t0 + 32 * u + src;
          if ((wp == 0.f && ws == 0.f) || i >= N) continue;
          const float* qi = qh + static_cast<size_t>(i) * d;
          const float* doi = doh + static_cast<size_t>(i) * d;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const int c = 32 * cc + lane;
            if (c < d) {
              acc_v[cc] = fmaf(wp, doi[c], acc_v[cc]);
              acc_k[cc] = fmaf(ws, qi[c], acc_k[cc]);
            }
          }
        }
      }
    }
  }
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    const int c = 32 * cc + lane;
    if (c < d) {
      dk[row_g * d + c] = acc_k[cc] * scale;
      dv[row_g * d + c] = acc_v[cc];
    }
  }
}

// Diagnostic: the two exp2 paths of the forward softmax side by side, for their tests.
__global__ void __launch_bounds__(256)
diag_exp2_kernel(const float* __restrict__ x, float* __restrict__ y_fma, float* __restrict__ y_mufu,
                 float* __restrict__ y_ref, int n) {
  const int i = (blockIdx.x * 256 + threadIdx.x) * 2;
  if (i + 1 < n) {
    float a, b;
    exp2_fma2(a, b, x[i], x[i + 1]);
    y_fma[i] = a;
    y_fma[i + 1] = b;
  } else if (i < n) {
    float a, b;
    exp2_fma2(a, b, x[i], 0.0f);
    y_fma[i] = a;
  }
  for (int k = i; k < min(i + 2, n); ++k) {
    y_mufu[k] = ex2_approx(x[k]);
    y_ref[k] = exp2f(x[k]);
  }
}

// Diagnostic: one CTA waits on an mbarrier that nothing ever arrives on, through the same
// bounded wait the attention kernels use.  The wait gives up after its time limit and records
// `site` in the status word, which fa_device_status() then reports.  Nothing faults or hangs.
__global__ void diag_wait_timeout_kernel(int site) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, site);
}

}  // namespace fa
