// fa_api.cu -- the C ABI of libfa (declared in include/fa.h): argument validation, TMA
// tensor-map encoding and kernel launches.  No allocation, no host synchronisation.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "fa.h"
#include "fa_bwd_dkdv_pair_sm100.cuh"
#include "fa_bwd_dkdv_sm100.cuh"
#include "fa_bwd_dq_sm100.cuh"
#include "fa_bwd_sm100.cuh"
#include "fa_fwd_sm100.cuh"
#include "fa_simt.cuh"
#include "ptx.cuh"

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

std::atomic<unsigned long long> g_launches{0};

int check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return FA_OK;
}

// overlap: launch with programmatic stream serialisation.  The kernel's CTAs may then start
// while the kernel before it on the stream finishes (once each of that kernel's CTAs has started
// and executed griddepcontrol.launch_dependents, or exited); the kernel executes
// griddepcontrol.wait before it reads or writes anything that kernel touches.  Otherwise a plain
// launch.
template <typename... Exp, typename... Act>
cudaError_t launch_ex(bool overlap, void (*kern)(Exp...), unsigned grid, unsigned block,
                      size_t smem, cudaStream_t s, Act&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = overlap ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Act>(args)...);
}

// ---- optional per-kernel timing (fa_kernel_timing): two events around each tensor-core launch
struct TimingRecord {
  const char* kernel;
  cudaEvent_t start, stop;
};
std::mutex g_timing_mu;
std::atomic<bool> g_timing_on{false};
std::vector<TimingRecord> g_timing;      // recorded, not yet read
std::vector<cudaEvent_t> g_event_pool;   // created once, reused

cudaEvent_t pooled_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// Brackets one launch with events on its stream while timing is enabled; otherwise inert.
class TimedLaunch {
 public:
  TimedLaunch(const char* kernel, cudaStream_t s) : kernel_(kernel), s_(s) {
    if (!g_timing_on.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lock(g_timing_mu);
    start_ = pooled_event();
    stop_ = pooled_event();
    if (start_ != nullptr && stop_ != nullptr) cudaEventRecord(start_, s_);
  }
  ~TimedLaunch() {
    if (start_ == nullptr || stop_ == nullptr) return;
    cudaEventRecord(stop_, s_);
    std::lock_guard<std::mutex> lock(g_timing_mu);
    g_timing.push_back({kernel_, start_, stop_});
  }

 private:
  const char* kernel_;
  cudaStream_t s_;
  cudaEvent_t start_ = nullptr, stop_ = nullptr;
};

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qres) ==
            cudaSuccess &&
        qres == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 3-D view [B*H][N][d] bf16 of a contiguous tensor, 128-byte swizzled boxes of 64 x rows.
int make_map(CUtensorMap* map, const void* base, int BH, int N, int d, int box_rows,
             const char* name) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                                 static_cast<cuuint64_t>(N) * d * 2};
  const cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(box_rows), 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "tensor map for %s failed (%d)", name, (int)r);
  return FA_OK;
}

// 3-D view [B*H][N][d] of the fp32 dQ accumulator for TMA reduce-adds: boxes of 32 columns x
// `box_rows` rows, unswizzled (d = 128) or 128-byte swizzled (d = 64).
int make_dq_map(CUtensorMap* map, float* base, int BH, int N, int d, int box_rows, bool swz) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 4,
                                 static_cast<cuuint64_t>(N) * d * 4};
  const cuuint32_t box[3] = {32u, static_cast<cuuint32_t>(box_rows), 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE,
                         swz ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "tensor map for the dQ accumulator failed (%d)", (int)r);
  return FA_OK;
}

template <typename Kernel>
int set_smem(Kernel kernel, int bytes) {
  const cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "smem attribute: %s", cudaGetErrorString(e));
  return FA_OK;
}

int common_checks(const void* q, const void* k, const void* v, const void* o, const float* lse,
                  int B, int H, int N, int d, float scale) {
  if (!q || !k || !v || !o || !lse) return fail(FA_ERR_INVALID, "null tensor pointer");
  if (B < 1 || H < 1 || N < 1 || d < 1) return fail(FA_ERR_INVALID, "B, H, N, d must be >= 1");
  if (!(std::isfinite(scale) && scale > 0.f)) return fail(FA_ERR_INVALID, "scale must be finite and > 0");
  if (static_cast<long long>(B) * H > (1ll << 24)) return fail(FA_ERR_UNSUPPORTED, "B*H too large");
  if (N > (1 << 24)) return fail(FA_ERR_UNSUPPORTED, "N too large");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return fail(FA_ERR_ALIGN, "tensor pointers must be 16-byte aligned");
  return FA_OK;
}

constexpr float kLog2e = 1.4426950408889634f;

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct BwdWs {
  size_t lse2, dvec, dq, total;
  int n_pad;
};
BwdWs bwd_ws(int B, int H, int N, int d) {
  BwdWs w;
  w.n_pad = (N + 127) / 128 * 128;
  const size_t bh = static_cast<size_t>(B) * H;
  w.lse2 = 0;
  w.dvec = round256(bh * w.n_pad * 4);
  w.dq = w.dvec + round256(bh * w.n_pad * 4);
  w.total = w.dq + round256(bh * static_cast<size_t>(N) * d * 4);
  return w;
}

// BN: keys per KV tile; O32: o is fp32 O/l (deviation study) instead of bf16 O; RANKED: the
// CTAs order the Q tiles by their unmasked blocks (needs a block mask and N <= 16384).
template <int D, int BN = fa::fwd_bn<D>(), bool O32 = false, bool RANKED = false>
int launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
               int H_kv, int N, float scale, int causal, const uint8_t* bm,
               const int32_t* kv_len, cudaStream_t stream) {
  using L = fa::FwdLayout<D, BN>;
  CUtensorMap mq, mk, mv, mo;
  const int BH = B * H;
  int rc;
  if ((rc = make_map(&mq, q, BH, N, D, 128, "q")) != FA_OK) return rc;
  if ((rc = make_map(&mk, k, B * H_kv, N, D, L::BN, "k")) != FA_OK) return rc;
  if ((rc = make_map(&mv, v, B * H_kv, N, D, L::BN, "v")) != FA_OK) return rc;
  // bf16 O: one warp's [32 rows][64 d] boxes (the fp32 O/l of the deviation study is stored
  // per lane, so its map is never used: it is built over o with the bf16 layout only to fill
  // the parameter)
  if ((rc = make_map(&mo, o, BH, N, D, 32, "o")) != FA_OK) return rc;
  if ((rc = set_smem(fa::fa_fwd_sm100_kernel<D, BN, O32, RANKED>, L::SMEM_ALLOC)) != FA_OK) return rc;
  fa::FwdParams p;
  p.block_mask = bm;
  p.kv_len = kv_len;
  p.o = O32 ? nullptr : static_cast<__nv_bfloat16*>(o);
  p.o32 = O32 ? static_cast<float*>(o) : nullptr;
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.H_kv = H_kv;
  p.N = N;
  p.n_mtiles = (N + 255) / 256;
  // Query heads per CTA-order group: Q, K, V and O of the group (8 bytes per element of each
  // query head, K and V counted per query head) within half of the 126 MB L2.
  p.hgroup = static_cast<int>(
      std::max(1ll, std::min((64ll << 20) / (8ll * N * D), static_cast<long long>(BH))));
  p.scale2 = scale * kLog2e;
  p.causal = causal ? 1 : 0;
  const long long grid = static_cast<long long>(p.n_mtiles) * BH;
  if (grid > 0x7fffffffll) return fail(FA_ERR_UNSUPPORTED, "grid too large");
  TimedLaunch tl("fa_fwd_sm100_kernel", stream);
  fa::fa_fwd_sm100_kernel<D, BN, O32, RANKED><<<static_cast<unsigned>(grid), 320, L::SMEM_ALLOC, stream>>>(mq, mk, mv, mo, p);
  return check_launch("fa_fwd_sm100_kernel");
}

template <int D>
int launch_bwd(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv,
               int B, int H, int H_kv, int N, float scale, int causal, const uint8_t* bm,
               const int32_t* kv_len, const BwdWs& ws, uint8_t* wsb, cudaStream_t stream) {
  using L = fa::BwdLayout<D>;
  CUtensorMap mq, mk, mv, mdo, mdq, mdk, mdv;
  const int BH = B * H;
  int rc;
  if ((rc = make_map(&mq, q, BH, N, D, L::BM, "q")) != FA_OK) return rc;
  if ((rc = make_map(&mk, k, B * H_kv, N, D, 128, "k")) != FA_OK) return rc;
  if ((rc = make_map(&mv, v, B * H_kv, N, D, 128, "v")) != FA_OK) return rc;
  if ((rc = make_map(&mdo, dO, BH, N, D, L::BM, "dO")) != FA_OK) return rc;
  // dK, dV: one warp's [32 rows][64 d] boxes
  if ((rc = make_map(&mdk, dk, B * H_kv, N, D, 32, "dK")) != FA_OK) return rc;
  if ((rc = make_map(&mdv, dv, B * H_kv, N, D, 32, "dV")) != FA_OK) return rc;
  // d = 128: [64 rows][32 d] boxes staged in the V tile; d = 64: swizzled [32 rows][32 d] boxes
  if ((rc = make_dq_map(&mdq, reinterpret_cast<float*>(wsb + ws.dq), BH, N, D,
                        L::V_IN_TMEM ? 64 : 32, !L::V_IN_TMEM)) != FA_OK)
    return rc;
  if ((rc = set_smem(fa::fa_bwd_sm100_kernel<D>, L::SMEM_ALLOC)) != FA_OK) return rc;
  fa::BwdParams p;
  p.block_mask = bm;
  p.kv_len = kv_len;
  p.lse2 = reinterpret_cast<const float*>(wsb + ws.lse2);
  p.dvec = reinterpret_cast<const float*>(wsb + ws.dvec);
  p.dq_acc = reinterpret_cast<float*>(wsb + ws.dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.B = B;
  p.H = H;
  p.H_kv = H_kv;
  p.N = N;
  p.N_pad = ws.n_pad;
  p.n_ktiles = (N + 127) / 128;
  p.scale = scale;
  p.scale2 = scale * kLog2e;
  p.causal = causal ? 1 : 0;
  {
    // K/V heads per CTA-order group: the group's dQ accumulator (fp32), Q and dO, 8 bytes per
    // element of its G query heads, within half of the 126 MB L2.
    const long long per_head = 8ll * (H / H_kv) * N * D;
    const long long fit = (64ll << 20) / per_head;
    p.hgroup = static_cast<int>(std::max(1ll, std::min(fit, static_cast<long long>(B) * H_kv)));
  }
  const long long grid = static_cast<long long>(p.n_ktiles) * B * H_kv;  // one CTA per K/V tile
  if (grid > 0x7fffffffll) return fail(FA_ERR_UNSUPPORTED, "grid too large");
  TimedLaunch tl("fa_bwd_sm100_kernel", stream);
  const cudaError_t le =
      launch_ex(L::OVERLAP_PREV, fa::fa_bwd_sm100_kernel<D>, static_cast<unsigned>(grid),
                L::THREADS, L::SMEM_ALLOC, stream, mq, mk, mv, mdo, mdq, mdk, mdv, p);
  if (le != cudaSuccess) return fail(FA_ERR_CUDA, "fa_bwd_sm100_kernel: %s", cudaGetErrorString(le));
  return check_launch("fa_bwd_sm100_kernel");
}

// dK and dV only, scores double-buffered (fa_bwd_dkdv_sm100.cuh).
template <int D>
int launch_bwd_dkdv(const void* q, const void* k, const void* v, const void* dO, void* dk,
                    void* dv, int B, int H, int H_kv, int N, float scale, int causal,
                    const uint8_t* bm, const int32_t* kv_len, const BwdWs& ws, uint8_t* wsb,
                    cudaStream_t stream) {
  using L = fa::BwdDkdvLayout<D>;
  CUtensorMap mq, mk, mv, mdo, mdk, mdv;
  const int BH = B * H;
  int rc;
  if ((rc = make_map(&mq, q, BH, N, D, L::BM, "q")) != FA_OK) return rc;
  if ((rc = make_map(&mk, k, B * H_kv, N, D, 128, "k")) != FA_OK) return rc;
  if ((rc = make_map(&mv, v, B * H_kv, N, D, 128, "v")) != FA_OK) return rc;
  if ((rc = make_map(&mdo, dO, BH, N, D, L::BM, "dO")) != FA_OK) return rc;
  if ((rc = make_map(&mdk, dk, B * H_kv, N, D, 32, "dK")) != FA_OK) return rc;  // [32][64] boxes
  if ((rc = make_map(&mdv, dv, B * H_kv, N, D, 32, "dV")) != FA_OK) return rc;
  if ((rc = set_smem(fa::fa_bwd_dkdv_sm100_kernel<D>, L::SMEM_ALLOC)) != FA_OK) return rc;
  fa::BwdParams p;
  p.block_mask = bm;
  p.kv_len = kv_len;
  p.lse2 = reinterpret_cast<const float*>(wsb + ws.lse2);
  p.dvec = reinterpret_cast<const float*>(wsb + ws.dvec);
  p.dq_acc = nullptr;
  {
    // K/V heads per CTA-order group: the group's Q and dO, 4 bytes per element of its G query
    // heads, within half of the 126 MB L2.
    const long long per_head = 4ll * (H / H_kv) * N * D;
    p.hgroup = static_cast<int>(
        std::max(1ll, std::min((64ll << 20) / per_head, static_cast<long long>(B) * H_kv)));
  }
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.B = B;
  p.H = H;
  p.H_kv = H_kv;
  p.N = N;
  p.N_pad = ws.n_pad;
  p.n_ktiles = (N + 127) / 128;
  p.scale = scale;
  p.scale2 = scale * kLog2e;
  p.causal = causal ? 1 : 0;
  const long long grid = static_cast<long long>(p.n_ktiles) * B * H_kv;
  if (grid > 0x7fffffffll) return fail(FA_ERR_UNSUPPORTED, "grid too large");
  TimedLaunch tl("fa_bwd_dkdv_sm100_kernel", stream);
  fa::fa_bwd_dkdv_sm100_kernel<D><<<static_cast<unsigned>(grid), L::THREADS, L::SMEM_ALLOC, stream>>>(mq, mk, mv, mdo, mdk, mdv, p);
  return check_launch("fa_bwd_dkdv_sm100_kernel");
}

// dK and dV at d = 128 on CTA pairs with 2-CTA MMAs (fa_bwd_dkdv_pair_sm100.cuh); the same sums
// in the same order as launch_bwd_dkdv<128>.
int launch_bwd_dkdv_pair(const void* q, const void* k, const void* v, const void* dO, void* dk,
                         void* dv, int B, int H, int H_kv, int N, float scale, int causal,
                         const uint8_t* bm, const int32_t* kv_len, const BwdWs& ws, uint8_t* wsb,
                         cudaStream_t stream) {
  using L = fa::BwdPairLayout;
  constexpr int D = L::D;
  CUtensorMap mq, mk, mv, mdo;
  const int BH = B * H;
  int rc;
  if ((rc = make_map(&mq, q, BH, N, D, 64, "q")) != FA_OK) return rc;
  if ((rc = make_map(&mk, k, B * H_kv, N, D, 128, "k")) != FA_OK) return rc;
  if ((rc = make_map(&mv, v, B * H_kv, N, D, 128, "v")) != FA_OK) return rc;
  if ((rc = make_map(&mdo, dO, BH, N, D, 64, "dO")) != FA_OK) return rc;
  if ((rc = set_smem(fa::fa_bwd_dkdv_pair_sm100_kernel, L::SMEM_ALLOC)) != FA_OK) return rc;
  fa::BwdParams p;
  p.block_mask = bm;
  p.kv_len = kv_len;
  p.lse2 = reinterpret_cast<const float*>(wsb + ws.lse2);
  p.dvec = reinterpret_cast<const float*>(wsb + ws.dvec);
  p.dq_acc = nullptr;
  {
    // K/V heads per CTA-order group: the group's Q and dO, 4 bytes per element of its G query
    // heads, within half of the 126 MB L2.
    const long long per_head = 4ll * (H / H_kv) * N * D;
    p.hgroup = static_cast<int>(
        std::max(1ll, std::min((64ll << 20) / per_head, static_cast<long long>(B) * H_kv)));
  }
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.B = B;
  p.H = H;
  p.H_kv = H_kv;
  p.N = N;
  p.N_pad = ws.n_pad;
  p.n_ktiles = (N + 127) / 128;
  p.scale = scale;
  p.scale2 = scale * kLog2e;
  p.causal = causal ? 1 : 0;
  // two CTAs (one cluster) per pair of KV tiles
  const long long grid = 2ll * ((p.n_ktiles + 1) / 2) * B * H_kv;
  if (grid > 0x7fffffffll) return fail(FA_ERR_UNSUPPORTED, "grid too large");
  TimedLaunch tl("fa_bwd_dkdv_pair_sm100_kernel", stream);
  fa::fa_bwd_dkdv_pair_sm100_kernel<<<static_cast<unsigned>(grid), 320, L::SMEM_ALLOC, stream>>>(
      mq, mk, mv, mdo, p);
  return check_launch("fa_bwd_dkdv_pair_sm100_kernel");
}

// dQ without atomics: one CTA per 128 query rows walks the KV tiles (fa_bwd_dq_sm100.cuh).
template <int D>
int launch_bwd_dq(const void* q, const void* k, const void* v, const void* dO, void* dq, int B,
                  int H, int H_kv, int N, float scale, int causal, const uint8_t* bm,
                  const int32_t* kv_len, const BwdWs& ws, uint8_t* wsb, cudaStream_t stream) {
  using L = fa::BwdDqLayout<D>;
  CUtensorMap mq, mk, mv, mdo;
  const int BH = B * H;
  int rc;
  if ((rc = make_map(&mq, q, BH, N, D, 128, "q")) != FA_OK) return rc;
  if ((rc = make_map(&mk, k, B * H_kv, N, D, 128, "k")) != FA_OK) return rc;
  if ((rc = make_map(&mv, v, B * H_kv, N, D, 128, "v")) != FA_OK) return rc;
  if ((rc = make_map(&mdo, dO, BH, N, D, 128, "dO")) != FA_OK) return rc;
  if ((rc = set_smem(fa::fa_bwd_dq_sm100_kernel<D>, L::SMEM_ALLOC)) != FA_OK) return rc;
  fa::BwdDqParams p;
  p.block_mask = bm;
  p.kv_len = kv_len;
  p.lse2 = reinterpret_cast<const float*>(wsb + ws.lse2);
  p.dvec = reinterpret_cast<const float*>(wsb + ws.dvec);
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.B = B;
  p.H = H;
  p.H_kv = H_kv;
  p.N = N;
  p.N_pad = ws.n_pad;
  p.n_mtiles = (N + 127) / 128;
  // Query heads per CTA-order group: the K and V they read (4 bytes per element, counted per
  // query head) within a quarter of the 126 MB L2 (in interleaved timings of the deterministic
  // call at long_causal: 3.06 ms against 3.15 ms with half of L2, 3.18 ms with an eighth).
  p.hgroup = static_cast<int>(
      std::max(1ll, std::min((32ll << 20) / (4ll * N * D), static_cast<long long>(BH))));
  p.scale = scale;
  p.scale2 = scale * kLog2e;
  p.causal = causal ? 1 : 0;
  const long long grid = static_cast<long long>(p.n_mtiles) * BH;
  if (grid > 0x7fffffffll) return fail(FA_ERR_UNSUPPORTED, "grid too large");
  TimedLaunch tl("fa_bwd_dq_sm100_kernel", stream);
  fa::fa_bwd_dq_sm100_kernel<D><<<static_cast<unsigned>(grid), 320, L::SMEM_ALLOC, stream>>>(mq, mk, mv, mdo, p);
  return check_launch("fa_bwd_dq_sm100_kernel");
}

}  // namespace

extern "C" {

const char* fa_get_last_error(void) { return g_err; }

int fa_device_status(unsigned int* code) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "device synchronise: %s", cudaGetErrorString(e));
  unsigned int v = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&v, fa::g_status, sizeof(v));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(fa::g_status, &zero, sizeof(zero));
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "status word: %s", cudaGetErrorString(e));
  if (code) *code = v;
  if (v != 0) return fail(FA_ERR_TIMEOUT, "device wait gave up: site %u block %u", v >> 16, v & 0xffffu);
  return FA_OK;
}

}  // extern "C"

namespace {

int check_groups(int H, int H_kv) {
  if (H_kv < 1 || H_kv > H || H % H_kv != 0)
    return fail(FA_ERR_INVALID, "H = %d must be a positive multiple of H_kv = %d", H, H_kv);
  return FA_OK;
}

int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
             int H_kv, int N, int d, float scale, int causal, const uint8_t* block_mask,
             const int32_t* kv_len, int dtype, void* stream) {
  int rc = common_checks(q, k, v, o, lse, B, H, N, d, scale);
  if (rc != FA_OK) return rc;
  if ((rc = check_groups(H, H_kv)) != FA_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == FA_BF16) {
    if (d == 64) {
      // block masks: the Q tiles are taken heaviest first (a block-sparse mask need not make
      // the last rows the longest, as a causal one does)
      if (block_mask != nullptr && (N + 255) / 256 <= fa::FWD_RANK_TILES)
        return launch_fwd<64, 64, false, true>(q, k, v, o, lse, B, H, H_kv, N, scale, causal, block_mask, kv_len, s);
      return launch_fwd<64>(q, k, v, o, lse, B, H, H_kv, N, scale, causal, block_mask, kv_len, s);
    }
    if (d == 128)
      return launch_fwd<128>(q, k, v, o, lse, B, H, H_kv, N, scale, causal, block_mask, kv_len, s);
    return fail(FA_ERR_UNSUPPORTED, "bf16 forward supports d in {64, 128}, got %d", d);
  }
  if (dtype == FA_F32) {
    if (d > 128) return fail(FA_ERR_UNSUPPORTED, "fp32 forward supports d <= 128, got %d", d);
    const long long rows = static_cast<long long>(B) * H * N;
    fa::fa_fwd_rowwarp_kernel<float, false><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, s>>>(
        static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
        static_cast<float*>(o), lse, block_mask, kv_len, B, H, N, d, scale, causal ? 1 : 0, 128, 0,
        H_kv, nullptr);
    return check_launch("fa_fwd_rowwarp_kernel<f32>");
  }
  return fail(FA_ERR_INVALID, "unknown dtype %d", dtype);
}

// fa_bwd_deterministic_ex options: which dK/dV kernel runs at d = 128.
constexpr bool kPairDkdvDefault = false;  // measured slower (see the kernel header)
bool use_pair_dkdv(int options) {
  if (options & FA_BWD_DKDV_SINGLE) return false;
  if (options & FA_BWD_DKDV_PAIR) return true;
  return kPairDkdvDefault;
}

// Argument checks shared by every backward entry point (everything but the workspace).
int bwd_checks(const void* q, const void* k, const void* v, const void* o, const float* lse,
               const void* dO, const void* dq, const void* dk, const void* dv, int B, int H,
               int H_kv, int N, int d, float scale, int dtype) {
  int rc = common_checks(q, k, v, o, lse, B, H, N, d, scale);
  if (rc != FA_OK) return rc;
  if ((rc = check_groups(H, H_kv)) != FA_OK) return rc;
  if (!dO || !dq || !dk || !dv) return fail(FA_ERR_INVALID, "null gradient pointer");
  if (!aligned16(dO) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return fail(FA_ERR_ALIGN, "gradient pointers must be 16-byte aligned");
  if (dtype != FA_BF16 && dtype != FA_F32) return fail(FA_ERR_INVALID, "unknown dtype %d", dtype);
  if (dtype == FA_F32 && d > 128)
    return fail(FA_ERR_UNSUPPORTED, "fp32 backward supports d <= 128, got %d", d);
  if (dtype == FA_BF16 && d != 64 && d != 128)
    return fail(FA_ERR_UNSUPPORTED, "bf16 backward supports d in {64, 128}, got %d", d);
  return FA_OK;
}

int bwd_impl(const void* q, const void* k, const void* v, const void* o, const float* lse,
             const void* dO, void* dq, void* dk, void* dv, int B, int H, int H_kv, int N, int d,
             float scale, int causal, const uint8_t* block_mask, const int32_t* kv_len,
             int dtype, void* workspace, size_t workspace_bytes, void* stream,
             bool deterministic, int options = 0) {
  int rc = bwd_checks(q, k, v, o, lse, dO, dq, dk, dv, B, H, H_kv, N, d, scale, dtype);
  if (rc != FA_OK) return rc;
  const BwdWs ws = bwd_ws(B, H, N, d);
  if (workspace == nullptr || workspace_bytes < ws.total)
    return fail(FA_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", ws.total, workspace_bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(FA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  const int BH = B * H;
  if (dtype == FA_F32) {
    // CUDA-core fp32 backward: Dvec, then dQ per query row and dK/dV per key row (no atomics)
    const long long qrows = static_cast<long long>(BH) * N;
    const long long krows = static_cast<long long>(B) * H_kv * N;
    float* dvec = reinterpret_cast<float*>(wsb + ws.dvec);
    fa::bwd_dvec_f32_kernel<<<static_cast<unsigned>((qrows + 7) / 8), 256, 0, s>>>(
        static_cast<const float*>(o), static_cast<const float*>(dO), dvec, qrows, d);
    if ((rc = check_launch("bwd_dvec_f32_kernel")) != FA_OK) return rc;
    fa::fa_bwd_f32_dq_kernel<<<static_cast<unsigned>((qrows + 7) / 8), 256, 0, s>>>(
        static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
        static_cast<const float*>(dO), lse, dvec, static_cast<float*>(dq), block_mask, kv_len, B,
        H, H_kv, N, d, scale, causal ? 1 : 0);
    if ((rc = check_launch("fa_bwd_f32_dq_kernel")) != FA_OK) return rc;
    fa::fa_bwd_f32_dkdv_kernel<<<static_cast<unsigned>((krows + 7) / 8), 256, 0, s>>>(
        static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
        static_cast<const float*>(dO), lse, dvec, static_cast<float*>(dk), static_cast<float*>(dv),
        block_mask, kv_len, B, H, H_kv, N, d, scale, causal ? 1 : 0);
    return check_launch("fa_bwd_f32_dkdv_kernel");
  }
  {
    // d / 8 threads per row, 256 threads per block
    const long long pre_threads = static_cast<long long>(BH) * ws.n_pad * (d / 8);
    const unsigned blocks = static_cast<unsigned>((pre_threads + 255) / 256);
    auto* pre = d == 64 ? fa::bwd_preprocess_kernel<64> : fa::bwd_preprocess_kernel<128>;
    pre<<<blocks, 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), lse,
        reinterpret_cast<float*>(wsb + ws.lse2), reinterpret_cast<float*>(wsb + ws.dvec),
        deterministic ? nullptr : reinterpret_cast<float*>(wsb + ws.dq), BH, N, ws.n_pad);
    if ((rc = check_launch("bwd_preprocess_kernel")) != FA_OK) return rc;
  }
  if (deterministic) {
    // dK and dV by the dK/dV kernel, dQ by the query-stationary kernel: no atomics.  At d = 128
    // the dK/dV kernel runs on CTA pairs (2-CTA MMAs) unless the caller asks for one CTA.
    if (d == 64)
      rc = launch_bwd_dkdv<64>(q, k, v, dO, dk, dv, B, H, H_kv, N, scale, causal, block_mask, kv_len, ws, wsb, s);
    else if (use_pair_dkdv(options))
      rc = launch_bwd_dkdv_pair(q, k, v, dO, dk, dv, B, H, H_kv, N, scale, causal, block_mask, kv_len, ws, wsb, s);
    else
      rc = launch_bwd_dkdv<128>(q, k, v, dO, dk, dv, B, H, H_kv, N, scale, causal, block_mask, kv_len, ws, wsb, s);
    if (rc != FA_OK) return rc;
    if (d == 64)
      return launch_bwd_dq<64>(q, k, v, dO, dq, B, H, H_kv, N, scale, causal, block_mask, kv_len, ws, wsb, s);
    return launch_bwd_dq<128>(q, k, v, dO, dq, B, H, H_kv, N, scale, causal, block_mask, kv_len, ws, wsb, s);
  }
  if (d == 64)
    rc = launch_bwd<64>(q, k, v, dO, dk, dv, B, H, H_kv, N, scale, causal, block_mask, kv_len, ws, wsb, s);
  else
    rc = launch_bwd<128>(q, k, v, dO, dk, dv, B, H, H_kv, N, scale, causal, block_mask, kv_len, ws, wsb, s);
  if (rc != FA_OK) return rc;
  const long long n = static_cast<long long>(BH) * N * d;
  // overlapping the main kernel where that kernel overlaps the preprocess
  const cudaError_t le = launch_ex(
      d == 64 ? fa::BwdLayout<64>::OVERLAP_PREV : fa::BwdLayout<128>::OVERLAP_PREV,
      fa::dq_convert_kernel, static_cast<unsigned>((n / 8 + 255) / 256 + 1), 256, 0, s,
      reinterpret_cast<const float*>(wsb + ws.dq), static_cast<__nv_bfloat16*>(dq), n, scale);
  if (le != cudaSuccess) return fail(FA_ERR_CUDA, "dq_convert_kernel: %s", cudaGetErrorString(le));
  return check_launch("dq_convert_kernel");
}

}  // namespace

extern "C" {

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
           int N, int d, float scale, int causal, const uint8_t* block_mask,
           const int32_t* kv_len, int dtype, void* stream) {
  return fwd_impl(q, k, v, o, lse, B, H, H, N, d, scale, causal, block_mask, kv_len, dtype,
                  stream);
}

int fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
               int H_kv, int N, int d, float scale, int causal, const uint8_t* block_mask,
               const int32_t* kv_len, int dtype, void* stream) {
  return fwd_impl(q, k, v, o, lse, B, H, H_kv, N, d, scale, causal, block_mask, kv_len, dtype,
                  stream);
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || d < 1) return 0;
  return bwd_ws(B, H, N, d).total;
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dO, void* dq, void* dk, void* dv, int B, int H, int N, int d,
           float scale, int causal, const uint8_t* block_mask, const int32_t* kv_len,
           int dtype, void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_impl(q, k, v, o, lse, dO, dq, dk, dv, B, H, H, N, d, scale, causal, block_mask,
                  kv_len, dtype, workspace, workspace_bytes, stream, false);
}

int fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const float* lse,
               const void* dO, void* dq, void* dk, void* dv, int B, int H, int H_kv, int N,
               int d, float scale, int causal, const uint8_t* block_mask,
               const int32_t* kv_len, int dtype, void* workspace, size_t workspace_bytes,
               void* stream) {
  return bwd_impl(q, k, v, o, lse, dO, dq, dk, dv, B, H, H_kv, N, d, scale, causal, block_mask,
                  kv_len, dtype, workspace, workspace_bytes, stream, false);
}

int fa_bwd_deterministic(const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* dO, void* dq, void* dk, void* dv, int B,
                         int H, int H_kv, int N, int d, float scale, int causal,
                         const uint8_t* block_mask, const int32_t* kv_len, int dtype,
                         void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_impl(q, k, v, o, lse, dO, dq, dk, dv, B, H, H_kv, N, d, scale, causal, block_mask,
                  kv_len, dtype, workspace, workspace_bytes, stream, true);
}

int fa_bwd_deterministic_ex(const void* q, const void* k, const void* v, const void* o,
                            const float* lse, const void* dO, void* dq, void* dk, void* dv, int B,
                            int H, int H_kv, int N, int d, float scale, int causal,
                            const uint8_t* block_mask, const int32_t* kv_len, int dtype,
                            void* workspace, size_t workspace_bytes, int options, void* stream) {
  if ((options & ~(FA_BWD_DKDV_PAIR | FA_BWD_DKDV_SINGLE)) != 0 ||
      (options & (FA_BWD_DKDV_PAIR | FA_BWD_DKDV_SINGLE)) == (FA_BWD_DKDV_PAIR | FA_BWD_DKDV_SINGLE))
    return fail(FA_ERR_INVALID, "unknown or contradictory backward options 0x%x", options);
  return bwd_impl(q, k, v, o, lse, dO, dq, dk, dv, B, H, H_kv, N, d, scale, causal, block_mask,
                  kv_len, dtype, workspace, workspace_bytes, stream, true, options);
}

int fa_fwd_tile_reference(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int H, int N, int d, float scale, int causal,
                          const uint8_t* block_mask, const int32_t* kv_len, int bc, int flags,
                          void* stream) {
  int rc = common_checks(q, k, v, o, lse, B, H, N, d, scale);
  if (rc != FA_OK) return rc;
  if (d > 128) return fail(FA_ERR_UNSUPPORTED, "d <= 128 required, got %d", d);
  if ((flags & ~(FA_TILE_REVERSE | FA_TILE_L_ROUNDED | FA_TILE_TENSOR_CORE | FA_TILE_O_F32)) != 0)
    return fail(FA_ERR_INVALID, "unknown tile-reference flags 0x%x", flags);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool o32 = (flags & FA_TILE_O_F32) != 0;
  if (flags & FA_TILE_TENSOR_CORE) {
    // the tcgen05 forward itself, with bc-key tiles (its own lazy rescale and fp32-P normaliser)
    if (flags & (FA_TILE_REVERSE | FA_TILE_L_ROUNDED))
      return fail(FA_ERR_INVALID, "the tensor-core forward has no reverse or rounded-l variant");
    if (d != 64 || (bc != 64 && bc != 128))
      return fail(FA_ERR_UNSUPPORTED, "tensor-core tile sweep: d = 64 and bc in {64, 128}");
    if (bc == 64)
      return o32 ? launch_fwd<64, 64, true>(q, k, v, o, lse, B, H, H, N, scale, causal, block_mask, kv_len, s)
                 : launch_fwd<64, 64, false>(q, k, v, o, lse, B, H, H, N, scale, causal, block_mask, kv_len, s);
    return o32 ? launch_fwd<64, 128, true>(q, k, v, o, lse, B, H, H, N, scale, causal, block_mask, kv_len, s)
               : launch_fwd<64, 128, false>(q, k, v, o, lse, B, H, H, N, scale, causal, block_mask, kv_len, s);
  }
  if (bc < 32 || bc > 256 || (bc % 32) != 0) return fail(FA_ERR_INVALID, "bc must be 32..256 in steps of 32");
  const long long rows = static_cast<long long>(B) * H * N;
  fa::fa_fwd_rowwarp_kernel<__nv_bfloat16, true>
      <<<static_cast<unsigned>((rows + 7) / 8), 256, 0, s>>>(
          static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
          static_cast<const __nv_bfloat16*>(v), o32 ? nullptr : static_cast<__nv_bfloat16*>(o),
          lse, block_mask, kv_len, B, H, N, d, scale, causal ? 1 : 0, bc, flags, H,
          o32 ? static_cast<float*>(o) : nullptr);
  return check_launch("fa_fwd_rowwarp_kernel<bf16>");
}

int fa_diag_exp2(const float* x, float* y_fma, float* y_mufu, float* y_ref, int n, void* stream) {
  if (!x || !y_fma || !y_mufu || !y_ref) return fail(FA_ERR_INVALID, "null pointer");
  if (n < 1) return fail(FA_ERR_INVALID, "n must be >= 1");
  const int blocks = (n + 511) / 512;
  fa::diag_exp2_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y_fma, y_mufu, y_ref, n);
  return check_launch("diag_exp2_kernel");
}

unsigned long long fa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int fa_kernel_timing(int enable) {
  g_timing_on.store(enable != 0, std::memory_order_relaxed);
  return FA_OK;
}

int fa_kernel_timing_read(const char* name, int* launches, double* total_ms) {
  if (name == nullptr || launches == nullptr || total_ms == nullptr)
    return fail(FA_ERR_INVALID, "null pointer");
  std::vector<TimingRecord> mine;
  {
    std::lock_guard<std::mutex> lock(g_timing_mu);
    std::vector<TimingRecord> rest;
    for (const TimingRecord& r : g_timing)
      (std::strstr(r.kernel, name) != nullptr ? mine : rest).push_back(r);
    g_timing.swap(rest);
  }
  int n = 0;
  double ms = 0.0;
  int rc = FA_OK;
  for (const TimingRecord& r : mine) {
    float t = 0.f;
    cudaError_t e = cudaEventSynchronize(r.stop);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t, r.start, r.stop);
    if (e != cudaSuccess && rc == FA_OK)
      rc = fail(FA_ERR_CUDA, "kernel timing: %s", cudaGetErrorString(e));
    ++n;
    ms += t;
  }
  {
    std::lock_guard<std::mutex> lock(g_timing_mu);
    for (const TimingRecord& r : mine) {
      g_event_pool.push_back(r.start);
      g_event_pool.push_back(r.stop);
    }
  }
  *launches = n;
  *total_ms = ms;
  return rc;
}

int fa_diag_wait_timeout(int site, void* stream) {
  if (site < 1 || site > 0x7fff) return fail(FA_ERR_INVALID, "site must be in [1, 32767]");
  fa::diag_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(site);
  return check_launch("diag_wait_timeout_kernel");
}

size_t fa_naive_workspace_size(int B, int H, int N) {
  if (B < 1 || H < 1 || N < 1) return 0;
  return static_cast<size_t>(B) * H * N * N * 2;
}

int fa_naive_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int N, int d, float scale, int causal, const uint8_t* block_mask,
                 const int32_t* kv_len, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = common_checks(q, k, v, o, lse, B, H, N, d, scale);
  if (rc != FA_OK) return rc;
  if (d > 128) return fail(FA_ERR_UNSUPPORTED, "d <= 128 required, got %d", d);
  const size_t need = fa_naive_workspace_size(B, H, N);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(FA_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", need, workspace_bytes);
  if (N > 65535 * 16) return fail(FA_ERR_UNSUPPORTED, "N too large for the naive kernel");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
  if (BH > 65535) return fail(FA_ERR_UNSUPPORTED, "B*H too large for the naive kernel");
  __nv_bfloat16* sm = static_cast<__nv_bfloat16*>(workspace);
  const dim3 g1((N + 15) / 16, (N + 15) / 16, BH);
  fa::naive_scores_kernel<<<g1, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(q),
                                             static_cast<const __nv_bfloat16*>(k), sm, block_mask,
                                             kv_len, H, N, d, scale, causal ? 1 : 0);
  if ((rc = check_launch("naive_scores_kernel")) != FA_OK) return rc;
  const long long rows = static_cast<long long>(BH) * N;
  fa::naive_softmax_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, s>>>(sm, lse, rows, N);
  if ((rc = check_launch("naive_softmax_kernel")) != FA_OK) return rc;
  const dim3 g3(1, (N + 15) / 16, BH);
  fa::naive_pv_kernel<<<g3, 256, 0, s>>>(sm, static_cast<const __nv_bfloat16*>(v),
                                         static_cast<__nv_bfloat16*>(o), N, d);
  return check_launch("naive_pv_kernel");
}

}  // extern "C"

// ---------------------------------------------------------------------------------------------
// Backward pass without any caller-provided or library-allocated workspace.
//
// Some callers cannot hand the library a device buffer: they run inside a host framework that
// owns every device allocation (a plugin interface that passes in only the input and output
// tensors, a fixed-budget memory pool), or they must not call cudaMalloc / cudaFree because
// those calls can synchronise the whole device.  fa_bwd_noalloc serves them: its scratch (the
// log2-scaled lse, Dvec and the fp32 dQ accumulator) lives in the fixed-size array below, which
// the CUDA driver places on every device that loads this library and keeps there until the
// process exits.  Nothing is allocated per call.
namespace {

constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(32) << 20;  // 32 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
struct NoallocSlot {
  void* ptr = nullptr;           // device address of g_noalloc_scratch in context `ctx_id`
  unsigned long long ctx_id = 0;
  bool have_id = false;
};
NoallocSlot g_noalloc[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult qres;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &qres) != cudaSuccess ||
      qres != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(p);
}

// Unique id of the CUDA context current on this thread (a context made after cudaDeviceReset
// gets a new id even if it lands at the same handle value); false if there is none or the
// driver cannot say.
bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_cur = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (get_cur == nullptr || get_id == nullptr) return false;
  CUcontext ctx = nullptr;
  if (get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_noalloc_scratch in the current context.  The host-side name of the array
// is only a stand-in, never a device address, so the address is looked up with the device
// current.  It is cached per device together with the id of the context it was looked up in,
// and looked up again whenever another context is current (after cudaDeviceReset, or with a
// context the caller made): the module -- and the array with it -- is loaded anew per context.
int noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(FA_ERR_UNSUPPORTED, "device ordinal %d", dev);
  unsigned long long id = 0;
  const bool have_id = current_context_id(&id);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoallocSlot& slot = g_noalloc[dev];
  if (slot.ptr == nullptr || !have_id || !slot.have_id || slot.ctx_id != id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(FA_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    slot.ptr = p;
    // the lookup made the device's context current if none was: record the id it has now
    slot.have_id = current_context_id(&slot.ctx_id);
  }
  *out = slot.ptr;
  return FA_OK;
}

}  // namespace

extern "C" int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                              const float* lse, const void* dO, void* dq, void* dk, void* dv,
                              int B, int H, int N, int d, float scale, int causal,
                              const uint8_t* block_mask, const int32_t* kv_len, int dtype,
                              void* stream) {
  int rc = bwd_checks(q, k, v, o, lse, dO, dq, dk, dv, B, H, H, N, d, scale, dtype);
  if (rc != FA_OK) return rc;
  const BwdWs ws = bwd_ws(B, H, N, d);
  if (ws.total > kNoAllocScratchBytes)
    return fail(FA_ERR_WORKSPACE,
                "fa_bwd_noalloc: this problem needs %zu bytes of scratch but the built-in "
                "scratch holds %zu; use fa_bwd with a caller-provided workspace",
                ws.total, kNoAllocScratchBytes);
  void* scratch = nullptr;
  if ((rc = noalloc_scratch(&scratch)) != FA_OK) return rc;
  // fa_bwd's path on the built-in scratch.  Its first kernel rewrites lse2 / Dvec and zeroes the
  // dQ accumulator, so whatever the previous call left in the scratch never leaks into this one.
  return bwd_impl(q, k, v, o, lse, dO, dq, dk, dv, B, H, H, N, d, scale, causal, block_mask,
                  kv_len, dtype, scratch, kNoAllocScratchBytes, stream, false);
}
