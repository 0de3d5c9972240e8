// Host side of libfa_b200.so: argument checks, TMA tensor maps and kernel
// launches behind the C ABI declared in include/fa.h.  The whole library is
// this one translation unit (the kernels are included below).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <mutex>
#include <utility>

#include "fa.h"
#include "sm100.cuh"
#include "fa_fwd.cuh"
#include "fa_fwd_fp8.cuh"
#include "fa_bwd.cuh"
#include "fa_decode.cuh"

namespace {

using fa::FwdLayout;
using fa::FwdParams;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

// 3-D tiled map over a dense [outer][rows][cols] tensor (cols contiguous),
// copied in boxes of box_rows x box_cols with 128-byte swizzle.  Out-of-range
// rows read as zero and are skipped on stores.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, uint64_t cols,
              uint64_t rows, uint64_t outer, uint32_t box_cols, uint32_t box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {cols, rows, outer};
  cuuint64_t strides[2] = {cols * esize, cols * rows * esize};
  cuuint32_t box[3] = {box_cols, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Events bracketing the launches of one kernel (see fa_set_profile_events).
cudaEvent_t g_prof_start[8] = {nullptr};
cudaEvent_t g_prof_stop[8] = {nullptr};

void prof_begin(int id, cudaStream_t st) {
  if (g_prof_start[id]) cudaEventRecord(g_prof_start[id], st);
}
void prof_end(int id, cudaStream_t st) {
  if (g_prof_stop[id]) cudaEventRecord(g_prof_stop[id], st);
}

// Cap on the persistent blocks of the backward main pass (0: one per SM).
std::atomic<int> g_bwd_max_blocks{0};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device must be sm_100 (B200 class); checked once per device.
fa_status_t check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  static std::atomic<int> ok_dev[64] = {};  // 0 unknown, 1 ok, 2 not ok (calls may race)
  if (dev < 0 || dev >= 64) return FA_ERR_UNSUPPORTED;
  if (ok_dev[dev].load() == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return FA_ERR_CUDA;
    ok_dev[dev].store((major == 10 && minor == 0) ? 1 : 2);
  }
  return ok_dev[dev].load() == 1 ? FA_OK : FA_ERR_UNSUPPORTED;
}

// Number of SMs of the current device (cached per device); 0 on error.
int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  static std::atomic<int> n_sm[64] = {};  // 0: not yet queried (calls may race)
  if (n_sm[dev].load() == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    n_sm[dev].store(n);
  }
  return n_sm[dev].load();
}

// Dropout probability -> 8-bit threshold t = round(256 p): a key is dropped
// when its random byte is below t.  p must be finite, 0 <= p and t <= 255.
bool drop_threshold(float p, int* t) {
  if (!std::isfinite(p) || p < 0.f) return false;
  const long r = std::lround(static_cast<double>(p) * 256.0);
  if (r > 255) return false;
  *t = static_cast<int>(r);
  return true;
}

// Checks shared by fa_fwd and fa_bwd.  Sets *empty for a problem with no work.
fa_status_t check_common(int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                         fa_dtype_t dtype, bool* empty) {
  if (B < 0 || N < 0 || Hq <= 0 || Hkv <= 0) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (dtype != FA_BF16 && dtype != FA_FP16) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  // sizes the kernels index with 32-bit block counts and TMA coordinates
  const int64_t tiles = (static_cast<int64_t>(N) + 127) / 128;
  if (static_cast<int64_t>(B) * Hq * tiles > INT32_MAX) return FA_ERR_UNSUPPORTED;
  *empty = (B == 0 || N == 0);
  return FA_OK;
}

// Opt a kernel into `smem` bytes of dynamic shared memory, once per kernel
// and device (the attribute belongs to the device's context).
template <typename K>
fa_status_t opt_in_smem(K kernel, int smem) {
  static std::mutex mu;
  static const void* done_fn[256];
  static int done_dev[256];
  static int n_done = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n_done; ++i)
    if (done_fn[i] == reinterpret_cast<const void*>(kernel) && done_dev[i] == dev) return FA_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return FA_ERR_CUDA;
  if (n_done < 256) {
    done_fn[n_done] = reinterpret_cast<const void*>(kernel);
    done_dev[n_done++] = dev;
  }
  return FA_OK;
}

// Launches `kernel` as a programmatic dependent of the kernel before it on the
// stream: it may be scheduled while that kernel still runs, and waits
// (griddepcontrol.wait) before it touches global memory.  Used for the decode
// pair (split, then merge), whose launch gap is a visible part of a step; on
// the training path it measured slower and is not used.
template <typename... Params, typename... Args>
cudaError_t launch_dependent(void (*kernel)(Params...), unsigned grid, unsigned block, int smem,
                             cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <int HD, bool BF, bool CA, bool DR, bool BM = false>
fa_status_t launch_fwd(const FwdParams& prm, cudaStream_t st) {
  auto kern = fa::fa_fwd_kernel<HD, BF, CA, DR, BM>;
  const int smem = FwdLayout<HD>::kDynSmem;
  fa_status_t s = opt_in_smem(kern, smem);
  if (s != FA_OK) return s;
  // one block per (head, couple of query pairs) or per (head, query pair)
  const int grid = (prm.fold ? (prm.n_pairs + 1) / 2 : prm.n_pairs) * prm.BH;
  prof_begin(fa::kKernFwd, st);
  kern<<<grid, fa::kFwdThreads, smem, st>>>(prm);
  const bool ok = cudaGetLastError() == cudaSuccess;
  prof_end(fa::kKernFwd, st);
  return ok ? FA_OK : FA_ERR_CUDA;
}

template <int HD, bool BF>
fa_status_t launch_fwd_c(const FwdParams& prm, int causal, cudaStream_t st) {
  if (prm.bmask != nullptr)
    return causal ? launch_fwd<HD, BF, true, false, true>(prm, st) : launch_fwd<HD, BF, false, false, true>(prm, st);
  if (prm.drop_t > 0)
    return causal ? launch_fwd<HD, BF, true, true>(prm, st) : launch_fwd<HD, BF, false, true>(prm, st);
  return causal ? launch_fwd<HD, BF, true, false>(prm, st) : launch_fwd<HD, BF, false, false>(prm, st);
}

// The FP8 forward kernel; its launches are bracketed by the forward's
// profiling events.
template <bool OB, bool CA>
fa_status_t launch_fwd_fp8(const fa::Fp8FwdParams& prm, cudaStream_t st) {
  auto kern = fa::fa_fwd_fp8_kernel<OB, CA>;
  const int smem = fa::Fp8FwdLayout::kDynSmem;
  fa_status_t s = opt_in_smem(kern, smem);
  if (s != FA_OK) return s;
  // one block per (head, couple of query pairs) or per (head, query pair)
  const int grid = (prm.fold ? (prm.n_pairs + 1) / 2 : prm.n_pairs) * prm.BH;
  prof_begin(fa::kKernFwd, st);
  kern<<<grid, fa::kFwdFp8Threads, smem, st>>>(prm);
  const bool ok = cudaGetLastError() == cudaSuccess;
  prof_end(fa::kKernFwd, st);
  return ok ? FA_OK : FA_ERR_CUDA;
}

template <int HD, bool BF, bool CA, bool DR, bool BM = false>
fa_status_t launch_bwd_main(const fa::BwdParams& prm, int grid, cudaStream_t st) {
  auto kern = fa::fa_bwd_kernel<HD, BF, CA, DR, BM>;
  const int smem = fa::BwdLayout<HD>::kDynSmem;
  fa_status_t s = opt_in_smem(kern, smem);
  if (s != FA_OK) return s;
  prof_begin(fa::kKernBwd, st);
  kern<<<grid, fa::kBwdThreads, smem, st>>>(prm);
  const bool ok = cudaGetLastError() == cudaSuccess;
  prof_end(fa::kKernBwd, st);
  return ok ? FA_OK : FA_ERR_CUDA;
}

template <int HD, bool BF>
fa_status_t bwd_run(const void* q, const void* k, const void* v, const void* o, const void* dout,
                    const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N,
                    float scale, int causal, int window, uint32_t drop_t, uint64_t seed,
                    void* workspace, cudaStream_t st, const uint8_t* bmask = nullptr,
                    long long bm_hstride = 0) {
  const int64_t Np = fa::bwd_padded_rows(N);
  const int64_t BHq = static_cast<int64_t>(B) * Hq, BHkv = static_cast<int64_t>(B) * Hkv;
  float* Dvec = static_cast<float*>(workspace);
  float* lse2 = Dvec + BHq * Np;
  float* dqacc = lse2 + BHq * Np;
  const int64_t rows = BHq * Np;
  unsigned* work_counter = reinterpret_cast<unsigned*>(dqacc + rows * HD);
  const int n_ktiles = (N + 127) / 128;

  // 1. D, lse2, zeroed accumulator and work counter
  fa::BwdPreParams pre;
  std::memset(&pre, 0, sizeof(pre));
  pre.o = o;
  pre.dout = dout;
  pre.lse = lse;
  pre.Dvec = Dvec;
  pre.lse2 = lse2;
  pre.dqacc = dqacc;
  pre.work_counter = work_counter;
  pre.N = N;
  pre.Np = static_cast<int>(Np);
  pre.total_rows = rows;
  {
    // HD / 8 threads a row; a grid of 16 blocks of 256 threads per SM, each
    // thread taking rows in turn
    const int64_t groups = rows * (HD / 8);
    int n_sm = sm_count();
    if (n_sm <= 0) return FA_ERR_CUDA;
    const int64_t blocks = std::min<int64_t>((groups + 255) / 256, static_cast<int64_t>(n_sm) * 16);
    fa::fa_bwd_pre_kernel<HD, BF><<<static_cast<unsigned>(blocks), 256, 0, st>>>(pre);
  }
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;

  // 1b. block mask: the walk of every work item
  uint16_t* plan_list = nullptr;
  int* plan_steps = nullptr;
  const int plan_cap = (Hq / Hkv) * n_ktiles;
  if (bmask != nullptr) {
    plan_steps = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(workspace) + fa::bwd_workspace_bytes(B, Hq, N, HD));
    plan_list = reinterpret_cast<uint16_t*>(plan_steps + BHkv * n_ktiles);
    fa::BwdPlanParams pl;
    std::memset(&pl, 0, sizeof(pl));
    pl.bmask = bmask;
    pl.bm_hstride = bm_hstride;
    pl.list = plan_list;
    pl.steps = plan_steps;
    pl.N = N;
    pl.Hq = Hq;
    pl.Hkv = Hkv;
    pl.group = Hq / Hkv;
    pl.n_ktiles = n_ktiles;
    pl.n_qtiles = (N + 63) / 64;
    pl.causal = causal;
    pl.window = window;
    pl.cap = plan_cap;
    pl.n_items = static_cast<int>(BHkv * n_ktiles);
    fa::fa_bwd_plan_kernel<<<static_cast<unsigned>((pl.n_items + 7) / 8), 256, 0, st>>>(pl);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }

  // 2. main pass
  const CUtensorMapDataType dt = BF ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  fa::BwdParams prm;
  std::memset(&prm, 0, sizeof(prm));
  if (!make_map(&prm.tm_q, q, dt, 2, HD, N, BHq, 64, 64) ||
      !make_map(&prm.tm_do, dout, dt, 2, HD, N, BHq, 64, 64) ||
      !make_map(&prm.tm_k, k, dt, 2, HD, N, BHkv, 64, 128) ||
      !make_map(&prm.tm_v, v, dt, 2, HD, N, BHkv, 64, 128))
    return FA_ERR_CUDA;
  prm.lse2 = lse2;
  prm.Dvec = Dvec;
  prm.dqacc = dqacc;
  prm.plan_list = plan_list;
  prm.plan_steps = plan_steps;
  prm.plan_cap = plan_cap;
  prm.dk = dk;
  prm.dv = dv;
  prm.work_counter = work_counter;
  prm.N = N;
  prm.Np = static_cast<int>(Np);
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.group = Hq / Hkv;
  prm.n_ktiles = (N + 127) / 128;
  prm.n_qtiles = (N + 63) / 64;
  prm.BHkv = static_cast<int>(BHkv);
  prm.scale = scale;
  prm.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  prm.window = window;
  prm.drop_t = drop_t;
  prm.drop_scale = drop_t ? 256.0f / static_cast<float>(256u - drop_t) : 1.0f;
  prm.seed_lo = static_cast<uint32_t>(seed);
  prm.seed_hi = static_cast<uint32_t>(seed >> 32);
  prm.n_items = prm.n_ktiles * prm.BHkv;
  {
    // kv heads per chunk of the item order: Q, dO (group query heads), K, V
    // and the fp32 dQ accumulator of a chunk stay within about 48 MB of L2
    const double head_bytes = static_cast<double>(prm.group) * N * HD * 2.0 * 2.0 +
                              static_cast<double>(prm.group) * Np * HD * 4.0 +
                              static_cast<double>(N) * HD * 2.0 * 2.0;
    const double c = std::floor(48.0 * 1024.0 * 1024.0 / head_bytes);
    prm.chunk_heads = static_cast<int>(std::max(1.0, std::min(c, static_cast<double>(prm.BHkv))));
  }
  int n_sm = 0;
  if ((n_sm = sm_count()) <= 0) return FA_ERR_CUDA;
  const int cap = g_bwd_max_blocks.load();
  const int grid = std::min(prm.n_items, cap > 0 ? std::min(cap, n_sm) : n_sm);  // persistent
  fa_status_t s;
  if (bmask != nullptr)
    s = causal ? launch_bwd_main<HD, BF, true, false, true>(prm, grid, st)
               : launch_bwd_main<HD, BF, false, false, true>(prm, grid, st);
  else if (prm.drop_t > 0)
    s = causal ? launch_bwd_main<HD, BF, true, true>(prm, grid, st)
               : launch_bwd_main<HD, BF, false, true>(prm, grid, st);
  else
    s = causal ? launch_bwd_main<HD, BF, true, false>(prm, grid, st)
               : launch_bwd_main<HD, BF, false, false>(prm, grid, st);
  if (s != FA_OK) return s;

  // 3. dQ = scale * accumulator
  const int64_t total_vec = BHq * N * (HD / 8);
  const int64_t blocks = std::min<int64_t>((total_vec + 255) / 256, 148 * 16);
  fa::fa_bwd_post_kernel<HD, BF><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
      dqacc, dq, N, static_cast<int>(Np), total_vec, scale);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

extern "C" {

}  // extern "C"

namespace {

fa_status_t fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int Hq, int Hkv, int N, int d, float scale, int causal, int window,
                     uint32_t drop_t, uint64_t seed, fa_dtype_t dtype, void* stream,
                     const uint8_t* bmask = nullptr, long long bm_hstride = 0) {
  bool empty = false;
  fa_status_t s = check_common(B, Hq, Hkv, N, d, scale, causal, dtype, &empty);
  if (s != FA_OK) return s;
  if (empty) return FA_OK;
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return FA_ERR_MISALIGNED;
  if ((s = check_device()) != FA_OK) return s;

  const bool bf = dtype == FA_BF16;
  const CUtensorMapDataType dt = bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  FwdParams prm;
  std::memset(&prm, 0, sizeof(prm));
  const uint64_t BHq = static_cast<uint64_t>(B) * Hq, BHkv = static_cast<uint64_t>(B) * Hkv;
  if (!make_map(&prm.tm_q, q, dt, 2, d, N, BHq, 64, 128) ||
      !make_map(&prm.tm_k, k, dt, 2, d, N, BHkv, 64, 128) ||
      !make_map(&prm.tm_v, v, dt, 2, d, N, BHkv, 64, 128))
    return FA_ERR_CUDA;
  prm.o = o;
  prm.lse = lse;
  prm.N = N;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.group = Hq / Hkv;
  prm.BH = static_cast<int>(BHq);
  prm.n_pairs = (N + 255) / 256;
  // fold two query pairs into a block while a pair is short (its fixed costs
  // then weigh most): up to 64 pairs (N <= 16384)
  prm.fold = prm.n_pairs <= 64 ? 1 : 0;
  prm.n_ktiles = (N + 127) / 128;
  prm.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  prm.window = window;
  prm.drop_t = drop_t;
  prm.drop_scale = drop_t ? 256.0f / static_cast<float>(256u - drop_t) : 1.0f;
  prm.seed_lo = static_cast<uint32_t>(seed);
  prm.seed_hi = static_cast<uint32_t>(seed >> 32);
  prm.bmask = bmask;
  prm.bm_hstride = bm_hstride;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (d == 128) return bf ? launch_fwd_c<128, true>(prm, causal, st) : launch_fwd_c<128, false>(prm, causal, st);
  return bf ? launch_fwd_c<64, true>(prm, causal, st) : launch_fwd_c<64, false>(prm, causal, st);
}

}  // namespace

extern "C" {

fa_status_t fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                   int Hq, int Hkv, int N, int d, float scale, int causal, fa_dtype_t dtype,
                   void* stream) {
  return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal, 0, 0, 0, dtype, stream);
}

fa_status_t fa_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                          int Hq, int Hkv, int N, int d, float scale, int window, fa_dtype_t dtype,
                          void* stream) {
  if (window < 1) return FA_ERR_INVALID_ARG;
  return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, 1, window, 0, 0, dtype, stream);
}

fa_status_t fa_fwd_dropout(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                           int Hq, int Hkv, int N, int d, float scale, int causal, float p_drop,
                           uint64_t seed, fa_dtype_t dtype, void* stream) {
  int t = 0;
  if (!drop_threshold(p_drop, &t)) return FA_ERR_INVALID_ARG;
  return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal, 0, static_cast<uint32_t>(t),
                  seed, dtype, stream);
}

fa_status_t fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                       int Hq, int Hkv, int N, int d, float scale, float descale_q,
                       float descale_k, float descale_v, int causal, fa_dtype_t out_dtype,
                       void* stream) {
  bool empty = false;
  fa_status_t s = check_common(B, Hq, Hkv, N, d, scale, causal, out_dtype, &empty);
  if (s != FA_OK) return s;
  for (float f : {descale_q, descale_k, descale_v})
    if (!std::isfinite(f) || !(f > 0.f)) return FA_ERR_INVALID_ARG;
  const double c = static_cast<double>(scale) * descale_q * descale_k * 1.4426950408889634;
  if (!(c >= 1.2e-38) || c > 3.0e38) return FA_ERR_INVALID_ARG;  // a normal fp32 factor
  if (d != 128) return FA_ERR_UNSUPPORTED;
  if (empty) return FA_OK;
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return FA_ERR_MISALIGNED;
  if ((s = check_device()) != FA_OK) return s;

  const bool bf = out_dtype == FA_BF16;
  const CUtensorMapDataType dt16 = bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  fa::Fp8FwdParams prm;
  std::memset(&prm, 0, sizeof(prm));
  const uint64_t BHq = static_cast<uint64_t>(B) * Hq, BHkv = static_cast<uint64_t>(B) * Hkv;
  if (!make_map(&prm.tm_q, q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 128, N, BHq, 128, 128) ||
      !make_map(&prm.tm_k, k, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 128, N, BHkv, 128, 128) ||
      !make_map(&prm.tm_v, v, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 128, N, BHkv, 128, 128) ||
      !make_map(&prm.tm_o, o, dt16, 2, 128, N, BHq, 64, 128))
    return FA_ERR_CUDA;
  prm.lse = lse;
  prm.N = N;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.group = Hq / Hkv;
  prm.BH = static_cast<int>(BHq);
  prm.n_pairs = (N + 255) / 256;
  prm.fold = prm.n_pairs <= 64 ? 1 : 0;  // as in the 16-bit forward
  prm.n_ktiles = (N + 127) / 128;
  prm.scale_log2 = static_cast<float>(c);
  prm.delta_v = descale_v;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (causal) return bf ? launch_fwd_fp8<true, true>(prm, st) : launch_fwd_fp8<false, true>(prm, st);
  return bf ? launch_fwd_fp8<true, false>(prm, st) : launch_fwd_fp8<false, false>(prm, st);
}

size_t fa_bwd_workspace_bytes(int B, int Hq, int Hkv, int N, int d) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || d <= 0) return 0;
  return fa::bwd_workspace_bytes(B, Hq, N, d);
}

}  // extern "C"

namespace {

// Block-mask additions to the backward workspace: the step count and the
// walk of every work item (see fa_bwd_plan_kernel).
size_t bwd_mask_plan_bytes(int B, int Hq, int Hkv, int N) {
  const int64_t n_ktiles = (static_cast<int64_t>(N) + 127) / 128;
  const int64_t items = static_cast<int64_t>(B) * Hkv * n_ktiles;
  const int64_t cap = static_cast<int64_t>(Hq / Hkv) * n_ktiles;
  return static_cast<size_t>(items) * 4u + static_cast<size_t>(items * cap) * 2u;
}

// Sizes a block mask supports: the walk entries hold the group head in 4
// bits and the query block in 12.
bool bmask_supported(int Hq, int Hkv, int N) {
  return Hq / Hkv <= 16 && (static_cast<int64_t>(N) + 127) / 128 <= 4096;
}

fa_status_t bwd_impl(const void* q, const void* k, const void* v, const void* o, const void* dout,
                     const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N,
                     int d, float scale, int causal, int window, uint32_t drop_t, uint64_t seed,
                     fa_dtype_t dtype, void* workspace, size_t workspace_bytes, void* stream,
                     const uint8_t* bmask = nullptr, long long bm_hstride = 0) {
  bool empty = false;
  fa_status_t s = check_common(B, Hq, Hkv, N, d, scale, causal, dtype, &empty);
  if (s != FA_OK) return s;
  if (empty) return FA_OK;
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !workspace)
    return FA_ERR_INVALID_ARG;
  size_t need = fa::bwd_workspace_bytes(B, Hq, N, d);
  if (bmask != nullptr) {
    if (!bmask_supported(Hq, Hkv, N)) return FA_ERR_UNSUPPORTED;
    need += bwd_mask_plan_bytes(B, Hq, Hkv, N);
  }
  if (workspace_bytes < need) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(lse) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      !aligned16(workspace))
    return FA_ERR_MISALIGNED;
  if ((s = check_device()) != FA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf = dtype == FA_BF16;
  if (d == 128)
    return bf ? bwd_run<128, true>(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, N, scale, causal, window, drop_t, seed, workspace, st, bmask, bm_hstride)
              : bwd_run<128, false>(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, N, scale, causal, window, drop_t, seed, workspace, st, bmask, bm_hstride);
  return bf ? bwd_run<64, true>(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, N, scale, causal, window, drop_t, seed, workspace, st, bmask, bm_hstride)
            : bwd_run<64, false>(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, N, scale, causal, window, drop_t, seed, workspace, st, bmask, bm_hstride);
}

}  // namespace

extern "C" {

fa_status_t fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                   const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N,
                   int d, float scale, int causal, fa_dtype_t dtype, void* workspace,
                   size_t workspace_bytes, void* stream) {
  return bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, N, d, scale, causal, 0, 0, 0,
                  dtype, workspace, workspace_bytes, stream);
}

fa_status_t fa_bwd_window(const void* q, const void* k, const void* v, const void* o,
                          const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                          int Hq, int Hkv, int N, int d, float scale, int window, fa_dtype_t dtype,
                          void* workspace, size_t workspace_bytes, void* stream) {
  if (window < 1) return FA_ERR_INVALID_ARG;
  return bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, N, d, scale, 1, window, 0, 0,
                  dtype, workspace, workspace_bytes, stream);
}

fa_status_t fa_bwd_dropout(const void* q, const void* k, const void* v, const void* o,
                           const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                           int Hq, int Hkv, int N, int d, float scale, int causal, float p_drop,
                           uint64_t seed, fa_dtype_t dtype, void* workspace,
                           size_t workspace_bytes, void* stream) {
  int t = 0;
  if (!drop_threshold(p_drop, &t)) return FA_ERR_INVALID_ARG;
  return bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, N, d, scale, causal, 0,
                  static_cast<uint32_t>(t), seed, dtype, workspace, workspace_bytes, stream);
}

fa_status_t fa_fwd_blockmask(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                             int Hq, int Hkv, int N, int d, float scale, int causal,
                             const uint8_t* block_mask, int mask_per_head, fa_dtype_t dtype,
                             void* stream) {
  if (block_mask == nullptr || (mask_per_head != 0 && mask_per_head != 1)) return FA_ERR_INVALID_ARG;
  if (Hq > 0 && Hkv > 0 && Hq % Hkv == 0 && !bmask_supported(Hq, Hkv, N)) return FA_ERR_UNSUPPORTED;
  const long long nb = (static_cast<long long>(N) + 127) / 128;
  return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal, 0, 0, 0, dtype, stream, block_mask,
                  mask_per_head ? nb * nb : 0);
}

size_t fa_bwd_blockmask_workspace_bytes(int B, int Hq, int Hkv, int N, int d) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || d <= 0 || Hq % Hkv != 0) return 0;
  return fa::bwd_workspace_bytes(B, Hq, N, d) + bwd_mask_plan_bytes(B, Hq, Hkv, N);
}

fa_status_t fa_bwd_blockmask(const void* q, const void* k, const void* v, const void* o,
                             const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                             int Hq, int Hkv, int N, int d, float scale, int causal,
                             const uint8_t* block_mask, int mask_per_head, fa_dtype_t dtype,
                             void* workspace, size_t workspace_bytes, void* stream) {
  if (block_mask == nullptr || (mask_per_head != 0 && mask_per_head != 1)) return FA_ERR_INVALID_ARG;
  const long long nb = (static_cast<long long>(N) + 127) / 128;
  return bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, N, d, scale, causal, 0, 0, 0, dtype,
                  workspace, workspace_bytes, stream, block_mask, mask_per_head ? nb * nb : 0);
}

fa_status_t fa_get_device_status(void* stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return FA_ERR_CUDA;
  uint32_t word = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&word, fa::g_device_status, sizeof(word)) != cudaSuccess)
    return FA_ERR_CUDA;
  if (word == 0) return FA_OK;
  if (cudaMemcpyToSymbol(fa::g_device_status, &zero, sizeof(zero)) != cudaSuccess)
    return FA_ERR_CUDA;
  const uint32_t code = word & 0xFFu;
  if (code == fa::kStatusTimeout) return FA_ERR_TIMEOUT;
  if (code == fa::kStatusBadInput) return FA_ERR_INVALID_ARG;
  return FA_ERR_CUDA;
}

uint32_t fa_peek_device_status_word(void* stream) {
  cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  uint32_t word = 0;
  cudaMemcpyFromSymbol(&word, fa::g_device_status, sizeof(word));
  return word;
}

fa_status_t fa_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
  fa_status_t s = check_device();
  if (s != FA_OK) return s;
  if (limit_ns == 0 || limit_ns > 10ull * 1000 * 1000 * 1000) return FA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // clear any earlier status, shorten the limit, run, restore
  if ((s = fa_get_device_status(stream)) == FA_ERR_CUDA) return s;
  const uint64_t dflt = 2000000000ull;
  if (cudaMemcpyToSymbolAsync(fa::g_wait_limit_ns, &limit_ns, sizeof(limit_ns), 0,
                              cudaMemcpyHostToDevice, st) != cudaSuccess)
    return FA_ERR_CUDA;
  fa::wait_timeout_selftest_kernel<<<1, 32, 0, st>>>();
  const bool launched = cudaGetLastError() == cudaSuccess;
  cudaMemcpyToSymbolAsync(fa::g_wait_limit_ns, &dflt, sizeof(dflt), 0, cudaMemcpyHostToDevice, st);
  if (!launched) return FA_ERR_CUDA;
  return fa_get_device_status(stream);
}

fa_status_t fa_set_profile_events(int kernel_id, void* start, void* stop) {
  if (kernel_id != static_cast<int>(fa::kKernFwd) && kernel_id != static_cast<int>(fa::kKernBwd))
    return FA_ERR_INVALID_ARG;
  if ((start == nullptr) != (stop == nullptr)) return FA_ERR_INVALID_ARG;
  g_prof_start[kernel_id] = reinterpret_cast<cudaEvent_t>(start);
  g_prof_stop[kernel_id] = reinterpret_cast<cudaEvent_t>(stop);
  return FA_OK;
}

size_t fa_decode_workspace_bytes(int B, int Hq, int Hkv, int Nq, int d, int max_pages) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || d <= 0 || max_pages <= 0) return 0;
  return fa::decode_workspace_bytes(B, Hq, Hkv, Nq, d, max_pages);
}

fa_status_t fa_decode_paged(const void* q, const void* k_cache, const void* v_cache,
                            const int* block_table, const int* seq_lens, void* o, float* lse, int B,
                            int Hq, int Hkv, int Nq, int d, int page_size, int max_pages,
                            int num_pages, float scale, fa_dtype_t dtype, void* workspace,
                            size_t workspace_bytes, void* stream) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || Nq <= 0 || max_pages <= 0 ||
      num_pages <= 0)
    return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (dtype != FA_BF16 && dtype != FA_FP16) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (page_size != 16 && page_size != 32 && page_size != 64 && page_size != 128)
    return FA_ERR_UNSUPPORTED;
  if ((Hq / Hkv) * Nq > fa::kDecodeMaxRows) return FA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(max_pages) * page_size > INT32_MAX) return FA_ERR_UNSUPPORTED;
  if (B == 0) return FA_OK;
  if (!q || !k_cache || !v_cache || !block_table || !seq_lens || !o || !lse || !workspace)
    return FA_ERR_INVALID_ARG;
  if (workspace_bytes < fa::decode_workspace_bytes(B, Hq, Hkv, Nq, d, max_pages))
    return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
      !aligned16(workspace) || (reinterpret_cast<uintptr_t>(lse) & 3u) ||
      (reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return FA_ERR_MISALIGNED;
  fa_status_t s = check_device();
  if (s != FA_OK) return s;
  fa::DecodeParams prm;
  std::memset(&prm, 0, sizeof(prm));
  prm.q = q;
  prm.table = block_table;
  prm.lens = seq_lens;
  prm.o = o;
  prm.lse = lse;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.Nq = Nq;
  prm.P = page_size;
  prm.max_pages = max_pages;
  prm.num_pages = num_pages;
  // the caches as [num_pages * Hkv][P][d]: one box = 64 features of the P
  // rows of one (page, kv head)
  if (static_cast<int64_t>(num_pages) * Hkv > INT32_MAX) return FA_ERR_UNSUPPORTED;
  const CUtensorMapDataType tdt = dtype == FA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  if (!make_map(&prm.tm_k, k_cache, tdt, 2, d, page_size, static_cast<uint64_t>(num_pages) * Hkv, 64, page_size) ||
      !make_map(&prm.tm_v, v_cache, tdt, 2, d, page_size, static_cast<uint64_t>(num_pages) * Hkv, 64, page_size))
    return FA_ERR_CUDA;
  prm.S = fa::decode_splits(B, Hkv, d, max_pages);
  // a split holds whole tiles of 128 keys
  const int ppt = fa::kDecodeTile / page_size;
  prm.pages_per_split = ((max_pages + prm.S - 1) / prm.S + ppt - 1) / ppt * ppt;
  prm.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  const int64_t rows = static_cast<int64_t>(B) * Hq * Nq;
  prm.part_o = static_cast<float*>(workspace);
  prm.part_ml = prm.part_o + rows * prm.S * d;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf = dtype == FA_BF16;
  const int R = (Hq / Hkv) * Nq;
  const int rb = R <= 4 ? 4 : R <= 8 ? 8 : R <= 16 ? 16 : 32;
  // q as [B * Hq * Nq][d]; a box is the NP (rows padded to 16 or 32) rows
  // that start at an item's first row
  const int np = rb < 16 ? 16 : rb;
  if (!make_map(&prm.tm_q, q, tdt, 2, d, static_cast<uint64_t>(B) * Hq * Nq, 1, 64, np)) return FA_ERR_CUDA;
  const int64_t n_work = static_cast<int64_t>(B) * Hkv * prm.S;
  if (n_work > INT32_MAX) return FA_ERR_UNSUPPORTED;
  const int sms = sm_count();
  if (sms <= 0) return FA_ERR_CUDA;
  auto run = [&](auto split_kern, auto merge_kern, int smem) -> fa_status_t {
    fa_status_t r = opt_in_smem(split_kern, smem);
    if (r != FA_OK) return r;
    // persistent: as many blocks as fit on the GPU at once, each taking
    // work items (splits) in turn
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, split_kern, fa::kDecodeThreads, smem) !=
            cudaSuccess ||
        per_sm <= 0)
      return FA_ERR_CUDA;
    const int grid = static_cast<int>(std::min<int64_t>(n_work, static_cast<int64_t>(sms) * per_sm));
    if (launch_dependent(split_kern, static_cast<unsigned>(grid), fa::kDecodeThreads, smem, st, prm) !=
        cudaSuccess)
      return FA_ERR_CUDA;
    return launch_dependent(merge_kern, static_cast<unsigned>(rows), static_cast<unsigned>(d), 0, st, prm) ==
                   cudaSuccess
               ? FA_OK
               : FA_ERR_CUDA;
  };
#define FA_DECODE_RUN(HD, BFV, RBV)                                                                  \
  run(fa::fa_decode_split_kernel<HD, BFV, RBV>, fa::fa_decode_merge_kernel<HD, BFV>, \
      fa::DecodeLayout<HD, RBV>::kDynSmem)
#define FA_DECODE_RB(HD, BFV)                                                        \
  (rb == 4 ? FA_DECODE_RUN(HD, BFV, 4) : rb == 8 ? FA_DECODE_RUN(HD, BFV, 8)        \
             : rb == 16 ? FA_DECODE_RUN(HD, BFV, 16) : FA_DECODE_RUN(HD, BFV, 32))
  fa_status_t rs;
  if (d == 128)
    rs = bf ? FA_DECODE_RB(128, true) : FA_DECODE_RB(128, false);
  else
    rs = bf ? FA_DECODE_RB(64, true) : FA_DECODE_RB(64, false);
#undef FA_DECODE_RB
#undef FA_DECODE_RUN
  return rs;
}

fa_status_t fa_set_bwd_max_blocks(int max_blocks) {
  if (max_blocks < 0) return FA_ERR_INVALID_ARG;
  g_bwd_max_blocks.store(max_blocks);
  return FA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Fixed scratch for fa_bwd_noalloc: reserved in the device memory of every GPU
// that loads this library, for the life of the process.  Host code must not
// pass `g_bwd_noalloc_scratch` itself to a kernel (on the host the name is
// only a stand-in); its device address is looked up once per device with
// cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_bwd_noalloc_scratch[FA_BWD_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {nullptr};

// Device address of the scratch array on the current device (looked up on
// the first call per device).
fa_status_t noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev < 0 || dev >= 64) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_noalloc_scratch) != cudaSuccess || p == nullptr)
      return FA_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return FA_OK;
}
}  // namespace

extern "C" {

fa_status_t fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                           const void* dout, const float* lse, void* dq, void* dk, void* dv,
                           int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                           fa_dtype_t dtype, void* stream) {
  bool empty = false;
  fa_status_t s = check_common(B, Hq, Hkv, N, d, scale, causal, dtype, &empty);
  if (s != FA_OK) return s;
  if (empty) return FA_OK;
  const size_t need = fa::bwd_workspace_bytes(B, Hq, N, d);
  if (need > FA_BWD_NOALLOC_SCRATCH_BYTES) return FA_ERR_UNSUPPORTED;
  if ((s = check_device()) != FA_OK) return s;
  void* scratch = nullptr;
  if ((s = noalloc_scratch(&scratch)) != FA_OK) return s;
  return fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, N, d, scale, causal, dtype,
                scratch, FA_BWD_NOALLOC_SCRATCH_BYTES, stream);
}

const char* fa_status_string(fa_status_t status) {
  switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported configuration or device";
    case FA_ERR_MISALIGNED: return "tensor pointer not 16-byte aligned";
    case FA_ERR_CUDA: return "CUDA error";
    case FA_ERR_TIMEOUT: return "device-side barrier wait timed out";
  }
  return "unknown status";
}

}  // extern "C"
