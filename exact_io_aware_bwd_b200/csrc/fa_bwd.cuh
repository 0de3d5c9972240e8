// Backward pass of exact attention on sm_100a, by recomputation.
//
// The pages keep only the softmax statistics from the forward pass and
// recompute the scores on chip in the backward pass ("FlashAttention"
// glossary, recomputation paragraph), and let one thread block own a block of
// keys so that dK and dV need no atomics ("FlashAttention" glossary,
// FlashAttention-2 list, backward-pass item).  The gradient formulas are the
// calculus of softmax (the pages print none):
//   P_ij  = exp(scale s_ij - lse_i)            (recomputed, s = q.k)
//   dV_j  = sum_i P_ij dO_i
//   dP_ij = dO_i . v_j
//   D_i   = sum_j P_ij dP_ij = dO_i . O_i
//   dS_ij = P_ij (dP_ij - D_i)
//   dQ_i  = scale sum_j dS_ij k_j,   dK_j = scale sum_i dS_ij q_i
//
// Three kernels:
//   bwd_pre   d/8 threads per query row: D_i = dO_i . O_i, lse2_i = lse_i log2(e)
//             (+inf for padding rows, which makes their P exactly 0), and a
//             zeroed fp32 dQ accumulator row.
//   bwd_main  persistent: one thread block per SM takes work items (128-row
//             key block j, kv head) one after another from a counter in the
//             workspace, head-major and, within a head, the key blocks with
//             the most query blocks first.  For an item, K_j and V_j stay in
//             shared memory; the block walks every query head of the group
//             and every 64-row query block i (causal: i >= the diagonal).
//             Per step, all products on the tensor cores with fp32
//             accumulators in tensor memory:
//               S^T  = K_j Q_i^T        (128 x 64)
//               dP^T = V_j dO_i^T       (128 x 64)
//               softmax warps: P^T, dS^T = P^T o (dP^T - D)
//               dQ_i^T = K_j^T dS^T     (d x 64) -> registers -> red.global.add.f32
//                                        into the fp32 dQ accumulator (in L2)
//               dV  += P^T dO_i         (P^T read from tensor memory)
//               dK  += dS^T Q_i
//             dK, dV stay in tensor memory for the whole walk and are written
//             once at the end: no atomics on them.  The steps of consecutive
//             items run through the same rings without a break: the next
//             item's Q / dO loads start while the last steps of the previous
//             one run, and its dK / dV are written out while the next item's
//             first steps run.
//   bwd_post  dQ = scale * accumulator, converted to the I/O dtype (rows
//             that no key block reaches, possible under a block mask, keep
//             their zeroed accumulator: dQ = 0).
//
// Warp roles of bwd_main (768 threads, at most 80 registers each: 24 warps,
// six per SM sub-partition, share its 16 384 registers):
//   warps 0-15  softmax-gradient: warp w owns key rows 32(w%4)..+31 (tensor
//               memory lanes) and query columns 16(w/4)..+15 of each step.
//   warps 16-19 dQ drain (lane = feature index of dQ^T) and, after each
//               item, the dK / dV epilogue (lane = key row).
//   warp 20     TMA producer; it also claims the work items and passes them
//               to the other roles through a small ring in shared memory.
//   warp 21     MMA issuer (the whole warp runs the loop, one elected lane
//               issues).
//   warps 22-23 idle (they round the block up to six warps per sub-partition).
// Tensor memory: dV [0,128), dK [128,256), and two step buffers b = 0, 1:
// S^T at 256+128b (64 columns; P^T of each 16-query group is written as
// 16-bit pairs over the first 8 columns of that group) and dP^T at
// 256+128b+64 (dQ^T is written over it once the softmax warps have read
// dP^T).  The step buffers let the tensor cores compute step t+1's S^T /
// dP^T while the softmax warps work on step t.
#pragma once

#include <type_traits>

#include "sm100.cuh"

namespace fa {

constexpr uint32_t kKernBwdPre = 2;
constexpr uint32_t kKernBwd = 3;
constexpr uint32_t kKernBwdPost = 4;
constexpr uint32_t kKernSelftest = 9;

__host__ __device__ inline int64_t bwd_padded_rows(int N) { return (static_cast<int64_t>(N) + 127) / 128 * 128; }

// Workspace: D [rows], lse2 [rows], dQ accumulator [rows][d] (fp32), then
// 256 bytes holding the work-item counter of bwd_main.
constexpr size_t kBwdWorkspaceTail = 256;

inline size_t bwd_workspace_bytes(int B, int Hq, int N, int d) {
  const int64_t rows = static_cast<int64_t>(B) * Hq * bwd_padded_rows(N);
  return static_cast<size_t>(rows) * 4u * static_cast<size_t>(2 + d) + kBwdWorkspaceTail;
}

// ---------------------------------------------------------------------------
// bwd_pre

struct BwdPreParams {
  const void* o;
  const void* dout;
  const float* lse;
  float* Dvec;            // [B*Hq][Np]
  float* lse2;            // [B*Hq][Np]
  float* dqacc;           // [B*Hq][Np][d], zeroed here
  unsigned* work_counter;
  int N, Np;
  long long total_rows;
};

// One group of HD / 8 threads per query row, each thread 8 elements (16
// bytes) of O and dO and 8 of the zeroed accumulator (two 16-byte stores);
// the group's partial dot products are summed by shuffles.  Grid-stride over
// the rows, so that every thread keeps several rows' loads in flight; a
// warp's lanes take 32 / (HD / 8) consecutive rows and the row count (a
// multiple of 128) and the stride are multiples of that, so all lanes of a
// warp run the same iterations and the shuffles see every lane.
template <int HD, bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const __grid_constant__ BwdPreParams p) {
  using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
  constexpr int kTpr = HD / 8;  // threads per row: 16 or 8
  const int64_t gtid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int c8 = static_cast<int>(gtid % kTpr);
  if (gtid == 0) *p.work_counter = 0u;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x / kTpr;
  for (int64_t row = gtid / kTpr; row < p.total_rows; row += stride) {
    const int64_t bh = row / p.Np;
    const int n = static_cast<int>(row % p.Np);
    float acc = 0.f;
    if (n < p.N) {
      const int64_t base = (bh * p.N + n) * HD + c8 * 8;
      const uint4 ov = *reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.o) + base);
      const uint4 dv = *reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.dout) + base);
      const T* o8 = reinterpret_cast<const T*>(&ov);
      const T* d8 = reinterpret_cast<const T*>(&dv);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc = fmaf(static_cast<float>(o8[e]), static_cast<float>(d8[e]), acc);
    }
#pragma unroll
    for (int off = kTpr / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (c8 == 0) {
      p.Dvec[row] = acc;
      p.lse2[row] = n < p.N ? p.lse[bh * p.N + n] * 1.4426950408889634f : INFINITY;
    }
    float4* z = reinterpret_cast<float4*>(p.dqacc + row * HD + c8 * 8);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// ---------------------------------------------------------------------------
// bwd_plan (block masks only): for every work item (kv head, 128-row key
// block jt), the (group head, 128-row query block) pairs that see the key
// block, in walk order, and the number of 64-row steps they make.  One warp
// per item.  Entry = group head << 12 | query block.

struct BwdPlanParams {
  const uint8_t* bmask;
  long long bm_hstride;
  uint16_t* list;   // [BHkv * n_ktiles][cap]
  int* steps;       // [BHkv * n_ktiles]
  int N, Hq, Hkv, group, n_ktiles, n_qtiles, causal, window, cap, n_items;
};

__global__ void __launch_bounds__(256) fa_bwd_plan_kernel(const __grid_constant__ BwdPlanParams p) {
  const int item = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (item >= p.n_items) return;
  const int kvh = item / p.n_ktiles, jt = item % p.n_ktiles;
  const int g = kvh % p.Hkv;
  const int i0 = p.causal ? 2 * jt : 0;
  const int i_end = (p.causal && p.window > 0)
                        ? min(p.n_qtiles, (min(p.N - 1, jt * 128 + 126 + p.window)) / 64 + 1)
                        : p.n_qtiles;
  const int qb_lo = i0 >> 1, qb_hi = (i_end - 1) >> 1;
  uint16_t* list = p.list + static_cast<long long>(item) * p.cap;
  int pos = 0, steps = 0;
  for (int hg = 0; hg < p.group; ++hg) {
    const uint8_t* col = p.bmask + static_cast<long long>(g * p.group + hg) * p.bm_hstride + jt;
    for (int qb0 = qb_lo; qb0 <= qb_hi; qb0 += 32) {
      const int qb = qb0 + lane;
      const bool vis = qb <= qb_hi && __ldg(col + static_cast<long long>(qb) * p.n_ktiles) != 0;
      const unsigned m = __ballot_sync(0xffffffffu, vis);
      if (vis) list[pos + __popc(m & ((1u << lane) - 1u))] = static_cast<uint16_t>((hg << 12) | qb);
      int mine = 0;
      if (vis) mine = (2 * qb >= i0 && 2 * qb < i_end) + (2 * qb + 1 >= i0 && 2 * qb + 1 < i_end);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, off);
      steps += mine;
      pos += __popc(m);
    }
  }
  if (lane == 0) p.steps[item] = steps;
}

// ---------------------------------------------------------------------------
// bwd_main

struct BwdParams {
  CUtensorMap tm_q;      // [B*Hq][N][d], box 64 cols x 64 rows
  CUtensorMap tm_do;     // [B*Hq][N][d], box 64 x 64
  CUtensorMap tm_k;      // [B*Hkv][N][d], box 64 x 128
  CUtensorMap tm_v;      // [B*Hkv][N][d], box 64 x 128
  const float* lse2;     // [B*Hq][Np]
  const float* Dvec;     // [B*Hq][Np]
  float* dqacc;          // [B*Hq][Np][d] fp32 accumulator
  void* dk;              // [B*Hkv][N][d]
  void* dv;
  unsigned* work_counter;  // next work item (zeroed by bwd_pre)
  // block mask (kernels instantiated with BMASK): the walk of each item, from bwd_plan
  const uint16_t* plan_list;
  const int* plan_steps;
  int plan_cap;
  int N, Np, Hq, Hkv, group, n_ktiles, n_qtiles, BHkv, n_items;
  int chunk_heads;         // kv heads per chunk of the item order
  int window;              // causal sliding window of this many keys; 0: none
  // dropout (kernel instantiated with DROP), as in the forward pass
  uint32_t seed_lo, seed_hi, drop_t;
  float drop_scale;
  float scale_log2, scale;
};

template <int HD>
struct BwdLayout {
  static constexpr int kStages = 4;                     // Q / dO / lse2 / D ring
  static constexpr int kChunks = HD / 64;
  static constexpr int kKVBox = 128 * 128;              // 128 rows x 64 cols x 2 B
  static constexpr int kQBox = 64 * 128;                // 64 rows x 64 cols x 2 B
  static constexpr int kKVTile = kChunks * kKVBox;
  static constexpr int kQTile = kChunks * kQBox;
  static constexpr int kDsBytes = 128 * 128;            // dS^T: 128 key rows x 64 query cols x 2 B
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kKVTile;
  static constexpr int kOffQ = kOffV + kKVTile;
  static constexpr int kOffDO = kOffQ + kStages * kQTile;
  static constexpr int kOffDS = kOffDO + kStages * kQTile;
  static constexpr int kOffLse = kOffDS + 2 * kDsBytes;
  static constexpr int kOffD = kOffLse + kStages * 256;
  static constexpr int kOffBar = kOffD + kStages * 256;
  static constexpr int kSched = 4;                      // work-item ring slots
  // kv_full, q_full[S], step_done[S], sdp_full[2], ds_full[2], dq_full[2],
  // dq_drained[2], acc_done, acc_free, done, sched_full[4], sched_empty[4]
  static constexpr int kNumBars = 1 + 2 * kStages + 4 * 2 + 3 + 2 * kSched;
  static constexpr int kOffSched = kOffBar + kNumBars * 8;
  static constexpr int kOffTmemPtr = kOffSched + kSched * 4;
  static constexpr int kOffAbort = kOffTmemPtr + 4;
  static constexpr int kSmemBytes = kOffAbort + 4;
  // Tiles must sit on 1024-byte boundaries (128-byte swizzle atoms).  The
  // dynamic shared memory of a block without static shared memory starts on
  // such a boundary on sm_100; the d = 64 layout keeps spare bytes for
  // re-alignment anyway, the d = 128 layout has none to spare and checks.
  static constexpr int kDynSmem = kSmemBytes + (232448 - kSmemBytes >= 1024 ? 1024 : 0);
  static_assert(kDynSmem <= 232448, "shared memory budget");
};

// One work item of bwd_main: key block jt (128 rows) of kv head kvh.
struct BwdItem {
  int kvh;    // b * Hkv + kv head
  int kv0;    // first key row
  int i0;     // first query block (64 rows) that sees the key block
  int i_end;  // one past the last
  int nq;     // query blocks per query head
  int T;      // steps: group * nq (block mask: the visible ones)
  int bh0;    // first query head of the group (b * Hq + g * group)
  const uint16_t* plan;  // block mask: the item's walk
};

// The steps of an item in walk order, as (query head, 64-row query block):
// every query block of every group head, or under a block mask those of
// the item's plan (each visible 128-row block gives its 64-row halves that
// lie in [i0, i_end)).  Every role walks the same sequence.
template <bool BMASK>
struct BwdWalk {
  int t = 0, e = 0, half = 0;
  __device__ __forceinline__ void next(const BwdItem& it, int* bh, int* qt) {
    if constexpr (!BMASK) {
      *bh = it.bh0 + t / it.nq;
      *qt = it.i0 + t % it.nq;
      ++t;
    } else {
      for (;;) {
        const uint32_t ent = it.plan[e];
        const int q = 2 * static_cast<int>(ent & 0xFFFu) + half;
        const int hg = static_cast<int>(ent >> 12);
        if (++half == 2) {
          half = 0;
          ++e;
        }
        if (q >= it.i0 && q < it.i_end) {
          *bh = it.bh0 + hg;
          *qt = q;
          return;
        }
      }
    }
  }
};

// Item order: kv heads are taken in chunks of chunk_heads (as many as keep
// their Q, dO, K, V and dQ accumulator within part of L2); inside a chunk the
// key blocks go in order (under a causal mask the first ones see the most
// query blocks), each across the chunk's heads.  The blocks running at one
// time then share few heads, and the items claimed last are short ones, so
// the blocks finish close together.
template <bool CAUSAL, bool BMASK>
__device__ __forceinline__ BwdItem bwd_item(const BwdParams& p, int item) {
  BwdItem it;
  const int per_chunk = p.chunk_heads * p.n_ktiles;
  const int chunk = item / per_chunk;
  const int r = item - chunk * per_chunk;
  const int h0 = chunk * p.chunk_heads;
  const int nh = p.BHkv - h0 < p.chunk_heads ? p.BHkv - h0 : p.chunk_heads;
  it.kvh = h0 + r % nh;
  const int jt = r / nh;
  const int b = it.kvh / p.Hkv, g = it.kvh % p.Hkv;
  it.kv0 = jt * 128;
  it.i0 = CAUSAL ? 2 * jt : 0;
  // under a sliding window of W keys the block's keys are seen by queries
  // up to kv0 + 127 + W - 1 only
  const int i_end = (CAUSAL && p.window > 0)
                        ? min(p.n_qtiles, (min(p.N - 1, it.kv0 + 126 + p.window)) / 64 + 1)
                        : p.n_qtiles;
  it.i_end = i_end;
  it.nq = i_end - it.i0;
  it.T = p.group * it.nq;
  it.bh0 = b * p.Hq + g * p.group;
  it.plan = nullptr;
  if constexpr (BMASK) {
    const int idx = it.kvh * p.n_ktiles + jt;
    it.T = __ldg(p.plan_steps + idx);
    it.plan = p.plan_list + static_cast<long long>(idx) * p.plan_cap;
  }
  return it;
}

constexpr int kBwdThreads = 768;

template <int HD, bool BF16, bool CAUSAL, bool DROP, bool BMASK>
__global__ void __launch_bounds__(kBwdThreads, 1) fa_bwd_kernel(const __grid_constant__ BwdParams p) {
  static_assert(!(DROP && BMASK), "dropout and block masks are not combined");
  using L = BwdLayout<HD>;
  using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint8_t* sK = sm + L::kOffK;
  uint8_t* sV = sm + L::kOffV;
  uint8_t* sQ = sm + L::kOffQ;
  uint8_t* sDO = sm + L::kOffDO;
  uint8_t* sDS = sm + L::kOffDS;
  float* sLse = reinterpret_cast<float*>(sm + L::kOffLse);
  float* sD = reinterpret_cast<float*>(sm + L::kOffD);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kOffBar);
  uint64_t* kv_full = bars;
  uint64_t* q_full = kv_full + 1;
  // step_done[s]: every MMA of the step held in stage s has completed, so
  // the stage may be refilled and the step's dS^T buffer rewritten
  uint64_t* step_done = q_full + L::kStages;
  uint64_t* sdp_full = step_done + L::kStages;  // S^T and dP^T of a step buffer ready
  uint64_t* ds_full = sdp_full + 2;
  uint64_t* dq_full = ds_full + 2;
  uint64_t* dq_drained = dq_full + 2;
  uint64_t* acc_done = dq_drained + 2;  // every MMA of an item has completed
  uint64_t* acc_free = acc_done + 1;    // the epilogue has read an item's dK, dV
  uint64_t* done_bar = acc_free + 1;
  uint64_t* sched_full = done_bar + 1;
  uint64_t* sched_empty = sched_full + L::kSched;
  volatile int* sched_item = reinterpret_cast<volatile int*>(sm + L::kOffSched);
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(sm + L::kOffTmemPtr);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kOffAbort);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  if (sm + L::kSmemBytes > smem_raw + L::kDynSmem) {  // no room to re-align: refuse
    if (tid == 0) record_error(kStatusSmemAlign, kKernBwd, 0, 0);
    return;
  }
  constexpr int kDrainThreads = HD == 128 ? 128 : 64;
  constexpr int kSchedReaders = 1 + 16 + 4;  // MMA warp, softmax warps, drain warps

  if (tid == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&step_done[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sdp_full[i], 1);
      mbar_init(&ds_full[i], 512);
      mbar_init(&dq_full[i], 1);
      mbar_init(&dq_drained[i], kDrainThreads);
    }
    mbar_init(acc_done, 1);
    mbar_init(acc_free, 128);
    mbar_init(done_bar, 1);
    for (int i = 0; i < L::kSched; ++i) {
      mbar_init(&sched_full[i], 1);
      mbar_init(&sched_empty[i], kSchedReaders);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 21) {
    tmem_alloc(tmem_ptr, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr;
  const uint32_t tm_dV = tmem;
  const uint32_t tm_dK = tmem + 128;
  auto tm_S = [&](int buf) { return tmem + 256 + 128 * buf; };
  auto tm_dP = [&](int buf) { return tmem + 256 + 128 * buf + 64; };

  // Reads the n-th work item from the ring (a whole warp, or one thread with
  // `whole_warp` false); -1 ends the walk, -2 reports an abort.
  auto sched_read = [&](int n, bool whole_warp, uint32_t role) -> int {
    const int slot = n % L::kSched;
    const bool ok = mbar_wait(&sched_full[slot], (n / L::kSched) & 1, abort_flag, kKernBwd, role, 6);
    if (whole_warp ? !__all_sync(0xffffffffu, ok) : !ok) return -2;
    const int item = sched_item[slot];
    if (whole_warp) __syncwarp();
    if (!whole_warp || lane == 0) mbar_arrive(&sched_empty[slot]);
    return item;
  };

  // Steps are numbered across the items a block takes (g); the Q / dO ring
  // stage is g % kStages, the tensor-memory step buffer g & 1.
  if (warp == 20) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&p.tm_q);
      prefetch_tensormap(&p.tm_do);
      prefetch_tensormap(&p.tm_k);
      prefetch_tensormap(&p.tm_v);
      int gt = 0;
      for (int n = 0;; ++n) {
        const int slot = n % L::kSched;
        if (n >= L::kSched &&
            !mbar_wait(&sched_empty[slot], ((n / L::kSched) - 1) & 1, abort_flag, kKernBwd, 12, 1))
          break;
        int item = static_cast<int>(atomicAdd(p.work_counter, 1u));
        if (item >= p.n_items) item = -1;
        sched_item[slot] = item;
        mbar_arrive(&sched_full[slot]);
        if (item < 0) break;
        const BwdItem it = bwd_item<CAUSAL, BMASK>(p, item);
        if (it.T == 0) {
          // No step (block mask): no loads; the epilogue writes zeros.  The
          // wait on the previous item's completion is still taken, so that
          // every wait on acc_done stays within one phase of the barrier
          // (a parity wait two phases behind would pass at once).
          if (n > 0 && !mbar_wait(acc_done, (n - 1) & 1, abort_flag, kKernBwd, 12, 2)) break;
          continue;
        }
        BwdWalk<BMASK> walk;
        auto load_step = [&](int t) -> bool {
          const int g = gt + t, s = g % L::kStages;
          if (g >= L::kStages &&
              !mbar_wait(&step_done[s], ((g / L::kStages) - 1) & 1, abort_flag, kKernBwd, 12, 0))
            return false;
          int bh, qt;
          walk.next(it, &bh, &qt);
          mbar_expect_tx(&q_full[s], 2 * L::kQTile + 512);
          for (int c = 0; c < L::kChunks; ++c) {
            tma_load_3d(sQ + s * L::kQTile + c * L::kQBox, &p.tm_q, &q_full[s], c * 64, qt * 64, bh);
            tma_load_3d(sDO + s * L::kQTile + c * L::kQBox, &p.tm_do, &q_full[s], c * 64, qt * 64,
                        bh);
          }
          const int64_t row0 = static_cast<int64_t>(bh) * p.Np + qt * 64;
          bulk_load(sLse + s * 64, p.lse2 + row0, 256, &q_full[s]);
          bulk_load(sD + s * 64, p.Dvec + row0, 256, &q_full[s]);
          return true;
        };
        // Q / dO of the first steps may land while the previous item is
        // still running; K and V only once its MMAs (the last readers of
        // sK and sV) have completed.
        const int early = it.T < L::kStages ? it.T : L::kStages;
        bool ok = true;
        int t = 0;
        for (; ok && t < early; ++t) ok = load_step(t);
        if (ok && n > 0) ok = mbar_wait(acc_done, (n - 1) & 1, abort_flag, kKernBwd, 12, 2);
        if (!ok) break;
        mbar_expect_tx(kv_full, 2 * L::kKVTile);
        for (int c = 0; c < L::kChunks; ++c) {
          tma_load_3d(sK + c * L::kKVBox, &p.tm_k, kv_full, c * 64, it.kv0, it.kvh);
          tma_load_3d(sV + c * L::kKVBox, &p.tm_v, kv_full, c * 64, it.kv0, it.kvh);
        }
        for (; ok && t < it.T; ++t) ok = load_step(t);
        if (!ok) break;
        gt += it.T;
      }
    }
  } else if (warp == 21) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop with warp-uniform values; one elected
    // lane issues each MMA and commit.  Descriptors are formed once and
    // moved by constant offsets.
    constexpr uint32_t kIdS = idesc_f16(BF16, 128, 64, false, false);    // S^T, dP^T
    constexpr uint32_t kIdDQ = idesc_f16(BF16, 128, 64, true, true);     // dQ^T = K^T dS^T
    constexpr uint32_t kIdAcc = idesc_f16(BF16, 128, HD, false, true);   // dV, dK
    const uint32_t dsb = smem_u32(sDS);
    const uint64_t dK_k = sdesc_sw128(smem_u32(sK), 16, 1024);           // K, K-major
    const uint64_t dV_k = sdesc_sw128(smem_u32(sV), 16, 1024);           // V, K-major
    const uint64_t dK_mn = sdesc_sw128(smem_u32(sK), L::kKVBox, 1024);   // K^T, MN-major
    const uint64_t dQ_k = sdesc_sw128(smem_u32(sQ), 16, 1024);           // Q stage 0, K-major
    const uint64_t dQ_mn = sdesc_sw128(smem_u32(sQ), L::kQBox, 1024);    // Q stage 0, MN-major
    const uint64_t dO_k = sdesc_sw128(smem_u32(sDO), 16, 1024);
    const uint64_t dO_mn = sdesc_sw128(smem_u32(sDO), L::kQBox, 1024);
    const uint64_t dS_mn = sdesc_sw128(dsb, 8192, 1024);                 // dS^T buffer 0, MN-major
    const uint64_t dS_k = sdesc_sw128(dsb, 16, 1024);                    // dS^T buffer 0, K-major
    auto wait_all = [&](uint64_t* bar, uint32_t parity, uint32_t site) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, kKernBwd, 13, site));
    };
    auto issue_s = [&](int g) -> bool {
      const int s = g % L::kStages;
      if (!wait_all(&q_full[s], (g / L::kStages) & 1, 1)) return false;
      tc_fence_after();
      const uint32_t qs = s * L::kQTile;
#pragma unroll
      for (int k = 0; k < HD / 16; ++k)
        umma_ss_w(tm_S(g & 1), sdesc_add(dK_k, (k >> 2) * L::kKVBox + (k & 3) * 32),
                  sdesc_add(dQ_k, qs + (k >> 2) * L::kQBox + (k & 3) * 32), kIdS, k > 0);
      return true;
    };
    auto issue_dp = [&](int g) {
      const uint32_t os = (g % L::kStages) * L::kQTile;
#pragma unroll
      for (int k = 0; k < HD / 16; ++k)
        umma_ss_w(tm_dP(g & 1), sdesc_add(dV_k, (k >> 2) * L::kKVBox + (k & 3) * 32),
                  sdesc_add(dO_k, os + (k >> 2) * L::kQBox + (k & 3) * 32), kIdS, k > 0);
      umma_commit_w(&sdp_full[g & 1]);
    };
    int gt = 0;
    int n_loaded = 0;  // items whose K and V were loaded (every item with a step)
    bool ok = true;
    for (int n = 0; ok; ++n) {
      const int item = sched_read(n, true, 13);
      if (item < 0) break;
      const BwdItem it = bwd_item<CAUSAL, BMASK>(p, item);
      if (it.T == 0) {
        // Nothing to compute (block mask); the epilogue writes zero dK, dV.
        // As for every item, acc_done is committed only once the previous
        // item's epilogue has read its accumulators, which keeps the
        // epilogue's waits on acc_done within one phase.
        if (n > 0 && !wait_all(acc_free, (n - 1) & 1, 7)) break;
        umma_commit_w(acc_done);
        continue;
      }
      if (!wait_all(kv_full, n_loaded & 1, 0)) break;
      ++n_loaded;
      tc_fence_after();
      // S^T, dP^T of the item's first two steps.  dP^T of step g lands on
      // the columns that held dQ^T of step g-2 (the previous item's): wait
      // for its drain.
      for (int t = 0; ok && t < 2 && t < it.T; ++t) {
        const int g = gt + t;
        ok = issue_s(g);
        if (ok && g >= 2) {
          ok = wait_all(&dq_drained[g & 1], ((g - 2) >> 1) & 1, 4);
          tc_fence_after();
        }
        if (ok) issue_dp(g);
      }
      for (int t = 0; ok && t < it.T; ++t) {
        const int g = gt + t, buf = g & 1, s = g % L::kStages;
        if (!wait_all(&ds_full[buf], (g >> 1) & 1, 2)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t qs = s * L::kQTile;
        const uint32_t ds = buf * L::kDsBytes;
        // dQ^T (d x 64) = K^T dS^T over the 128 keys, into the dP^T columns.
        // K^T is K read MN-major; its second 64-feature half sits kKVBox
        // bytes further (for d = 64 that is V: rows 64..127 of the product
        // are unused).
#pragma unroll
        for (int k = 0; k < 8; ++k)
          umma_ss_w(tm_dP(buf), sdesc_add(dK_mn, k * 2048), sdesc_add(dS_mn, ds + k * 2048), kIdDQ,
                    k > 0);
        umma_commit_w(&dq_full[buf]);
        if (t == 0 && n > 0) {
          // this item's dV, dK start afresh in the accumulators that the
          // epilogue of the previous item reads
          if (!wait_all(acc_free, (n - 1) & 1, 7)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        // dV += P^T dO: P^T from tensor memory (the 16 queries of MMA k sit
        // in the first 8 columns of their own 16-column group), dO read
        // MN-major.
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_ts_w(tm_dV, tm_S(buf) + k * 16, sdesc_add(dO_mn, qs + k * 2048),
                    kIdAcc, (t > 0 || k > 0) ? 1u : 0u);
        // dK += dS^T Q: dS^T K-major from shared memory, Q read MN-major.
#pragma unroll
        for (int k = 0; k < 4; ++k)
          umma_ss_w(tm_dK, sdesc_add(dS_k, ds + k * 32), sdesc_add(dQ_mn, qs + k * 2048), kIdAcc,
                    (t > 0 || k > 0) ? 1u : 0u);
        umma_commit_w(&step_done[s]);
        if (t + 2 < it.T) {
          // S^T_{g+2} overwrites P^T_g, which dV_g (issued just before by
          // this warp) reads: the tensor core runs one thread's MMAs in issue
          // order, reading an MMA's operands before a later MMA writes its
          // result, so no wait is needed (a wait for an MMA's completion
          // costs several hundred idle tensor-core cycles on B200).
          // dP^T_{g+2} overwrites dQ^T_g: wait for the drain warps to read it.
          if (!issue_s(g + 2)) {
            ok = false;
            break;
          }
          if (!wait_all(&dq_drained[buf], (g >> 1) & 1, 4)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_dp(g + 2);
        }
      }
      if (!ok) break;
      umma_commit_w(acc_done);
      gt += it.T;
    }
    // every MMA this warp issued completes before tensor memory is freed
    umma_commit_w(done_bar);
    mbar_wait_drain(done_bar, 0, kKernBwd, 13, 5);
  } else if (warp < 16) {
    // ------------------------------------------------------------ softmax gradient
    // Every step is shared by the sixteen warps: warp w takes key rows
    // 32(w%4)..+31 and query columns 16(w/4)..+15.
    const int quarter = warp & 3, qq = warp >> 2;
    const int r = quarter * 32 + lane;                 // key row within the block
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float c_log2 = p.scale_log2;
    int gt = 0;
    for (int n = 0;; ++n) {
      const int item = sched_read(n, true, 0);
      if (item < 0) break;
      const BwdItem it = bwd_item<CAUSAL, BMASK>(p, item);
      const int kv_row = it.kv0 + r;
      const bool row_valid = kv_row < p.N;
      bool ok = true;
      BwdWalk<BMASK> walk;
      for (int t = 0; t < it.T; ++t) {
        const int g = gt + t, buf = g & 1, s = g % L::kStages;
        int bh_step, qt_step;                            // query head and block of the step
        walk.next(it, &bh_step, &qt_step);
        const int q_step = qt_step * 64;                 // first query of the step
        if (!__all_sync(0xffffffffu, mbar_wait(&sdp_full[buf], (g >> 1) & 1, abort_flag, kKernBwd, 0, 0))) {
          ok = false;
          break;
        }
        tc_fence_after();
        // S^T and dP^T of this warp's 16 query columns.  P^T of them is
        // packed into the first 8 of those tensor-memory columns of the S^T
        // buffer, where the dV product reads it.
        uint32_t v[16], vd[16];
        tmem_ld16(tm_S(buf) + lane_off + 16 * qq, v);
        tmem_ld16(tm_dP(buf) + lane_off + 16 * qq, vd);
        tmem_ld_wait();
        {
          const int q_first = q_step + qq * 16;          // first query of these 16 columns
          const float4* lse4 = reinterpret_cast<const float4*>(sLse + s * 64 + qq * 16);
          const float4* d4 = reinterpret_cast<const float4*>(sD + s * 64 + qq * 16);
          float pr[16];
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const float4 l4 = lse4[c4];
            pr[4 * c4 + 0] = ex2_approx(fmaf(__uint_as_float(v[4 * c4 + 0]), c_log2, -l4.x));
            pr[4 * c4 + 1] = ex2_approx(fmaf(__uint_as_float(v[4 * c4 + 1]), c_log2, -l4.y));
            pr[4 * c4 + 2] = ex2_approx(fmaf(__uint_as_float(v[4 * c4 + 2]), c_log2, -l4.z));
            pr[4 * c4 + 3] = ex2_approx(fmaf(__uint_as_float(v[4 * c4 + 3]), c_log2, -l4.w));
          }
          // causal: key kv_row is hidden from queries before it; padding keys
          // (kv_row >= N) carry no probability
          if (!row_valid) {
#pragma unroll
            for (int c = 0; c < 16; ++c) pr[c] = 0.f;
          } else {
            if (CAUSAL && q_first < kv_row) {
#pragma unroll
              for (int c = 0; c < 16; ++c)
                if (q_first + c < kv_row) pr[c] = 0.f;
            }
            // sliding window: query q sees key kv_row only while q < kv_row + W
            if (CAUSAL && p.window > 0 && q_first + 15 >= kv_row + p.window) {
#pragma unroll
              for (int c = 0; c < 16; ++c)
                if (q_first + c >= kv_row + p.window) pr[c] = 0.f;
            }
          }
          uint32_t pk[8];
          float fd[16];  // dropout factor of each of the 16 queries (1 without dropout)
          if constexpr (DROP) {
            // One Philox call covers 4 queries x 4 keys (word = query % 4,
            // byte = key % 4).  The 4 lanes of a quad hold 4 consecutive keys:
            // lane g of the quad draws the block of queries 4g..4g+3 of these
            // 16 and offers each lane its byte column (that lane's key, 4
            // queries); four rotations of a shuffle collect them.
            const int ql = lane & 3;
            const uint4 rnd = philox4x32_10(
                make_uint4(static_cast<uint32_t>(kv_row >> 2), static_cast<uint32_t>((q_first + 4 * ql) >> 2),
                           static_cast<uint32_t>(bh_step), 0u),
                p.seed_lo, p.seed_hi);
            uint32_t cols[4] = {0, 0, 0, 0};  // cols[g]: bytes of queries 4g..4g+3 for this key
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) {
              const uint32_t b = static_cast<uint32_t>((ql - rr) & 3);  // column the reader needs
              const uint32_t lo = __byte_perm(rnd.x, rnd.y, b | ((4u + b) << 4));
              const uint32_t hi = __byte_perm(rnd.z, rnd.w, b | ((4u + b) << 4));
              const uint32_t col = __byte_perm(lo, hi, 0x5410u);
              const uint32_t got = __shfl_sync(0xffffffffu, col, (lane & ~3) | ((ql + rr) & 3));
              const int g = (ql + rr) & 3;
              cols[0] = g == 0 ? got : cols[0];
              cols[1] = g == 1 ? got : cols[1];
              cols[2] = g == 2 ? got : cols[2];
              cols[3] = g == 3 ? got : cols[3];
            }
#pragma unroll
            for (int g = 0; g < 4; ++g)
#pragma unroll
              for (int u = 0; u < 4; ++u)
                fd[4 * g + u] = ((cols[g] >> (8 * u)) & 0xFFu) >= p.drop_t ? p.drop_scale : 0.f;
            // Z P for the dV product: the factor 1/(1-p) of the kept
            // probabilities is applied to dV once, in its epilogue, rather
            // than before P is rounded to 16 bits
#pragma unroll
            for (int i = 0; i < 8; ++i)
              pk[i] = pack2<BF16>(fd[2 * i] != 0.f ? pr[2 * i] : 0.f, fd[2 * i + 1] != 0.f ? pr[2 * i + 1] : 0.f);
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) pk[i] = pack2<BF16>(pr[2 * i], pr[2 * i + 1]);
          }
          tmem_st8(tm_S(buf) + lane_off + 16 * qq, pk);
          float dp[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) dp[c] = __uint_as_float(vd[c]);
          if constexpr (DROP) {
            // dP of P is dP' times the dropout factor
#pragma unroll
            for (int c = 0; c < 16; ++c) dp[c] *= fd[c];
          }
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const float4 dd = d4[c4];
            pr[4 * c4 + 0] *= dp[4 * c4 + 0] - dd.x;
            pr[4 * c4 + 1] *= dp[4 * c4 + 1] - dd.y;
            pr[4 * c4 + 2] *= dp[4 * c4 + 2] - dd.z;
            pr[4 * c4 + 3] *= dp[4 * c4 + 3] - dd.w;
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) pk[i] = pack2<BF16>(pr[2 * i], pr[2 * i + 1]);
          // dS^T buffer `buf` was last read by dQ_{g-2} and dK_{g-2}.  Both
          // were issued before dP_g, and the commit that completed sdp_full
          // for step g above arrives only once every MMA issued before it has
          // completed: the buffer is free.
          uint8_t* row_base = sDS + buf * L::kDsBytes + r * 128;
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int chunk = (qq * 2 + u) ^ (r & 7);
            *reinterpret_cast<uint4*>(row_base + chunk * 16) =
                make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
          }
        }
        fence_proxy_async_smem();
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&ds_full[buf]);
      }
      if (!ok) break;
      gt += it.T;
    }
  } else if (warp < 20) {
    // ------------------------------------------------------------ dQ drain, dK/dV epilogue
    // Lane f of drain warp w holds feature f = 32w + lane of dQ^T: 64 query
    // values.  They are added into the fp32 accumulator straight from
    // registers; for a fixed query the 32 lanes of a warp touch 128
    // consecutive bytes, so every reduction is one coalesced request.
    const int dw = warp - 16;                          // 0..3 == lane quarter
    const uint32_t lane_off = static_cast<uint32_t>(dw * 32) << 16;
    const bool drains = dw * 32 < HD;                  // warp holds real dQ^T rows
    int gt = 0;
    for (int n = 0;; ++n) {
      const int item = sched_read(n, true, 8);
      if (item < 0) break;
      const BwdItem it = bwd_item<CAUSAL, BMASK>(p, item);
      bool ok = true;
      BwdWalk<BMASK> walk;
      for (int t = 0; drains && t < it.T; ++t) {
        const int g = gt + t, buf = g & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&dq_full[buf], (g >> 1) & 1, abort_flag, kKernBwd, 8, 0))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t v0[32], v1[32];
        tmem_ld32(tm_dP(buf) + lane_off, v0);
        tmem_ld32(tm_dP(buf) + lane_off + 32, v1);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&dq_drained[buf]);
        int bh, qt;
        walk.next(it, &bh, &qt);
        float* dst = p.dqacc + (static_cast<size_t>(bh) * p.Np + qt * 64) * HD + dw * 32 + lane;
#pragma unroll
        for (int q = 0; q < 32; ++q) atomicAdd(dst + q * HD, __uint_as_float(v0[q]));
#pragma unroll
        for (int q = 0; q < 32; ++q) atomicAdd(dst + (32 + q) * HD, __uint_as_float(v1[q]));
      }
      if (!ok) break;
      gt += it.T;
      // epilogue: dV, dK (times scale) rows -> I/O dtype, written once
      if (!__all_sync(0xffffffffu, mbar_wait(acc_done, n & 1, abort_flag, kKernBwd, 8, 1))) break;
      tc_fence_after();
      const int r = dw * 32 + lane;
      const int kv_row = it.kv0 + r;
      const size_t row_off = (static_cast<size_t>(it.kvh) * p.N + kv_row) * HD;
      // an item without steps (block mask: no query sees the key block) has
      // dK = dV = 0 and never touched the accumulators
      const bool zero = it.T == 0;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t src = (which ? tm_dK : tm_dV) + lane_off;
        const float mul = which ? p.scale : (DROP ? p.drop_scale : 1.0f);
        T* dst = reinterpret_cast<T*>(which ? p.dk : p.dv) + row_off;
#pragma unroll
        for (int c = 0; c < HD; c += 32) {
          uint32_t v[32];
          if (!zero) {
            tmem_ld32(src + c, v);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0u;
          }
          if (kv_row < p.N) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              uint4 w;
              w.x = pack2<BF16>(__uint_as_float(v[8 * u + 0]) * mul, __uint_as_float(v[8 * u + 1]) * mul);
              w.y = pack2<BF16>(__uint_as_float(v[8 * u + 2]) * mul, __uint_as_float(v[8 * u + 3]) * mul);
              w.z = pack2<BF16>(__uint_as_float(v[8 * u + 4]) * mul, __uint_as_float(v[8 * u + 5]) * mul);
              w.w = pack2<BF16>(__uint_as_float(v[8 * u + 6]) * mul, __uint_as_float(v[8 * u + 7]) * mul);
              *reinterpret_cast<uint4*>(dst + c + 8 * u) = w;
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(acc_free);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 21) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// bwd_post: dQ = scale * accumulator -> I/O dtype (8 elements per thread)

template <int HD, bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_post_kernel(const float* __restrict__ dqacc,
                                                          void* __restrict__ dq_, int N, int Np,
                                                          int64_t total_vec, float scale) {
  using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
  constexpr int kVecPerRow = HD / 8;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total_vec;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = i / kVecPerRow;  // row of the [B*Hq][N] output
    const int cv = static_cast<int>(i % kVecPerRow);
    const int64_t bh = row / N;
    const int64_t n = row % N;
    const float4* src = reinterpret_cast<const float4*>(dqacc + (bh * Np + n) * HD + cv * 8);
    const float4 a = src[0], c = src[1];
    uint4 w;
    w.x = pack2<BF16>(a.x * scale, a.y * scale);
    w.y = pack2<BF16>(a.z * scale, a.w * scale);
    w.z = pack2<BF16>(c.x * scale, c.y * scale);
    w.w = pack2<BF16>(c.z * scale, c.w * scale);
    reinterpret_cast<uint4*>(reinterpret_cast<T*>(dq_) + row * HD)[cv] = w;
  }
}

// ---------------------------------------------------------------------------
// failure-path self test: one barrier that nobody signals

__global__ void wait_timeout_selftest_kernel() {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, kKernSelftest, 0, 0);
  __syncthreads();
}

}  // namespace fa
