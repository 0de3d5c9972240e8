// Decode over a paged key/value cache: a few new query tokens per sequence
// attend to every cached token of their sequence ("Paper digest:
// FlashAttention", section "Limits": decode-time attention over a KV cache;
// "Flash Attention" glossary, PagedAttention entry: the cache is held in
// fixed-size blocks found through a block table).
//
// Sequence b holds L = seq_lens[b] cached tokens whose last Nq are the new
// queries: query t (position L - Nq + t) sees keys 0 .. L - Nq + t.  Key k of
// sequence b sits in physical page block_table[b][k / P], slot k % P, of
// caches laid out [num_pages][Hkv][P][d].  The rows of one thread block are
// the G = Hq / Hkv query heads of a kv head times the Nq tokens (R = G * Nq
// <= 32 rows), so every key and value read from memory serves all of them.
//
// The work is bound by memory (each cached byte is read once, a handful of
// flops per byte), so it is split along the cache: a block takes one split
// of the pages of one (sequence, kv head), keeps an online softmax over it
// and writes its unnormalised O with the row reference max m and sum l
// (base 2); a second kernel merges the splits: m* = max m_s, l* = sum l_s
// 2^(m_s - m*), O = sum O_s 2^(m_s - m*) / l*, lse = ln 2 (m* + log2 l*).
//
// Inside a block the cache is walked in tiles of 128 keys (128 / P pages):
//   warp 4     TMA loads of each page's K and V rows (two 128-byte-swizzled
//              boxes of 64 features per page at d = 128) into a ring of
//              tile slots; a page outside the sequence or with a bad table
//              entry is loaded from outside the tensor (zeros) and hidden;
//   warp 5     tcgen05.mma, one elected lane: S^T = K Q^T (M = 128 keys,
//              N = the rows padded to 16 or 32, K = d) into tensor memory,
//              then O^T += V^T P^T (M = d, N = rows, K = 128 keys), V read
//              MN-major straight from its [key][d] rows;
//   warps 0-3  one thread per key (its tensor-memory lane): scores of the R
//              rows, the online-softmax reference max, the probabilities
//              written to shared memory as the B operand of the P V product.
// The reference max of a row moves only when a tile's scores exceed it by
// more than 8 (log2), so the running O^T is rescaled in tensor memory only
// then (exact: O and l share the reference).
#pragma once

#include <type_traits>

#include "sm100.cuh"

namespace fa {

constexpr uint32_t kKernDecode = 10;
constexpr uint32_t kKernDecodeMerge = 11;
constexpr uint32_t kStatusBadInput = 7;  // a block-table entry or sequence length out of range
constexpr int kDecodeThreads = 192;      // softmax warps 0-3, TMA warp 4, MMA warp 5
constexpr int kDecodeMaxRows = 32;
constexpr int kDecodeMaxPage = 128;
constexpr int kDecodeTile = 128;         // keys per tile: the M of S^T = K Q^T
constexpr int kDecodeSMs = 148;          // B200

struct DecodeParams {
  CUtensorMap tm_k;       // K cache as [num_pages * Hkv][P][d], box 64 features x P rows
  CUtensorMap tm_v;       // V cache, the same
  CUtensorMap tm_q;       // q as [B * Hq * Nq][d], box 64 features x NP rows
  const void* q;          // [B][Hq][Nq][d]
  const int* table;       // [B][max_pages]
  const int* lens;        // [B]
  float* part_o;          // [B][Hq][Nq][S][d]   unnormalised partial outputs
  float* part_ml;         // [B][Hq][Nq][S][2]   (m, l) in base 2
  void* o;                // [B][Hq][Nq][d]
  float* lse;             // [B][Hq][Nq]
  int B, Hq, Hkv, Nq, P, max_pages, num_pages, S, pages_per_split;
  float scale_log2;
};

// Splits of each (sequence, kv head), for a grid of B * Hkv * S blocks: at
// least four waves of the blocks that fit on a B200 at once (one per SM at
// d = 128, two at d = 64); among S0 .. 2 S0 the count whose last wave is the
// fullest; at least 4 pages a split.
inline int decode_splits(int B, int Hkv, int d, int max_pages) {
  const int64_t bh = static_cast<int64_t>(B) * Hkv > 0 ? static_cast<int64_t>(B) * Hkv : 1;
  const int64_t slots = kDecodeSMs * (d == 64 ? 2 : 1);
  const int64_t s0 = (4 * slots + bh - 1) / bh;
  const int64_t cap = max_pages / 4 > 1 ? max_pages / 4 : 1;
  int64_t best = s0 < cap ? s0 : cap;
  double best_eff = -1.0;
  for (int64_t s = s0; s <= 2 * s0 && s <= cap; ++s) {
    const int64_t blocks = bh * s;
    const int64_t waves = (blocks + slots - 1) / slots;
    const double eff = static_cast<double>(blocks) / static_cast<double>(waves * slots);
    if (eff > best_eff + 1e-9) {
      best = s;
      best_eff = eff;
    }
  }
  return static_cast<int>(best < 1 ? 1 : best);
}

inline size_t decode_workspace_bytes(int B, int Hq, int Hkv, int Nq, int d, int max_pages) {
  const int64_t S = decode_splits(B, Hkv, d, max_pages);
  const int64_t rows = static_cast<int64_t>(B) * Hq * Nq * S;
  return static_cast<size_t>(rows) * 4u * static_cast<size_t>(d + 2);
}

// Shared memory of the split kernel for head dimension HD and row bound RB
// (offsets from a 1024-byte-aligned base).
template <int HD, int RB>
struct DecodeLayout {
  static constexpr int NP = RB < 16 ? 16 : RB;           // MMA N: rows padded to 16 or 32
  static constexpr int kChunks = HD / 64;                // 64-feature boxes per row
  static constexpr int kChunkBytes = kDecodeTile * 128;  // 128 keys x 128 bytes
  // a slot: the V chunks, then the K chunks (at d = 64 the unused upper half
  // of the product V^T P^T reads the K chunk that follows: finite data)
  static constexpr int kSlotBytes = 2 * kChunks * kChunkBytes;
  static constexpr int kSlots = 3;
  static constexpr int kQChunk = NP * 128;               // Q rows of one feature box
  static constexpr int kPChunk = NP * 128;               // P rows of 64 keys
  static constexpr int kPBytes = 2 * kPChunk;            // one buffer: 128 keys
  static constexpr int kOffQ = kSlots * kSlotBytes;
  static constexpr int kOffP = kOffQ + kChunks * kQChunk;
  static constexpr int kOffFlag = kOffP + 2 * kPBytes;   // int [2][4]
  static constexpr int kOffMax = kOffFlag + 8 * 4;       // float [2][4][32]
  static constexpr int kOffSum = kOffMax + 2 * 4 * 32 * 4;  // float [2][4][32]
  static constexpr int kOffBar = kOffSum + 2 * 4 * 32 * 4;
  // kv_full[slots], kv_empty[slots], s_full[2], p_full[2], pv_done[2], done,
  // q_full, q_empty
  static constexpr int kNumBars = 2 * kSlots + 9;
  static constexpr int kOffTmemPtr = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmemPtr + 4;
  static constexpr int kBytes = kOffAbort + 4;
  static constexpr int kDynSmem = kBytes + 1024;         // room to align the base
  static_assert(kOffQ % 1024 == 0 && kOffP % 1024 == 0 && kQChunk % 1024 == 0, "swizzle atoms");
  static_assert(kDynSmem <= 232448, "shared memory budget");
};

// tensor memory <-> registers, 32 lanes x N 32-bit columns (N = 4 .. 32)
template <int N>
__device__ __forceinline__ void tmem_ld_n(uint32_t taddr, uint32_t* r) {
  if constexpr (N == 4) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
  } else if constexpr (N == 8) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
  } else if constexpr (N == 16) {
    tmem_ld16(taddr, r);
  } else {
    static_assert(N == 32, "column count");
    tmem_ld32(taddr, r);
  }
}

template <int N>
__device__ __forceinline__ void tmem_st_n(uint32_t taddr, const uint32_t* r) {
  if constexpr (N == 4) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3])
                 : "memory");
  } else if constexpr (N == 8) {
    tmem_st8(taddr, r);
  } else if constexpr (N == 16) {
    tmem_st16(taddr, r);
  } else {
    static_assert(N == 32, "column count");
    tmem_st16(taddr, r);
    tmem_st16(taddr + 16, r + 16);
  }
}

// One work item: a split of the pages of one sequence and kv head.
struct DecodeItem {
  int b, g, split, Lb, pg0, pg1, n_tiles;
  bool len_ok;
};

__device__ __forceinline__ DecodeItem decode_item(const DecodeParams& p, int w) {
  DecodeItem it;
  it.split = w % p.S;
  it.g = (w / p.S) % p.Hkv;
  it.b = w / (p.S * p.Hkv);
  const int P = p.P, ppt = kDecodeTile / P;
  it.Lb = p.lens[it.b];
  it.len_ok = it.Lb >= p.Nq && it.Lb <= p.max_pages * P;
  const int n_pages = it.len_ok ? (it.Lb + P - 1) / P : 0;
  it.pg0 = it.split * p.pages_per_split;  // pages_per_split is a multiple of ppt
  it.pg1 = min(n_pages, it.pg0 + p.pages_per_split);
  it.n_tiles = it.pg1 > it.pg0 ? (it.pg1 - it.pg0 + ppt - 1) / ppt : 0;
  return it;
}

// Persistent: a block takes work items blockIdx.x, blockIdx.x + gridDim.x,
// ...  The tile ring, the tensor-memory buffers and the barrier phases run on
// across items (tiles are numbered over the block's items), so the fill of
// the ring and the pipeline's start are paid once per block, not per split.
// RB: compile-time bound on the rows (4, 8, 16 or 32, the smallest >= R), so
// the per-row loops unroll to the rows that exist.
// Programmatic dependent launch: the split and merge kernels are launched as
// dependents of the kernel before them on the stream, so that each may be
// scheduled (and run its set-up) while that kernel still runs.
// Lets the next kernel, if launched as a dependent, be scheduled now.
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Waits until the kernels this one depends on have completed and their
// memory is visible (returns at once when launched without the dependency).
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

template <int HD, bool BF16, int RB>
__global__ void __launch_bounds__(kDecodeThreads, 1) fa_decode_split_kernel(const __grid_constant__ DecodeParams p) {
  using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
  using L = DecodeLayout<HD, RB>;
  constexpr int NP = L::NP;
  constexpr int NS = L::kSlots;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = sm + L::kOffQ;
  uint8_t* sP = sm + L::kOffP;
  volatile int* sFlag = reinterpret_cast<volatile int*>(sm + L::kOffFlag);
  float* sMax = reinterpret_cast<float*>(sm + L::kOffMax);
  float* sSum = reinterpret_cast<float*>(sm + L::kOffSum);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kOffBar);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + NS;
  uint64_t* s_full = kv_empty + NS;
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* done_bar = pv_done + 2;
  uint64_t* q_full = done_bar + 1;   // the q rows of an item landed
  uint64_t* q_empty = q_full + 1;    // the S products of an item (readers of sQ) completed
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(sm + L::kOffTmemPtr);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::kOffAbort);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.Hq / p.Hkv, R = G * p.Nq, P = p.P;
  const int ppt = kDecodeTile / P;  // pages per tile
  const int n_work = p.B * p.Hkv * p.S;

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(done_bar, 1);
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_ptr, 128);
    tmem_relinquish();
  }
  // The set-up above may overlap the previous kernel on the stream; no
  // global memory is touched before this wait.
  grid_dependency_wait();
  grid_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr;
  const uint32_t tm_O = tmem + 2 * NP;  // O^T: lanes = features, columns = rows

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&p.tm_k);
      prefetch_tensormap(&p.tm_v);
      prefetch_tensormap(&p.tm_q);
      int j = 0;   // tiles issued, over the block's items
      int qi = 0;  // items with tiles so far
      bool ok = true;
      for (int w = blockIdx.x; ok && w < n_work; w += gridDim.x) {
        const DecodeItem I = decode_item(p, w);
        if (!I.len_ok && I.split == 0 && I.g == 0) record_error(kStatusBadInput, kKernDecode, 4, 0);
        if (I.n_tiles == 0) continue;
        // the item's q rows (row r: head g*G + r / Nq, token r % Nq; rows
        // past R are the next heads' or zeros, and their columns of S^T and
        // O^T are never read), once the previous item's S products are done
        if (qi > 0 && !(ok = mbar_wait(q_empty, (qi - 1) & 1, abort_flag, kKernDecode, 4, 3))) break;
        mbar_expect_tx(q_full, static_cast<uint32_t>(L::kChunks * L::kQChunk));
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_3d(sQ + c * L::kQChunk, &p.tm_q, q_full, c * 64, (I.b * p.Hq + I.g * G) * p.Nq, 0);
        ++qi;
        for (int jj = 0; jj < I.n_tiles; ++jj) {
          const int s = j % NS;
          if (j >= NS && !(ok = mbar_wait(&kv_empty[s], ((j / NS) - 1) & 1, abort_flag, kKernDecode, 4, 0)))
            break;
          mbar_expect_tx(&kv_full[s], static_cast<uint32_t>(L::kSlotBytes));
          uint8_t* slot = sm + s * L::kSlotBytes;
          for (int pp = 0; pp < ppt; ++pp) {
            const int pg = I.pg0 + jj * ppt + pp;
            int outer = -1;  // outside the tensor: the box reads as zeros
            if (pg < I.pg1) {
              const int phys = p.table[static_cast<size_t>(I.b) * p.max_pages + pg];
              if (phys >= 0 && phys < p.num_pages)
                outer = phys * p.Hkv + I.g;
              else
                record_error(kStatusBadInput, kKernDecode, 4, 1);
            }
#pragma unroll
            for (int c = 0; c < L::kChunks; ++c) {
              tma_load_3d(slot + c * L::kChunkBytes + pp * P * 128, &p.tm_v, &kv_full[s], c * 64, 0, outer);
              tma_load_3d(slot + (L::kChunks + c) * L::kChunkBytes + pp * P * 128, &p.tm_k, &kv_full[s],
                          c * 64, 0, outer);
            }
          }
          ++j;
        }
      }
      // the copies of the last tile issued into each slot, and the last q
      // rows, land before the block exits (all earlier ones were waited for
      // by the MMA warp)
      for (int jx = j > NS ? j - NS : 0; jx < j; ++jx)
        mbar_wait_drain(&kv_full[jx % NS], (jx / NS) & 1, kKernDecode, 4, 2);
      if (qi > 0) mbar_wait_drain(q_full, (qi - 1) & 1, kKernDecode, 4, 4);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t kIdS = idesc_f16(BF16, 128, NP, false, false);  // S^T = K Q^T
    constexpr uint32_t kIdO = idesc_f16(BF16, 128, NP, true, false);   // O^T += V^T P^T
    const uint64_t dK = sdesc_sw128(smem_u32(sm) + L::kChunks * L::kChunkBytes, 16, 1024);  // slot 0 K
    const uint64_t dVt = sdesc_sw128(smem_u32(sm), L::kChunkBytes, 1024);  // slot 0 V, MN-major
    const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t dP = sdesc_sw128(smem_u32(sP), 16, 1024);
    auto wait_all = [&](uint64_t* bar, uint32_t parity, uint32_t site) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, kKernDecode, 5, site));
    };
    // O^T += V^T P^T of tile t (over the block's items); `first`: the item's
    // first tile, which starts O^T afresh
    auto issue_pv = [&](int t, bool first) -> bool {
      if (!wait_all(&p_full[t & 1], (t >> 1) & 1, 1)) return false;
      tc_fence_after();
      const uint32_t so = (t % NS) * L::kSlotBytes, po = (t & 1) * L::kPBytes;
#pragma unroll
      for (int k = 0; k < kDecodeTile / 16; ++k)
        umma_ss_w(tm_O, sdesc_add(dVt, so + k * 2048), sdesc_add(dP, po + (k >> 2) * L::kPChunk + (k & 3) * 32),
                  kIdO, (!first || k > 0) ? 1u : 0u);
      umma_commit_w(&kv_empty[t % NS]);
      umma_commit_w(&pv_done[t & 1]);
      return true;
    };
    bool ok = true;
    int j = 0;   // tiles, over the block's items
    int qi = 0;  // items with tiles so far
    for (int w = blockIdx.x; ok && w < n_work; w += gridDim.x) {
      const DecodeItem I = decode_item(p, w);
      if (I.n_tiles == 0) continue;
      if (!(ok = wait_all(q_full, qi & 1, 2))) break;
      tc_fence_after();
      ++qi;
      for (int jj = 0; jj < I.n_tiles; ++jj, ++j) {
        const int s = j % NS;
        if (!(ok = wait_all(&kv_full[s], (j / NS) & 1, 0))) break;
        tc_fence_after();
        const uint32_t so = s * L::kSlotBytes;
        // S^T_j lands in buffer j % 2, last read by the softmax of tile j - 2,
        // whose P the PV product issued before this one waited for
#pragma unroll
        for (int k = 0; k < HD / 16; ++k)
          umma_ss_w(tmem + (j & 1) * NP, sdesc_add(dK, so + (k >> 2) * L::kChunkBytes + (k & 3) * 32),
                    sdesc_add(dQ, (k >> 2) * L::kQChunk + (k & 3) * 32), kIdS, k > 0 ? 1u : 0u);
        umma_commit_w(&s_full[j & 1]);
        if (jj + 1 == I.n_tiles) umma_commit_w(q_empty);  // the item's last S: sQ may be refilled
        if (jj > 0 && !(ok = issue_pv(j - 1, jj == 1))) break;
      }
      if (ok) ok = issue_pv(j - 1, I.n_tiles == 1);
    }
    // every MMA this warp issued completes before tensor memory is freed
    umma_commit_w(done_bar);
    mbar_wait_drain(done_bar, 0, kKernDecode, 5, 3);
  } else {
    // ------------------------------------------------------------ softmax (warps 0-3)
    // Thread i owns key i of every tile (tensor-memory lane i of S^T) and,
    // for the rescales and the epilogue, feature i of O^T.
    const int i = tid;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float c_log2 = p.scale_log2;
    bool ok = true;
    int j = 0;   // tiles, over the block's items
    int ei = 0;  // items, over the block
    for (int w = blockIdx.x; ok && w < n_work; w += gridDim.x, ++ei) {
      const DecodeItem I = decode_item(p, w);
      float ref[RB], lp[RB];
#pragma unroll
      for (int r = 0; r < RB; ++r) {
        ref[r] = -INFINITY;
        lp[r] = 0.f;
      }
      // whether this thread's key of the item's tile jj sits in a page that was loaded
      auto page_loaded = [&](int jj) -> bool {
        const int pg = I.pg0 + jj * ppt + i / P;
        if (pg >= I.pg1) return false;
        const int phys = __ldg(p.table + static_cast<size_t>(I.b) * p.max_pages + pg);
        return phys >= 0 && phys < p.num_pages;
      };
      bool loaded_next = I.n_tiles > 0 ? page_loaded(0) : false;
      for (int jj = 0; jj < I.n_tiles; ++jj, ++j) {
        const int buf = j & 1;
        const bool loaded = loaded_next;
        if (jj + 1 < I.n_tiles) loaded_next = page_loaded(jj + 1);
        // warp-uniform, as the tensor-memory loads below must be
        const bool fail = !__all_sync(0xffffffffu, mbar_wait(&s_full[buf], (j >> 1) & 1, abort_flag, kKernDecode, 0, 0));
        tc_fence_after();
        uint32_t sv[RB];
        if (!fail) {
          tmem_ld_n<RB>(tmem + buf * NP + lane_off, sv);
          tmem_ld_wait();
        }
        const int key = (I.pg0 + jj * ppt) * P + i;
        float t[RB];
        bool need = false;
#pragma unroll
        for (int r = 0; r < RB; ++r) {
          t[r] = -INFINITY;
          if (r < R && !fail) {
            const bool vis = loaded && key <= I.Lb - p.Nq + r % p.Nq;
            t[r] = vis ? __uint_as_float(sv[r]) * c_log2 : -INFINITY;
            need |= t[r] > ref[r] + 8.f;
          }
        }
        // One decision for all 128 threads: whether a reference max moves (and
        // whether a wait failed).  Every softmax thread reaches every barrier.
        const bool wneed = __any_sync(0xffffffffu, need), wfail = __any_sync(0xffffffffu, fail);
        if (lane == 0) sFlag[buf * 4 + warp] = (wneed ? 1 : 0) | (wfail ? 2 : 0);
        named_barrier_sync(1, 128);
        const int f = sFlag[buf * 4 + 0] | sFlag[buf * 4 + 1] | sFlag[buf * 4 + 2] | sFlag[buf * 4 + 3];
        if (f & 2) {
          ok = false;
          break;
        }
        if (f & 1) {
          // per-row maxima of the tile over the 128 keys
#pragma unroll
          for (int r = 0; r < RB; ++r) {
            if (r < R) {
              float m = t[r];
#pragma unroll
              for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
              if (lane == 0) sMax[(buf * 4 + warp) * 32 + r] = m;
            }
          }
          named_barrier_sync(1, 128);
          float fac[RB];
#pragma unroll
          for (int r = 0; r < RB; ++r) {
            fac[r] = 1.f;
            if (r < R) {
              const float* mr = sMax + buf * 4 * 32 + r;
              const float nm = fmaxf(fmaxf(ref[r], fmaxf(mr[0], mr[32])), fmaxf(mr[64], mr[96]));
              if (nm != ref[r]) fac[r] = ref[r] == -INFINITY ? 0.f : ex2_approx(ref[r] - nm);
              ref[r] = nm;
              lp[r] *= fac[r];
            }
          }
          // O^T holds the products of the item's tiles before this one: once
          // they are complete, scale its row columns (this thread: feature lane i)
          if (jj > 0) {
            if (__all_sync(0xffffffffu, mbar_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag, kKernDecode, 0, 1))) {
              tc_fence_after();
              uint32_t ov[RB];
              tmem_ld_n<RB>(tm_O + lane_off, ov);
              tmem_ld_wait();
#pragma unroll
              for (int r = 0; r < RB; ++r) ov[r] = __float_as_uint(__uint_as_float(ov[r]) * fac[r]);
              tmem_st_n<RB>(tm_O + lane_off, ov);
              tmem_st_wait();
            }
          }
        }
        // P of this thread's key for every row; buffer `buf` was last read by
        // the PV product of tile j - 2
        float pr[RB];
#pragma unroll
        for (int r = 0; r < RB; ++r) {
          pr[r] = 0.f;
          if (r < R && t[r] != -INFINITY) {
            pr[r] = ex2_approx(t[r] - ref[r]);
            lp[r] += pr[r];
          }
        }
        if (j >= 2) mbar_wait(&pv_done[buf], ((j - 2) >> 1) & 1, abort_flag, kKernDecode, 0, 2);
        // P[row][key] in the K-major, 128-byte-swizzled B operand of V^T P^T:
        // 64 keys (128 bytes) per row and box; the 32 lanes of a warp write 64
        // consecutive bytes of one row at a time
        uint8_t* pb = sP + buf * L::kPBytes + (i >> 6) * L::kPChunk + (i & 7) * 2;
#pragma unroll
        for (int r = 0; r < RB; ++r)
          if (r < R) *reinterpret_cast<T*>(pb + r * 128 + ((((i & 63) >> 3) ^ (r & 7)) << 4)) = static_cast<T>(pr[r]);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&p_full[buf]);
      }
      // ---------------------------------------------------------------- epilogue of the item
      // l of each row: the sum of the 128 threads' partial sums (sSum is
      // double-buffered by item, so no thread still reads the previous one's)
      float* ss = sSum + (ei & 1) * 4 * 32;
#pragma unroll
      for (int r = 0; r < RB; ++r) {
        if (r < R) {
          float sum = lp[r];
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
          if (lane == 0) ss[warp * 32 + r] = sum;
        }
      }
      named_barrier_sync(1, 128);
      bool have = ok && I.n_tiles > 0;
      if (have) {
        have = mbar_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag, kKernDecode, 0, 3);
        tc_fence_after();
      }
      uint32_t ov[RB];
#pragma unroll
      for (int r = 0; r < RB; ++r) ov[r] = 0u;
      if (__all_sync(0xffffffffu, have)) {
        tmem_ld_n<RB>(tm_O + lane_off, ov);
        tmem_ld_wait();
      }
      if (i < HD) {
#pragma unroll
        for (int r = 0; r < RB; ++r) {
          if (r < R) {
            const int h = I.g * G + r / p.Nq, tq = r % p.Nq;
            const size_t row = ((static_cast<size_t>(I.b) * p.Hq + h) * p.Nq + tq) * p.S + I.split;
            p.part_o[row * HD + i] = __uint_as_float(ov[r]);
          }
        }
      }
      if (i < R) {
        float m = -INFINITY;
#pragma unroll
        for (int r = 0; r < RB; ++r)
          if (r == i) m = ref[r];
        const float l = ss[i] + ss[32 + i] + ss[64 + i] + ss[96 + i];
        const int h = I.g * G + i / p.Nq, tq = i % p.Nq;
        const size_t row = ((static_cast<size_t>(I.b) * p.Hq + h) * p.Nq + tq) * p.S + I.split;
        p.part_ml[row * 2 + 0] = l > 0.f ? m : -INFINITY;
        p.part_ml[row * 2 + 1] = l;
      }
      // this item's O^T has been read: the next item's first P V (after
      // this thread's next arrival on p_full) may overwrite it
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// Merge of the splits of one (sequence, query head, token): one block of HD
// threads, thread c owns output column c.
template <int HD, bool BF16>
__global__ void __launch_bounds__(HD) fa_decode_merge_kernel(const __grid_constant__ DecodeParams p) {
  using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
  const size_t row = blockIdx.x;  // (b * Hq + h) * Nq + t
  const int c = threadIdx.x;
  grid_dependency_wait();  // the splits' partial rows are complete and visible
  grid_launch_dependents();
  const float* ml = p.part_ml + row * p.S * 2;
  float m_star = -INFINITY;
  for (int s = 0; s < p.S; ++s) m_star = fmaxf(m_star, ml[2 * s]);
  float l_star = 0.f, o = 0.f;
  if (m_star != -INFINITY) {
    for (int s = 0; s < p.S; ++s) {
      const float m = ml[2 * s];
      if (m == -INFINITY) continue;  // an empty split
      const float w = ex2_approx(m - m_star);
      l_star += ml[2 * s + 1] * w;
      o += p.part_o[(row * p.S + s) * HD + c] * w;
    }
  }
  const float out = l_star > 0.f ? o / l_star : 0.f;
  reinterpret_cast<T*>(p.o)[row * HD + c] = static_cast<T>(out);
  if (c == 0)
    p.lse[row] = l_star > 0.f ? (m_star + __log2f(l_star)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace fa
